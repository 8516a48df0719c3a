"""Weight arena and opt-in L2 residency on the GPU: packed weights give bit-identical results,
and clearing the window restores the context's persisting-L2 set-aside."""
import pytest
import torch

from draft_block_causal_b200 import domino, synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from tests import gpu_common as G
else:
    G = None


def _case(B, seed):
    wl = dict(B=B, L=16, d=512, Hs=256, r=256, V=12000, dtype=1, weight_seed=seed, input_seed=seed + 1,
              s0_std=0.2, peak=2.0, name="arena")
    return synth.make_workload(wl)


@pytest.mark.parametrize("B", [1, 32], ids=["fused", "per-phase"])
def test_packed_weights_give_identical_results(B):
    data = _case(B, 400 + B)
    w, lb, h, S0 = G.device_inputs(data)
    packed = domino.pack_weights(w)
    for n in ("W2", "W1", "W_hh", "W_ih", "b_ih", "b_hh"):
        assert torch.equal(getattr(packed, n), getattr(w, n))
    # one contiguous range, in the documented order
    ptrs = [getattr(packed, n).data_ptr() for n in ("W2", "W1", "W_hh", "W_ih", "b_ih", "b_hh")]
    assert ptrs == sorted(ptrs) and ptrs[-1] - ptrs[0] < domino.arena_bytes(w)
    a = domino.draft_greedy(w, lb, h, S0, logits_out=True, states_out=True)
    b = domino.draft_greedy(packed, lb, h, S0, logits_out=True, states_out=True)
    torch.cuda.synchronize()
    # every summation order is fixed (split-K pieces in order; fixed-point atomics in the fused
    # kernels): the packed copy gives the same bits
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def _persisting_limit():
    try:
        from cuda.bindings import runtime as rt
    except ImportError:
        return None
    err, v = rt.cudaDeviceGetLimit(rt.cudaLimit.cudaLimitPersistingL2CacheSize)
    return int(v) if int(err) == 0 else None


def test_persistence_window_set_and_cleared():
    import dataclasses
    data = _case(1, 410)
    w, lb, h, S0 = G.device_inputs(data)
    packed = domino.pack_weights(w)
    before = _persisting_limit()
    s = torch.cuda.Stream()
    ref = domino.draft_greedy(packed, lb, h, S0, logits_out=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        domino.set_l2_persistence(packed, s, 1.0)
        during = _persisting_limit()
        got = domino.draft_greedy(packed, lb, h, S0, logits_out=True, stream=s)
        again = domino.draft_greedy(packed, lb, h, S0, logits_out=True, stream=s)
        domino.set_l2_persistence(packed, s, 0.0)
    torch.cuda.synchronize()
    assert torch.equal(ref[0], got[0]) and torch.equal(ref[0], again[0])
    assert torch.equal(ref[1], got[1]) and torch.equal(ref[1], again[1])
    if before is not None:
        assert during is not None and during > 0
        assert _persisting_limit() == before
    # weights 64 MB apart are not one window: W2 at the start of a buffer, the rest after a gap
    gap = 64 << 20
    nb = [packed.W2.numel() * 2, packed.W1.numel() * 2, packed.W_hh.numel() * 2, packed.W_ih.numel() * 2]
    buf = torch.empty(sum(nb) + gap + 4096, dtype=torch.uint8, device="cuda")
    off = [0, nb[0] + gap]
    off += [off[1] + nb[1], off[1] + nb[1] + nb[2]]
    parts = {}
    for name, o, n in zip(("W2", "W1", "W_hh", "W_ih"), off, nb):
        t = buf[o:o + n].view(torch.bfloat16).view(getattr(packed, name).shape)
        t.copy_(getattr(packed, name))
        parts[name] = t
    far = dataclasses.replace(packed, **parts)
    with pytest.raises(domino.DominoError):
        domino.set_l2_persistence(far, s, 1.0)
