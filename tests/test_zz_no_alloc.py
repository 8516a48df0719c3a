"""The workspace-free greedy entry point (domino_draft_greedy_noalloc).

It exists for callers that cannot allocate device memory when they draft -- e.g. a server that
gave all free device memory to its weight and KV-cache pools at start-up, or a plugin whose
host runtime owns the allocator.  Its scratch is a fixed array inside the library.  These tests
call it through the C ABI and hold it to the same tolerances as every other parity test,
against the workspace entry point on the same inputs, on two calls in a row (the second call
finds the previous call's leftovers in the shared array).  This file is named to be collected
last.
"""
import ctypes

import numpy as np
import pytest
import torch

from draft_block_causal_b200 import domino, synth

pytestmark = pytest.mark.gpu

LOGIT_ATOL, LOGIT_RTOL, STATE_ATOL, MARGIN = 1e-2, 1e-2, 5e-3, 2e-2


def _case(B, L, seed):
    wl = dict(B=B, L=L, d=512, Hs=256, r=256, V=12000, dtype=synth.BF16, weight_seed=seed, input_seed=seed + 1,
              s0_std=0.2, peak=2.0, name="noalloc")
    data = synth.make_workload(wl)
    sh = data["shape"]
    w = domino.to_device_weights(data["weights"], sh["dtype"])
    lb = domino.to_device(data["base_logits"], sh["dtype"])
    h = domino.to_device(data["hidden"], sh["dtype"])
    S0 = torch.from_numpy(data["S0"]).cuda()
    return w, lb, h, S0


def _top2_margin(logits):
    top = torch.topk(logits, 2, dim=-1).values
    return (top[..., 0] - top[..., 1]).cpu().numpy()


@pytest.mark.parametrize("B,L", [(1, 16), (3, 16), (4, 9)])
def test_noalloc_matches_workspace_entry_point_twice(B, L):
    w, lb, h, S0 = _case(B, L, 400 + B)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t_ref, l_ref, s_ref = domino.draft_greedy(w, lb, h, S0, logits_out=True, states_out=True, status=status)
    torch.cuda.synchronize()
    margin = _top2_margin(l_ref)
    ref_l = l_ref.cpu().numpy().astype(np.float64)
    ref_s = s_ref.cpu().numpy()
    tok = torch.empty((B, L), dtype=torch.int32, device="cuda")
    lg = torch.empty_like(l_ref)
    st = torch.empty_like(s_ref)
    for call in range(2):
        tok.fill_(-1)
        lg.fill_(float("nan"))
        st.fill_(float("nan"))
        domino.draft_greedy_noalloc(w, lb, h, S0, tokens_out=tok, logits_out=lg, states_out=st, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: {domino.status_string(int(status.item()))}"
        got_l = lg.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got_l - ref_l) <= LOGIT_ATOL + LOGIT_RTOL * np.abs(ref_l)), f"call {call}: logits"
        assert np.abs(st.cpu().numpy() - ref_s).max() <= STATE_ATOL, f"call {call}: states"
        t = tok.cpu().numpy()
        tr = t_ref.cpu().numpy()
        # identical tokens up to each row's first near-tie position of the reference
        for b in range(B):
            for i in range(L):
                if margin[b, i] <= MARGIN:
                    break
                assert t[b, i] == tr[b, i], f"call {call}: row {b} position {i}"


@pytest.mark.parametrize("B", [1, 4])
def test_noalloc_tmem_kernel_against_oracle_twice(B):
    """The Qwen3-8B widths (d = 4096, Hs = 1024) take the TMEM-resident fused kernel, the one behind
    the headline shape; through the fixed scratch array its tokens, logits and states must match
    the fp64 oracle (replayed on the GPU's tokens) on two calls in a row, and the second call must
    repeat the first bit for bit despite the leftovers the first left in the array."""
    from tests import gpu_common as G
    wl = dict(B=B, L=16, d=4096, Hs=1024, r=256, V=6000, dtype=synth.BF16, weight_seed=450 + B,
              input_seed=451 + B, s0_std=0.2, peak=2.0, name="noalloc-tmem")
    data = synth.make_workload(wl)
    w, lb, h, S0 = G.device_inputs(data)
    assert "k_greedy_tmem" in domino.greedy_plan(domino.make_shape(w, B, 16))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    first = None
    for call in range(2):
        tok, lg, st = domino.draft_greedy_noalloc(w, lb, h, S0, logits_out=True, states_out=True, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: {domino.status_string(int(status.item()))}"
        t = tok.cpu().numpy()
        ref = G.oracle.head(data["shape"], data["weights"], data["base_logits"], data["hidden"], data["S0"],
                            tokens=np.ascontiguousarray(t))
        G.check_logits_states(lg.cpu().numpy(), st.cpu().numpy(), ref, f"noalloc call {call}")
        G.check_tokens_against_replay(t, ref, f"noalloc call {call}")
        if first is None:
            first = (tok.clone(), lg.clone(), st.clone())
        else:
            for x, y in zip(first, (tok, lg, st)):
                assert torch.equal(x, y), f"call {call} differs from call 0"


def test_noalloc_without_status_pointer_or_optional_outputs():
    w, lb, h, S0 = _case(2, 16, 420)
    t_ref, l_ref, _ = domino.draft_greedy(w, lb, h, S0, logits_out=True)
    t, l, s = domino.draft_greedy_noalloc(w, lb, h, S0)
    torch.cuda.synchronize()
    assert l is None and s is None
    margin = _top2_margin(l_ref)
    t, tr = t.cpu().numpy(), t_ref.cpu().numpy()
    for b in range(2):
        for i in range(16):
            if margin[b, i] <= MARGIN:
                break
            assert t[b, i] == tr[b, i]


def test_noalloc_long_block_that_still_fits():
    # B = 2 rows of 64 positions: about 180 KB of keys, projections and accumulators, within the array
    w, lb, h, S0 = _case(2, 64, 440)
    t_ref, l_ref, s_ref = domino.draft_greedy(w, lb, h, S0, logits_out=True, states_out=True)
    t, l, s = domino.draft_greedy_noalloc(w, lb, h, S0, logits_out=True, states_out=True)
    torch.cuda.synchronize()
    ref = l_ref.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(l.cpu().numpy() - ref) <= LOGIT_ATOL + LOGIT_RTOL * np.abs(ref))
    assert np.abs(s.cpu().numpy() - s_ref.cpu().numpy()).max() <= STATE_ATOL


def test_noalloc_rejects_shapes_beyond_its_scratch_and_unsupported_shapes():
    w, lb, h, S0 = _case(1, 16, 430)
    L = domino.lib()
    ws = w.c_struct()
    p = ctypes.c_void_p(lb.data_ptr())  # never dereferenced: the checks fail before any launch
    # B = 4 rows of 64 positions need more than the 256 KiB array
    big = domino.Shape(4, 64, 512, 256, 256, 12000, 1)
    assert L.domino_draft_greedy_noalloc(ctypes.byref(big), ctypes.byref(ws), p, p, p, p, None, None,
                                         None, None) == domino.ERR_SCRATCH_LIMIT
    assert "scratch" in domino.status_string(domino.ERR_SCRATCH_LIMIT)
    # a batch the fused kernel does not take
    b32 = domino.Shape(32, 16, 512, 256, 256, 12000, 1)
    assert L.domino_draft_greedy_noalloc(ctypes.byref(b32), ctypes.byref(ws), p, p, p, p, None, None,
                                         None, None) == domino.ERR_UNSUPPORTED
    # missing weights
    ok = domino.Shape(1, 16, 512, 256, 256, 12000, 1)
    assert L.domino_draft_greedy_noalloc(ctypes.byref(ok), None, p, p, p, p, None, None, None,
                                         None) == domino.ERR_INVALID_ARGUMENT
