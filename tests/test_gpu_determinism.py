"""Run-to-run reproducibility on the GPU: the same call on the same inputs gives the same bits.

Every sum that several threads, warps or CTAs add into -- the fused kernels' W1 state-block
accumulators and GRU gate sums, the split-K reductions of the tensor-core path -- is formed in an
order that does not depend on scheduling (fixed-point integer atomics, or a fixed piece order),
so tokens, logits and states must repeat exactly, not merely within a tolerance."""
import pytest
import torch

from draft_block_causal_b200 import domino, synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from tests import gpu_common as G
else:
    G = None


def _case(B, L, d, Hs, V, seed):
    wl = dict(B=B, L=L, d=d, Hs=Hs, r=256, V=V, dtype=synth.BF16, weight_seed=seed, input_seed=seed + 1,
              s0_std=0.5, peak=1.0, name="repeat")
    return synth.make_workload(wl, with_tokens=True)


CASES = [  # (B, L, d, Hs, V, plan substring)
    (1, 16, 512, 256, 12000, "k_greedy_persistent"),
    (4, 9, 768, 256, 33000, "k_greedy_persistent"),
    (1, 16, 4096, 1024, 20000, "k_greedy_tmem"),
    (3, 16, 1024, 512, 9000, "k_greedy_tmem"),
    (4, 16, 2560, 1024, 20000, "k_greedy_tmem"),
    (32, 16, 1024, 512, 9000, "k_greedy_batched"),
    (136, 4, 512, 256, 3000, "per-phase"),
]


@pytest.mark.parametrize("B,L,d,Hs,V,plan", CASES, ids=lambda v: str(v))
def test_greedy_repeats_bit_for_bit(B, L, d, Hs, V, plan):
    data = _case(B, L, d, Hs, V, 600 + B + d)
    w, lb, h, S0 = G.device_inputs(data)
    assert plan in domino.greedy_plan(domino.make_shape(w, B, L))
    runs = []
    for _ in range(3):
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = domino.draft_greedy(w, lb, h, S0, logits_out=True, states_out=True, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        runs.append(out)
    for other in runs[1:]:
        for x, y in zip(runs[0], other):
            assert torch.equal(x, y)


@pytest.mark.parametrize("B", [1, 4])
def test_greedy_with_projection_table_repeats_bit_for_bit(B):
    data = _case(B, 16, 4096, 1024, 20000, 640 + B)
    w, lb, h, S0 = G.device_inputs(data)
    w.embed_proj = domino.project_embeddings(w)
    a = domino.draft_greedy(w, lb, h, S0, logits_out=True, states_out=True)
    b = domino.draft_greedy(w, lb, h, S0, logits_out=True, states_out=True)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("B,d,Hs", [(1, 4096, 1024), (4, 1024, 512), (2, 512, 256), (32, 1024, 1024), (100, 512, 256)])
def test_teacher_forced_repeats_bit_for_bit(B, d, Hs):
    data = _case(B, 16, d, Hs, 9000, 660 + B)
    w, lb, h, S0 = G.device_inputs(data)
    y = torch.from_numpy(data["tokens"]).cuda()
    a = domino.teacher_forced(w, lb, h, S0, y, states_out=True)
    b = domino.teacher_forced(w, lb, h, S0, y, states_out=True)
    torch.cuda.synchronize()
    for x, y2 in zip(a, b):
        assert torch.equal(x, y2)
