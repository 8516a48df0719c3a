"""The optional input-projection table (embed . W_ih^T, domino_project_embeddings): the table
itself against an fp64 product on sampled rows, then greedy drafting and teacher forcing with the
table in use against the fp64 oracle (oracle replay, the same tolerances as every parity test)."""
import numpy as np
import pytest
import torch

from draft_block_causal_b200 import domino, synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from tests import gpu_common as G
else:
    G = None


def _wl(B, L, d, Hs, r, V, dtype, seed, s0_std=0.2, peak=2.0):
    return dict(B=B, L=L, d=d, Hs=Hs, r=r, V=V, dtype=dtype, weight_seed=seed, input_seed=seed + 1,
                s0_std=s0_std, peak=peak, name=f"proj-{seed}")


@pytest.mark.parametrize("wl", [_wl(1, 4, 64, 32, 16, 1000, 0, 500),          # fp32, CUDA-core projection
                                _wl(2, 8, 512, 256, 256, 3000, 1, 510),        # bf16, tensor cores, ragged V
                                _wl(1, 16, 4096, 1024, 256, 151936, 1, 520)],  # Qwen3-8B widths
                         ids=["f32", "bf16-small", "bf16-8b"])
def test_projection_table_matches_fp64_product(wl):
    data = synth.make_workload(wl)
    sh = data["shape"]
    w = domino.to_device_weights(data["weights"], sh["dtype"])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    xp = domino.project_embeddings(w, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    V = sh["V"]
    rows = np.unique(np.r_[0, 1, 127, 128, V - 1, np.random.default_rng(0).integers(0, V, 60)])
    emb = synth.to_f32(data["weights"]["embed"][rows], sh["dtype"]).astype(np.float64)
    wih = synth.to_f32(data["weights"]["W_ih"], sh["dtype"]).astype(np.float64)
    ref = emb @ wih.T
    got = xp[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64)
    # fp32 accumulation of d exact bf16/fp32 products
    tol = 1e-5 * np.abs(emb).max() * np.abs(wih).max() * sh["d"] ** 0.5 + 1e-7
    assert np.abs(got - ref).max() <= tol


SHAPES = [
    _wl(1, 4, 64, 32, 16, 1000, 0, 530),            # fp32: per-phase kernels
    _wl(2, 16, 512, 256, 256, 12000, 1, 540),       # fused L2-streamed kernel
    _wl(3, 16, 1024, 512, 256, 9000, 1, 550),       # fused TMEM kernel
    _wl(12, 6, 512, 512, 256, 5000, 1, 560),        # per-phase kernels, bf16
    _wl(1, 16, 4096, 1024, 256, 151936, 1, 570),    # Qwen3-8B shapes, fused TMEM kernel
]


@pytest.mark.parametrize("wl", SHAPES, ids=lambda w: f"{w['name']}-B{w['B']}")
def test_greedy_and_teacher_forcing_with_projection_table(wl):
    data = synth.make_workload(wl, with_tokens=True)
    sh = data["shape"]
    w, lb, h, S0 = G.device_inputs(data)
    w.embed_proj = domino.project_embeddings(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tok, lg, st = domino.draft_greedy(w, lb, h, S0, logits_out=True, states_out=True, status=status)
    y = torch.from_numpy(data["tokens"]).cuda()
    tlg, tst = domino.teacher_forced(w, lb, h, S0, y, states_out=True, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    import oracle
    tok = tok.cpu().numpy()
    ref = oracle.head(sh, data["weights"], data["base_logits"], data["hidden"], data["S0"],
                      tokens=np.ascontiguousarray(tok))
    G.check_logits_states(lg.cpu().numpy(), st.cpu().numpy(), ref, "greedy+proj")
    G.check_tokens_against_replay(tok, ref, "greedy+proj")
    tref = oracle.head(sh, data["weights"], data["base_logits"], data["hidden"], data["S0"], tokens=data["tokens"])
    G.check_logits_states(tlg.cpu().numpy(), tst.cpu().numpy(), tref, "teacher-forced+proj")
