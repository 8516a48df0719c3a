"""GPU boundary behaviour of the C ABI: device status codes, optional outputs, stream ordering,
and the bounded-wait error path (driven from the host by a tiny spin limit -- nothing is made
to fault or hang)."""
import time

import numpy as np
import pytest
import torch

from draft_block_causal_b200 import domino, synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from tests import gpu_common as G
else:
    G = None


def _small(B=2, L=6, dtype=1, seed=200):
    wl = dict(B=B, L=L, d=128, Hs=64, r=32, V=2000, dtype=dtype, weight_seed=seed, input_seed=seed + 1,
              s0_std=0.2, peak=2.0, name="small")
    return synth.make_workload(wl, with_tokens=True)


@pytest.mark.parametrize("shape", ["per-phase", "unit-owned"])
def test_bad_teacher_forcing_token_sets_status(shape):
    if shape == "per-phase":
        data = _small()
    else:  # the unit-owned recurrence (5 <= B <= 128, Hs a multiple of 128 up to 1024)
        data = synth.make_workload(dict(B=8, L=6, d=256, Hs=128, r=128, V=2000, dtype=1, weight_seed=260,
                                        input_seed=261, s0_std=0.2, peak=2.0, name="bad-token"), with_tokens=True)
        w, _, _, _ = G.device_inputs(data)
        assert "k_tf_units" in domino.teacher_forced_plan(domino.make_shape(w, 8, 6))
    w, lb, h, S0 = G.device_inputs(data)
    y = torch.from_numpy(data["tokens"]).cuda()
    y[1, 2] = 5000  # V = 2000
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    domino.teacher_forced(w, lb, h, S0, y, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == domino.STATUS_BAD_TOKEN
    # row 0 is unaffected and still matches the oracle
    y0 = torch.from_numpy(data["tokens"]).cuda()
    status.zero_()
    lg, _ = domino.teacher_forced(w, lb, h, S0, y0, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_optional_outputs_and_no_status_pointer():
    data = _small()
    w, lb, h, S0 = G.device_inputs(data)
    t1, l1, s1 = domino.draft_greedy(w, lb, h, S0)  # no logits, no states, status in workspace
    t2, l2, s2 = domino.draft_greedy(w, lb, h, S0, logits_out=True, states_out=True)
    torch.cuda.synchronize()
    assert l1 is None and s1 is None and l2 is not None and s2 is not None
    assert torch.equal(s2[:, 0], S0)  # the state consumed at position 0 is S0


def test_calls_are_asynchronous_and_ordered_on_the_callers_stream():
    data = _small(B=4, L=8)
    w, lb, h, S0 = G.device_inputs(data)
    ref_tok, _, _ = domino.draft_greedy(w, lb, h, S0)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    lb2 = torch.zeros_like(lb)
    with torch.cuda.stream(s):
        # outputs and workspace allocated up front: a first allocation on a new stream may wait for
        # the device inside the caching allocator, which is not the library's call
        tok_out = torch.empty_like(ref_tok)
        ws = domino.alloc_workspace(domino.workspace_bytes(w, 4, 8))
        torch.cuda.synchronize()
        torch.cuda._sleep(200_000_000)  # ~0.1 s of GPU time on this stream
        lb2.copy_(lb)                   # the inputs only become valid after the sleep
        t0 = time.perf_counter()
        tok, _, _ = domino.draft_greedy(w, lb2, h, S0, tokens_out=tok_out, workspace=ws, stream=s)
        host_s = time.perf_counter() - t0
    s.synchronize()
    assert host_s < 0.05, f"call blocked the host for {host_s:.3f} s"
    assert torch.equal(tok, ref_tok)


def test_accept_len_workspace_from_head_sizing():
    data = _small(B=3, L=5)
    w, lb, h, S0 = G.device_inputs(data)
    ws = domino.alloc_workspace(domino.workspace_bytes(w, 3, 5))
    tok, _, _ = domino.draft_greedy(w, lb, h, S0, workspace=ws)
    T = torch.randn(3, 5, 2000, device="cuda")
    acc = domino.accept_len(tok, T, workspace=ws)
    want = []
    am = T.argmax(-1).cpu().numpy()
    tk = tok.cpu().numpy()
    for b in range(3):
        k = 0
        while k < 5 and tk[b, k] == am[b, k]:
            k += 1
        want.append(k)
    assert acc.cpu().numpy().tolist() == want


def _persistent_case(B=1, seed=300, Hs=256):
    wl = dict(B=B, L=16, d=512, Hs=Hs, r=256, V=12000, dtype=1, weight_seed=seed, input_seed=seed + 1,
              s0_std=0.2, peak=2.0, name="persistent")
    return synth.make_workload(wl)


def test_plan_names_the_kernel_of_each_batch_size():
    data = _persistent_case()
    w, lb, h, S0 = G.device_inputs(data)
    assert "k_greedy_persistent" in domino.greedy_plan(domino.make_shape(w, 1, 16))
    assert "k_greedy_persistent" in domino.greedy_plan(domino.make_shape(w, 4, 16))
    assert "k_greedy_batched" in domino.greedy_plan(domino.make_shape(w, 32, 16))
    assert "per-phase" in domino.greedy_plan(domino.make_shape(w, 200, 16))
    data = _persistent_case(Hs=512)
    w, lb, h, S0 = G.device_inputs(data)
    assert "k_greedy_tmem" in domino.greedy_plan(domino.make_shape(w, 2, 16))


@pytest.mark.parametrize("B,Hs,plan", [(2, 256, "k_greedy_persistent"), (2, 512, "k_greedy_tmem"),
                                       (8, 128, "k_greedy_batched")],
                         ids=["l2-streamed", "tmem-resident", "batched"])
def test_bounded_barrier_gives_up_with_status_and_the_context_survives(B, Hs, plan):
    """A spin limit of one poll makes the waits give up at once: the kernels must report
    DOMINO_STATUS_DEVICE_TIMEOUT and return (letting their own copies and MMAs finish and freeing
    their tensor memory first); the next call with the default limit is correct."""
    data = _persistent_case(B=B, Hs=Hs)
    w, lb, h, S0 = G.device_inputs(data)
    assert plan in domino.greedy_plan(domino.make_shape(w, B, 16))
    good, _, _ = domino.draft_greedy(w, lb, h, S0)
    torch.cuda.synchronize()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    domino.set_spin_limit(1)
    try:
        domino.draft_greedy(w, lb, h, S0, status=status)
        torch.cuda.synchronize()
    finally:
        domino.set_spin_limit(0)
    assert int(status.item()) == domino.STATUS_DEVICE_TIMEOUT
    status.zero_()
    again, _, _ = domino.draft_greedy(w, lb, h, S0, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(again, good)


@pytest.mark.parametrize("Hs,plan", [(128, "k_tf_units"), (1280, "k_greedy_batched")], ids=["unit-owned", "batched"])
def test_teacher_forced_bounded_waits_give_up_with_status(Hs, plan):
    """The teacher-forced recurrence kernels under a spin limit of one poll: the call reports
    DOMINO_STATUS_DEVICE_TIMEOUT, and the next call with the default limit repeats the first
    call's logits and states bit for bit."""
    data = synth.make_workload(dict(B=8, L=6, d=256, Hs=Hs, r=128, V=2000, dtype=1, weight_seed=270,
                                    input_seed=271, s0_std=0.2, peak=2.0, name="tf-timeout"), with_tokens=True)
    w, lb, h, S0 = G.device_inputs(data)
    assert plan in domino.teacher_forced_plan(domino.make_shape(w, 8, 6))
    y = torch.from_numpy(data["tokens"]).cuda()
    good, good_s = domino.teacher_forced(w, lb, h, S0, y, states_out=True)
    torch.cuda.synchronize()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    domino.set_spin_limit(1)
    try:
        domino.teacher_forced(w, lb, h, S0, y, status=status)
        torch.cuda.synchronize()
    finally:
        domino.set_spin_limit(0)
    assert int(status.item()) == domino.STATUS_DEVICE_TIMEOUT
    status.zero_()
    again, again_s = domino.teacher_forced(w, lb, h, S0, y, states_out=True, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(again, good) and torch.equal(again_s, good_s)


def test_persistent_and_per_phase_paths_agree():
    """B = 4 runs the fused kernel; the same rows drafted inside a B = 32 batch run the per-phase
    kernels.  Tokens agree wherever the oracle replay margin is above 2e-2."""
    import oracle
    data4 = _persistent_case(B=4, seed=310)
    w, lb, h, S0 = G.device_inputs(data4)
    t4, l4, _ = domino.draft_greedy(w, lb, h, S0, logits_out=True)
    lb32, h32, S032 = lb.repeat(8, 1, 1), h.repeat(8, 1, 1), S0.repeat(8, 1)
    t32, l32, _ = domino.draft_greedy(w, lb32, h32, S032, logits_out=True)
    torch.cuda.synchronize()
    t4 = t4.cpu().numpy()
    t32 = t32.cpu().numpy()[:4]
    ref = oracle.head(data4["shape"], data4["weights"], data4["base_logits"], data4["hidden"], data4["S0"],
                      tokens=np.ascontiguousarray(t4))
    firm = ref["margin"] > G.MARGIN
    # identical up to the first position where either path met a near-tie
    for b in range(4):
        for i in range(16):
            if not firm[b, i]:
                break
            assert t4[b, i] == t32[b, i]
    err = np.abs(l4.cpu().numpy() - ref["logits"])
    assert (err <= G.LOGIT_ATOL + G.LOGIT_RTOL * np.abs(ref["logits"])).all()


def test_split_k_products_are_reproducible():
    """At B = 64 the GRU and activation products run split-K, the partial tiles summed in a fixed
    order by whichever piece arrives last: repeated calls give bit-identical results, and the
    arrival counters are back at zero for the next call."""
    data = _persistent_case(B=64, seed=320)
    w, lb, h, S0 = G.device_inputs(data)
    runs = [domino.draft_greedy(w, lb, h, S0, logits_out=True, states_out=True) for _ in range(3)]
    y = torch.from_numpy(data["tokens"]).cuda() if "tokens" in data else runs[0][0]
    tf = [domino.teacher_forced(w, lb, h, S0, y, states_out=True) for _ in range(2)]
    torch.cuda.synchronize()
    for t, lg, st in runs[1:]:
        assert torch.equal(t, runs[0][0])
        assert torch.equal(lg, runs[0][1])
        assert torch.equal(st, runs[0][2])
    assert torch.equal(tf[1][0], tf[0][0]) and torch.equal(tf[1][1], tf[0][1])


def test_fused_teacher_forcing_reports_bad_tokens():
    """Teacher forcing at a TMEM-resident shape runs the fused recurrence: an out-of-range given
    token sets DOMINO_STATUS_BAD_TOKEN there too, and valid tokens match the oracle."""
    import oracle
    data = _persistent_case(B=2, seed=330, Hs=512)
    w, lb, h, S0 = G.device_inputs(data)
    y = torch.randint(0, data["shape"]["V"], (2, 16), dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lg, st = domino.teacher_forced(w, lb, h, S0, y, states_out=True, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle.head(data["shape"], data["weights"], data["base_logits"], data["hidden"], data["S0"],
                      tokens=y.cpu().numpy())
    err = np.abs(lg.cpu().numpy() - ref["logits"])
    assert (err <= G.LOGIT_ATOL + G.LOGIT_RTOL * np.abs(ref["logits"])).all()
    assert np.abs(st.cpu().numpy() - ref["states"]).max() <= G.STATE_ATOL
    y[1, 3] = data["shape"]["V"] + 5
    domino.teacher_forced(w, lb, h, S0, y, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == domino.STATUS_BAD_TOKEN


def test_batched_teacher_forcing_reports_bad_tokens():
    """B = 8 (beyond the TMEM kernel): the batched tensor-core recurrence gives the oracle's logits
    and states, and an out-of-range given token sets DOMINO_STATUS_BAD_TOKEN."""
    import oracle
    data = _persistent_case(B=8, seed=340, Hs=256)
    w, lb, h, S0 = G.device_inputs(data)
    y = torch.randint(0, data["shape"]["V"], (8, 16), dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lg, st = domino.teacher_forced(w, lb, h, S0, y, states_out=True, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle.head(data["shape"], data["weights"], data["base_logits"], data["hidden"], data["S0"],
                      tokens=y.cpu().numpy())
    err = np.abs(lg.cpu().numpy() - ref["logits"])
    assert (err <= G.LOGIT_ATOL + G.LOGIT_RTOL * np.abs(ref["logits"])).all()
    assert np.abs(st.cpu().numpy() - ref["states"]).max() <= G.STATE_ATOL
    y[5, 7] = -3
    domino.teacher_forced(w, lb, h, S0, y, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == domino.STATUS_BAD_TOKEN


@pytest.mark.parametrize("B", [1, 8], ids=["vocabulary-major", "row-major"])
def test_bf16_teacher_forced_logits_are_the_fp32_ones_rounded(B):
    """domino_teacher_forced_ex with bf16 logits writes exactly the fp32 logits of the same call
    rounded to nearest even (both logits epilogues: B*L < 64 and >= 64), and those bf16 logits lie
    within the stated tolerance of the fp64 oracle, widened by the rounding to bf16 (2^-9 of the
    value)."""
    data = _persistent_case(B=B, seed=350 + B, Hs=256)
    w, lb, h, S0 = G.device_inputs(data)
    y = torch.randint(0, data["shape"]["V"], (B, 16), dtype=torch.int32, device="cuda")
    lg32, _ = domino.teacher_forced(w, lb, h, S0, y)
    lg16, _ = domino.teacher_forced(w, lb, h, S0, y, logits_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert lg16.dtype == torch.bfloat16
    assert torch.equal(lg16, lg32.to(torch.bfloat16))
    data["tokens"] = y.cpu().numpy()
    res = G.tf_parity_rows(data, logits_dtype=torch.bfloat16)
    print("bf16 teacher-forced logits against the oracle", res)


def test_bf16_teacher_forced_logits_8b_b32_against_oracle():
    """bf16 logits at the Qwen3-8B shape, B = 32 (the row-major epilogue), every row against the
    oracle."""
    wl = synth.workload("qwen3-8b-head-b32")
    data = synth.make_workload(wl, with_tokens=True)
    print(G.tf_parity_rows(data, logits_dtype=torch.bfloat16))
