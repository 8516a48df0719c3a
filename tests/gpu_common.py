"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and compare it
with the fp64 oracle on the same seeded inputs.

Parity procedure ("oracle replay"):
  1. the oracle runs teacher-forced on the GPU's own draft tokens; GPU logits and states must
     lie within |d| <= 1e-2 + 1e-2 |ref| (logits) and |d| <= 5e-3 (states) of it;
  2. each GPU draft token must equal the replay's argmax wherever the replay's top-2 margin
     exceeds 2e-2; smaller-margin disagreements are counted and reported, not failed (both
     tokens are then correct to within the arithmetic's error);
  3. the oracle's own greedy path must agree with the GPU's up to the first position whose
     oracle margin is at most 2e-2;
  4. accept lengths on identical draft tokens are bit-exact.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from draft_block_causal_b200 import domino, synth

LOGIT_ATOL = 1e-2
LOGIT_RTOL = 1e-2
STATE_ATOL = 5e-3
MARGIN = 2e-2


def device_inputs(data: dict):
    sh = data["shape"]
    dt = sh["dtype"]
    w = domino.to_device_weights(data["weights"], dt)
    lb = domino.to_device(data["base_logits"], dt)
    h = domino.to_device(data["hidden"], dt)
    S0 = torch.from_numpy(data["S0"]).cuda()
    return w, lb, h, S0


def check_logits_states(got_logits, got_states, ref, what=""):
    """Element-wise comparison against the oracle replay; returns (max logit err, max state err)."""
    rl = ref["logits"]
    gl = got_logits.astype(np.float64)
    err = np.abs(gl - rl)
    bad = err > LOGIT_ATOL + LOGIT_RTOL * np.abs(rl)
    assert not bad.any(), f"{what}: {bad.sum()} logits out of tolerance, max err {err.max():.3e}"
    s_err = 0.0
    if got_states is not None:
        s = np.abs(got_states.astype(np.float64) - ref["states"])
        s_err = float(s.max())
        assert s_err <= STATE_ATOL, f"{what}: state error {s_err:.3e} > {STATE_ATOL}"
    return float(err.max()), s_err


def check_tokens_against_replay(tokens, ref, what=""):
    """Step 2 of the procedure; returns the number of small-margin divergences."""
    am = np.argmax(ref["logits"], axis=-1)  # first maximal index
    diff = tokens != am
    firm = diff & (ref["margin"] > MARGIN)
    assert not firm.any(), f"{what}: {firm.sum()} draft tokens differ where the replay margin > {MARGIN}"
    return int(diff.sum())


def check_against_oracle_greedy(tokens, og, what=""):
    """Step 3: the oracle's own greedy path agrees up to its first small-margin position."""
    B, L = tokens.shape
    for b in range(B):
        for i in range(L):
            if og["margin"][b, i] <= MARGIN:
                break
            assert tokens[b, i] == og["tokens"][b, i], f"{what}: row {b} position {i} differs from oracle greedy"


def greedy_parity(data: dict, rows=None, nthreads: int = 0):
    """Run the GPU greedy path (with logits and states) and check it by oracle replay."""
    sh = data["shape"]
    w, lb, h, S0 = device_inputs(data)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tok, lg, st = domino.draft_greedy(w, lb, h, S0, logits_out=True, states_out=True, status=status)
    tok2, _, _ = domino.draft_greedy(w, lb, h, S0, status=status)  # fused-argmax path, no logits written
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    tok = tok.cpu().numpy()
    tok2 = tok2.cpu().numpy()
    rows = list(range(sh["B"])) if rows is None else list(rows)
    gl = lg[rows].cpu().numpy()
    gs = st[rows].cpu().numpy()
    bl, hh, s0 = data["base_logits"], data["hidden"], data["S0"]
    ref = oracle.head(sh, data["weights"], bl, hh, s0, tokens=np.ascontiguousarray(tok), rows=rows,
                      nthreads=nthreads)
    le, se = check_logits_states(gl, gs, ref, "greedy")
    ndiv = check_tokens_against_replay(tok[rows], ref, "greedy")
    # the no-logits call must draft the same block, up to small-margin divergences of its own
    ref2 = oracle.head(sh, data["weights"], bl, hh, s0, tokens=np.ascontiguousarray(tok2), rows=rows,
                       want_states=False, nthreads=nthreads)
    ndiv2 = check_tokens_against_replay(tok2[rows], ref2, "greedy (no logits)")
    og = oracle.head(sh, data["weights"], bl, hh, s0, rows=rows, want_logits=False, want_states=False,
                     nthreads=nthreads)
    check_against_oracle_greedy(tok[rows], og, "greedy")
    return {"tokens": tok, "max_logit_err": le, "max_state_err": se, "small_margin_divergences": ndiv + ndiv2}


def tf_parity(data: dict, rows=None, nthreads: int = 0):
    sh = data["shape"]
    w, lb, h, S0 = device_inputs(data)
    y = torch.from_numpy(data["tokens"]).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lg, st = domino.teacher_forced(w, lb, h, S0, y, states_out=True, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rows = list(range(sh["B"])) if rows is None else list(rows)
    ref = oracle.head(sh, data["weights"], data["base_logits"], data["hidden"], data["S0"], tokens=data["tokens"],
                      rows=rows, nthreads=nthreads)
    le, se = check_logits_states(lg[rows].cpu().numpy(), st[rows].cpu().numpy(), ref, "teacher-forced")
    return {"max_logit_err": le, "max_state_err": se}


def accept_parity(draft_tokens: np.ndarray, target: np.ndarray):
    d = torch.from_numpy(np.ascontiguousarray(draft_tokens, dtype=np.int32)).cuda()
    T = torch.from_numpy(target).cuda()
    got = domino.accept_len(d, T).cpu().numpy()
    want = oracle.accept_len(np.ascontiguousarray(draft_tokens, dtype=np.int32), target)
    assert np.array_equal(got, want), f"accept length mismatch: {got} vs {want}"
    return got


def greedy_parity_rows(data: dict, chunk: int = 16, nthreads: int = 0):
    """Oracle replay of every row of a large greedy case, in chunks of rows.

    The GPU drafts with logits and states written, and again with neither (the fused-argmax path).
    Each chunk of rows is replayed teacher-forced on the GPU's tokens and compared element by
    element (steps 1 and 2).  The no-logits call is replayed only on rows whose tokens differ from
    the first call's.  Step 3 needs no separate oracle run here: where every earlier token matched
    the replay's argmax at a margin above MARGIN, the replay of that prefix is the oracle's own
    greedy path, so the oracle's greedy tokens equal the GPU's up to the first small margin.
    """
    sh = data["shape"]
    B = sh["B"]
    w, lb, h, S0 = device_inputs(data)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tok, lg, st = domino.draft_greedy(w, lb, h, S0, logits_out=True, states_out=True, status=status)
    tok2, _, _ = domino.draft_greedy(w, lb, h, S0, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    tok = tok.cpu().numpy()
    tok2 = tok2.cpu().numpy()
    bl, hh, s0 = data["base_logits"], data["hidden"], data["S0"]
    le = se = 0.0
    ndiv = 0
    for r0 in range(0, B, chunk):
        rows = list(range(r0, min(B, r0 + chunk)))
        ref = oracle.head(sh, data["weights"], bl, hh, s0, tokens=np.ascontiguousarray(tok), rows=rows,
                          nthreads=nthreads)
        e1, e2 = check_logits_states(lg[r0:rows[-1] + 1].cpu().numpy(), st[r0:rows[-1] + 1].cpu().numpy(), ref,
                                     f"greedy rows {rows[0]}..{rows[-1]}")
        le, se = max(le, e1), max(se, e2)
        ndiv += check_tokens_against_replay(tok[rows], ref, f"greedy rows {rows[0]}..{rows[-1]}")
        del ref
    other = [b for b in range(B) if not np.array_equal(tok[b], tok2[b])]
    for r0 in range(0, len(other), chunk):
        rows = other[r0:r0 + chunk]
        ref2 = oracle.head(sh, data["weights"], bl, hh, s0, tokens=np.ascontiguousarray(tok2), rows=rows,
                           want_states=False, nthreads=nthreads)
        ndiv += check_tokens_against_replay(tok2[rows], ref2, "greedy (no logits)")
    return {"tokens": tok, "max_logit_err": le, "max_state_err": se, "small_margin_divergences": ndiv,
            "rows_replayed_twice": len(other)}


def tf_parity_rows(data: dict, chunk: int = 16, nthreads: int = 0, logits_dtype=torch.float32):
    """Teacher-forced parity on every row, in chunks of rows.  With bf16 logits the bound widens by
    the rounding of the fp32 value to bf16 (at most 2^-9 of its magnitude)."""
    sh = data["shape"]
    B = sh["B"]
    w, lb, h, S0 = device_inputs(data)
    y = torch.from_numpy(data["tokens"]).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lg, st = domino.teacher_forced(w, lb, h, S0, y, states_out=True, status=status, logits_dtype=logits_dtype)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rtol = LOGIT_RTOL + (2.0 ** -9 if logits_dtype == torch.bfloat16 else 0.0)
    le = se = 0.0
    for r0 in range(0, B, chunk):
        rows = list(range(r0, min(B, r0 + chunk)))
        ref = oracle.head(sh, data["weights"], data["base_logits"], data["hidden"], data["S0"],
                          tokens=data["tokens"], rows=rows, nthreads=nthreads)
        gl = lg[r0:rows[-1] + 1].float().cpu().numpy().astype(np.float64)
        err = np.abs(gl - ref["logits"])
        bad = err > LOGIT_ATOL + rtol * np.abs(ref["logits"])
        assert not bad.any(), f"teacher-forced rows {rows[0]}..: {bad.sum()} logits out of tolerance"
        s = float(np.abs(st[r0:rows[-1] + 1].cpu().numpy().astype(np.float64) - ref["states"]).max())
        assert s <= STATE_ATOL, f"teacher-forced rows {rows[0]}..: state error {s:.3e}"
        le, se = max(le, float(err.max())), max(se, s)
        del ref
    return {"max_logit_err": le, "max_state_err": se}
