"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test fixes the oracle to something independent: a hand-worked example, a closed form, a
library routine (torch.nn.GRUCell, numpy.argmax), an invariant of the equations, or brute-force
enumeration.  Together they catch a dropped term, a swapped concat order, a transposed
operand, an off-by-one position index and a wrong tie rule.

Source of the equations: Domino review page (paper.oopus.info), section 二 -- the head
equation L_final = L_base + W2 . sigma(W1 . [H_i ; S_{i-1}]), the GRU causal encoder that
reads the drafted embeddings, the SiLU named in the low-rank-head bullet.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from draft_block_causal_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f32_weights(d, Hs, r, V, rng, scale=1.0):
    return {
        "embed": (rng.standard_normal((V, d)) * scale).astype(np.float32),
        "W_ih": (rng.uniform(-1, 1, (3 * Hs, d)) * scale).astype(np.float32),
        "W_hh": (rng.uniform(-1, 1, (3 * Hs, Hs)) * scale).astype(np.float32),
        "b_ih": (rng.uniform(-1, 1, (3 * Hs,)) * scale).astype(np.float32),
        "b_hh": (rng.uniform(-1, 1, (3 * Hs,)) * scale).astype(np.float32),
        "W1": (rng.uniform(-1, 1, (r, d + Hs)) * scale).astype(np.float32),
        "W2": (rng.uniform(-2, 2, (V, r)) * scale).astype(np.float32),
    }


def _shape(B, L, d, Hs, r, V, dtype=0):
    return dict(B=B, L=L, d=d, Hs=Hs, r=r, V=V, dtype=dtype)


def _silu(x):
    return x / (1.0 + math.exp(-x))


# ---------------------------------------------------------------------------------------------
# 1. Hand-worked example: 2 positions, V = 5, d = Hs = r = 2.
#    W1 picks H_i[0] into a[0] and S_{i-1}[1] into a[1]; the GRU has only its n-gate input
#    weights (identity), every bias zero, so r = z = 1/2 and S_i = (tanh(x) + S_{i-1}) / 2.
# ---------------------------------------------------------------------------------------------
def test_hand_example_two_positions_v5():
    d = Hs = r = 2
    V, L = 5, 2
    w = {
        "embed": np.array([[0, 0], [0.5, 0], [0, 1.0], [1, 0.5], [-0.5, 1]], np.float32),
        "W_ih": np.zeros((6, 2), np.float32),
        "W_hh": np.zeros((6, 2), np.float32),
        "b_ih": np.zeros(6, np.float32),
        "b_hh": np.zeros(6, np.float32),
        "W1": np.array([[1, 0, 0, 0], [0, 0, 0, 1]], np.float32),
        "W2": np.array([[1, 0], [0, 1], [1, 1], [-1, 0], [0, 2]], np.float32),
    }
    w["W_ih"][4:6] = np.eye(2, dtype=np.float32)  # n-gate rows (gate order r | z | n)
    H = np.array([[[2, 7], [-1, 5]]], np.float32)
    Lb = np.array([[[0, 0.5, 0.25, 1, 0], [0, 0, 0, 0.125, 0]]], np.float32)
    S0 = np.zeros((1, 2), np.float32)
    out = oracle.head(_shape(1, L, d, Hs, r, V), w, Lb, H, S0)

    # position 0: a = (H_0[0], S0[1]) = (2, 0);  u = (silu 2, 0)
    u0 = _silu(2.0)
    z0 = [0 + u0, 0.5 + 0, 0.25 + u0, 1 - u0, 0 + 0]
    # argmax is index 2 (0.25 + silu 2); the GRU then reads embed[2] = (0, 1)
    s1 = [0.5 * math.tanh(0.0), 0.5 * math.tanh(1.0)]
    # position 1: a = (H_1[0], S_0[1]) = (-1, tanh(1)/2)
    v0, v1 = _silu(-1.0), _silu(s1[1])
    z1 = [v0, v1, v0 + v1, 0.125 - v0, 2 * v1]

    assert out["tokens"].tolist() == [[2, 4]]
    np.testing.assert_allclose(out["logits"][0, 0], z0, rtol=0, atol=1e-15)
    np.testing.assert_allclose(out["logits"][0, 1], z1, rtol=0, atol=1e-15)
    np.testing.assert_allclose(out["states"][0, 0], [0, 0], rtol=0, atol=0)
    np.testing.assert_allclose(out["states"][0, 1], s1, rtol=0, atol=1e-15)
    # top-2 margins: position 0 is z[2] - z[0] = 0.25; position 1 is 2 v1 - (0.125 - v0)
    np.testing.assert_allclose(out["margin"][0], [0.25, 2 * v1 - (0.125 - v0)], rtol=0, atol=1e-15)


# ---------------------------------------------------------------------------------------------
# 2. The GRU cell against torch.nn.GRUCell in float64 (the library routine whose form the
#    oracle adopts: gates r | z | n, reset gate applied to W_hn h + b_hn).
# ---------------------------------------------------------------------------------------------
def _torch_cell(w, d, Hs):
    cell = torch.nn.GRUCell(d, Hs, bias=True, dtype=torch.float64)
    with torch.no_grad():
        cell.weight_ih.copy_(torch.from_numpy(w["W_ih"].astype(np.float64)))
        cell.weight_hh.copy_(torch.from_numpy(w["W_hh"].astype(np.float64)))
        cell.bias_ih.copy_(torch.from_numpy(w["b_ih"].astype(np.float64)))
        cell.bias_hh.copy_(torch.from_numpy(w["b_hh"].astype(np.float64)))
    return cell


def test_gru_step_matches_torch_grucell():
    rng = np.random.default_rng(11)
    d, Hs = 7, 5
    w = _f32_weights(d, Hs, 3, 9, rng)
    cell = _torch_cell(w, d, Hs)
    for _ in range(5):
        x = rng.standard_normal(d)
        h = rng.standard_normal(Hs)
        got = oracle.gru_step(d, Hs, 0, w, x, h)
        want = cell(torch.from_numpy(x)[None], torch.from_numpy(h)[None])[0].detach().numpy()
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-14)


def test_teacher_forced_states_follow_grucell_sequence():
    rng = np.random.default_rng(12)
    B, L, d, Hs, r, V = 2, 5, 6, 4, 3, 11
    w = _f32_weights(d, Hs, r, V, rng)
    Lb = rng.standard_normal((B, L, V)).astype(np.float32)
    H = rng.standard_normal((B, L, d)).astype(np.float32)
    S0 = rng.standard_normal((B, Hs)).astype(np.float32)
    y = rng.integers(0, V, (B, L)).astype(np.int32)
    out = oracle.head(_shape(B, L, d, Hs, r, V), w, Lb, H, S0, tokens=y)
    cell = _torch_cell(w, d, Hs)
    for b in range(B):
        h = torch.from_numpy(S0[b].astype(np.float64))[None]
        for i in range(L):
            # the state consumed at position i is S_{i-1}; S_{-1} = S0
            np.testing.assert_allclose(out["states"][b, i], h[0].detach().numpy(), rtol=0, atol=1e-13)
            x = torch.from_numpy(w["embed"][y[b, i]].astype(np.float64))[None]
            h = cell(x, h)
    assert out["tokens"].tolist() == y.tolist()


# ---------------------------------------------------------------------------------------------
# 3. Closed forms.
# ---------------------------------------------------------------------------------------------
def test_w2_zero_gives_base_logits_exactly_and_lowest_index_ties():
    rng = np.random.default_rng(13)
    B, L, d, Hs, r, V = 2, 4, 5, 3, 2, 17
    w = _f32_weights(d, Hs, r, V, rng)
    w["W2"][:] = 0
    Lb = rng.standard_normal((B, L, V)).astype(np.float32)
    # plant exact ties for the maximum at several positions
    Lb[0, 1, 3] = Lb[0, 1, 9] = 10.0
    Lb[1, 2, 16] = Lb[1, 2, 0] = Lb[1, 2, 5] = 7.5
    H = rng.standard_normal((B, L, d)).astype(np.float32)
    S0 = rng.standard_normal((B, Hs)).astype(np.float32)
    out = oracle.head(_shape(B, L, d, Hs, r, V), w, Lb, H, S0)
    assert np.array_equal(out["logits"], Lb.astype(np.float64))
    assert out["tokens"][0, 1] == 3 and out["tokens"][1, 2] == 0
    assert np.array_equal(out["tokens"], np.argmax(Lb, axis=-1))  # numpy: first maximal index
    assert out["margin"][0, 1] == 0.0 and out["margin"][1, 2] == 0.0


def test_zero_gru_halves_the_state_each_step():
    rng = np.random.default_rng(14)
    B, L, d, Hs, r, V = 2, 6, 4, 5, 3, 13
    w = _f32_weights(d, Hs, r, V, rng)
    for k in ("W_ih", "W_hh", "b_ih", "b_hh"):
        w[k][:] = 0
    Lb = rng.standard_normal((B, L, V)).astype(np.float32)
    H = rng.standard_normal((B, L, d)).astype(np.float32)
    S0 = rng.standard_normal((B, Hs)).astype(np.float32)
    out = oracle.head(_shape(B, L, d, Hs, r, V), w, Lb, H, S0)
    for i in range(L):
        assert np.array_equal(out["states"][:, i], S0.astype(np.float64) * 0.5 ** i)


def test_adding_a_constant_per_position_shifts_logits_and_keeps_tokens():
    rng = np.random.default_rng(15)
    B, L, d, Hs, r, V = 1, 4, 5, 3, 2, 19
    w = _f32_weights(d, Hs, r, V, rng)
    # multiples of 2^-10 within [-4, 4]: adding c in {1, -2, 0.5, 3} stays exact in fp32
    Lb = (rng.integers(-4096, 4096, (B, L, V)) / 1024.0).astype(np.float32)
    c = np.array([1.0, -2.0, 0.5, 3.0], np.float32)
    H = rng.standard_normal((B, L, d)).astype(np.float32)
    S0 = np.zeros((B, Hs), np.float32)
    sh = _shape(B, L, d, Hs, r, V)
    a = oracle.head(sh, w, Lb, H, S0)
    b = oracle.head(sh, w, Lb + c[None, :, None], H, S0)
    assert np.array_equal(a["tokens"], b["tokens"])
    np.testing.assert_allclose(b["logits"], a["logits"] + c[None, :, None], rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# 4. Invariants: causality and greedy == teacher forcing on the greedy tokens.
# ---------------------------------------------------------------------------------------------
def test_teacher_forcing_is_causal():
    rng = np.random.default_rng(16)
    B, L, d, Hs, r, V = 1, 5, 4, 3, 2, 7
    w = _f32_weights(d, Hs, r, V, rng)
    Lb = rng.standard_normal((B, L, V)).astype(np.float32)
    H = rng.standard_normal((B, L, d)).astype(np.float32)
    S0 = rng.standard_normal((B, Hs)).astype(np.float32)
    sh = _shape(B, L, d, Hs, r, V)
    y = rng.integers(0, V, (B, L)).astype(np.int32)
    base = oracle.head(sh, w, Lb, H, S0, tokens=y)
    for j in range(L):
        y2 = y.copy()
        y2[0, j] = (y2[0, j] + 3) % V
        alt = oracle.head(sh, w, Lb, H, S0, tokens=y2)
        # positions 0..j see only y_<i, so they are unchanged; later ones change
        assert np.array_equal(alt["logits"][0, : j + 1], base["logits"][0, : j + 1])
        assert np.array_equal(alt["states"][0, : j + 1], base["states"][0, : j + 1])
        if j < L - 1:
            assert not np.array_equal(alt["logits"][0, j + 1], base["logits"][0, j + 1])
    # the last token feeds nothing
    y3 = y.copy()
    y3[0, L - 1] = (y3[0, L - 1] + 1) % V
    last = oracle.head(sh, w, Lb, H, S0, tokens=y3)
    assert np.array_equal(last["logits"], base["logits"])
    assert np.array_equal(last["states"], base["states"])


@pytest.mark.parametrize("dtype", [0, 1])
def test_greedy_equals_teacher_forcing_on_its_own_tokens(dtype):
    shape = _shape(3, 6, 24, 16, 8, 40, dtype)
    w = synth.head_weights(shape, seed=5)
    inp = synth.block_inputs(shape, seed=6, peak=1.0, s0_std=0.3)
    g = oracle.head(shape, w, inp["base_logits"], inp["hidden"], inp["S0"])
    t = oracle.head(shape, w, inp["base_logits"], inp["hidden"], inp["S0"], tokens=g["tokens"])
    assert np.array_equal(g["logits"], t["logits"])
    assert np.array_equal(g["states"], t["states"])
    assert np.array_equal(g["tokens"], t["tokens"])


def test_row_subset_matches_full_batch():
    shape = _shape(4, 5, 16, 8, 4, 30, 1)
    w = synth.head_weights(shape, seed=7)
    inp = synth.block_inputs(shape, seed=8, s0_std=0.2)
    full = oracle.head(shape, w, inp["base_logits"], inp["hidden"], inp["S0"])
    sub = oracle.head(shape, w, inp["base_logits"], inp["hidden"], inp["S0"], rows=[3, 1])
    assert np.array_equal(sub["logits"], full["logits"][[3, 1]])
    assert np.array_equal(sub["tokens"], full["tokens"][[3, 1]])


def test_thread_count_does_not_change_results():
    shape = _shape(2, 4, 32, 16, 8, 300, 1)
    w = synth.head_weights(shape, seed=9)
    inp = synth.block_inputs(shape, seed=10, s0_std=0.2)
    one = oracle.head(shape, w, inp["base_logits"], inp["hidden"], inp["S0"], nthreads=1)
    many = oracle.head(shape, w, inp["base_logits"], inp["hidden"], inp["S0"], nthreads=4)
    for k in ("tokens", "logits", "states", "margin"):
        assert np.array_equal(one[k], many[k])


# ---------------------------------------------------------------------------------------------
# 5. Brute force: every token sequence of a tiny vocabulary.  Greedy drafting must return the
#    unique sequence that is its own argmax at every position under teacher forcing.
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("seed", [21, 22, 23])
def test_greedy_is_the_unique_fixed_point_of_teacher_forcing(seed):
    rng = np.random.default_rng(seed)
    B, L, d, Hs, r, V = 1, 4, 3, 3, 2, 5
    w = _f32_weights(d, Hs, r, V, rng, scale=3.0)
    Lb = (0.3 * rng.standard_normal((B, L, V))).astype(np.float32)
    H = rng.standard_normal((B, L, d)).astype(np.float32)
    S0 = rng.standard_normal((B, Hs)).astype(np.float32)
    sh = _shape(B, L, d, Hs, r, V)
    greedy = oracle.head(sh, w, Lb, H, S0)
    fixed = []
    steered = set()
    for y in itertools.product(range(V), repeat=L):
        yy = np.array([y], np.int32)
        tf = oracle.head(sh, w, Lb, H, S0, tokens=yy, want_states=False)
        am = [min(np.flatnonzero(tf["logits"][0, i] == tf["logits"][0, i].max())) for i in range(L)]
        steered.add(tuple(am[1:]))
        if list(y) == am:
            fixed.append(y)
    assert fixed == [tuple(greedy["tokens"][0].tolist())]
    # the test is only meaningful if the prefix actually steers the later argmax
    assert len(steered) > 1


# ---------------------------------------------------------------------------------------------
# 6. Accept length against numpy.argmax (first maximal index) and hand cases.
# ---------------------------------------------------------------------------------------------
def test_accept_len_matches_numpy_first_argmax():
    rng = np.random.default_rng(31)
    B, L, V = 64, 16, 37
    T = rng.integers(-3, 4, (B, L, V)).astype(np.float32)  # many exact ties
    am = np.argmax(T, axis=-1).astype(np.int32)
    draft = am.copy()
    cut = rng.integers(0, L + 1, B)
    for b in range(B):
        if cut[b] < L:
            draft[b, cut[b]] = (draft[b, cut[b]] + 1 + rng.integers(0, V - 1)) % V
            draft[b, cut[b] + 1:] = rng.integers(0, V, L - cut[b] - 1)
    want = np.array([next((j for j in range(L) if draft[b, j] != am[b, j]), L) for b in range(B)])
    got = oracle.accept_len(draft, T)
    assert np.array_equal(got, want)
    assert np.array_equal(got, np.minimum(cut, L))


def test_accept_len_hand_cases():
    T = np.zeros((3, 3, 4), np.float32)
    T[:, :, 2] = 1.0          # argmax 2 everywhere
    T[1, 1, 0] = 1.0          # tie 0/2 at row 1 position 1 -> argmax 0
    draft = np.array([[2, 2, 2], [2, 2, 2], [1, 2, 2]], np.int32)
    assert oracle.accept_len(draft, T).tolist() == [3, 1, 0]


# ---------------------------------------------------------------------------------------------
# 7. Shapes against the pages' printed parameter count.
# ---------------------------------------------------------------------------------------------
def test_parameter_count_matches_the_pages():
    with open(os.path.join(GOLDEN, "paper_facts.json")) as f:
        facts = json.load(f)
    sh = synth.shape_of(synth.workload("qwen3-8b-head-b1"))
    assert sh["Hs"] == facts["gru_hidden"]["value"]
    assert sh["r"] == facts["rank"]["value"]
    assert sh["L"] == facts["block_size"]["value"]
    n = synth.param_count(sh)
    assert n == 55_941_120
    # "about 56 million" -- rounds to 5600 ten-thousands
    assert round(n / 1e4 / 100) * 100 == facts["head_params_wan"]["value"]
