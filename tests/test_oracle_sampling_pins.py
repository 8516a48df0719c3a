"""Pins of the oracle's sampled (temperature > 0) verification rule, on the CPU.

The rule is speculative sampling's acceptance test (Leviathan, Kalman and Matias, ICML 2023; Chen
et al. 2023): the pages call Domino's verification lossless (review page, section 一;
researchpapers.dev summary) without restating it.  What pins the oracle here is not its formula
but what the rule must achieve:
  - identical draft and target distributions accept every position, whatever the draws;
  - a draft token the target gives no mass is always rejected, and the replacement comes from
    the target's own support;
  - lossless: integrating the oracle over both of its random draws (exactly, by bisection on the
    fp32 uniforms where its decisions switch), the distribution of the token it emits at one
    position equals the target distribution softmax(target / T) -- for a sampled draft
    distribution and for a greedy (one-hot) draft alike;
  - as T -> 0 the rule becomes the greedy accept rule (oracle.accept_len) and the replacement the
    target's argmax.
"""
import numpy as np
import pytest

import oracle

ONE_MINUS = np.nextafter(np.float32(1.0), np.float32(0.0))  # the largest fp32 uniform below 1


def _sm(t, T):
    e = np.exp((t.astype(np.float64) - t.max()) / T)
    return e / e.sum()


def test_identical_distributions_accept_every_position():
    rng = np.random.default_rng(1)
    B, L, V = 4, 6, 50
    t = rng.standard_normal((B, L, V)).astype(np.float32)
    x = rng.integers(0, V, (B, L)).astype(np.int32)
    for u in (0.0, 0.5, float(ONE_MINUS)):
        uni = np.full((B, L + 1), u, np.float32)
        r = oracle.accept_sample(x, t, 0.8, uni, draft_logits=t.copy())
        assert (r["accept"] == L).all() and (r["next"] == -1).all()
        assert np.allclose(r["ratio"], 1.0, rtol=0, atol=1e-12)


def test_token_outside_the_target_support_is_rejected_and_replaced_from_it():
    V, L = 9, 3
    t = np.zeros((1, L, V), np.float32)
    t[0, :, 4] = 2000.0  # all target mass on token 4 (the other probabilities underflow to 0)
    x = np.array([[7, 4, 4]], np.int32)
    for draft in (None, np.zeros((1, L, V), np.float32)):  # one-hot greedy draft, or a uniform draft
        for u0 in (0.0, 0.3, float(ONE_MINUS)):
            uni = np.array([[u0, 0.1, 0.1, 0.77]], np.float32)
            r = oracle.accept_sample(x, t, 1.0, uni, draft_logits=draft)
            assert r["accept"][0] == 0 and r["next"][0] == 4
            assert r["ratio"][0, 0] == 0.0 and (r["ratio"][0, 1:] == -1.0).all()


def _threshold(f, lo=np.float32(0.0), hi=ONE_MINUS):
    """The first fp32 u in [lo, hi] at which the monotone predicate f switches to True (hi + ulp
    if never): bisection on the fp32 grid."""
    lo_i, hi_i = int(np.float32(lo).view(np.int32)), int(np.float32(hi).view(np.int32))
    if not f(np.float32(hi)):
        return float(np.nextafter(np.float32(hi), np.float32(2.0)))
    if f(np.float32(lo)):
        return float(lo)
    while hi_i - lo_i > 1:
        mid = (lo_i + hi_i) // 2
        if f(np.int32(mid).view(np.float32)):
            hi_i = mid
        else:
            lo_i = mid
    return float(np.int32(hi_i).view(np.float32))


def _emitted_distribution(t_row, draft_row, x, T):
    """Exact distribution of the token the oracle emits at a single position for draft token x,
    integrating over its acceptance draw u0 and its resampling draw u1."""
    V = t_row.shape[0]
    tl = t_row.reshape(1, 1, V)
    dl = None if draft_row is None else draft_row.reshape(1, 1, V)
    xs = np.array([[x]], np.int32)

    def run(u0, u1):
        r = oracle.accept_sample(xs, tl, T, np.array([[u0, u1]], np.float32), draft_logits=dl)
        return int(r["accept"][0]), int(r["next"][0])

    # P(accept) = measure of {u0 : accepted} = the first u0 that rejects (accepting is u0 < ratio)
    p_acc = min(1.0, _threshold(lambda u: run(u, 0.5)[0] == 0))
    out = np.zeros(V)
    out[x] += p_acc
    if p_acc < 1.0:
        # the replacement is a non-decreasing step function of u1: the measure of each token is
        # the gap between consecutive switch points
        starts = [_threshold(lambda u, v=v: run(ONE_MINUS, u)[1] >= v) for v in range(V)] + [1.0]
        starts = [min(1.0, s) for s in starts]
        starts[0] = 0.0
        for v in range(V):
            out[v] += (1.0 - p_acc) * max(0.0, starts[v + 1] - starts[v])
    return out


@pytest.mark.parametrize("T", [0.5, 1.0, 2.5])
def test_lossless_for_a_sampled_draft_on_five_tokens(T):
    """sum_x q(x) P(emit v | x) = p(v) for every v: the emitted token follows the target."""
    rng = np.random.default_rng(int(T * 10))
    V = 5
    t = (rng.standard_normal(V) * 1.5).astype(np.float32)
    dq = (rng.standard_normal(V) * 1.5).astype(np.float32)
    q = _sm(dq, T)
    total = np.zeros(V)
    for x in range(V):
        total += q[x] * _emitted_distribution(t, dq, x, T)
    assert np.abs(total - _sm(t, T)).max() < 2e-6, (total, _sm(t, T))


@pytest.mark.parametrize("x", [0, 2, 4])
def test_lossless_for_a_greedy_draft_on_five_tokens(x):
    """A greedy draft is a one-hot draft distribution: whatever fixed token it proposes, the
    emitted token follows the target."""
    rng = np.random.default_rng(40 + x)
    t = (rng.standard_normal(5) * 1.2).astype(np.float32)
    got = _emitted_distribution(t, None, x, 0.9)
    assert np.abs(got - _sm(t, 0.9)).max() < 2e-6, (got, _sm(t, 0.9))


def test_low_temperature_is_the_greedy_accept_rule():
    rng = np.random.default_rng(5)
    B, L, V = 24, 8, 40
    t = rng.standard_normal((B, L, V)).astype(np.float32)
    am = np.argmax(t, axis=-1)
    srt = np.sort(t, axis=-1)
    # widen every top-2 gap to at least 0.05, so that p(argmax) is 1 to within e^-50 at T = 1e-3
    for b in range(B):
        for j in range(L):
            if srt[b, j, -1] - srt[b, j, -2] < 0.05:
                t[b, j, am[b, j]] = np.float32(srt[b, j, -2] + 0.05)
    assert np.array_equal(np.argmax(t, axis=-1), am)
    draft = am.astype(np.int32).copy()
    for b in range(B):  # row b diverges at position b % (L + 1) (none when b % (L + 1) == L)
        k = b % (L + 1)
        if k < L:
            draft[b, k] = (draft[b, k] + 1 + b) % V
            if draft[b, k] == am[b, k]:
                draft[b, k] = (draft[b, k] + 1) % V
    uni = np.full((B, L + 1), 0.5, np.float32)
    r = oracle.accept_sample(draft, t, 1e-3, uni)
    assert np.array_equal(r["accept"], oracle.accept_len(draft, t))
    for b in range(B):
        k = r["accept"][b]
        assert r["next"][b] == (am[b, k] if k < L else -1)


def test_residual_cdf_is_the_resampling_mass():
    """The helper the GPU tests use to validate a replacement token: its running sums end at Z,
    and the oracle's replacement is where the running sum first exceeds u * Z."""
    rng = np.random.default_rng(9)
    V = 300
    t = rng.standard_normal(V).astype(np.float32)
    dq = rng.standard_normal(V).astype(np.float32)
    x = int(np.argmax(dq))
    cdf, z = oracle.residual_cdf(t, dq, x, 1.0)
    assert cdf[-1] == z and z > 0 and (np.diff(cdf) >= 0).all()
    for u1 in (0.0, 0.25, 0.9):
        uni = np.array([[ONE_MINUS, u1]], np.float32)
        r = oracle.accept_sample(np.array([[x]], np.int32), t.reshape(1, 1, V), 1.0, uni,
                                 draft_logits=dq.reshape(1, 1, V))
        if r["accept"][0] == 0:
            y = r["next"][0]
            assert cdf[y] > np.float32(u1) * z and (y == 0 or cdf[y - 1] <= np.float32(u1) * z)
