"""Sampled (temperature > 0) verification on the GPU (domino_accept_sample) against the oracle, on
the same inputs and the same uniform draws.

Decisions are floating-point comparisons (u < p/q) and an inverse-transform draw, computed in fp32
with fixed-order sums on the GPU and in fp64 in the oracle.  The accept length must equal the
oracle's unless the deciding draw lies within RTOL of the oracle's ratio at the first position where
they part (a near-tie, reported, not failed); the replacement token must equal the oracle's unless
the draw u * Z lies within RTOL * Z of a boundary of the oracle's running residual sum, and then it
must still be a token whose residual interval holds the draw to within that tolerance."""
import numpy as np
import pytest
import torch

import oracle
from draft_block_causal_b200 import domino

pytestmark = pytest.mark.gpu

RTOL = 1e-4


def _sample_tokens(logits, T, rng):
    """Draft tokens drawn from softmax(logits / T) (test set-up, fp64 on the host, row by row)."""
    B, L, V = logits.shape
    out = np.empty((B, L), np.int32)
    for b in range(B):
        for j in range(L):
            z = logits[b, j].astype(np.float64) / T
            c = np.exp(z - z.max()).cumsum()
            out[b, j] = min(int(np.searchsorted(c, rng.random() * c[-1], side="right")), V - 1)
    return out


def _check(draft, target, T, uni, dl, got_acc, got_next):
    ref = oracle.accept_sample(draft, target, T, uni, draft_logits=dl)
    B, L, V = target.shape
    near = 0
    for b in range(B):
        ko, kg = int(ref["accept"][b]), int(got_acc[b])
        if ko != kg:
            m = min(ko, kg)
            ratio = ref["ratio"][b, m]
            assert abs(float(uni[b, m]) - ratio) <= RTOL * max(1.0, ratio), \
                f"row {b}: accept {kg} vs oracle {ko}, u={uni[b, m]} ratio={ratio}"
            near += 1
            continue
        if ko == L:
            assert got_next[b] == -1 and ref["next"][b] == -1
            continue
        yg, yo = int(got_next[b]), int(ref["next"][b])
        if yg == yo:
            continue
        n = ko
        cdf, z = oracle.residual_cdf(target[b, n], None if dl is None else dl[b, n], int(draft[b, n]), T)
        tz = float(uni[b, L]) * z
        lo = cdf[yg - 1] if yg > 0 else 0.0
        assert 0 <= yg < V and cdf[yg] > lo, f"row {b}: replacement {yg} has no residual mass"
        assert lo - RTOL * z <= tz <= cdf[yg] + RTOL * z, f"row {b}: replacement {yg} vs oracle {yo}"
        near += 1
    return ref, near


@pytest.mark.parametrize("B,L,V,T,sampled", [
    (32, 16, 151936, 1.0, True),     # the B = 32 serving shape, a sampled draft distribution
    (32, 16, 151936, 0.7, False),    # greedy drafts (one-hot draft distribution)
    (5, 7, 1000, 1.3, True),         # one chunk, odd B and L
    (3, 4, 20008, 0.9, True),        # a ragged last chunk
    (70, 2, 8192, 1.0, False),       # exactly one chunk, many rows
])
def test_accept_sample_against_oracle(B, L, V, T, sampled):
    rng = np.random.default_rng(B * 1000 + V % 997)
    base = (rng.standard_normal((B, L, V)) * 2.5).astype(np.float32)
    target = (base + rng.standard_normal((B, L, V)).astype(np.float32) * 0.4).astype(np.float32)
    dl = base if sampled else None
    draft = _sample_tokens(base, T, rng) if sampled else np.argmax(base, axis=-1).astype(np.int32)
    uni = rng.random((B, L + 1)).astype(np.float32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    acc, nxt = domino.accept_sample(torch.from_numpy(draft).cuda(), torch.from_numpy(target).cuda(), T,
                                    torch.from_numpy(uni).cuda(),
                                    draft_logits=None if dl is None else torch.from_numpy(dl).cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, near = _check(draft, target, T, uni, dl, acc.cpu().numpy(), nxt.cpu().numpy())
    print(f"B={B} L={L} V={V} T={T} sampled={sampled}: mean accept {ref['accept'].mean():.2f}, "
          f"near-tie divergences {near}")
    assert near <= max(1, B // 16)


def test_accept_sample_closed_forms():
    B, L, V = 4, 5, 4096
    rng = np.random.default_rng(3)
    t = rng.standard_normal((B, L, V)).astype(np.float32)
    tt = torch.from_numpy(t).cuda()
    x = torch.from_numpy(rng.integers(0, V, (B, L)).astype(np.int32)).cuda()
    # identical draft and target distributions: every position is accepted, whatever the draws
    uni = torch.full((B, L + 1), float(np.nextafter(np.float32(1), np.float32(0))), device="cuda")
    acc, nxt = domino.accept_sample(x, tt, 0.8, uni, draft_logits=tt.clone())
    torch.cuda.synchronize()
    assert (acc == L).all() and (nxt == -1).all()
    # all target mass on token 7 and draft tokens elsewhere: rejected at once, replaced by 7
    t2 = np.zeros((B, L, V), np.float32)
    t2[:, :, 7] = 2000.0
    x2 = torch.full((B, L), 9, dtype=torch.int32, device="cuda")
    for dl in (None, torch.zeros((B, L, V), device="cuda")):
        acc, nxt = domino.accept_sample(x2, torch.from_numpy(t2).cuda(), 1.0, torch.rand((B, L + 1), device="cuda"),
                                        draft_logits=dl)
        torch.cuda.synchronize()
        assert (acc == 0).all() and (nxt == 7).all()


def test_accept_sample_bad_token_and_host_checks():
    B, L, V = 2, 3, 64
    t = torch.randn((B, L, V), device="cuda")
    x = torch.zeros((B, L), dtype=torch.int32, device="cuda")
    x[1, 0] = V + 5
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    acc, nxt = domino.accept_sample(x, t, 1.0, torch.zeros((B, L + 1), device="cuda"), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == domino.STATUS_BAD_TOKEN and int(acc[1]) == 0
    for bad_t in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(domino.DominoError):
            domino.accept_sample(x, t, bad_t, torch.zeros((B, L + 1), device="cuda"))
