"""The tensor-core GEMM engine behind the batched paths, on its own (domino_debug_gemm): every
tile width and K split against a float64 product of the same bf16 operands, ragged edges, the
K-wrap used for two-term state splits, and bit-identical repeats of split products."""
import math

import pytest
import torch

from draft_block_causal_b200 import domino

pytestmark = pytest.mark.gpu


def _operands(M, N, K, seed, kwrap=0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    A = torch.randn(M, kwrap or K, generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, generator=g).to(torch.bfloat16)
    return A.cuda(), B.cuda()


def _reference(A, B, kwrap=0):
    a = A.double()
    if kwrap:
        a = a.repeat(1, B.shape[1] // kwrap)
    return a @ B.double().T


def _check(got, ref, K):
    tol = 1e-4 * math.sqrt(K) + 1e-6 * K
    err = (got.double() - ref).abs().max().item()
    assert err <= tol, (err, tol)


@pytest.mark.parametrize("bn", [16, 32, 64, 128])
@pytest.mark.parametrize("ks", [1, 2, 3, 5, 8])
def test_forced_plans_match_float64(bn, ks):
    M, N, K = 300, 70, 512
    A, B = _operands(M, N, K, seed=bn * 10 + ks)
    ref = _reference(A, B)
    got = domino.debug_gemm(A, B, trans=True, bn=bn, ks=ks)
    torch.cuda.synchronize()
    _check(got.T, ref, K)
    if ks > 1:  # the split partials are added in piece order: repeats are bit-identical
        again = domino.debug_gemm(A, B, trans=True, bn=bn, ks=ks)
        torch.cuda.synchronize()
        assert torch.equal(got, again)


@pytest.mark.parametrize("M,N,K,trans", [(3072, 128, 4096, True), (3328, 32, 2048, True), (1000, 20, 192, False),
                                         (1000, 20, 192, True), (128, 1, 64, True), (256, 256, 1024, False),
                                         (3072, 480, 4096, True)])
def test_automatic_plan_matches_float64(M, N, K, trans):
    A, B = _operands(M, N, K, seed=M + N + K)
    ref = _reference(A, B)
    got = domino.debug_gemm(A, B, trans=trans)
    torch.cuda.synchronize()
    _check(got.T if trans else got, ref, K)


@pytest.mark.parametrize("ks", [1, 4])
def test_k_wrap_applies_a_to_both_halves(ks):
    M, N, K, kw = 256, 33, 2048, 1024
    A, B = _operands(M, N, K, seed=77 + ks, kwrap=kw)
    ref = _reference(A, B, kwrap=kw)
    got = domino.debug_gemm(A, B, trans=True, a_kwrap=kw, bn=64, ks=ks)
    torch.cuda.synchronize()
    _check(got.T, ref, K)


def test_invalid_plans_are_refused_on_the_host():
    A, B = _operands(128, 16, 128, seed=1)
    for bn, ks in ((48, 1), (16, 9), (0, 2), (128, 0)):
        with pytest.raises(domino.DominoError):
            domino.debug_gemm(A, B, bn=bn, ks=ks)


def test_read_passes_runs_and_counts_one_launch():
    buf = torch.ones(1 << 22, dtype=torch.uint8, device="cuda")
    n0 = domino.launch_count()
    domino.debug_read_passes(buf, 3)
    torch.cuda.synchronize()
    assert domino.launch_count() == n0 + 1
