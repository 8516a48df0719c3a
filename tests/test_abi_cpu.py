"""The C-ABI library on a machine without a GPU: it loads, exports every symbol that
include/domino.h declares, and its host-side logic (workspace sizing, argument checks, status
strings) answers without touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

from draft_block_causal_b200 import domino

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", f)).read()
            names |= set(re.findall(r"DOMINO_API\s+[\w\s\*]+?\b(domino_\w+)\s*\(", txt))
    return names


@pytest.fixture(scope="module")
def L():
    from draft_block_causal_b200 import build
    build.build()
    return domino.lib()


def test_every_declared_symbol_is_exported(L):
    declared = _declared()
    assert set(domino.EXPORTS) <= declared
    out = subprocess.run(["nm", "-D", "--defined-only", domino.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (domino_\w+)", out))
    assert declared <= exported, declared - exported
    for n in declared:
        assert hasattr(L, n)


def test_abi_version_and_status_strings(L):
    assert domino.abi_version() == 2
    for code in (0, -1, -2, -3, -4, -5, 1, 2):
        s = domino.status_string(code)
        assert s and s != "unknown code"
    assert domino.status_string(12345) == "unknown code"


def _shape(**kw):
    base = dict(B=1, L=16, d=4096, Hs=1024, r=256, V=151936, dtype=1)
    base.update(kw)
    return domino.Shape(*(base[k] for k in ("B", "L", "d", "Hs", "r", "V", "dtype")))


def test_workspace_bytes_host_logic(L):
    n1 = L.domino_workspace_bytes(ctypes.byref(_shape()))
    n32 = L.domino_workspace_bytes(ctypes.byref(_shape(B=32)))
    assert n1 > 0 and n32 > n1 and n1 % 256 == 0
    # invalid shapes give 0
    for bad in (dict(B=0), dict(L=0), dict(L=65), dict(d=12), dict(V=1001), dict(dtype=7), dict(r=2048)):
        assert L.domino_workspace_bytes(ctypes.byref(_shape(**bad))) == 0, bad
    # a d whose 16-byte vector count is neither a multiple of 32 nor a power of two up to 32
    assert L.domino_workspace_bytes(ctypes.byref(_shape(d=8 * 40))) == 0
    assert L.domino_workspace_bytes(ctypes.byref(_shape(d=2560))) > 0  # 320 vectors = 10 x 32
    assert L.domino_accept_workspace_bytes(32, 16) > 0
    assert L.domino_accept_workspace_bytes(0, 16) == 0
    # B * L up to 65535 rows (launches with one row per block along grid y), and 32-bit element
    # loops over B * L * Hs
    assert L.domino_workspace_bytes(ctypes.byref(_shape(B=4095))) > 0
    assert L.domino_workspace_bytes(ctypes.byref(_shape(B=4096))) == 0
    assert L.domino_workspace_bytes(ctypes.byref(_shape(B=65535, L=1))) > 0
    assert L.domino_workspace_bytes(ctypes.byref(_shape(B=8, Hs=1 << 24))) == 0


def test_invalid_arguments_are_rejected_before_any_launch(L):
    sh = _shape()
    fake = ctypes.c_void_p(0x10000)  # 16-byte aligned, never dereferenced
    w = domino.Weights(*([0x10000] * 7))
    ws_bytes = L.domino_workspace_bytes(ctypes.byref(sh))
    # null shape / weights
    assert L.domino_draft_greedy(None, ctypes.byref(w), fake, fake, fake, fake, None, None, fake, ws_bytes, None,
                                 None) == domino.ERR_INVALID_ARGUMENT
    assert L.domino_draft_greedy(ctypes.byref(sh), None, fake, fake, fake, fake, None, None, fake, ws_bytes, None,
                                 None) == domino.ERR_INVALID_ARGUMENT
    # null required outputs / inputs
    assert L.domino_draft_greedy(ctypes.byref(sh), ctypes.byref(w), fake, fake, fake, None, None, None, fake,
                                 ws_bytes, None, None) == domino.ERR_INVALID_ARGUMENT
    assert L.domino_teacher_forced(ctypes.byref(sh), ctypes.byref(w), fake, fake, fake, fake, None, None, fake,
                                   ws_bytes, None, None) == domino.ERR_INVALID_ARGUMENT
    # misaligned pointer
    mis = ctypes.c_void_p(0x10004)
    assert L.domino_draft_greedy(ctypes.byref(sh), ctypes.byref(w), mis, fake, fake, fake, None, None, fake,
                                 ws_bytes, None, None) == domino.ERR_INVALID_ARGUMENT
    w_mis = domino.Weights(*([0x10000] * 6 + [0x10008]))
    assert L.domino_draft_greedy(ctypes.byref(sh), ctypes.byref(w_mis), fake, fake, fake, fake, None, None, fake,
                                 ws_bytes, None, None) == domino.ERR_INVALID_ARGUMENT
    # workspace missing, misaligned or too small
    assert L.domino_draft_greedy(ctypes.byref(sh), ctypes.byref(w), fake, fake, fake, fake, None, None, None,
                                 ws_bytes, None, None) == domino.ERR_WORKSPACE
    assert L.domino_draft_greedy(ctypes.byref(sh), ctypes.byref(w), fake, fake, fake, fake, None, None,
                                 ctypes.c_void_p(0x10010), ws_bytes, None, None) == domino.ERR_WORKSPACE
    assert L.domino_draft_greedy(ctypes.byref(sh), ctypes.byref(w), fake, fake, fake, fake, None, None, fake,
                                 ws_bytes - 256, None, None) == domino.ERR_WORKSPACE
    # bad shapes
    for bad in (dict(B=0), dict(L=100), dict(V=999), dict(dtype=3)):
        assert L.domino_draft_greedy(ctypes.byref(_shape(**bad)), ctypes.byref(w), fake, fake, fake, fake, None,
                                     None, fake, ws_bytes, None, None) == domino.ERR_INVALID_ARGUMENT
    # accept length
    i32 = ctypes.c_int32
    assert L.domino_accept_len(i32(0), i32(16), i32(151936), fake, fake, fake, fake, 1 << 20, None,
                               None) == domino.ERR_INVALID_ARGUMENT
    assert L.domino_accept_len(i32(1), i32(16), i32(151936), None, fake, fake, fake, 1 << 20, None,
                               None) == domino.ERR_INVALID_ARGUMENT
    assert L.domino_accept_len(i32(1), i32(16), i32(151936), fake, fake, fake, fake, 16, None,
                               None) == domino.ERR_WORKSPACE
    assert L.domino_accept_len(i32(4096), i32(16), i32(151936), fake, fake, fake, fake, 1 << 30, None,
                               None) == domino.ERR_UNSUPPORTED


def test_arena_host_logic(L):
    sh = _shape()
    n = L.domino_arena_bytes(ctypes.byref(sh))
    # W2, W1, W_hh, W_ih, b_ih, b_hh at the 8B shapes, bf16, each region rounded up to 256 bytes
    parts = [151936 * 256, 256 * (4096 + 1024), 3072 * 1024, 3072 * 4096, 3072, 3072]
    assert n == sum((2 * p + 255) // 256 * 256 for p in parts)
    assert L.domino_arena_bytes(ctypes.byref(_shape(V=999))) == 0
    w = domino.Weights(*([0x10000] * 7))
    out = domino.Weights()
    fake = ctypes.c_void_p(0x100000)
    # arena missing, misaligned or too small: rejected before any copy
    assert L.domino_pack_weights(ctypes.byref(sh), ctypes.byref(w), None, n, ctypes.byref(out),
                                 None) == domino.ERR_WORKSPACE
    assert L.domino_pack_weights(ctypes.byref(sh), ctypes.byref(w), ctypes.c_void_p(0x100010), n,
                                 ctypes.byref(out), None) == domino.ERR_WORKSPACE
    assert L.domino_pack_weights(ctypes.byref(sh), ctypes.byref(w), fake, n - 256, ctypes.byref(out),
                                 None) == domino.ERR_WORKSPACE
    assert L.domino_pack_weights(ctypes.byref(sh), ctypes.byref(w), fake, n, None,
                                 None) == domino.ERR_INVALID_ARGUMENT
    # persistence: the legacy default stream and out-of-range ratios are refused on the host
    assert L.domino_set_l2_persistence(ctypes.byref(sh), ctypes.byref(w), None,
                                       ctypes.c_float(1.0)) == domino.ERR_INVALID_ARGUMENT
    assert L.domino_set_l2_persistence(ctypes.byref(sh), ctypes.byref(w), ctypes.c_void_p(0x1000),
                                       ctypes.c_float(1.5)) == domino.ERR_INVALID_ARGUMENT


def test_read_passes_argument_checks(L):
    assert L.domino_debug_read_passes(None, 1 << 20, 1, None) == domino.ERR_INVALID_ARGUMENT
    assert L.domino_debug_read_passes(ctypes.c_void_p(0x10004), 1 << 20, 1, None) == domino.ERR_INVALID_ARGUMENT
    assert L.domino_debug_read_passes(ctypes.c_void_p(0x10000), 1 << 20, 0, None) == domino.ERR_INVALID_ARGUMENT
    assert L.domino_debug_read_passes(ctypes.c_void_p(0x10000), 8, 1, None) == domino.ERR_INVALID_ARGUMENT


def test_teacher_forced_ex_rejects_a_bad_logits_dtype(L):
    sh = _shape()
    fake = ctypes.c_void_p(0x10000)
    w = domino.Weights(*([0x10000] * 7))
    n = L.domino_workspace_bytes(ctypes.byref(sh))
    for bad in (-1, 2, 7):
        assert L.domino_teacher_forced_ex(ctypes.byref(sh), ctypes.byref(w), fake, fake, fake, fake, fake,
                                          ctypes.c_int32(bad), None, fake, n, None,
                                          None) == domino.ERR_INVALID_ARGUMENT
    # bf16 logits with fp32 storage: unsupported, refused on the host
    sh32 = _shape(dtype=0)
    n32 = L.domino_workspace_bytes(ctypes.byref(sh32))
    assert L.domino_teacher_forced_ex(ctypes.byref(sh32), ctypes.byref(w), fake, fake, fake, fake, fake,
                                      ctypes.c_int32(1), None, fake, n32, None, None) == domino.ERR_UNSUPPORTED


def test_noalloc_limits_are_checked_on_the_host(L):
    w = domino.Weights(*([0x10000] * 7))
    p = ctypes.c_void_p(0x10000)  # never dereferenced: every case fails before any launch
    # B = 4 rows of 64 positions need more than the 256 KiB scratch array
    big = domino.Shape(4, 64, 512, 256, 256, 12000, 1)
    assert L.domino_draft_greedy_noalloc(ctypes.byref(big), ctypes.byref(w), p, p, p, p, None, None, None,
                                         None) == domino.ERR_SCRATCH_LIMIT
    # shapes the fused small-batch kernel does not take: a larger batch, fp32 storage, another rank
    for bad in (domino.Shape(8, 16, 512, 256, 256, 12000, 1), domino.Shape(1, 16, 512, 256, 256, 12000, 0),
                domino.Shape(1, 16, 512, 256, 128, 12000, 1)):
        assert L.domino_draft_greedy_noalloc(ctypes.byref(bad), ctypes.byref(w), p, p, p, p, None, None, None,
                                             None) == domino.ERR_UNSUPPORTED
    ok = domino.Shape(1, 16, 512, 256, 256, 12000, 1)
    assert L.domino_draft_greedy_noalloc(ctypes.byref(ok), None, p, p, p, p, None, None, None,
                                         None) == domino.ERR_INVALID_ARGUMENT
    assert L.domino_draft_greedy_noalloc(ctypes.byref(ok), ctypes.byref(w), p, p, p, None, None, None, None,
                                         None) == domino.ERR_INVALID_ARGUMENT  # tokens_out is required
    # the optional projection table is checked like every other weight: a misaligned one is refused on
    # the host by both greedy entry points (the fused kernels read it with vector loads)
    wp = domino.Weights(*([0x10000] * 7 + [0x10004]))
    assert L.domino_draft_greedy_noalloc(ctypes.byref(ok), ctypes.byref(wp), p, p, p, p, None, None, None,
                                         None) == domino.ERR_INVALID_ARGUMENT
    n = L.domino_workspace_bytes(ctypes.byref(ok))
    assert L.domino_draft_greedy(ctypes.byref(ok), ctypes.byref(wp), p, p, p, p, None, None, p, n, None,
                                 None) == domino.ERR_INVALID_ARGUMENT


def test_accept_sample_checks_its_arguments_on_the_host(L):
    p = ctypes.c_void_p(0x10000)  # never dereferenced: every case fails before any launch
    n = L.domino_accept_sample_workspace_bytes(4, 16, 151936)
    assert n > 0 and n % 256 == 0
    assert L.domino_accept_sample_workspace_bytes(0, 16, 1000) == 0
    assert L.domino_accept_sample_workspace_bytes(4, 65, 1000) == 0
    assert L.domino_accept_sample_workspace_bytes(4, 16, 1001) == 0
    ok = (4, 16, 151936)
    # temperature must be positive and finite
    for t in (0.0, -0.5, float("inf"), float("nan")):
        assert L.domino_accept_sample(*ok, p, None, p, t, p, p, p, p, n, None, None) == domino.ERR_INVALID_ARGUMENT
    # required pointers, aligned logits, the workspace
    assert L.domino_accept_sample(*ok, None, None, p, 1.0, p, p, p, p, n, None, None) == domino.ERR_INVALID_ARGUMENT
    assert L.domino_accept_sample(*ok, p, None, p, 1.0, None, p, p, p, n, None, None) == domino.ERR_INVALID_ARGUMENT
    assert L.domino_accept_sample(*ok, p, ctypes.c_void_p(0x10004), p, 1.0, p, p, p, p, n, None,
                                  None) == domino.ERR_INVALID_ARGUMENT
    assert L.domino_accept_sample(*ok, p, None, p, 1.0, p, p, p, p, n - 256, None, None) == domino.ERR_WORKSPACE
    assert L.domino_accept_sample(*ok, p, None, p, 1.0, p, p, p, ctypes.c_void_p(0x10010), n, None,
                                  None) == domino.ERR_WORKSPACE
    assert L.domino_accept_sample(5000, 16, 1000, p, None, p, 1.0, p, p, p, p, 1 << 40, None,
                                  None) == domino.ERR_UNSUPPORTED


def test_projection_and_debug_entry_points_check_their_arguments(L):
    sh = _shape()
    w = domino.Weights(*([0x10000] * 7))
    assert L.domino_embed_proj_bytes(ctypes.byref(sh)) == 151936 * 3 * 1024 * 4
    assert L.domino_embed_proj_bytes(ctypes.byref(_shape(V=999))) == 0
    # the table pointer is required and must be 16-byte aligned
    assert L.domino_project_embeddings(ctypes.byref(sh), ctypes.byref(w), None, None,
                                       None) == domino.ERR_INVALID_ARGUMENT
    assert L.domino_project_embeddings(ctypes.byref(sh), ctypes.byref(w), ctypes.c_void_p(0x10004), None,
                                       None) == domino.ERR_INVALID_ARGUMENT
    a = ctypes.c_void_p(0x10000)
    i64 = ctypes.c_int64
    # K must be a positive multiple of 64, the wrap a divisor of K and a multiple of 64
    for M, N, K, wrap in ((128, 16, 100, 0), (128, 16, 0, 0), (128, 16, 256, 96), (128, 16, 192, 128), (0, 16, 64, 0)):
        assert L.domino_debug_gemm(a, a, M, N, K, wrap, a, i64(128), 0, 0, 0, None,
                                   None) == domino.ERR_INVALID_ARGUMENT, (M, N, K, wrap)
    # output stride shorter than a row, misaligned output, unknown tile width or split
    assert L.domino_debug_gemm(a, a, 128, 16, 64, 0, a, i64(8), 0, 0, 0, None, None) == domino.ERR_INVALID_ARGUMENT
    assert L.domino_debug_gemm(a, a, 128, 16, 64, 0, ctypes.c_void_p(0x10008), i64(16), 0, 0, 0, None,
                               None) == domino.ERR_INVALID_ARGUMENT
    for bn, ks in ((48, 1), (64, 0), (64, 9), (0, 2)):
        assert L.domino_debug_gemm(a, a, 128, 16, 64, 0, a, i64(16), 0, bn, ks, None,
                                   None) == domino.ERR_INVALID_ARGUMENT, (bn, ks)
    # the trace hook wants an 8-byte aligned buffer and a positive length; NULL turns it off
    assert L.domino_debug_set_trace(ctypes.c_void_p(0x10004), 16) == domino.ERR_INVALID_ARGUMENT
    assert L.domino_debug_set_trace(ctypes.c_void_p(0x10000), 0) == domino.ERR_INVALID_ARGUMENT
    assert L.domino_debug_set_trace(None, 0) == domino.OK
    # the plan text of an invalid shape, and the CUDA-core kernels of fp32 storage
    assert L.domino_greedy_plan(ctypes.byref(_shape(B=0))) == b"invalid shape"
    assert b"k_w2" in L.domino_greedy_plan(ctypes.byref(_shape(dtype=0)))
    assert L.domino_teacher_forced_plan(ctypes.byref(_shape(B=0))) == b"invalid shape"
    assert b"k_gru" in L.domino_teacher_forced_plan(ctypes.byref(_shape(dtype=0)))
