"""fp64 CPU oracle of the Domino head -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference leg may
import this package.  The product path (``draft_block_causal_b200``) never imports it, and this
package never imports the product: the two share only the seeded input arrays.

The arithmetic lives in ``domino_oracle.c`` (plain C, double precision, OpenMP over independent
outputs).  This module builds it with gcc and marshals numpy arrays through ctypes.

Source of the equations: the Domino review page (paper.oopus.info), section 二, the head
equation ``L_final = L_base + W2 . sigma(W1 . [H_i ; S_{i-1}])`` with the GRU causal encoder
(hidden 1024) and the rank-256 SiLU correction described beside it.  The readings taken where
the pages are silent are listed in the header of ``domino_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import time

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "domino_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32 = 0
BF16 = 1


class _Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "L", "d", "Hs", "r", "V", "dtype")]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE semantics: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = f"{_LIB}.{os.getpid()}.{time.time_ns()}.tmp"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def configure(lib: ctypes.CDLL) -> ctypes.CDLL:
    """Declare the C entry points' argument types on a loaded oracle library."""
    vp = ctypes.c_void_p
    lib.oracle_head.argtypes = [ctypes.POINTER(_Shape)] + [vp] * 10 + [vp, vp, vp, vp, vp, ctypes.c_int]
    lib.oracle_head.restype = ctypes.c_int
    lib.oracle_accept_len.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp]
    lib.oracle_accept_len.restype = ctypes.c_int
    lib.oracle_gru_step.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int] + [vp] * 7
    lib.oracle_gru_step.restype = None
    lib.oracle_accept_sample.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp, ctypes.c_float, vp,
                                         vp, vp, vp]
    lib.oracle_accept_sample.restype = ctypes.c_int
    lib.oracle_residual_cdf.argtypes = [ctypes.c_int, vp, vp, ctypes.c_int, ctypes.c_float, vp]
    lib.oracle_residual_cdf.restype = ctypes.c_double
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = configure(ctypes.CDLL(build()))
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(a, dtype, shape, name):
    if a.dtype != dtype or tuple(a.shape) != tuple(shape) or not a.flags.c_contiguous:
        raise ValueError(f"oracle: {name} must be a C-contiguous {np.dtype(dtype)} array of shape {shape},"
                         f" got {a.dtype} {a.shape}")


def _wdtype(dtype: int):
    return np.float32 if dtype == F32 else np.uint16


def head(shape: dict, w: dict, base_logits, hidden, S0, tokens=None, rows=None,
         want_logits: bool = True, want_states: bool = True, nthreads: int = 0) -> dict:
    """Run the head over a block (greedy when ``tokens`` is None, else teacher-forced).

    ``shape`` holds B, L, d, Hs, r, V and dtype (0 = fp32 storage, 1 = bf16 bit patterns in
    uint16 arrays).  ``rows`` optionally restricts the run to a subset of batch rows (the rows
    are independent); the outputs then have ``len(rows)`` rows.
    """
    B, L, d, Hs, r, V, dt = (int(shape[k]) for k in ("B", "L", "d", "Hs", "r", "V", "dtype"))
    wd = _wdtype(dt)
    _check(w["embed"], wd, (V, d), "embed")
    _check(w["W_ih"], wd, (3 * Hs, d), "W_ih")
    _check(w["W_hh"], wd, (3 * Hs, Hs), "W_hh")
    _check(w["b_ih"], wd, (3 * Hs,), "b_ih")
    _check(w["b_hh"], wd, (3 * Hs,), "b_hh")
    _check(w["W1"], wd, (r, d + Hs), "W1")
    _check(w["W2"], wd, (V, r), "W2")
    _check(base_logits, wd, (B, L, V), "base_logits")
    _check(hidden, wd, (B, L, d), "hidden")
    _check(S0, np.float32, (B, Hs), "S0")
    if tokens is not None:
        _check(tokens, np.int32, (B, L), "tokens")
    if rows is not None:
        rows = np.asarray(rows, dtype=np.int64)
        base_logits = np.ascontiguousarray(base_logits[rows])
        hidden = np.ascontiguousarray(hidden[rows])
        S0 = np.ascontiguousarray(S0[rows])
        if tokens is not None:
            tokens = np.ascontiguousarray(tokens[rows])
        B = len(rows)
    sh = _Shape(B, L, d, Hs, r, V, dt)
    tok_out = np.empty((B, L), np.int32)
    logits = np.empty((B, L, V), np.float64) if want_logits else None
    states = np.empty((B, L, Hs), np.float64) if want_states else None
    margin = np.empty((B, L), np.float64)
    rc = _load().oracle_head(ctypes.byref(sh), _ptr(w["embed"]), _ptr(w["W_ih"]), _ptr(w["W_hh"]),
                             _ptr(w["b_ih"]), _ptr(w["b_hh"]), _ptr(w["W1"]), _ptr(w["W2"]),
                             _ptr(base_logits), _ptr(hidden), _ptr(S0), _ptr(tokens), _ptr(tok_out),
                             _ptr(logits), _ptr(states), _ptr(margin), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_head failed with code {rc}")
    return {"tokens": tok_out, "logits": logits, "states": states, "margin": margin}


def accept_len(draft_tokens, target_logits) -> np.ndarray:
    """Greedy accept length per row (see ``oracle_accept_len`` in domino_oracle.c)."""
    B, L, V = target_logits.shape
    _check(draft_tokens, np.int32, (B, L), "draft_tokens")
    _check(target_logits, np.float32, (B, L, V), "target_logits")
    out = np.empty((B,), np.int32)
    rc = _load().oracle_accept_len(B, L, V, _ptr(draft_tokens), _ptr(target_logits), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_accept_len failed with code {rc}")
    return out


def accept_sample(draft_tokens, target_logits, temperature: float, uniforms, draft_logits=None) -> dict:
    """Sampled verification of a block (see ``oracle_accept_sample`` in domino_oracle.c):
    accept lengths [B], replacement tokens [B] (-1 when every position was accepted) and the
    acceptance ratios p/q [B, L] of the decisions taken (-1 after)."""
    B, L, V = target_logits.shape
    _check(draft_tokens, np.int32, (B, L), "draft_tokens")
    _check(target_logits, np.float32, (B, L, V), "target_logits")
    _check(uniforms, np.float32, (B, L + 1), "uniforms")
    if draft_logits is not None:
        _check(draft_logits, np.float32, (B, L, V), "draft_logits")
    acc = np.empty((B,), np.int32)
    nxt = np.empty((B,), np.int32)
    ratio = np.empty((B, L), np.float64)
    rc = _load().oracle_accept_sample(B, L, V, _ptr(draft_tokens), _ptr(draft_logits), _ptr(target_logits),
                                      float(temperature), _ptr(uniforms), _ptr(acc), _ptr(nxt), _ptr(ratio))
    if rc != 0:
        raise ValueError(f"oracle_accept_sample failed with code {rc}")
    return {"accept": acc, "next": nxt, "ratio": ratio}


def residual_cdf(target_row, draft_row, draft_token: int, temperature: float):
    """Running sums of the resampling residual at one position (``oracle_residual_cdf``):
    returns (cdf [V] float64, Z)."""
    V = target_row.shape[0]
    _check(target_row, np.float32, (V,), "target_row")
    if draft_row is not None:
        _check(draft_row, np.float32, (V,), "draft_row")
    cdf = np.empty((V,), np.float64)
    z = _load().oracle_residual_cdf(V, _ptr(target_row), _ptr(draft_row), int(draft_token), float(temperature),
                                    _ptr(cdf))
    return cdf, float(z)


def gru_step(d: int, Hs: int, dtype: int, w: dict, x, h) -> np.ndarray:
    """One GRU step on double inputs ``x`` [d] and ``h`` [Hs] with the stored GRU weights."""
    wd = _wdtype(dtype)
    _check(w["W_ih"], wd, (3 * Hs, d), "W_ih")
    _check(w["W_hh"], wd, (3 * Hs, Hs), "W_hh")
    _check(w["b_ih"], wd, (3 * Hs,), "b_ih")
    _check(w["b_hh"], wd, (3 * Hs,), "b_hh")
    x = np.ascontiguousarray(x, dtype=np.float64)
    h = np.ascontiguousarray(h, dtype=np.float64)
    out = np.empty((Hs,), np.float64)
    _load().oracle_gru_step(d, Hs, dtype, _ptr(w["W_ih"]), _ptr(w["W_hh"]), _ptr(w["b_ih"]),
                            _ptr(w["b_hh"]), _ptr(x), _ptr(h), _ptr(out))
    return out
