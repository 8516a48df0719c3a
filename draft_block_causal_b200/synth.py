"""Seeded synthetic inputs for the Domino head (weights, backbone outputs, tokens, targets).

This module is shared by the tests, the bench and the smoke check: it feeds the CUDA library
and the CPU oracle the same arrays.  It holds none of the head's arithmetic -- only random
draws, the bf16 rounding of stored values, and the workload table.

Shapes follow the pages' two target models (Qwen3-4B and Qwen3-8B, Domino review page,
section 三) with block size 16 (section 二, "block size=16"), GRU hidden 1024 and rank 256
(section 二, the two bullets above the head equation).  The embedding width d equals the
model's hidden size (2560 for Qwen3-4B, 4096 for Qwen3-8B) and V = 151936 (the Qwen3
vocabulary); with these, GRU(d->1024) + W1((d+1024)->256) + W2(256->V) holds 55,941,120
parameters at d=4096, the "about 56 million" the review quotes.

Value recipe (the pages print no data; these are synthetic stand-ins for trained weights and
for the datasets the pages evaluate on):
  weights   U(-1/sqrt(fan_in), +1/sqrt(fan_in)), fan_in = d (W_ih, b_ih), Hs (W_hh, b_hh),
            d+Hs (W1), r (W2)
  embed     N(0, 0.02)  (standard deviation)
  hidden H  N(0, 1)
  L_base    N(0, 1), plus ``peak`` added at one uniformly drawn token per (row, position)
  S0        zero, or N(0, s0_std) per row
  tokens    uniform on [0, V) (teacher forcing)
  target    L_base (widened exactly) + N(0, 0.5), stored fp32
bf16 tensors are rounded to nearest-even from the fp32 draw and stored as uint16 bit patterns.

Every tensor draws from its own stream, seeded by (seed, crc32(tensor name)) through
numpy's SeedSequence, so the order in which tensors are generated does not matter.
"""
from __future__ import annotations

import zlib
from functools import lru_cache

import numpy as np

F32 = 0
BF16 = 1

# Workloads: name -> shape and seeds.  Batch sweeps override B.
WORKLOADS = {
    # small fp32 head the oracle finishes instantly; greedy drafting
    "tiny-f32-b1": dict(B=1, L=4, d=64, Hs=32, r=16, V=1000, dtype=F32,
                        weight_seed=0, input_seed=0, s0_std=0.0, peak=4.0),
    # Qwen3-4B-shaped head, bf16, one row; greedy and teacher-forced
    "qwen3-4b-head-b1": dict(B=1, L=16, d=2560, Hs=1024, r=256, V=151936, dtype=BF16,
                             weight_seed=0, input_seed=1, s0_std=0.0, peak=4.0),
    # Qwen3-8B-shaped head, bf16, one row; greedy plus accept length
    "qwen3-8b-head-b1": dict(B=1, L=16, d=4096, Hs=1024, r=256, V=151936, dtype=BF16,
                             weight_seed=0, input_seed=2, s0_std=0.0, peak=4.0),
    # Qwen3-8B-shaped head, serving batch of 32 rows with independent S0
    "qwen3-8b-head-b32": dict(B=32, L=16, d=4096, Hs=1024, r=256, V=151936, dtype=BF16,
                              weight_seed=0, input_seed=3, s0_std=0.1, peak=4.0),
    # Qwen3-8B-shaped head, batch sweep (B and peak overridden per point)
    "qwen3-8b-head-sweep": dict(B=1, L=16, d=4096, Hs=1024, r=256, V=151936, dtype=BF16,
                                weight_seed=0, input_seed=4, s0_std=0.1, peak=4.0),
    # Qwen3-4B-shaped head, the same batch sweep
    "qwen3-4b-head-sweep": dict(B=1, L=16, d=2560, Hs=1024, r=256, V=151936, dtype=BF16,
                                weight_seed=0, input_seed=5, s0_std=0.1, peak=4.0),
    # a narrower head (d = 512, Hs = 256) over the full vocabulary, two rows: the GRU rows do not fill
    # TMEM's layout, so the fused kernel streams them from L2 (profiling of that variant)
    "narrow-head-b2": dict(B=2, L=16, d=512, Hs=256, r=256, V=151936, dtype=BF16,
                           weight_seed=0, input_seed=6, s0_std=0.1, peak=4.0),
}
SWEEP_BATCHES = (1, 4, 16, 64, 128, 256)
SWEEP_PEAKS = (1.0, 2.0, 4.0)


def workload(name: str, **override) -> dict:
    w = dict(WORKLOADS[name])
    w.update(override)
    w["name"] = name
    return w


def shape_of(wl: dict) -> dict:
    return {k: int(wl[k]) for k in ("B", "L", "d", "Hs", "r", "V", "dtype")}


def _rng(seed: int, name: str) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), zlib.crc32(name.encode())]))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); return the 16-bit patterns as uint16."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_f32(a: np.ndarray, dtype: int) -> np.ndarray:
    return a.astype(np.float32) if dtype == F32 else bf16_bits_to_f32(a)


def _store(x: np.ndarray, dtype: int) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float32) if dtype == F32 else f32_to_bf16_bits(x)


def _uniform(seed, name, shape, bound, dtype, chunk=1 << 24):
    rng = _rng(seed, name)
    n = int(np.prod(shape))
    out = np.empty(n, np.float32 if dtype == F32 else np.uint16)
    for s in range(0, n, chunk):
        m = min(chunk, n - s)
        x = rng.random(m, dtype=np.float32)
        x = (x * np.float32(2.0) - np.float32(1.0)) * np.float32(bound)
        out[s:s + m] = _store(x, dtype)
    return out.reshape(shape)


def _normal(seed, name, shape, std, dtype, chunk=1 << 24):
    rng = _rng(seed, name)
    n = int(np.prod(shape))
    out = np.empty(n, np.float32 if dtype == F32 else np.uint16)
    for s in range(0, n, chunk):
        m = min(chunk, n - s)
        x = rng.standard_normal(m, dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        out[s:s + m] = _store(x, dtype)
    return out.reshape(shape)


def head_weights(shape: dict, seed: int) -> dict:
    """Embedding table and head weights, row-major: embed [V,d], W_ih [3Hs,d], W_hh [3Hs,Hs],
    b_ih/b_hh [3Hs] (gate blocks r|z|n), W1 [r, d+Hs] (H columns first), W2 [V, r]."""
    d, Hs, r, V, dt = shape["d"], shape["Hs"], shape["r"], shape["V"], shape["dtype"]
    return {
        "embed": _normal(seed, "embed", (V, d), 0.02, dt),
        "W_ih": _uniform(seed, "W_ih", (3 * Hs, d), d ** -0.5, dt),
        "W_hh": _uniform(seed, "W_hh", (3 * Hs, Hs), Hs ** -0.5, dt),
        "b_ih": _uniform(seed, "b_ih", (3 * Hs,), d ** -0.5, dt),
        "b_hh": _uniform(seed, "b_hh", (3 * Hs,), Hs ** -0.5, dt),
        "W1": _uniform(seed, "W1", (r, d + Hs), (d + Hs) ** -0.5, dt),
        "W2": _uniform(seed, "W2", (V, r), r ** -0.5, dt),
    }


def block_inputs(shape: dict, seed: int, peak: float = 4.0, s0_std: float = 0.0) -> dict:
    """Backbone outputs for one block: base_logits [B,L,V], hidden [B,L,d], S0 [B,Hs] fp32."""
    B, L, d, Hs, V, dt = shape["B"], shape["L"], shape["d"], shape["Hs"], shape["V"], shape["dtype"]
    rng_l = _rng(seed, "base_logits")
    peaks = _rng(seed, "base_logits.peak").integers(0, V, size=(B, L))
    lb = np.empty((B, L, V), np.float32 if dt == F32 else np.uint16)
    for b in range(B):
        for i in range(L):
            x = rng_l.standard_normal(V, dtype=np.float32)
            x[peaks[b, i]] += np.float32(peak)
            lb[b, i] = _store(x, dt)
    hidden = _normal(seed, "hidden", (B, L, d), 1.0, dt)
    if s0_std > 0.0:
        S0 = _rng(seed, "S0").standard_normal((B, Hs), dtype=np.float32) * np.float32(s0_std)
    else:
        S0 = np.zeros((B, Hs), np.float32)
    return {"base_logits": lb, "hidden": hidden, "S0": np.ascontiguousarray(S0, dtype=np.float32)}


def teacher_tokens(shape: dict, seed: int) -> np.ndarray:
    return _rng(seed, "tokens").integers(0, shape["V"], size=(shape["B"], shape["L"])).astype(np.int32)


def target_logits(base_logits: np.ndarray, shape: dict, seed: int, noise_std: float = 0.5) -> np.ndarray:
    """Synthetic target-model logits: the base logits (widened exactly) plus N(0, noise_std)."""
    B, L, V = base_logits.shape
    rng = _rng(seed, "target_logits")
    out = np.empty((B, L, V), np.float32)
    for b in range(B):
        for i in range(L):
            out[b, i] = to_f32(base_logits[b, i], shape["dtype"]) + \
                rng.standard_normal(V, dtype=np.float32) * np.float32(noise_std)
    return out


@lru_cache(maxsize=2)
def _cached_weights(key):
    shape = dict(key[0])
    return head_weights(shape, key[1])


def cached_head_weights(shape: dict, seed: int) -> dict:
    """``head_weights`` memoised per (shape, seed) -- the 8B embedding table takes seconds."""
    key = (tuple(sorted((k, shape[k]) for k in ("d", "Hs", "r", "V", "dtype"))), int(seed))
    return _cached_weights(key)


def make_workload(wl: dict, with_tokens: bool = False, with_target: bool = False) -> dict:
    """All arrays for a workload: weights, block inputs and (optionally) tokens and targets."""
    shape = shape_of(wl)
    out = {"shape": shape, "weights": cached_head_weights(shape, wl["weight_seed"])}
    out.update(block_inputs(shape, wl["input_seed"], peak=wl["peak"], s0_std=wl["s0_std"]))
    if with_tokens:
        out["tokens"] = teacher_tokens(shape, wl["input_seed"])
    if with_target:
        out["target_logits"] = target_logits(out["base_logits"], shape, wl["input_seed"])
    return out


def param_count(shape: dict) -> int:
    """Head parameters: GRU (with both biases), W1 and W2 (embedding table excluded)."""
    d, Hs, r, V = shape["d"], shape["Hs"], shape["r"], shape["V"]
    return 3 * Hs * d + 3 * Hs * Hs + 6 * Hs + r * (d + Hs) + V * r
