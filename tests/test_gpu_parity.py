"""GPU parity: the CUDA path, called through the C ABI, against the fp64 oracle on the same
seeded inputs (procedure in gpu_common).  Every case is checked on every row and every output;
the large ones row chunk by row chunk."""
import numpy as np
import pytest
import torch

from draft_block_causal_b200 import synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from tests import gpu_common as G
else:  # collected but skipped on machines without a GPU
    G = None


def _custom(B, L, d, Hs, r, V, dtype, seed, s0_std=0.2, peak=2.0):
    wl = dict(B=B, L=L, d=d, Hs=Hs, r=r, V=V, dtype=dtype, weight_seed=seed, input_seed=seed + 1,
              s0_std=s0_std, peak=peak, name=f"custom-{seed}")
    return wl


SMALL = [
    synth.workload("tiny-f32-b1"),
    _custom(3, 5, 256, 128, 64, 4104, 1, 100),            # ragged vocab tail, several rows
    _custom(5, 7, 64, 32, 16, 1000, 0, 110),              # fp32, odd B and L
    _custom(2, 16, 512, 256, 256, 20008, 1, 120),         # bf16, full block, r = 256
    _custom(1, 1, 64, 64, 32, 64, 1, 130),                # a single position: no GRU update
    _custom(17, 3, 128, 64, 32, 3000, 1, 140),            # B not a multiple of the row tiles
    # shapes the fused persistent kernel takes (bf16, r = 256, d and Hs multiples of 256, B <= 4)
    _custom(3, 16, 256, 256, 256, 1000, 1, 150),          # odd B, vocabulary smaller than 8 rows/CTA
    _custom(4, 9, 768, 512, 256, 33000, 1, 160),          # B = 4, odd L, ragged vocabulary slices
    _custom(1, 1, 256, 256, 256, 5000, 1, 170),           # one position: no GRU update at all
    _custom(2, 16, 1024, 256, 256, 40000, 1, 180, s0_std=1.0, peak=0.5),  # weak peaks: many near-ties
    # shapes the TMEM-resident variant takes (d and Hs multiples of 512)
    _custom(3, 16, 1024, 512, 256, 9000, 1, 190),         # odd B, several GRU units per CTA
    _custom(2, 5, 512, 512, 256, 3000, 1, 200),           # short block, small vocabulary
    _custom(4, 16, 2560, 1024, 256, 20000, 1, 210),       # Qwen3-4B widths, B = 4
    _custom(1, 16, 4096, 1024, 256, 7992, 1, 220, s0_std=1.0, peak=0.5),  # 8B widths, many near-ties
    # the batched tensor-core path (B > 4) and its W2 argmax kernel: ragged 16-column units, every
    # supported rank, two batch bands, fewer vocabulary units than SMs, a one-unit vocabulary
    _custom(7, 5, 256, 128, 64, 1000, 1, 300),            # r = 64, V % 16 = 8
    _custom(130, 3, 256, 256, 128, 5000, 1, 310),         # bands of 128 and 2 rows, r = 128
    _custom(40, 16, 512, 256, 256, 2056, 1, 320, s0_std=1.0, peak=0.5),  # 129 units: 129 CTAs
    _custom(9, 4, 128, 64, 64, 16, 1, 330),               # V = 16: one unit, one CTA
    # the persistent batched kernel (5 <= B <= 128, Hs a multiple of 128): its smallest batch with a
    # short block, a single position (no GRU update), r = 128 and a vocabulary of 65 units
    _custom(5, 2, 256, 128, 128, 1000, 1, 340),
    _custom(100, 1, 256, 128, 128, 1040, 1, 350),
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w["name"] + f"-B{w['B']}")
def test_greedy_small(wl):
    data = synth.make_workload(wl)
    res = G.greedy_parity(data)
    print(wl["name"], {k: v for k, v in res.items() if k != "tokens"})


TF_CASES = SMALL[1:4] + [
    _custom(20, 16, 512, 256, 256, 3000, 1, 230),   # B*L = 320: two column tiles, ragged vocabulary tile
    _custom(1, 7, 256, 256, 128, 1024, 1, 240),     # exactly 8 vocabulary tiles, 7 positions
    # the unit-owned recurrence (k_tf_units): four, two and one row groups per A tile, a W_hh chunk
    # count that halves the row groups (Hs = 128), a single update, a single position
    _custom(5, 9, 256, 256, 128, 2000, 1, 250),
    _custom(40, 6, 256, 256, 128, 3000, 1, 252),
    _custom(100, 5, 256, 512, 128, 2000, 1, 254),
    _custom(30, 4, 128, 128, 128, 1504, 1, 256),
    _custom(12, 2, 256, 256, 128, 1000, 1, 258),
    _custom(12, 1, 256, 256, 128, 1000, 1, 260),
    # Hs above the unit-owned kernel's limit: the batched kernel's teacher-forced mode
    _custom(9, 4, 256, 1280, 128, 2000, 1, 262),
    # logits GEMM with three row bands over more vocabulary tiles than SMs (a CTA meets several bands)
    _custom(20, 16, 256, 256, 256, 24008, 1, 264),
]
TF_PLANS = {250: "k_tf_units", 252: "k_tf_units", 254: "k_tf_units", 256: "k_tf_units", 258: "k_tf_units",
            260: "k_tf_units", 262: "k_greedy_batched", 230: "k_tf_units", 264: "k_tf_units"}


@pytest.mark.parametrize("wl", TF_CASES, ids=lambda w: w["name"] + f"-B{w['B']}")
def test_teacher_forced_small(wl):
    data = synth.make_workload(wl, with_tokens=True)
    seed = wl["weight_seed"]
    if seed in TF_PLANS:
        from draft_block_causal_b200 import domino
        w, _, _, _ = G.device_inputs(data)
        assert TF_PLANS[seed] in domino.teacher_forced_plan(domino.make_shape(w, wl["B"], wl["L"]))
    res = G.tf_parity(data)
    print(wl["name"], res)


def test_greedy_and_teacher_forced_4b_shapes():
    wl = synth.workload("qwen3-4b-head-b1")
    data = synth.make_workload(wl, with_tokens=True)
    print("greedy", {k: v for k, v in G.greedy_parity(data).items() if k != "tokens"})
    print("tf", G.tf_parity(data))


def test_greedy_and_accept_8b_b1():
    wl = synth.workload("qwen3-8b-head-b1")
    data = synth.make_workload(wl, with_target=True)
    res = G.greedy_parity(data)
    acc = G.accept_parity(res["tokens"], data["target_logits"])
    print({k: v for k, v in res.items() if k != "tokens"}, "accept", acc)


def test_greedy_tf_accept_8b_b32_every_row():
    """Qwen3-8B shapes at B = 32 (per-row S0 ~ N(0, 0.1)): greedy, teacher forcing and the accept
    length against the oracle on every row and every output."""
    wl = synth.workload("qwen3-8b-head-b32")
    data = synth.make_workload(wl, with_tokens=True, with_target=True)
    res = G.greedy_parity_rows(data)
    print("greedy", {k: v for k, v in res.items() if k != "tokens"})
    print("tf", G.tf_parity_rows(data))
    acc = G.accept_parity(res["tokens"], data["target_logits"])
    print("accept", acc)


@pytest.mark.parametrize("B,peak", [(B, p) for B in synth.SWEEP_BATCHES for p in synth.SWEEP_PEAKS],
                         ids=lambda v: str(v))
def test_greedy_batch_sweep_every_row(B, peak):
    """The batch sweep, B in {1, 4, 16, 64, 128, 256} crossed with base-logit peaks {+1, +2, +4}:
    every row replayed by the oracle, with and without logits written."""
    wl = synth.workload("qwen3-8b-head-sweep", B=B, peak=peak)
    data = synth.make_workload(wl)
    res = G.greedy_parity_rows(data)
    print(B, peak, {k: v for k, v in res.items() if k != "tokens"})


@pytest.mark.parametrize("B", [16, 64, 128])
def test_teacher_forced_sweep_every_row(B):
    """Teacher forcing at the Qwen3-8B widths with four, two and one row groups per A tile of the
    unit-owned recurrence: every row's logits and states against the oracle."""
    from draft_block_causal_b200 import domino
    wl = synth.workload("qwen3-8b-head-sweep", B=B, peak=2.0)
    data = synth.make_workload(wl, with_tokens=True)
    w, _, _, _ = G.device_inputs(data)
    assert "k_tf_units" in domino.teacher_forced_plan(domino.make_shape(w, B, wl["L"]))
    res = G.tf_parity_rows(data)
    print(B, res)


def test_accept_length_constructed_prefixes():
    rng = np.random.default_rng(7)
    B, L, V = 40, 16, 151936
    T = rng.standard_normal((B, L, V)).astype(np.float32)
    am = np.argmax(T, axis=-1).astype(np.int32)
    draft = am.copy()
    for b in range(B):
        k = b % (L + 1)
        if k < L:
            draft[b, k] = (draft[b, k] + 1) % V
    # exact ties: the lowest index must win
    T[3, 0, 10] = T[3, 0, 20] = 100.0
    draft[3, 0] = 10
    got = G.accept_parity(draft, T)
    assert got[0] == 0 and got[16] == 16


def test_accept_length_small_vocab_and_single_position():
    rng = np.random.default_rng(8)
    for B, L, V in [(1, 1, 8), (3, 4, 24), (65, 16, 1000)]:
        T = rng.integers(-2, 3, (B, L, V)).astype(np.float32)  # ties everywhere
        draft = np.argmax(T, axis=-1).astype(np.int32)
        draft[::2, L // 2] = (draft[::2, L // 2] + 1) % V
        G.accept_parity(draft, T)
