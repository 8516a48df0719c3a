"""The bench's roofline arithmetic on CPU, against figures worked out by hand from the
Qwen3-8B-shaped head (16-token block, Hs = 1024, r = 256, V = 151936): algorithmic bytes of a
greedy call with no reuse, unique (first-touch) bytes, and FLOPs per call."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from draft_block_causal_b200 import synth  # noqa: E402


def _sh(B):
    return dict(B=B, L=16, d=4096, Hs=1024, r=256, V=151936, dtype=synth.BF16)


def test_greedy_bytes_match_the_worked_figures():
    # W2 16 x 77.79 MB, GRU 15 x 31.46 MB, W1 (H block) once, W1 (state block) 16 x 0.52 MB, plus per
    # row the base logits, hidden states, embedding rows, S0 and tokens: 1.732 GB at B = 1
    assert bench.greedy_bytes(_sh(1)) == 1_732_309_056
    w2 = 16 * 151936 * 256 * 2
    gru = 15 * (3 * 1024 * 4096 + 3 * 1024 * 1024 + 6 * 1024) * 2
    assert w2 == 1_244_659_712 and gru == 472_043_520  # 16 x 77.79 MB, 15 x 31.47 MB
    # the per-row part grows linearly with B
    per_row = bench.greedy_bytes(_sh(2)) - bench.greedy_bytes(_sh(1))
    assert bench.greedy_bytes(_sh(128)) == bench.greedy_bytes(_sh(1)) + 127 * per_row


def test_unique_bytes_are_the_weights_once():
    # every weight byte once plus the per-row inputs: about 117 MB at B = 1
    assert bench.unique_bytes(_sh(1)) == 117_002_304
    assert bench.unique_bytes(_sh(1)) < bench.greedy_bytes(_sh(1)) / 14


def test_flops_match_the_worked_table():
    # total GFLOP per call: 1.76 (B = 1), 56.3 (B = 32), 225.1 (B = 128)
    for B, gflop in ((1, 1.76), (32, 56.3), (128, 225.1)):
        assert bench.greedy_flops(_sh(B)) / 1e9 == pytest.approx(gflop, rel=2e-3)
    # the W2 part alone at B = 128: 159.3 GFLOP
    assert 2 * 128 * 16 * 256 * 151936 / 1e9 == pytest.approx(159.3, rel=1e-3)


def test_projection_table_variant_reads_less():
    # the projection table replaces the W_ih stream by a 3Hs-float row gather: 1.355 GB at B = 1
    assert bench.greedy_bytes_proj(_sh(1)) == 1_354_883_136


def test_teacher_forcing_bytes():
    # W_ih, W1, W2 once, W_hh per update, given tokens' rows, base logits in, fp32 logits out
    assert bench.tf_bytes(_sh(1)) == 214_806_592
    assert bench.tf_bytes(_sh(32)) - bench.tf_bytes(_sh(1)) == 31 * (
        16 * 151936 * 2 + 16 * 4096 * 2 + 15 * 4096 * 2 + 1024 * 4 + 16 * 4 + 16 * 151936 * 4)


def test_near_gpu_placement_leaves_the_affinity_as_it_found_it(monkeypatch):
    """The e2e pinned-buffer placement: with a fake NVML that names half of the allowed CPUs as the
    GPU's nearest, the block runs on those and the previous affinity comes back afterwards; when the
    query fails, nothing changes."""
    import types
    before = os.sched_getaffinity(0)
    allowed = sorted(before)
    near = set(allowed[: max(1, len(allowed) // 2)])
    mask = [0] * ((max(allowed) // 64) + 1)
    for c in near:
        mask[c // 64] |= 1 << (c % 64)

    class Props:
        pci_domain_id = pci_bus_id = pci_device_id = 0

    fake_torch = types.SimpleNamespace(cuda=types.SimpleNamespace(get_device_properties=lambda i: Props()))
    fake_nvml = types.SimpleNamespace(nvmlInit=lambda: None, nvmlDeviceGetHandleByPciBusId=lambda bus: "h",
                                      nvmlDeviceGetHandleByIndex=lambda i: "h",
                                      nvmlDeviceGetCpuAffinity=lambda h, n: mask[:n] + [0] * max(0, n - len(mask)))
    monkeypatch.setitem(sys.modules, "pynvml", fake_nvml)
    monkeypatch.setitem(sys.modules, "torch", fake_torch)
    with bench.NearGpu(0) as g:
        inside = os.sched_getaffinity(0)
    assert os.sched_getaffinity(0) == before
    if near != before:
        assert inside == near and "nearest the GPU" in g.describe()

    def broken(*a):
        raise RuntimeError("no NVML")

    fake_nvml.nvmlInit = broken
    with bench.NearGpu(0) as g:
        assert os.sched_getaffinity(0) == before
    assert g.describe() == "process CPU affinity unchanged"
