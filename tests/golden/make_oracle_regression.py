"""Writes oracle_regression.json: a digest of the fp64 oracle's outputs on small seeded workloads.

    python tests/golden/make_oracle_regression.py

This is a regression fixture, not a pin: the oracle is pinned to the pages and to the mathematics
by tests/test_oracle_pins.py.  The digest makes any later change to the oracle's arithmetic (or to
the seeded input generator) visible as a failing test, so that such a change is made on purpose.
Every value here comes from oracle/ alone, on inputs from the seeded generator.
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from draft_block_causal_b200 import synth  # noqa: E402

# logit columns sampled for the digest (taken modulo V)
SAMPLE_COLS = [0, 1, 7, 64, 123, 255, 500, 777, 999, 1024, 1500, 1999]

CASES = {
    "tiny-f32-b1": synth.workload("tiny-f32-b1"),
    "small-bf16-b2": dict(B=2, L=6, d=128, Hs=64, r=32, V=2000, dtype=synth.BF16, weight_seed=200,
                          input_seed=201, s0_std=0.2, peak=2.0, name="small-bf16-b2"),
}


def digest(out: dict, V: int) -> dict:
    lg = out["logits"]
    cols = sorted({c % V for c in SAMPLE_COLS})
    return {
        "tokens": out["tokens"].tolist(),
        "margin": out["margin"].tolist(),
        "logit_sum": lg.sum(axis=-1).tolist(),
        "logit_sumsq": (lg * lg).sum(axis=-1).tolist(),
        "logit_cols": cols,
        "logit_samples": lg[:, :, cols].tolist(),
        "state_sum": out["states"].sum(axis=-1).tolist(),
        "states_last_position": out["states"][:, -1, :].tolist(),
    }


def compute() -> dict:
    res = {}
    for name, wl in CASES.items():
        data = synth.make_workload(wl, with_tokens=True, with_target=True)
        sh = data["shape"]
        args = (sh, data["weights"], data["base_logits"], data["hidden"], data["S0"])
        greedy = oracle.head(*args)
        tf = oracle.head(*args, tokens=data["tokens"])
        acc = oracle.accept_len(greedy["tokens"], data["target_logits"])
        res[name] = {"workload": {k: wl[k] for k in ("B", "L", "d", "Hs", "r", "V", "dtype", "weight_seed",
                                                     "input_seed", "s0_std", "peak")},
                     "greedy": digest(greedy, sh["V"]), "teacher_forced": digest(tf, sh["V"]),
                     "accept_len_of_greedy_tokens": acc.tolist()}
    return res


if __name__ == "__main__":
    out = {"note": "digest of the fp64 oracle on seeded workloads; written by make_oracle_regression.py",
           "cases": compute()}
    with open(os.path.join(HERE, "oracle_regression.json"), "w") as f:
        f.write(json.dumps(out, separators=(",", ":")).replace(',"', ',\n"') + "\n")
