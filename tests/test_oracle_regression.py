"""The fp64 oracle against its stored digest (tests/golden/oracle_regression.json, written by
tests/golden/make_oracle_regression.py from the oracle alone).

Not a pin to the pages -- those are in test_oracle_pins.py -- but a guard: a change to the oracle's
arithmetic or to the seeded inputs fails here until the digest is rewritten on purpose.  Integers
(tokens, accept lengths) must match exactly; floating-point values to 1e-12 relative (libm's exp
and tanh may differ in the last place between C libraries)."""
import json
import os

import numpy as np
import pytest

from tests.golden import make_oracle_regression as gen

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def stored_and_now():
    with open(os.path.join(HERE, "golden", "oracle_regression.json")) as f:
        stored = json.load(f)["cases"]
    return stored, gen.compute()


@pytest.mark.parametrize("case", sorted(gen.CASES))
def test_oracle_matches_its_stored_digest(stored_and_now, case):
    stored, now = stored_and_now
    s, n = stored[case], now[case]
    assert s["workload"] == n["workload"]
    assert s["accept_len_of_greedy_tokens"] == n["accept_len_of_greedy_tokens"]
    for mode in ("greedy", "teacher_forced"):
        a, b = s[mode], n[mode]
        assert a["tokens"] == b["tokens"], mode
        assert a["logit_cols"] == b["logit_cols"], mode
        for key in ("margin", "logit_sum", "logit_sumsq", "logit_samples", "state_sum", "states_last_position"):
            np.testing.assert_allclose(np.asarray(b[key]), np.asarray(a[key]), rtol=1e-12, atol=1e-12,
                                       err_msg=f"{case} {mode} {key}")
