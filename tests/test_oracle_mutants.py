"""The oracle's pins catch plausible mistakes: each mutant below is the oracle's C source with one
planted error (a sign, a gate, a bias, an index, an operand order, the tie rule, the accept count,
the sampled-verification rule's clamp, ratio, draw, temperature and residual),
built into a separate library on the CPU; at least one pin of tests/test_oracle_pins.py must fail
on it.  The oracle itself is never modified."""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins
from tests import test_oracle_sampling_pins as spins

SRC = os.path.join(os.path.dirname(oracle.__file__), "domino_oracle.c")

# (name, text in the oracle, planted replacement)
MUTANTS = [
    ("update gate sign", "double z = sigmoid(gi[1] + gh[1]);", "double z = sigmoid(gi[1] - gh[1]);"),
    ("reset gate row", "double r = sigmoid(gi[0] + gh[0]);", "double r = sigmoid(gi[1] + gh[1]);"),
    ("reset applied to the input half", "double n = tanh(gi[2] + r * gh[2]);", "double n = tanh(r * (gi[2] + gh[2]));"),
    ("update mix swapped", "h_out[j] = (1.0 - z) * n + z * h[j];", "h_out[j] = z * n + (1.0 - z) * h[j];"),
    ("hidden bias dropped", "double sh = elem(b_hh, row, dtype);", "double sh = 0.0;"),
    ("sigmoid for SiLU", "u[k] = silu(a);", "u[k] = sigmoid(a);"),
    ("state block at the wrong W1 column", "elem(W1, (size_t)k * W1cols + d + j, dt) * S[j]",
     "elem(W1, (size_t)k * W1cols + j, dt) * S[j]"),
    ("W2 transposed", "elem(W2, (size_t)v * r + q, dt)", "elem(W2, (size_t)q * V + v, dt)"),
    ("highest index on ties", "if (z[w] > z[best]) best = w;", "if (z[w] >= z[best]) best = w;"),
    ("embedding of the argmax under teacher forcing", "elem(embed, (size_t)t * d + c, dt)",
     "elem(embed, (size_t)best * d + c, dt)"),
    ("accept length counts a bonus token", "      k = j + 1;", "      k = j + 2;"),
    ("hidden state of the next position", "elem(hidden, pos * d + c, dt)",
     "elem(hidden, (pos + (i + 1 < L)) * d + c, dt)"),
    # sampled verification
    ("residual not clamped at zero", "res[v] = r > 0.0 ? r : 0.0;", "res[v] = r;"),
    ("acceptance ratio inverted", "const double ratio = p[x] / (q ? q[x] : 1.0);",
     "const double ratio = (q ? q[x] : 1.0) / p[x];"),
    ("resampled with the position's acceptance draw",
     "const double target = (double)uniforms[(size_t)b * (L + 1) + L] * z;",
     "const double target = (double)uniforms[(size_t)b * (L + 1) + j] * z;"),
    ("temperature ignored", "out[v] = exp(((double)t[v] - m) / T);", "out[v] = exp(((double)t[v] - m));"),
    ("replacement drawn from the target instead of the residual",
     "const double qv = q ? q[v] : (v == x ? 1.0 : 0.0);", "const double qv = 0.0 * (q ? q[v] : (double)x);"),
]

PIN_CALLS = [
    pins.test_hand_example_two_positions_v5,
    pins.test_gru_step_matches_torch_grucell,
    pins.test_teacher_forced_states_follow_grucell_sequence,
    pins.test_w2_zero_gives_base_logits_exactly_and_lowest_index_ties,
    pins.test_zero_gru_halves_the_state_each_step,
    pins.test_adding_a_constant_per_position_shifts_logits_and_keeps_tokens,
    pins.test_teacher_forcing_is_causal,
    lambda: pins.test_greedy_equals_teacher_forcing_on_its_own_tokens(0),
    lambda: pins.test_greedy_is_the_unique_fixed_point_of_teacher_forcing(21),
    pins.test_accept_len_matches_numpy_first_argmax,
    pins.test_accept_len_hand_cases,
    spins.test_identical_distributions_accept_every_position,
    spins.test_token_outside_the_target_support_is_rejected_and_replaced_from_it,
    lambda: spins.test_lossless_for_a_sampled_draft_on_five_tokens(0.5),
    lambda: spins.test_lossless_for_a_greedy_draft_on_five_tokens(2),
    spins.test_low_temperature_is_the_greedy_accept_rule,
]


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name!r} not found exactly once"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared",
                    "-fPIC", "-o", str(lib), str(path), "-lm"], check=True)
    return str(lib)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_every_planted_mistake_fails_a_pin(tmp_path, name, old, new):
    mutant = oracle.configure(ctypes.CDLL(_build_mutant(tmp_path, name, old, new)))
    oracle._load()
    saved = oracle._lib
    oracle._lib = mutant
    caught = None
    try:
        for call in PIN_CALLS:
            try:
                call()
            except AssertionError:
                caught = call
                break
    finally:
        oracle._lib = saved
    assert caught is not None, f"no pin catches the mutant {name!r}"
