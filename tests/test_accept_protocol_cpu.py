"""A model of the accept-length kernel's concurrency protocol (k_accept_early), run on the CPU.

The kernel has one block per (row b, position j, column chunk c), issued position-major. Each block:
  1. reads its row's first-mismatch word f[b] (stored as L - j, 0 = none) and skips its reads when
     f[b] > L - j, i.e. when a mismatch before j has been recorded;
  2. otherwise folds its chunk's argmax key into key[b, j] (atomicMax);
  3. counts itself done for (b, j) (atomicAdd); the block that completes the count
  4. compares the finished argmax with the draft token and, on a mismatch, does f[b] = max(f[b], L - j).
The last block of the grid writes accept[b] = L - f[b].

The claim is that the result never depends on scheduling: a position can only be skipped once an
earlier mismatch of its row is recorded, and that earlier mismatch then wins the max. This test
interleaves the four steps of many blocks at random (with ties in the logits) and checks the
outcome against the plain definition: the number of leading positions whose draft token equals
the lowest-index argmax of the target row.
"""
import random

import numpy as np


def _model(T, draft, chunk, rng):
    B, L, V = T.shape
    nch = -(-V // chunk)
    keys, count, first = {}, {}, [0] * B

    def block(c, y):
        j, b = y // B, y % B
        skip = first[b] > L - j
        yield
        if not skip:
            lo, hi = c * chunk, min(V, c * chunk + chunk)
            best = max((T[b, j, v], -v) for v in range(lo, hi))  # larger value, then lower index
            keys[(b, j)] = max(keys.get((b, j), (-np.inf, 0)), best)
        yield
        count[(b, j)] = count.get((b, j), 0) + 1
        last = count[(b, j)] == nch
        yield
        if last and draft[b, j] != -keys.get((b, j), (-np.inf, 0))[1]:
            first[b] = max(first[b], L - j)
        yield

    pending = [block(c, y) for y in range(B * L) for c in range(nch)]  # issue order: position-major
    running = []
    while pending or running:
        while pending and len(running) < rng.randint(1, 12):  # a varying number of resident blocks
            running.append(pending.pop(0))
        g = rng.choice(running)
        try:
            next(g)
        except StopIteration:
            running.remove(g)
    return [L - f for f in first]


def _plain(T, draft):
    out = []
    for b in range(T.shape[0]):
        k = 0
        while k < T.shape[1] and draft[b, k] == int(np.argmax(T[b, k])):  # numpy: first maximal index
            k += 1
        out.append(k)
    return out


def test_early_exit_protocol_matches_the_definition_under_random_interleavings():
    rng = random.Random(7)
    nrng = np.random.default_rng(8)
    for _ in range(1500):
        B, L = rng.randint(1, 4), rng.randint(1, 6)
        V, chunk = rng.choice([8, 16, 24, 40]), rng.choice([8, 16])
        T = nrng.integers(0, 4, size=(B, L, V)).astype(np.float64)  # few levels: many exact ties
        am = T.argmax(-1)
        draft = am.copy()
        for b in range(B):
            m = rng.randint(0, L)  # first mismatch, or none when m == L
            if m < L:
                draft[b, m] = (am[b, m] + rng.randint(1, V - 1)) % V
            for j in range(m + 1, L):
                if rng.random() < 0.5:
                    draft[b, j] = rng.randint(0, V - 1)
        assert _model(T, draft, chunk, rng) == _plain(T, draft)
