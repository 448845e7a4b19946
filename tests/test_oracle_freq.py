"""Pins for the oracle's frequency tables: sums, support, the largest-remainder property
(brute-forced as the least-squares apportionment on small alphabets), hand-worked golden
examples, and the single-token rule (every frequency below M)."""
import itertools
import os

import numpy as np

M = 2048
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "freq_example.txt")


def test_golden(oracle):
    lines = [ln for ln in open(GOLDEN) if ln.strip() and not ln.startswith("#")]
    assert len(lines) % 2 == 0 and lines
    for a, b in zip(lines[::2], lines[1::2]):
        counts = [int(t) for t in a.split(":")[1].split()]
        expect = [int(t) for t in b.split(":")[1].split()]
        f, n = oracle.normalize_freqs(counts)
        assert list(f) == expect
        assert n == max(i + 1 for i, c in enumerate(expect) if c)


def test_sum_and_support(oracle):
    rng = np.random.default_rng(0)
    for trial in range(300):
        n = int(rng.integers(2, 200))
        kind = trial % 3
        if kind == 0:
            c = rng.integers(0, 1000, size=n)
        elif kind == 1:  # heavy skew: one dominant token and many singletons
            c = rng.integers(0, 2, size=n)
            c[int(rng.integers(0, n))] = 10 ** 9
        else:  # geometric, like lattice coordinates
            c = (1e7 * 0.7 ** np.arange(n)).astype(np.int64)
        if c.sum() == 0:
            c[0] = 1
        f, length = oracle.normalize_freqs(c)
        assert f.sum() == M and f.max() < M
        if np.count_nonzero(c) == 1:  # the phantom token
            only = int(np.flatnonzero(c)[0])
            phantom = 1 if only == 0 else 0
            assert f[only] == M - 1 and f[phantom] == 1 and np.count_nonzero(f) == 2
            assert length == max(only, phantom) + 1
        else:
            assert np.array_equal(f > 0, c > 0)
            assert length == np.flatnonzero(c).max() + 1


def test_largest_remainder_is_least_squares(oracle):
    """Without zero bumps, largest remainders minimise sum (f_i - c_i M / n)^2 over integer
    vectors with sum M: brute force over the neighbourhood of the exact shares."""
    rng = np.random.default_rng(1)
    for _ in range(200):
        c = rng.integers(1, 5000, size=int(rng.integers(2, 5)))
        q = c * M / c.sum()
        f, _ = oracle.normalize_freqs(c)
        best, arg = None, None
        ranges = [range(int(np.floor(x)) - 1, int(np.floor(x)) + 3) for x in q[:-1]]
        for head in itertools.product(*ranges):
            last = M - sum(head)
            g = np.array(list(head) + [last])
            err = float(((g - q) ** 2).sum())
            if best is None or err < best - 1e-9:
                best, arg = err, g
        assert abs(float(((f - q) ** 2).sum()) - best) < 1e-9, (c, f, arg)
        assert np.all(np.abs(f - q) < 1.0)


def test_single_token_alphabet_rejected(oracle):
    f, n = oracle.normalize_freqs([5])
    assert n == -1
