"""Pin of the oracle's pair-table rule (paired coding) against hand-worked examples
(tests/golden/pair_table_example.txt): the pair base, the rare-pair and outside-the-base escapes,
and the normalisation to 2^12."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pair_table_example.txt")


def examples():
    cases, cur = [], {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, _, val = line.partition(":")
        cur[key.strip()] = val.strip()
        if key.startswith("freqs"):
            cases.append(cur)
            cur = {}
    return cases


def dense(spec, n):
    out = np.zeros(n, np.int64)
    for item in spec.split():
        i, v = item.split(":")
        out[int(i)] = int(v)
    return out


def test_pair_table_examples(oracle):
    cases = examples()
    assert len(cases) == 3
    for c in cases:
        A, N = int(c["A"]), int(c["N"])
        B = min(A, 40)
        if "inside" in c:
            inside = np.array([int(x) for x in c["inside"].split()], np.uint64)
            rare = np.array([int(x) for x in c["rare"].split()], np.uint8)
            freqs = np.array([int(x) for x in c["freqs"].split()], np.uint32)
        else:
            inside = dense(c["inside_sparse"], B * B).astype(np.uint64)
            rare = dense(c["rare_sparse"], B * B).astype(np.uint8)
            freqs = dense(c["freqs_sparse"], B * B + 1).astype(np.uint32)
        f, r = oracle.pair_table(inside, A, N)
        assert np.array_equal(f, freqs), (A, f[np.nonzero(f)])
        assert np.array_equal(r, rare)
        assert int(f.sum()) == 4096
