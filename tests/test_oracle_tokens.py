"""Pins for the symbol layer of the oracle: zigzag, the hybrid-integer tokens, the
conditional contexts and the resolution grid.  Checked by exhaustive round trips and by
counting properties that any correct binarization must have, not by retyping it."""
import numpy as np
import pytest


def test_zigzag_bijection(oracle):
    ys = list(range(-3000, 3001)) + [-(1 << 21), (1 << 21) - 1, 123456, -654321]
    us = [oracle.zigzag(y) for y in ys]
    assert len(set(us)) == len(us)
    assert all(oracle.unzigzag(u) == y for u, y in zip(us, ys))
    # small magnitudes get small codes: 0, -1, 1, -2, 2, ...
    assert [oracle.unzigzag(u) for u in range(7)] == [0, -1, 1, -2, 2, -3, 3]


@pytest.mark.parametrize("m", range(8))
def test_tokens_exhaustive(oracle, m):
    u = np.arange(1 << 22, dtype=np.uint32)
    tok, nbits, extra = oracle.tokenize(u, m)
    # exact inverse
    assert np.array_equal(oracle.detokenize_batch(tok, m, extra), u)
    # values below 2^m are their own token, with no extra bits
    assert np.array_equal(tok[: 1 << m], u[: 1 << m])
    assert not nbits[: 1 << m].any()
    # tokens are non-decreasing in u, and each token covers a contiguous run of 2^nbits values
    assert np.all(np.diff(tok.astype(np.int64)) >= 0)
    starts = np.flatnonzero(np.diff(tok.astype(np.int64))) + 1
    runs = np.diff(np.concatenate([[0], starts, [u.size]]))
    first = np.concatenate([[0], starts])
    assert np.array_equal(runs, 1 << nbits[first].astype(np.int64))
    assert np.all(extra < (1 << nbits.astype(np.int64)))
    # the alphabet stays within 8-bit tokens for every split
    assert tok.max() < 256
    # tokens are dense: every token index below the maximum is used
    assert np.unique(tok).size == tok.max() + 1


def test_resolution_grid(oracle):
    qs = np.array([oracle.q_of_k(k) for k in range(1280)])
    assert np.all(np.diff(qs) > 0)
    assert qs[0] == 2.0 ** -8 and qs[-1] < 2.0 ** 12
    # exact in fp32 (the grid value reaches the decoder only through f_r, but the encoder's
    # row factor must not depend on double-rounding of q)
    assert np.array_equal(qs.astype(np.float32).astype(np.float64), qs)
    # relative step between 1/128 and 1/64
    rel = np.diff(qs) / qs[:-1]
    assert rel.max() <= 1 / 64 + 1e-15 and rel.min() >= 1 / 128 - 1e-15
    # k_max keeps |v| below 2^21: sqrt(C) q (+1 for the rounding) <= 2^20
    for cols in (8, 256, 3072, 28672, 1 << 20):
        k = oracle.k_max(cols)
        assert oracle.q_of_k(k) * (np.sqrt(cols) + 1) <= 2 ** 20
        assert k == 1279 or oracle.q_of_k(k + 1) * (np.sqrt(cols) + 1) > 2 ** 20


def test_blocks_per_lane_rule(oracle):
    """tiles near 2048 for mid-size matrices, at most 256 blocks per lane, and a tile's
    expected payload (32 K x 8 coordinates x target bits, +10%) within 5952 bytes"""
    assert oracle.blocks_per_lane(1, 4.0) == 16
    assert oracle.blocks_per_lane(2 ** 20, 4.0) == 16
    assert oracle.blocks_per_lane(4096 * 4096 // 8, 4.0) == 32
    assert oracle.blocks_per_lane(8192 * 28672 // 8, 0.5) == 256
    assert oracle.blocks_per_lane(8192 * 28672 // 8, 4.0) == 32
    assert oracle.blocks_per_lane(8192 * 28672 // 8, 8.0) == 16
    assert oracle.blocks_per_lane(10 ** 12, 11.0) == 8
    for nb in (10, 10 ** 5, 10 ** 7, 10 ** 9):
        for t in (0.001, 0.5, 2.0, 4.0, 8.0, 11.0):
            k = oracle.blocks_per_lane(nb, t)
            assert k & (k - 1) == 0 and 1 <= k <= 256
            assert k == 1 or 32 * k * t * 1.1 <= 5952
