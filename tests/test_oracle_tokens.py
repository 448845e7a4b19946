"""Pins for the symbol layer of the oracle: zigzag, the hybrid-integer tokens (with the
value's low bits kept in the token), the conditional contexts and the resolution grid.  Checked by exhaustive round trips and by
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


SPLITS = [(m, low) for low in (0, 1, 2) for m in range(2 + low, 10)]


@pytest.mark.parametrize("m,low", SPLITS)
def test_tokens_exhaustive(oracle, m, low):
    s = np.arange(1 << 22, dtype=np.uint32)
    tok, nbits, extra = oracle.tokenize(s, m, low)
    # exact inverse
    assert np.array_equal(oracle.detokenize_batch(tok, m, low, extra), s)
    # values below 2^m are their own token, with no extra bits
    assert np.array_equal(tok[: 1 << m], s[: 1 << m])
    assert not nbits[: 1 << m].any()
    # the token keeps the value's `low` low bits, whatever the extra bits
    assert np.array_equal(tok & ((1 << low) - 1), s & ((1 << low) - 1))
    # every token owns the values {base + (e << low) : e < 2^nbits}: a token and its extra bits
    # name one value, and the values of a token differ only in the raw bits
    assert np.all(extra < (1 << nbits.astype(np.int64)))
    base = oracle.detokenize_batch(tok, m, low, np.zeros_like(extra))
    assert np.array_equal(base + (extra.astype(np.int64) << low), s)
    # tokens increase with the value's magnitude class: non-decreasing in floor(log2 s)
    top = s >= (1 << m)
    n = np.floor(np.log2(np.maximum(s, 1))).astype(np.int64)
    order = np.lexsort((tok[top], n[top]))
    assert np.all(np.diff(tok[top][order].astype(np.int64)) >= 0)
    # an escape token names n, the two bits below the leading one and the low bits
    esc = tok[top].astype(np.int64) - (1 << m)
    assert np.array_equal(n[top] - m, (esc >> low) >> 2)
    assert np.array_equal(nbits[top].astype(np.int64), n[top] - 2 - low)
    # the alphabet is dense and its size is the documented count
    assert np.unique(tok).size == tok.max() + 1 == oracle.alphabet_size(m, low)


def test_block_symbols_roundtrip(oracle):
    """every E8 point v = 2z in a box round trips through the coded values; the contexts
    follow the coset and the parity of y_0..y_6; the values' low bits carry them"""
    rng = np.random.default_rng(0)
    pts = []
    for _ in range(4000):
        c = int(rng.integers(0, 2))
        y = rng.integers(-300, 300, size=8)
        y[7] += (int(y[:7].sum()) - int(y[7])) % 2  # sum of y even: z in D8 (+ 1/2)
        pts.append(2 * y + c)
    pts += [np.zeros(8, np.int64), np.full(8, 1), np.array([-1] * 8), np.array([2, 0, 0, 0, 0, 0, 0, 2]),
            np.array([-(1 << 20) + 1] + [1] * 6 + [5])]
    for v in pts:
        v = np.asarray(v, np.int32)
        assert int(v.sum()) % 4 == 0 and len(set(int(x) & 1 for x in v)) == 1
        ctx, s = oracle.block_symbols(v)
        v2, ctx2 = oracle.block_values(s)
        assert np.array_equal(v2, v) and np.array_equal(ctx2, ctx)
        c = int(v[0]) & 1
        y = (v.astype(np.int64) - c) // 2
        p = int(y[:7].sum()) & 1
        assert list(ctx) == [0] + [1 + c] * 6 + [3 + 2 * c + p]
        assert int(s[0]) & 3 == int(v[0]) & 3
        assert all(int(s[i]) & 1 == int(y[i]) & 1 for i in range(1, 7))
        assert all(int(x) < (1 << 22) for x in s)


def test_direct_tokens_fit_decoder_field(oracle):
    """at the largest split of each context every direct token names a coordinate 0 with
    -256 <= v0 <= 255, and for coordinates 1..7 a y = (v - c) / 2 with -256 <= y <= 255 (the
    decoder's 9-bit value field); with the splits of the narrow range (8 for coordinates 1..6,
    7 for coordinate 7) the coordinates themselves stay within -256 <= v <= 255"""
    for ctx_kind, (low, mmax) in enumerate([(2, 9), (1, 9), (0, 8)]):
        vals = []
        for s in range(1 << mmax):
            if ctx_kind == 0:
                vals.append(4 * oracle.unzigzag(s >> 2) + (s & 3))
            elif ctx_kind == 1:
                vals.append(2 * oracle.unzigzag(s >> 1) + (s & 1))
            else:
                for p in (0, 1):
                    vals.append(2 * oracle.unzigzag(s) + p)
        assert min(vals) >= -256 and max(vals) <= 255
    for ctx_kind, mmax in ((1, 8), (2, 7)):
        vals = []
        for s in range(1 << mmax):
            for c in (0, 1):
                if ctx_kind == 1:
                    vals.append(2 * (2 * oracle.unzigzag(s >> 1) + (s & 1)) + c)
                else:
                    for p in (0, 1):
                        vals.append(2 * (2 * oracle.unzigzag(s) + p) + c)
        assert min(vals) >= -256 and max(vals) <= 255
    assert oracle.CTX_LOW == (2, 1, 1, 0, 0, 0, 0) and oracle.CTX_MAX_SPLIT == (9, 9, 9, 8, 8, 8, 8)


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
