"""Pins for the oracle's alphabet split rule and for the sampled storage estimate's metadata term,
both recomputed in numpy from the stated readings, not from the oracle's own functions.

The split rule (reading R10 of the conditional model the Abstract of "EntroPack: Fast and
Accurate Entropy-Coded Weight Compression at Arbitrary Bitrates" names but does not define):
each context codes small values directly and larger ones through an escape token; its split m
is the smallest m in [2 + low, max] with at least 99.9 % of the context's values below 2^m,
else max (low = 2, 1, 1, 0, 0, 0, 0 and max = 9, 9, 9, 8, 8, 8, 8 per context).  The values
come from the lattice points v = 2z of each block:
    c = v0 mod 2, y_i = (v_i - c) / 2, p = (y0 + ... + y6) mod 2,
    context 0:          4 zz(a0) + r0   with v0 = 4 a0 + r0, r0 in [0, 4)
    context 1 + c:      2 zz(a) + b     with y_i = 2 a + b, b in {0, 1}       (i = 1..6)
    context 3 + 2c + p: zz((y7 - p) / 2)
with zz(a) = 2a for a >= 0 and -2a - 1 otherwise.

The estimate (reading R22: the resolution comes from storage estimated on a sample, as the
Abstract says): on a tensor of fewer than 65,536 blocks the sample is every block, so the
estimate must equal the stream's exact metadata (header, row factors, scales, frequency
tables, tile directory) plus 168 bytes per tile plus the empirical conditional entropy of the
tokens and their raw extra bits."""
import math

import numpy as np
import pytest

from dit_weight_compression_tile_b200 import synth

BF16, INT8, FP8 = 1, 4, 5
LOW = [2, 1, 1, 0, 0, 0, 0]
MAX_SPLIT = [9, 9, 9, 8, 8, 8, 8]


def zz(a):
    return np.where(a >= 0, 2 * a, -2 * a - 1).astype(np.int64)


def context_values(v):
    """(context, value) of every coordinate of the blocks v (n, 8), from the formulas above"""
    v = v.astype(np.int64)
    c = v[:, 0] & 1
    y = (v - c[:, None]) >> 1                      # exact: v_i - c is even
    p = y[:, :7].sum(axis=1) & 1
    r0 = v[:, 0] & 3
    a0 = (v[:, 0] - r0) >> 2
    vals = np.empty_like(v)
    ctx = np.empty_like(v)
    vals[:, 0] = 4 * zz(a0) + r0
    ctx[:, 0] = 0
    b = y[:, 1:7] & 1
    vals[:, 1:7] = 2 * zz((y[:, 1:7] - b) >> 1) + b
    ctx[:, 1:7] = (1 + c)[:, None]
    vals[:, 7] = zz((y[:, 7] - p) >> 1)
    ctx[:, 7] = 3 + 2 * c + p
    return ctx.reshape(-1), vals.reshape(-1)


def split_rule(values, c):
    """R10: smallest m in [2 + low, max] with >= 99.9 % of the values below 2^m, else max"""
    n = values.size
    if n == 0:
        return 2 + LOW[c]
    for m in range(2 + LOW[c], MAX_SPLIT[c] + 1):
        if np.count_nonzero(values < (1 << m)) * 1000 >= n * 999:
            return m
    return MAX_SPLIT[c]


def tokens(values, m, low):
    """hybrid tokens: s < 2^m is its own token; else n = floor(log2 s) and the token keeps the
    2 bits below the leading one and the `low` lowest bits; n - 2 - low raw bits in between"""
    s = values.astype(np.int64)
    direct = s < (1 << m)
    n = np.zeros_like(s)
    big = ~direct
    n[big] = np.floor(np.log2(s[big].astype(np.float64))).astype(np.int64)
    # guard the float log against rounding at powers of two
    n[big] -= (1 << n[big]) > s[big]
    n[big] += (1 << (n[big] + 1)) <= s[big]
    top = np.where(big, (s >> np.maximum(n - 2, 0)) & 3, 0)
    lo = s & ((1 << low) - 1)
    tok = np.where(direct, s, (1 << m) + (((((n - m) << 2) | top) << low) | lo))
    nbits = np.where(direct, 0, n - 2 - low)
    return tok, nbits


def lattice_blocks(oracle, w, k, container):
    v = oracle.quantize(w, k, container=container)
    return v.reshape(-1, 8)


CASES = [
    # (name, factory, target, container)
    ("lognormal 256x1024 @4", lambda: synth.row_lognormal(256, 1024, seed=21), 4.0, 0),
    ("student-t 192x768 @2.5", lambda: synth.dit_layer(0, 1)[:192, :768].contiguous(), 2.5, 0),
    ("outliers 128x2048 @8", lambda: synth.gaussian_outliers(128, 2048, seed=22), 8.0, 0),
    ("outliers 128x2048 @11", lambda: synth.gaussian_outliers(128, 2048, seed=22), 11.0, 0),
    ("gaussian 128x1024 @0.5", lambda: synth.gaussian(128, 1024, 0.02, seed=23), 0.5, 0),
    ("int8 codes 96x808 @3", lambda: synth.gaussian(96, 808, 0.02, seed=24), 3.0, INT8),
    ("fp8 codes 96x808 @7", lambda: synth.gaussian(96, 808, 0.02, seed=24), 7.0, FP8),
]


@pytest.fixture(scope="module")
def split_cases(oracle):
    out = []
    for name, make, target, container in CASES:
        w = make()
        rc, blob = oracle.compress(w, target, container=container, coding=oracle.CODING_SINGLE)
        assert rc == 0, (name, rc)
        rc, info = oracle.parse(blob)
        assert rc == 0
        v = lattice_blocks(oracle, w, info.q_index, container or BF16)
        ctx, vals = context_values(v)
        out.append((name, info, ctx, vals))
    return out


def test_split_bytes_follow_the_rule(split_cases):
    """the header's seven split bytes are R10 applied to the whole tensor at the chosen resolution"""
    for name, info, ctx, vals in split_cases:
        want = [split_rule(vals[ctx == c], c) for c in range(7)]
        assert list(info.split) == want, name


def test_split_rule_cases_reach_every_branch(split_cases):
    """the cases above exercise the lower bound, the 99.9 % rule strictly inside the range and
    the cap (where fewer than 99.9 % of the values fit even at the largest split)"""
    floor = rule = cap = 0
    for name, info, ctx, vals in split_cases:
        for c in range(7):
            x = vals[ctx == c]
            m = info.split[c]
            if x.size == 0:
                continue
            frac_max = np.count_nonzero(x < (1 << MAX_SPLIT[c])) / x.size
            if m == MAX_SPLIT[c] and frac_max < 0.999:
                cap += 1
            elif m == 2 + LOW[c]:
                floor += 1
            else:
                rule += 1
    assert floor > 0 and rule > 0 and cap > 0, (floor, rule, cap)


@pytest.mark.parametrize("thr", [0.99, 0.9999])
def test_split_rule_threshold_is_decisive(split_cases, thr):
    """a 99 % or 99.99 % threshold would pick other splits on these cases: the pin above tells
    the stated threshold apart from its neighbours"""
    differs = False
    for name, info, ctx, vals in split_cases:
        for c in range(7):
            x = vals[ctx == c]
            if x.size == 0:
                continue
            m_alt = MAX_SPLIT[c]
            for m in range(2 + LOW[c], MAX_SPLIT[c] + 1):
                if np.count_nonzero(x < (1 << m)) >= thr * x.size:
                    m_alt = m
                    break
            differs |= m_alt != info.split[c]
    assert differs


@pytest.mark.parametrize("shape,target,container,K", [((128, 1024), 4.0, 0, 16), ((96, 808), 3.0, INT8, 8),
                                                      ((200, 512), 2.5, 0, 32), ((64, 2048), 6.0, 0, 4)])
def test_estimate_metadata_term(oracle, shape, target, container, K):
    """below 65,536 blocks the estimate is exact metadata + 168 B per tile + empirical conditional
    entropy of the tokens (natural splits of the whole tensor) + raw extra bits"""
    w = synth.row_lognormal(*shape, seed=shape[0] + shape[1])
    rc, blob = oracle.compress(w, target, container=container, blocks_per_lane=K, coding=oracle.CODING_SINGLE)
    assert rc == 0
    rc, info = oracle.parse(blob)
    k = info.q_index
    R, Cc = shape
    nb = R * ((Cc + 7) // 8)
    assert nb < 65536
    v = lattice_blocks(oracle, w, k, container or BF16)
    ctx, vals = context_values(v)
    bits = 0.0
    for c in range(7):
        x = vals[ctx == c]
        m = split_rule(x, c)
        assert m == info.split[c]
        tok, nbits = tokens(x, m, LOW[c])
        _, counts = np.unique(tok, return_counts=True)
        n = counts.sum()
        if n:
            bits += n * math.log2(n) - float(np.sum(counts * np.log2(counts)))
        bits += float(nbits.sum())
    # exact metadata: everything in front of the tile section of the stream coded at k
    meta = info.off_tiles
    tiles = -(-nb // (32 * K))
    assert info.n_tiles == tiles and info.blocks_per_lane == K
    want = 8.0 * (meta + 168.0 * tiles + bits / 8.0) / (R * Cc)
    got = oracle.estimate_bpp(w, k, container=container, blocks_per_lane=K, coding=oracle.CODING_SINGLE)
    assert got == pytest.approx(want, rel=1e-12, abs=1e-12)
    # the per-tile term is told apart from its neighbours
    for other in (160.0, 176.0, 192.0):
        alt = 8.0 * (meta + other * tiles + bits / 8.0) / (R * Cc)
        assert abs(alt - got) > 1e-6
