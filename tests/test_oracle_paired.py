"""Pins for the oracle's paired coding of coordinates 1..6 (three pair symbols per block, pair
tables of base B = min(A, 40) summing to 2^12, rare pairs and pairs outside the base escaped to
raw bits): exact round trips, the same lattice
points as single-token coding at the same resolution, the automatic choice, the escape rule
recomputed from the quantizer's points, the code length, the closed-form distortion and
damaged or malformed streams."""
import math
import struct

import numpy as np
import pytest
import torch

from dit_weight_compression_tile_b200 import synth

BF16, INT8, FP8 = 1, 4, 5
G_E8 = 929.0 / 12960.0


def zz(y):
    return np.where(y >= 0, 2 * y, -2 * y - 1).astype(np.int64)


def compress(oracle, w, target, coding, container=0, q=-1, K=0):
    rc, blob = oracle.compress(w, target, container=container, blocks_per_lane=K, q_override=q, coding=coding)
    assert rc == 0, rc
    rc, info = oracle.parse(blob)
    assert rc == 0
    return blob, info


@pytest.mark.parametrize("shape,target,container,K", [((64, 512), 4.0, 0, 0), ((300, 1000), 3.0, 0, 0),
                                                      ((137, 455), 3.5, 0, 3), ((128, 1024), 2.0, 0, 8),
                                                      ((96, 808), 4.0, INT8, 0), ((96, 808), 3.0, FP8, 0),
                                                      ((256, 256), 1.0, 0, 0)])
def test_paired_roundtrip(oracle, shape, target, container, K):
    w = synth.row_lognormal(*shape, seed=shape[1] + int(10 * target))
    blob, info = compress(oracle, w, target, oracle.CODING_PAIRED, container, K=K)
    assert info.paired == 1 and blob[43] == 1
    assert info.actual_bpp <= target
    rc, st, v, out = oracle.decode(blob)
    assert rc == 0 and st == 0
    assert np.array_equal(v, oracle.quantize(w, info.q_index, container=container or BF16))


def test_paired_and_single_give_the_same_points(oracle):
    w = synth.gaussian_outliers(200, 1024, seed=4)
    a, ia = compress(oracle, w, 3.0, oracle.CODING_PAIRED)
    q = ia.q_index
    b, ib = compress(oracle, w, 3.0, oracle.CODING_SINGLE, q=q)
    assert ia.paired == 1 and ib.paired == 0 and a[43] == 1 and b[43] == 0
    ra, sa, va, oa = oracle.decode(a)
    rb, sb, vb, ob = oracle.decode(b)
    assert sa == 0 and sb == 0
    assert np.array_equal(va, vb) and np.array_equal(oa, ob)
    assert np.array_equal(va, oracle.quantize(w, q))


def test_automatic_choice(oracle):
    """automatic coding pairs from 2^17 blocks on, when the tokens of contexts 1 and 2 concentrate
    below the base 40"""
    big = synth.row_lognormal(1024, 1024, seed=1)        # 131072 blocks
    small = synth.row_lognormal(1024, 1016, seed=1)      # 130048 blocks
    b1, i1 = compress(oracle, big, 4.0, oracle.CODING_AUTO)
    b2, i2 = compress(oracle, small, 4.0, oracle.CODING_AUTO)
    assert i1.paired == 1 and i2.paired == 0
    b3, i3 = compress(oracle, big, 8.0, oracle.CODING_AUTO)   # most tokens far beyond 40
    assert i3.paired == 0 and i3.ntok[1] > 40
    b4, i4 = compress(oracle, big, 8.0, oracle.CODING_PAIRED)  # asked for, but not possible
    assert i4.paired == 0
    for blob, info in ((b1, i1), (b3, i3)):
        rc, st, v, _ = oracle.decode(blob)
        assert st == 0 and np.array_equal(v, oracle.quantize(big, info.q_index))


def expected_escapes(oracle, v, info):
    """escaped pairs and token extra bits recomputed from the lattice points: a pair (t_a, t_b) of
    context c is escaped when a token is at or above B = min(A, 40) or when it is seen fewer than
    N_c / 2^16 times"""
    vb = v.reshape(-1, 8).astype(np.int64) if v.shape[1] % 8 == 0 else None
    assert vb is not None
    c = vb[:, 0] & 1
    y = (vb - c[:, None]) >> 1
    p = y[:, 1:7] & 1
    s16 = 2 * zz((y[:, 1:7] - p) // 2) + p
    escaped, rawbits = 0, 0
    for cc in (0, 1):
        m = int(info.split[1 + cc])
        A = int(info.ntok[1 + cc])
        sel = s16[c == cc]
        if sel.size == 0:
            continue
        tok, _, _ = oracle.tokenize(sel.reshape(-1).astype(np.uint32), m, 1)
        tok = tok.reshape(-1, 6).astype(np.int64)
        assert tok.max() < A
        Bb = min(A, 40)
        ta, tb = tok[:, 0::2].reshape(-1), tok[:, 1::2].reshape(-1)
        inside = (ta < Bb) & (tb < Bb)
        cnt = np.bincount((ta * Bb + tb)[inside], minlength=Bb * Bb)
        rare = (cnt > 0) & (cnt * 65536 < ta.size)
        e = int(cnt[rare].sum()) + int((~inside).sum())
        escaped += e
        rawbits += 2 * e * int(A - 1).bit_length()
    # extra bits of escape tokens, every coordinate with its own context's split
    extra = 0
    flat_ctx = np.zeros(vb.shape, np.uint32)
    flat_s = np.zeros(vb.shape, np.uint32)
    for b in range(vb.shape[0]):
        flat_ctx[b], flat_s[b] = oracle.block_symbols(vb[b])
    for cx in range(7):
        sel = flat_s[flat_ctx == cx]
        if sel.size:
            _, nb, _ = oracle.tokenize(sel, int(info.split[cx]), (2, 1, 1, 0, 0, 0, 0)[cx])
            extra += int(nb.sum())
    return escaped, rawbits, extra


ESCAPE_CASES = [  # (seed, target, outlier fraction, outlier size in sigmas)
    (2, 3.5, 0.001, 8.0), (3, 3.0, 0.001, 8.0),
    (5, 3.5, 0.0002, 40.0),  # sparse large spikes: tokens beyond the pair base B = 40
]


@pytest.mark.parametrize("seed,target,frac,sigmas", ESCAPE_CASES)
def test_escape_rule_and_symbol_count(oracle, seed, target, frac, sigmas):
    """rare pairs and pairs with a token beyond the base are escaped"""
    w = synth.gaussian_outliers(512, 2048, seed=seed, frac=frac, sigmas=sigmas)
    blob, info = compress(oracle, w, target, oracle.CODING_PAIRED)
    assert info.paired == 1
    if sigmas > 10:
        assert info.ntok[1] > 40 or info.ntok[2] > 40
    rc, st, v, _ = oracle.decode(blob)
    assert st == 0
    escaped, rawbits, extra = expected_escapes(oracle, v, info)
    assert escaped > 0  # the case exercises the escape path
    rc, cs = oracle.code_stats(blob)
    assert rc == 0
    nb = v.size // 8
    assert cs["n_symbols"] == 5 * nb
    assert cs["extra_bits"] == rawbits + extra
    # the escape symbol (last entry of each pair table) has a frequency exactly when used
    b = blob.tobytes()
    q = info.off_freq + 2 * info.ntok[0]
    for cc in (1, 2):
        Bb = min(info.ntok[cc], 40)
        tab = np.frombuffer(b, np.uint16, Bb * Bb + 1, q)
        assert int(tab.sum()) == 4096 and tab.max() < 4096
        q += 2 * (Bb * Bb + 1)


def test_paired_code_length(oracle):
    """words + final states carry the symbols' information (pair symbols at 2^-12 precision)"""
    w = synth.row_lognormal(256, 1024, seed=5)
    blob, info = compress(oracle, w, 4.0, oracle.CODING_PAIRED)
    rc, cs = oracle.code_stats(blob)
    assert rc == 0
    info_bits = cs["ideal_bits"] + cs["extra_bits"]
    b = blob.tobytes()
    st = []
    for t in range(info.n_tiles):
        off = info.off_tiles + 16 * struct.unpack_from("<I", b, info.off_dir + 4 * t)[0]
        st.extend(struct.unpack_from("<32I", b, off))
    st = np.array(st, np.float64)
    state_bits = float(np.log2(st).sum() - 16.0 * st.size)
    hi = 8.0 * cs["payload_bytes"] + state_bits
    lo = hi - 16 * 8 * info.n_tiles
    assert lo <= info_bits + 1e-3 * cs["n_symbols"]
    assert hi >= info_bits - 1.0
    kl = (cs["ideal_bits"] - cs["entropy_bits"]) / cs["n_symbols"]
    assert 0.0 <= kl < 0.05


@pytest.mark.parametrize("target", [3.0, 4.0])
def test_paired_rate_distortion_closed_form(oracle, target):
    w = synth.gaussian(512, 1024, 0.02, seed=8, dtype=torch.float32)
    blob, info = compress(oracle, w, target, oracle.CODING_PAIRED)
    assert info.paired == 1
    rc, st, v, out = oracle.decode(blob)
    rc, cs = oracle.code_stats(blob)
    r_payload = (cs["ideal_bits"] + cs["extra_bits"]) / w.numel()
    pred = math.sqrt(G_E8 * 2 * math.pi * math.e) * 2.0 ** (-r_payload)
    wf = w.numpy()
    rel = np.linalg.norm(wf - out) / np.linalg.norm(wf)
    assert 1.0 <= rel / pred < 1.15, (rel, pred, r_payload)


def test_pair_table_normalisation(oracle):
    rng = np.random.default_rng(3)
    for _ in range(20):
        n = int(rng.integers(2, 1602))
        counts = np.where(rng.random(n) < 0.3, 0, rng.integers(0, 10**6, n)).astype(np.uint64)
        counts[int(rng.integers(0, n))] += 1
        f, ln = oracle.normalize_freqs(counts, bits=12)
        assert int(f.sum()) == 4096 and f.max() < 4096
        assert np.array_equal(f[: n] > 0, counts > 0) or (counts > 0).sum() == 1
    f, ln = oracle.normalize_freqs(np.array([0, 0, 5, 0], np.uint64), bits=12)
    assert list(f) == [1, 0, 4095, 0]


def test_malformed_paired_streams_rejected(oracle):
    w = synth.row_lognormal(64, 512, seed=9)
    blob, info = compress(oracle, w, 4.0, oracle.CODING_PAIRED)
    bad = blob.copy()
    bad[43] = 2
    assert oracle.parse(bad)[0] == oracle.ERR_CORRUPT
    bad = blob.copy()
    bad[36 + 3] = 8  # a split beyond the narrow range is not allowed with pairs
    assert oracle.parse(bad)[0] == oracle.ERR_CORRUPT
    bad = blob.copy()
    q = info.off_freq + 2 * info.ntok[0]
    bad[q] ^= 1  # the first pair table no longer sums to 2^12
    assert oracle.parse(bad)[0] == oracle.ERR_CORRUPT
    bad = blob.copy()
    bad[43] = 0  # read as single coding, the tables no longer fit their lengths
    assert oracle.parse(bad)[0] == oracle.ERR_CORRUPT


def test_damaged_paired_tile_detected(oracle):
    w = synth.row_lognormal(64, 1024, seed=10)
    blob, info = compress(oracle, w, 4.0, oracle.CODING_PAIRED)
    rc, st, v0, _ = oracle.decode(blob)
    seen = 0
    for off in (info.off_tiles + 200, info.off_tiles + 700, blob.size - 40):
        bad = blob.copy()
        bad[off] ^= 0x24
        rc, st, v, _ = oracle.decode(bad)
        seen += int(st != 0 or not np.array_equal(v, v0))
        assert st != 0 or not np.array_equal(v, v0)
    assert seen == 3
