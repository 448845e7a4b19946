"""Pins for the oracle's second block order (reading R32): tiles that are the operand tiles of a
consumer GEMM, 128 output rows by 64 input columns, lane l taking row 32 (k mod 4) + l of the tile
at column block k / 4 ("EntroPack API reference", CompressedLinear: the weight is decoded for every
forward call; the order lets a decode feed a GEMM's K loop tile by tile).

Pinned from outside the oracle: the same resolution, lattice points and weights as the row order
(a block order cannot change what is coded, only where); one tile decoded alone writes exactly its
128 x 64 region (a sentinel-filled output shows which elements it touched); and every lane's coded
length matches the information content of exactly the blocks R32 gives it, recomputed in numpy
from the quantizer's points, the stated value formulas and the stream's own frequency tables."""
import math
import struct

import numpy as np
import pytest

from dit_weight_compression_tile_b200 import synth

from test_oracle_split import LOW, context_values, tokens


def compress(oracle, w, target, layout, coding=0):
    # the row order at the GEMM order's tile size (32 blocks per lane), so that both have the same tiles
    rc, blob = oracle.compress(w, target, coding=coding, layout=layout, blocks_per_lane=32)
    assert rc == 0, rc
    rc, info = oracle.parse(blob)
    assert rc == 0
    return blob, info


@pytest.mark.parametrize("shape,target,coding", [((256, 512), 4.0, 1), ((384, 1024), 3.0, 2), ((128, 192), 5.0, 1)])
def test_same_points_as_row_order(oracle, shape, target, coding):
    w = synth.row_lognormal(*shape, seed=shape[1])
    b0, i0 = compress(oracle, w, target, 0, coding)
    b1, i1 = compress(oracle, w, target, 1, coding)
    assert i1.layout == 1 and b1[58] == 1 and i1.blocks_per_lane == 32
    assert i1.q_index == i0.q_index and i1.n_tiles == i0.n_tiles
    rc0, st0, v0, o0 = oracle.decode(b0)
    rc1, st1, v1, o1 = oracle.decode(b1)
    assert st0 == st1 == 0
    assert np.array_equal(v1, oracle.quantize(w, i1.q_index)) and np.array_equal(v0, v1) and np.array_equal(o0, o1)
    assert i1.actual_bpp <= target


def test_layout_needs_whole_operand_tiles(oracle):
    w = synth.gaussian(128, 64 * 3, 0.02, seed=2)
    for bad in (synth.gaussian(100, 128, 0.02, seed=3), synth.gaussian(128, 100, 0.02, seed=4)):
        rc, _ = oracle.compress(bad, 4.0, layout=1)
        assert rc == oracle.ERR_INVALID_ARG
    rc, _ = oracle.compress(w, 4.0, blocks_per_lane=16, layout=1)
    assert rc == oracle.ERR_INVALID_ARG
    rc, blob = oracle.compress(w, 4.0, layout=1)
    assert rc == 0
    for byte, val in ((58, 2), (28, 16)):  # an unknown layout; a tile size other than 32
        bad = blob.copy()
        bad[byte] = val
        assert oracle.parse(bad)[0] == oracle.ERR_CORRUPT


def test_each_tile_is_one_operand_tile(oracle):
    w = synth.row_lognormal(256, 384, seed=5)
    blob, info = compress(oracle, w, 4.0, 1)
    kt = 384 // 64
    rc, st, v, full = oracle.decode(blob)
    for t in range(info.n_tiles):
        buf = np.full((256, 384), 0xFFFF, dtype=np.uint16)
        rc, st, _, out = oracle.decode(blob, t, t + 1, want_v=False, out_buf=buf)
        assert rc == 0 and st == 0
        r0, c0 = 128 * (t // kt), 64 * (t % kt)
        touched = out != 0xFFFF
        region = np.zeros_like(touched)
        region[r0:r0 + 128, c0:c0 + 64] = True
        # every element of the region is written (a decoded weight equal to the sentinel would be
        # a NaN, which the decode never produces) and nothing outside it
        assert np.array_equal(touched, region), t
        assert np.array_equal(out[region], full[region])


def test_lane_lengths_follow_the_lane_blocks(oracle):
    """16 W_front + log2(x) - 16 of every lane equals sum log2(M / f) over the tokens of the blocks
    R32 assigns to that lane (single-token coding; raw escape bits counted at the back)"""
    w = synth.row_lognormal(256, 512, seed=6)
    blob, info = compress(oracle, w, 4.0, 1, coding=1)
    b = blob.tobytes()
    v = oracle.quantize(w, info.q_index).reshape(-1, 8)
    ctx, vals = context_values(v)
    ctx, vals = ctx.reshape(-1, 8), vals.reshape(-1, 8)
    # the stream's frequency tables, contexts in order
    freqs, off = [], info.off_freq
    for c in range(7):
        freqs.append(np.frombuffer(b, np.uint16, count=info.ntok[c], offset=off).astype(np.float64))
        off += 2 * info.ntok[c]
    cost = np.zeros(ctx.shape)
    extra = np.zeros(ctx.shape)
    for c in range(7):
        sel = ctx == c
        tok, nbits = tokens(vals[sel], info.split[c], LOW[c])
        cost[sel] = np.log2(2048.0 / freqs[c][tok])
        extra[sel] = nbits
    cb, kt = 512 // 8, 512 // 64
    worst = 0.0
    for t in range(info.n_tiles):
        toff = info.off_tiles + 16 * struct.unpack_from("<I", b, info.off_dir + 4 * t)[0]
        states = struct.unpack_from("<32I", b, toff)
        lens = struct.unpack_from("<32H", b, toff + 128)
        for lane in range(32):
            blocks = [(128 * (t // kt) + 32 * (k % 4) + lane) * cb + 8 * (t % kt) + k // 4 for k in range(32)]
            want = float(cost[blocks].sum())
            raw_words = math.ceil(float(extra[blocks].sum()) / 16)
            got = 16.0 * (lens[lane] - raw_words) + math.log2(states[lane]) - 16.0
            worst = max(worst, abs(got - want))
    # rANS rounding: well under a bit per lane of 256 tokens
    assert worst < 1.0, worst


def test_lane_decode_order(oracle):
    """the order of a lane's blocks, seen from outside: damage one early word of lane 5's region; the
    blocks the lane decodes before reading it come out unchanged and every later one changes, so the
    unchanged blocks must be a prefix of R32's order (rows 5, 37, 69, 101 at column block 0, then
    the same rows at column block 1, ...)"""
    w = synth.row_lognormal(128, 128, seed=7)
    blob, info = compress(oracle, w, 4.0, 1, coding=1)
    b = blob.tobytes()
    rc, st, v_ok, _ = oracle.decode(blob)
    lane, word = 5, 6
    toff = info.off_tiles + 16 * struct.unpack_from("<I", b, info.off_dir)[0]
    lens = struct.unpack_from("<32H", b, toff + 128)
    start = sum(lens[:lane])
    bad = blob.copy()
    pos = toff + 192 + 2 * (start + word)
    bad[pos] ^= 0xA5
    bad[pos + 1] ^= 0x3C
    rc, st, v_bad, _ = oracle.decode(bad)
    order = [(32 * (k % 4) + lane, k // 4) for k in range(32)]  # (row, column block) in decode order
    same = [np.array_equal(v_ok[r, 8 * c:8 * c + 8], v_bad[r, 8 * c:8 * c + 8]) for r, c in order]
    first = same.index(False)
    assert 1 <= first < 16, same
    assert sum(same[first:]) <= 1, same  # after the damaged word the lane is out of step
    # the other lanes of the tile are untouched
    for other in range(32):
        if other != lane:
            for k in range(32):
                r, c = 32 * (k % 4) + other, k // 4
                assert np.array_equal(v_ok[r, 8 * c:8 * c + 8], v_bad[r, 8 * c:8 * c + 8])
