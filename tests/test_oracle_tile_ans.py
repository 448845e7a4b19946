"""Pins for the oracle's Tile-ANS lossless stream ("EntroPack README", Configuration: TileANSConfig,
lossless compression for BF16, FP16, FP32, FP8 and INT8 tensors; "EntroPack API reference",
decompress: lossless schemes restore every input bit).

What the pages fix is losslessness itself, so the first pin is the identity: every bit pattern of
every dtype (NaN payloads, infinities, signed zeros and subnormals included) comes back unchanged,
for ragged element counts and several tile sizes.  The readings that define the stream are pinned
from outside the oracle: the raw plane holds exactly the elements' low bytes (numpy slicing), the
frequency table is the stated normalisation of the histogram of the elements' top bytes (numpy
histogram), and the coded length matches the information content of the symbols under that table
(rANS spends log2(M / f) bits per symbol, up to a small per-step rounding), which in turn sits
just above the empirical entropy of the top bytes."""
import math
import struct

import numpy as np
import pytest
import torch

from dit_weight_compression_tile_b200 import synth

BF16, FP16, FP32, INT8, FP8 = 1, 2, 3, 4, 5
NP = {BF16: np.uint16, FP16: np.uint16, FP32: np.uint32, INT8: np.uint8, FP8: np.uint8}
ESZ = {BF16: 2, FP16: 2, FP32: 4, INT8: 1, FP8: 1}


def bits_of(t):
    """raw bit patterns of a torch tensor as a numpy array"""
    return {torch.bfloat16: lambda: t.view(torch.int16).numpy().view(np.uint16),
            torch.float16: lambda: t.view(torch.int16).numpy().view(np.uint16),
            torch.float32: lambda: t.numpy().view(np.uint32),
            torch.int8: lambda: t.numpy().view(np.uint8),
            torch.float8_e4m3fn: lambda: t.view(torch.uint8).numpy()}[t.dtype]()


def roundtrip(oracle, x, dt, K=0, shape=None):
    rc, blob = oracle.ta_compress(x, dt, shape=shape, blocks_per_lane=K)
    assert rc == 0, rc
    rc, st, y = oracle.ta_decode(blob)
    assert rc == 0 and st == 0
    assert y.dtype == x.dtype and np.array_equal(y.reshape(-1), x.reshape(-1))
    return blob


@pytest.mark.parametrize("dt", [BF16, FP16])
def test_every_16_bit_pattern(oracle, dt):
    """all 65,536 patterns (every NaN payload, both infinities and zeros, all subnormals), in a
    seeded order so that chunks mix them"""
    x = np.random.default_rng(1).permutation(np.arange(65536, dtype=np.uint32)).astype(np.uint16)
    roundtrip(oracle, x, dt)
    roundtrip(oracle, x[:12345], dt, K=2)


@pytest.mark.parametrize("dt", [INT8, FP8])
def test_every_byte(oracle, dt):
    x = np.tile(np.arange(256, dtype=np.uint8), 40)
    roundtrip(oracle, x, dt)
    roundtrip(oracle, np.random.default_rng(2).permutation(x), dt, K=1)


def test_fp32_special_and_random(oracle):
    special = np.array([0x00000000, 0x80000000, 0x7f800000, 0xff800000, 0x7fc00000, 0x7fa00001, 0xffffffff,
                        0x00000001, 0x807fffff, 0x3f800000, 0xbf800000, 0x7f7fffff], dtype=np.uint32)
    rnd = np.random.default_rng(3).integers(0, 2 ** 32, size=50000, dtype=np.uint64).astype(np.uint32)
    roundtrip(oracle, np.concatenate([special, rnd, special]), FP32)


@pytest.mark.parametrize("n", [1, 7, 8, 9, 255, 256, 257, 8191, 8192, 8193, 40000])
@pytest.mark.parametrize("dt", [BF16, FP32, INT8])
def test_ragged_counts(oracle, n, dt):
    x = np.random.default_rng(n).integers(0, 2 ** (8 * ESZ[dt]), size=n, dtype=np.uint64).astype(NP[dt])
    for K in (0, 1, 3):
        roundtrip(oracle, x, dt, K=K)


def test_shapes_kept(oracle):
    for shape in [(1,), (3, 5, 7), (2, 1, 1, 1, 1, 1, 1, 4), (64, 33)]:
        x = np.arange(math.prod(shape), dtype=np.uint16).reshape(shape)
        blob = roundtrip(oracle, x, BF16)
        rc, info = oracle.ta_parse(blob)
        assert tuple(info.shape[: info.ndim]) == shape
        rc, st, y = oracle.ta_decode(blob)
        assert y.shape == shape


def test_constant_tensor(oracle):
    """a lone symbol gets 4095 of the 4096 slots and a phantom symbol the last one"""
    x = np.full(100000, 0x3c00, dtype=np.uint16)
    blob = roundtrip(oracle, x, FP16)
    rc, info = oracle.ta_parse(blob)
    f = np.frombuffer(blob.tobytes(), np.uint16, count=256, offset=info.off_freq)
    assert f[0x3c] == 4095 and f[0] == 1 and f.sum() == 4096


def layout_checks(oracle, blob, x, dt):
    b = blob.tobytes()
    rc, info = oracle.ta_parse(blob)
    assert rc == 0
    magic, ver, dtype, ndim, n, T, K, pb = struct.unpack_from("<IHBBqIIB", b, 0)
    assert magic == 0x31415045 and ver == 1 and dtype == dt and n == x.size and pb == 12
    assert info.off_freq == 128 and info.off_dir == 640
    esz = ESZ[dt]
    # the raw plane is the elements' low bytes, in element order
    raw = np.frombuffer(b, np.uint8, count=x.size * (esz - 1), offset=info.off_raw)
    xb = x.reshape(-1).view(np.uint8).reshape(-1, esz)
    assert np.array_equal(raw.reshape(-1, esz - 1) if esz > 1 else raw, xb[:, : esz - 1] if esz > 1 else raw)
    # the table is the stated normalisation of the top bytes' histogram (zero padding included)
    top = xb[:, esz - 1]
    nc = -(-x.size // 8)
    hist = np.bincount(top, minlength=256).astype(np.uint64)
    hist[0] += nc * 8 - x.size
    want = np.zeros(256, np.uint32)
    import ctypes as C
    oracle.lib().or_normalize_freqs_to(oracle._ptr(np.ascontiguousarray(hist)), 256, 12, oracle._ptr(want))
    f = np.frombuffer(b, np.uint16, count=256, offset=info.off_freq)
    assert np.array_equal(f, want)
    return info, f, hist


def information_checks(oracle, blob, info, f, hist):
    """16 W + sum over lanes of (log2 x_l - 16) equals the symbols' information under the table,
    sum log2(4096 / f_s), up to the rANS rounding; that information exceeds the empirical entropy
    of the symbols by the table's KL divergence only"""
    b = blob.tobytes()
    words, state_bits = 0, 0.0
    for t in range(info.n_tiles):
        off = info.off_tiles + 16 * struct.unpack_from("<I", b, info.off_dir + 4 * t)[0]
        states = np.array(struct.unpack_from("<32I", b, off), dtype=np.float64)
        lens = struct.unpack_from("<32H", b, off + 128)
        words += sum(lens)
        state_bits += float(np.sum(np.log2(states) - 16.0))
    n_sym = float(hist.sum())
    nz = hist > 0
    info_bits = float(np.sum(hist[nz] * np.log2(4096.0 / f[nz])))
    entropy = float(-np.sum(hist[nz] * np.log2(hist[nz] / n_sym)))
    coded = 16.0 * words + state_bits
    assert abs(coded - info_bits) <= 1e-3 * n_sym + 64.0
    assert info_bits >= entropy - 1e-6
    return coded, info_bits, entropy, n_sym


@pytest.mark.parametrize("dt,make", [
    (BF16, lambda: synth.row_lognormal(512, 1024, seed=4)),
    (FP16, lambda: synth.gaussian(256, 1024, 0.02, seed=5).to(torch.float16)),
    (FP32, lambda: synth.dit_layer(1, 2)[:128, :1024].float().contiguous()),
    (INT8, lambda: torch.clamp(torch.round(synth.gaussian(256, 1024, 0.02, seed=6).float() / 0.0006), -127,
                               127).to(torch.int8)),
    (FP8, lambda: (synth.gaussian(256, 1024, 0.02, seed=7).float() * 100).to(torch.float8_e4m3fn)),
])
def test_layout_and_code_length(oracle, dt, make):
    t = make()
    x = bits_of(t).reshape(-1).copy()
    blob = roundtrip(oracle, x, dt)
    info, f, hist = layout_checks(oracle, blob, x, dt)
    coded, info_bits, entropy, n_sym = information_checks(oracle, blob, info, f, hist)
    # a 12-bit table costs little over the entropy: rare symbols still take one of 4096 slots
    # (measured: 0.012 bit per symbol on the INT8 codes, whose tails reach +-127; < 0.004 on the rest)
    assert (info_bits - entropy) / n_sym < 0.02
    # the whole stream: raw bytes + coded symbols + tile heads and tables, nothing else
    overhead = len(blob) * 8 - (coded + 8 * (ESZ[dt] - 1) * x.size)
    assert overhead <= 8 * (128 + 512 + 16 + 4 * (info.n_tiles + 1) + 16 + 208 * info.n_tiles)


def test_damaged_streams(oracle):
    x = bits_of(synth.row_lognormal(128, 1024, seed=8)).reshape(-1).copy()
    rc, blob = oracle.ta_compress(x, BF16)
    rc, info = oracle.ta_parse(blob)
    assert oracle.ta_parse(blob[:-16])[0] == oracle.ERR_CORRUPT
    for off in (0, 4, 6, 24, info.off_freq + 2 * 0x3c, info.off_dir + 4 * info.n_tiles):
        bad = blob.copy()
        bad[off] ^= 0x5A
        assert oracle.ta_parse(bad)[0] == oracle.ERR_CORRUPT, off
    # a moved inner directory entry passes the parser; the decoder's end checks see it
    bad = blob.copy()
    bad[info.off_dir + 4] += 1
    rc, st, y = oracle.ta_decode(bad)
    assert rc == 0 and st != 0
    # a flipped word inside a tile's regions: the decoder's end checks see it
    flagged = 0
    for t in range(info.n_tiles):
        off = info.off_tiles + 16 * struct.unpack_from("<I", blob.tobytes(), info.off_dir + 4 * t)[0] + 192 + 40
        bad = blob.copy()
        bad[off] ^= 0x40
        rc, st, y = oracle.ta_decode(bad)
        flagged += st != 0 or not np.array_equal(y.reshape(-1), x)
    assert flagged == info.n_tiles
