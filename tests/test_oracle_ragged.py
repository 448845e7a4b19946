"""Pins for rows whose length is not a multiple of 8.  Reading: each row is zero-padded to the next
multiple of 8 before it is cut into E8 blocks; the row statistics use the true columns only, the
padded coordinates are coded like any other and the decoder drops them.

* brute force: the kept coordinates of every block are those of the nearest E8 point (searched
  over both cosets in exact arithmetic) of x = w / (2 f_r) with zeros in the padded places, f_r
  from the row RMS over the true columns (computed here left to right in double);
* exact round trips through the stream on ragged shapes, and the rate counts true elements only;
* a stream whose rows are padded in the caller's data instead (extra zero columns) is a different
  tensor: its row RMS divides by the padded length."""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from dit_weight_compression_tile_b200 import synth


def brute_force_nearest(x):
    """the nearest point of E8 to x as v = 2z, and whether it is unique"""
    best, arg, ties = None, None, 0
    fx = [Fraction(float(a)) for a in x]
    for half in (Fraction(0), Fraction(1, 2)):
        lo = [math.floor(a - half) for a in fx]
        for bits in itertools.product((0, 1), repeat=8):
            z = [lo[i] + bits[i] for i in range(8)]
            if sum(z) % 2:
                continue
            d = sum((fx[i] - (z[i] + half)) ** 2 for i in range(8))
            if best is None or d < best:
                best, arg, ties = d, [int(2 * (z[i] + half)) for i in range(8)], 0
            elif d == best:
                ties += 1
    return arg, ties == 0


def rms_left_to_right(row):
    acc = 0.0
    for a in row:
        acc += float(a) * float(a)
    return np.float32(math.sqrt(acc / len(row)))


@pytest.mark.parametrize("shape,k", [((2, 13), 300), ((3, 7), 420), ((1, 21), 350)])
def test_padded_blocks_brute_force(oracle, shape, k):
    w = synth.gaussian(*shape, std=0.02, seed=shape[1], dtype=torch.float32)
    a = w.numpy().astype(np.float64)
    s, f = oracle.row_factors(w, k)
    v = oracle.quantize(w, k)
    R, Cc = shape
    cp = (Cc + 7) // 8 * 8
    checked = 0
    for r in range(R):
        assert s[r] == rms_left_to_right(a[r])
        assert f[r] == np.float32(float(s[r]) / (2.0 * oracle.q_of_k(k)))
        xr = np.zeros(cp)
        xr[:Cc] = a[r] / (2.0 * float(f[r]))
        for b in range(cp // 8):
            near, unique = brute_force_nearest(xr[8 * b: 8 * b + 8])
            if not unique:
                continue
            keep = min(8, Cc - 8 * b)
            assert list(v[r, 8 * b: 8 * b + keep]) == near[:keep], (r, b)
            checked += 1
    assert checked >= R * (cp // 8) - 1


@pytest.mark.parametrize("shape", [(5, 61), (3, 7), (17, 130), (1, 1), (40, 1001), (2, 9)])
@pytest.mark.parametrize("target", [1.0, 5.0])
def test_ragged_round_trip(oracle, shape, target):
    w = synth.row_lognormal(*shape, seed=sum(shape))
    rc, blob = oracle.compress(w, max(target, 8.0) if shape[0] * shape[1] < 64 else target, q_override=500)
    assert rc == 0
    rc, info = oracle.parse(blob)
    assert rc == 0 and (info.rows, info.cols) == shape
    rc, st, v, out = oracle.decode(blob)
    assert rc == 0 and st == 0 and v.shape == shape and out.shape == shape
    assert np.array_equal(v, oracle.quantize(w, info.q_index))
    assert info.actual_bpp == pytest.approx(8.0 * blob.size / (shape[0] * shape[1]))


def test_ragged_rate_control(oracle):
    w = synth.row_lognormal(96, 1001, seed=3)
    for target in (2.0, 4.0):
        rc, blob = oracle.compress(w, target)
        assert rc == 0
        rc, info = oracle.parse(blob)
        assert info.actual_bpp <= target
        rc, st, v, out = oracle.decode(blob)
        assert st == 0


def test_padding_is_not_extra_columns(oracle):
    w = synth.gaussian(4, 12, 0.02, seed=2, dtype=torch.float32)
    wide = torch.cat([w, torch.zeros(4, 4)], dim=1)
    s12, _ = oracle.row_factors(w, 400)
    s16, _ = oracle.row_factors(wide, 400)
    assert np.allclose(s16, s12 * np.sqrt(12.0 / 16.0), rtol=1e-6) and not np.array_equal(s12, s16)
