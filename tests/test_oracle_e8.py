"""Pins for the oracle's E8 quantizer, independent of its code.

* brute force: the nearest point is searched over every candidate of both cosets in the
  box of floor/ceil neighbours (all 2 x 256 sign patterns), in exact rational arithmetic;
* lattice invariants: all-even or all-odd v, sum v = 0 mod 4, distance <= covering radius 1,
  lattice points are fixed points;
* closed form: the normalized second moment of E8 is 929/12960 (Conway & Sloane), so the
  mean squared error per dimension over uniform inputs must approach it;
* the worked examples in tests/golden/e8_examples.txt, derived by hand from the definition.
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e8_examples.txt")


def brute_force_min_dist(x):
    """Exact minimum squared distance from x to E8 = D8 u (D8 + 1/2)."""
    best = None
    fx = [Fraction(float(a)) for a in x]
    for half in (Fraction(0), Fraction(1, 2)):
        lo = [math.floor(a - half) for a in fx]
        for bits in itertools.product((0, 1), repeat=8):
            z = [lo[i] + bits[i] for i in range(8)]
            if sum(z) % 2:
                continue
            d = sum((fx[i] - (z[i] + half)) ** 2 for i in range(8))
            if best is None or d < best:
                best = d
    return best


def exact_dist(x, v):
    return sum((Fraction(float(x[i])) - Fraction(int(v[i]), 2)) ** 2 for i in range(8))


def check_lattice(v):
    v = np.asarray(v, dtype=np.int64)
    par = v % 2
    assert np.all(par == par[..., :1]), "mixed cosets"
    assert np.all(v.sum(-1) % 4 == 0), "sum v must be 0 mod 4"


def test_golden_examples(oracle):
    n = 0
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        xs, vs, ds, _ = line.split("|")
        x = np.array([float(a) for a in xs.split()])
        v_expect = np.array([int(a) for a in vs.split()])
        v = oracle.e8_nearest(x)
        assert np.array_equal(v, v_expect), (x, v, v_expect)
        assert abs(float(exact_dist(x, v)) - float(ds)) < 1e-12
        n += 1
    assert n >= 9


@pytest.mark.parametrize("scale", [0.3, 1.0, 4.0, 100.0])
def test_brute_force_nearest(oracle, scale):
    rng = np.random.default_rng(int(scale * 10))
    x = rng.normal(size=(60, 8)) * scale
    v = oracle.e8_nearest(x)
    check_lattice(v)
    for i in range(x.shape[0]):
        assert exact_dist(x[i], v[i]) == brute_force_min_dist(x[i]), x[i]


def test_brute_force_ties(oracle):
    """Inputs on half-integers and quarter-integers, where rounding ties and coset ties occur."""
    rng = np.random.default_rng(7)
    x = rng.integers(-8, 9, size=(80, 8)) / 4.0
    v = oracle.e8_nearest(x)
    check_lattice(v)
    for i in range(x.shape[0]):
        assert exact_dist(x[i], v[i]) == brute_force_min_dist(x[i]), x[i]


def test_d8_brute_force(oracle):
    rng = np.random.default_rng(3)
    for _ in range(60):
        y = rng.normal(size=8) * 2
        r = oracle.d8_nearest(y)
        assert int(round(r.sum())) % 2 == 0
        fy = [Fraction(float(a)) for a in y]
        best = None
        lo = [math.floor(a) for a in fy]
        for bits in itertools.product((0, 1), repeat=8):
            z = [lo[i] + bits[i] for i in range(8)]
            if sum(z) % 2 == 0:
                d = sum((fy[i] - z[i]) ** 2 for i in range(8))
                best = d if best is None or d < best else best
        assert sum((fy[i] - Fraction(float(r[i]))) ** 2 for i in range(8)) == best


def test_invariants_large_batch(oracle):
    rng = np.random.default_rng(11)
    x = rng.normal(size=(200000, 8)) * rng.uniform(0.1, 50, size=(200000, 1))
    v = oracle.e8_nearest(x)
    check_lattice(v)
    d2 = ((x - v / 2.0) ** 2).sum(-1)
    assert d2.max() <= 1.0 + 1e-12  # covering radius of E8 (min norm sqrt 2) is 1


def test_lattice_points_fixed(oracle):
    rng = np.random.default_rng(5)
    z = rng.integers(-20, 21, size=(5000, 8))
    z[:, 7] += z.sum(-1) % 2  # make the sum even: a D8 point
    half = rng.integers(0, 2, size=(5000, 1))
    v = 2 * z + half  # D8 or D8 + 1/2, doubled
    check_lattice(v)
    assert np.array_equal(oracle.e8_nearest(v / 2.0), v)


def test_normalized_second_moment(oracle):
    """G(E8) = 929/12960 ~ 0.0716821 (Conway & Sloane, SPLAG table 2.3); cell volume 1."""
    rng = np.random.default_rng(2024)
    x = rng.uniform(-64, 64, size=(400000, 8))
    v = oracle.e8_nearest(x)
    mse = ((x - v / 2.0) ** 2).sum(-1).mean() / 8.0
    assert abs(mse - 929.0 / 12960.0) < 0.004 * (929.0 / 12960.0)
    # a quantizer that dropped the 1/2 coset (plain D8, cell volume 2) would give ~0.0902
