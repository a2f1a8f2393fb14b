"""Pins of the oracle's E8 quantiser (Conway & Sloane 1982; EntroPack paper §1).

The oracle must return a nearest point of E8 = D8 u (D8 + 1/2).  It is checked
against (a) brute force over all candidate lattice points near u, (b) an exact
dynamic program over coordinate parities, (c) the covering radius of E8 (1, at
minimal norm sqrt 2), (d) Q(y) = y on lattice points, (e) membership.
"""
import itertools

import numpy as np
import pytest

import oracle


def _is_e8(y):
    y2 = np.rint(2 * y)
    assert np.all(2 * y == y2)
    c = (y2[:, 0] % 2 != 0)
    same = np.all((y2 % 2 != 0) == c[:, None], axis=1)
    even = (np.sum(y, axis=1) % 2 == 0)
    return same & even


_OFFS = np.array(list(itertools.product((-1, 0, 1), repeat=8)), dtype=np.float64)  # 6561 x 8


def _brute_min_dist(u):
    """Minimum squared distance from each u to E8 by enumerating candidates."""
    best = np.full(u.shape[0], np.inf)
    for half in (0.0, 0.5):
        base = np.rint(u - half) + half                      # n x 8
        for i in range(u.shape[0]):
            cand = base[i][None, :] + _OFFS                  # 6561 x 8
            s = np.rint(np.sum(cand - half, axis=1))
            ok = (s % 2 == 0)
            d = np.sum((cand[ok] - u[i]) ** 2, axis=1)
            best[i] = min(best[i], d.min())
    return best


def _dp_min_dist(u):
    """Exact min distance to D8 and D8+1/2 by a parity DP (two states per coordinate)."""
    out = np.full(u.shape[0], np.inf)
    for half in (0.0, 0.5):
        v = u - half
        even = np.zeros(u.shape[0])
        odd = np.full(u.shape[0], np.inf)
        for k in range(8):
            f = np.floor(v[:, k])
            # best cost of an even / odd integer for this coordinate among floor-1..floor+2
            ce = np.full(u.shape[0], np.inf)
            co = np.full(u.shape[0], np.inf)
            for d in (-1, 0, 1, 2):
                a = f + d
                cost = (v[:, k] - a) ** 2
                is_even = (a % 2 == 0)
                ce = np.where(is_even, np.minimum(ce, cost), ce)
                co = np.where(~is_even, np.minimum(co, cost), co)
            even, odd = np.minimum(even + ce, odd + co), np.minimum(even + co, odd + ce)
        out = np.minimum(out, even)
    return out


def test_brute_force_nearest_random():
    rng = np.random.default_rng(11)
    u = np.concatenate([rng.normal(0, s, (300, 8)) for s in (0.3, 1.0, 3.0, 20.0)])
    y, c = oracle.quantize_e8(u)
    assert _is_e8(y).all()
    d = np.sum((u - y) ** 2, axis=1)
    np.testing.assert_allclose(d, _brute_min_dist(u), rtol=0, atol=1e-9)
    assert np.all(c == (np.rint(2 * y[:, 0]) % 2 != 0))


def test_brute_force_ties_and_boundaries():
    # points exactly between lattice points: half-integers, quarter points, deep holes
    rng = np.random.default_rng(12)
    pts = [np.zeros(8), np.full(8, 0.25), np.full(8, 0.5), np.full(8, -0.25),
           np.array([1, 0, 0, 0, 0, 0, 0, 0.0]), np.array([0.5, 0, 0, 0, 0, 0, 0, 0]),
           np.array([0.5, 0.5, 0, 0, 0, 0, 0, 0]), np.array([1, 1, 1, 1, 0, 0, 0, 0.0]) * 0.5,
           np.array([1, 0, 0, 0, 0, 0, 0, 0.0]) * 0.75]
    grid = rng.integers(-8, 9, size=(400, 8)) / 4.0   # many exact ties
    u = np.concatenate([np.array(pts), grid])
    y, _ = oracle.quantize_e8(u)
    assert _is_e8(y).all()
    d = np.sum((u - y) ** 2, axis=1)
    np.testing.assert_allclose(d, _brute_min_dist(u), rtol=0, atol=1e-12)


def test_parity_dp_large_sample():
    rng = np.random.default_rng(13)
    u = np.concatenate([rng.normal(0, s, (25000, 8)) for s in (0.5, 2.0, 7.0, 50.0)])
    y, _ = oracle.quantize_e8(u)
    assert _is_e8(y).all()
    d = np.sum((u - y) ** 2, axis=1)
    np.testing.assert_allclose(d, _dp_min_dist(u), rtol=1e-12, atol=1e-9)


def test_covering_radius():
    # E8 (minimal norm sqrt 2) has covering radius 1: no point is farther than 1.
    rng = np.random.default_rng(14)
    u = np.concatenate([rng.uniform(-4, 4, (200000, 8)), rng.normal(0, 100, (20000, 8))])
    y, _ = oracle.quantize_e8(u)
    d = np.sum((u - y) ** 2, axis=1)
    assert d.max() <= 1.0 + 1e-9
    # deep hole (1, 0, ..., 0) sits exactly at distance 1
    y, _ = oracle.quantize_e8(np.array([[1.0, 0, 0, 0, 0, 0, 0, 0]]))
    assert abs(np.sum((y[0] - np.array([1.0, 0, 0, 0, 0, 0, 0, 0])) ** 2) - 1.0) < 1e-12


def test_fixed_points():
    rng = np.random.default_rng(15)
    z = rng.integers(-50, 51, size=(50000, 8)).astype(np.float64)
    z[:, 7] += (z.sum(axis=1) % 2)          # even sum -> D8
    half = rng.integers(0, 2, size=(50000, 1))
    y0 = z + 0.5 * half
    y, c = oracle.quantize_e8(y0)
    np.testing.assert_array_equal(y, y0)
    np.testing.assert_array_equal(c, half[:, 0])
