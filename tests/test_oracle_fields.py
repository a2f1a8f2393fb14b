"""Pins of the invertible integer fields (EntroPack paper §1, App. A.3, the parity
reduction): (c, z1..z7, m) with z = y - c/2, p = (z1+...+z7) mod 2, m = (z8-p)/2.
"""
import itertools

import numpy as np

import oracle


def _e8_box(lim_int, lim_half):
    pts = []
    r = np.arange(-lim_int, lim_int + 1)
    g = np.array(list(itertools.product(r, repeat=8)), dtype=np.float64)
    pts.append(g[g.sum(axis=1) % 2 == 0])
    h = np.arange(-lim_half, lim_half + 1e-9, 1.0)    # -2.5, -1.5, ..., 2.5
    g = np.array(list(itertools.product(h, repeat=8)), dtype=np.float64)
    pts.append(g[np.rint(g.sum(axis=1)) % 2 == 0])
    return np.concatenate(pts)


def test_exhaustive_bijection_small_box():
    y = _e8_box(2, 2.5)          # every E8 point in [-2, 2]^8 and (Z+1/2)^8 cap [-2.5, 2.5]^8
    assert y.shape[0] > 800000
    c = (np.rint(2 * y[:, 0]) % 2 != 0).astype(np.int32)
    for direct in (False, True):
        f = oracle.fields_of(y, c, direct)
        y2 = oracle.points_of(f, direct)
        np.testing.assert_array_equal(y2, np.rint(2 * y).astype(np.int32))
        # fields -> point -> fields is the identity too
        f2 = oracle.fields_of(y2 / 2.0, f[:, 0], direct)
        np.testing.assert_array_equal(f2, f)
    # the map is injective on the box: distinct points give distinct field tuples
    f = oracle.fields_of(y, c)
    assert np.unique(f, axis=0).shape[0] == y.shape[0]


def test_field_definition_worked_examples():
    # worked by hand from the definitions
    cases = [
        # y                                   c  z1..z7                 m
        ([1, 1, 0, 0, 0, 0, 0, 0],            0, [1, 1, 0, 0, 0, 0, 0], 0),   # p=0, z8=0
        ([1, 0, 0, 0, 0, 0, 0, 1],            0, [1, 0, 0, 0, 0, 0, 0], 0),   # p=1, z8=1 -> m=0
        ([0, 0, 0, 0, 0, 0, 0, 2],            0, [0, 0, 0, 0, 0, 0, 0], 1),   # p=0, z8=2 -> m=1
        ([0, 0, 0, 0, 0, 0, 1, -3],           0, [0, 0, 0, 0, 0, 0, 1], -2),  # p=1, z8=-3 -> m=-2
        ([.5] * 8,                            1, [0] * 7, 0),                 # z=0
        ([-.5] * 8,                           1, [-1] * 7, -1),               # p=1, z8=-1 -> m=-1
        ([1.5, .5, .5, .5, .5, .5, .5, -.5],  1, [1, 0, 0, 0, 0, 0, 0], -1),  # p=1, z8=-1 -> m=-1
    ]
    y = np.array([c[0] for c in cases], np.float64)
    cc = np.array([c[1] for c in cases], np.int32)
    f = oracle.fields_of(y, cc)
    for i, (_, c, z, m) in enumerate(cases):
        assert f[i, 0] == c
        assert list(f[i, 1:8]) == z
        assert f[i, 8] == m, (i, f[i])


def test_parity_reduction_halves_last_field_range():
    # m carries one bit less than z8: on random lattice points its range is about half.
    rng = np.random.default_rng(3)
    y, c = oracle.quantize_e8(rng.normal(0, 6, (100000, 8)))
    f = oracle.fields_of(y, c)
    fz = oracle.fields_of(y, c, direct_z8=True)
    span_m = f[:, 8].max() - f[:, 8].min()
    span_z = fz[:, 8].max() - fz[:, 8].min()
    assert abs(span_z / span_m - 2.0) < 0.1
