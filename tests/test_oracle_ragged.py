"""Pins of the oracle on matrices whose width is not a multiple of 8.

Reading (the paper gives only 8-wide blocks of a row): each row is padded with
zeros to whole 8-vectors; the row normaliser (RMS) and the least-squares row
scale use the real entries only; the decoder writes the real entries of the
row-major matrix and drops the padding.  Checked against a brute-force nearest
E8 point of every padded vector, the closed-form least-squares scale over the
real entries, the coder round trip, rates and tile ranges.
"""
import itertools

import numpy as np
import pytest

import oracle

_OFFS = np.array(list(itertools.product((-1, 0, 1), repeat=8)), dtype=np.float64)


def _brute_nearest_dist(u):
    """Squared distance from u (8,) to the nearest E8 point, by enumeration."""
    best = np.inf
    for half in (0.0, 0.5):
        cand = (np.rint(u - half) + half)[None, :] + _OFFS
        ok = np.rint(np.sum(cand - half, axis=1)) % 2 == 0
        best = min(best, float(np.min(np.sum((cand[ok] - u) ** 2, axis=1))))
    return best


@pytest.mark.parametrize("rows,cols", [(3, 5), (2, 13), (4, 1), (2, 23)])
def test_padded_vectors_are_nearest_points(rows, cols):
    rng = np.random.default_rng(rows * 100 + cols)
    W = (rng.standard_normal((rows, cols)) * 0.3).astype(np.float32)
    ob = oracle.encode(W, 6.0, tile_vectors=2)
    nq = -(-cols // 8)
    assert ob.nvec == rows * nq
    y = oracle.points_of(ob.fields).astype(np.float64) / 2          # [nvec, 8], padding included
    norms = np.sqrt(np.mean(W.astype(np.float64) ** 2, axis=1))    # RMS over the real entries
    norms[norms == 0] = 1.0
    for r in range(rows):
        pad = np.zeros(8 * nq)
        pad[:cols] = (W[r].astype(np.float64) / norms[r]) / ob.s
        for q in range(nq):
            u = pad[8 * q:8 * q + 8]
            got = float(np.sum((y[r * nq + q] - u) ** 2))
            assert got <= _brute_nearest_dist(u) + 1e-12


@pytest.mark.parametrize("rows,cols", [(40, 60), (17, 1001), (64, 4097), (5, 3)])
def test_ragged_round_trip_scale_and_rate(rows, cols):
    rng = np.random.default_rng(cols)
    W = (rng.standard_t(5, (rows, cols)) * 0.02).astype(np.float32)
    ob = oracle.encode(W, 4.0, tile_vectors=37)
    nq = -(-cols // 8)
    # the stored fields decode back to the encoder's fields, every tile
    got = oracle.decode_fields(ob.payload, ob.tile_index, ob.freq_tables, ob.rows, ob.cols)
    np.testing.assert_array_equal(got, ob.fields.reshape(-1, 9))
    # the lattice output holds the real entries of the points, padding dropped
    y2 = oracle.points_of(ob.fields).reshape(rows, 8 * nq)[:, :cols]
    lat = oracle.decode_blob(ob, oracle.LATTICE)
    np.testing.assert_array_equal(lat, y2)
    # each row scale is the least-squares scale over the real entries
    y = y2.astype(np.float64) / 2
    for r in range(rows):
        den = float(np.dot(y[r], y[r]))
        want = np.float32(np.dot(W[r].astype(np.float64), y[r]) / den) if den else np.float32(0)
        assert ob.row_scales[r] == want
    # FP32 output = fl32(sigma * y) over the real entries
    np.testing.assert_array_equal(oracle.decode_blob(ob, oracle.FP32),
                                  (ob.row_scales[:, None] * y.astype(np.float32)))
    # the rate counts real weights
    assert ob.stored_bpp == pytest.approx(8.0 * ob.stored_bytes / (rows * cols))


def test_ragged_tile_ranges_concatenate():
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((33, 100)) * 0.02).astype(np.float32)
    ob = oracle.encode(W, 5.0, tile_vectors=19)
    full = oracle.decode_blob(ob, oracle.BF16).reshape(-1)
    parts = [oracle.decode(ob.payload, ob.tile_index, ob.freq_tables, ob.row_scales, ob.rows, ob.cols, oracle.BF16,
                           t, t + 1) for t in range(ob.ntiles)]
    np.testing.assert_array_equal(np.concatenate(parts), full)


def test_ragged_rate_and_distortion_behave():
    rng = np.random.default_rng(4)
    W = (rng.standard_t(6, (128, 1020)) * 0.02).astype(np.float32)
    prev = None
    for bpp in (2.0, 4.0, 6.0):
        ob = oracle.encode(W, bpp)
        assert abs(ob.stored_bpp / bpp - 1) < 0.05
        rel = float(np.linalg.norm(oracle.decode_blob(ob, oracle.FP32) - W) / np.linalg.norm(W))
        assert prev is None or rel < prev
        prev = rel
