"""Pins of the oracle's encoder against what the pages and lattice theory fix:
rate lands near the target (EntroPack paper §4.2: mean 0.80 %, max 2.13 % on real
weights), rel-L2 falls with rate, the E8 high-rate distortion law, the Table 4
ablation directions, least-squares refit, row-scale covariance, precision
escalation and coarsening (App. C.1)."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
G_E8 = 0.0716821                           # normalised second moment of E8 (Conway & Sloane)
H_GAUSS = 0.5 * np.log2(2 * np.pi * np.e)  # differential entropy of N(0,1), bits


@pytest.fixture(scope="module")
def gauss():
    rng = np.random.default_rng(0)
    return (rng.standard_normal((1024, 2048)) * 0.02).astype(np.float32)


@pytest.fixture(scope="module")
def sweep(gauss):
    return {t: oracle.encode(gauss, t) for t in (2, 3, 4, 5, 6, 7, 8)}


def _rel(bl, W):
    out = oracle.decode_blob(bl, oracle.FP32)
    return float(np.linalg.norm(out - W) / np.linalg.norm(W))


def test_rate_lands_near_target(sweep):
    for t, bl in sweep.items():
        assert abs(bl.stored_bpp / t - 1) <= 0.03, (t, bl.stored_bpp)


def test_rel_l2_falls_with_rate(gauss, sweep):
    rel = [_rel(sweep[t], gauss) for t in sorted(sweep)]
    assert all(a > b for a, b in zip(rel, rel[1:])), rel


def test_high_rate_e8_distortion_law(gauss, sweep):
    # entropy-coded E8 on i.i.d. Gaussian: rel-L2 ~ sqrt(G_E8) * 2^(h - R), R = payload bits per weight
    for t in (4, 5, 6, 7):
        bl = sweep[t]
        R = 16.0 * bl.payload.size / gauss.size
        pred = np.sqrt(G_E8) * 2 ** (H_GAUSS - R)
        assert abs(_rel(bl, gauss) / pred - 1) < 0.05, (t, _rel(bl, gauss), pred)


def _golden(name):
    rows = []
    for line in open(os.path.join(GOLDEN, name)):
        if line.strip() and not line.startswith("#"):
            rows.append([float(v) for v in line.split()])
    return rows


def test_table4_ablation_directions(sweep):
    # Table 4: coding z8 directly costs 0.10-0.13 bpp; dropping coset conditioning costs most at 2 bpp.
    g = _golden("table4_ablation.txt")
    dz_page = [r[2] - r[3] for r in g]
    pool_page = {int(r[0]): r[1] - r[3] for r in g}
    for t in (2, 4, 8):
        bl = sweep[t]
        y2 = oracle.points_of(bl.fields)
        fz = oracle.fields_of(y2 / 2.0, bl.fields[:, 0], direct_z8=True)
        bz = oracle.encode_fields(fz, bl.rows, bl.cols, bl.row_scales, bl.b, bl.V, flags=1)
        bp = oracle.encode_fields(bl.fields, bl.rows, bl.cols, bl.row_scales, bl.b, bl.V, flags=2)
        # both variants reconstruct the same weights
        np.testing.assert_array_equal(oracle.decode_blob(bz, oracle.LATTICE), oracle.decode_blob(bl, oracle.LATTICE))
        np.testing.assert_array_equal(oracle.decode_blob(bp, oracle.LATTICE), oracle.decode_blob(bl, oracle.LATTICE))
        dz = bz.stored_bpp - bl.stored_bpp
        assert min(dz_page) - 0.03 <= dz <= max(dz_page) + 0.03, (t, dz)
        if t == 2:
            dp = bp.stored_bpp - bl.stored_bpp
            assert dp >= 0.5 * pool_page[2], dp


def test_search_estimate_brackets_target(gauss):
    bl = oracle.encode(gauss, 4.0)
    r = oracle.estimate_rate(gauss, 4.0, bl.s, bl.b)
    assert abs(r / 4.0 - 1) < 0.01
    assert oracle.estimate_rate(gauss, 4.0, bl.s * 0.9, bl.b) > 4.0 > oracle.estimate_rate(gauss, 4.0, bl.s * 1.1, bl.b)


def test_refit_is_least_squares(gauss):
    bl = oracle.encode(gauss[:64], 3.0, tile_vectors=64)
    y = oracle.decode_blob(bl, oracle.LATTICE).astype(np.float64) / 2.0
    W = gauss[:64].astype(np.float64)
    for r in range(64):
        sig = float(bl.row_scales[r])
        e0 = np.sum((W[r] - sig * y[r]) ** 2)
        for f in (1 - 1e-4, 1 + 1e-4, 0.99, 1.01):
            assert e0 <= np.sum((W[r] - sig * f * y[r]) ** 2)
        # normal equation <w - sigma y, y> = 0 up to the FP32 rounding of sigma
        assert abs(np.dot(W[r] - sig * y[r], y[r])) <= 1e-6 * np.linalg.norm(W[r]) * np.linalg.norm(y[r])
        assert oracle.refit_row(gauss[r], y[r]) == bl.row_scales[r]
    assert oracle.refit_row(np.ones(8, np.float32), np.zeros(8)) == 0.0


def test_row_scale_covariance(gauss):
    # row normalisation: scaling a row by a power of two leaves every field unchanged and scales sigma
    W = gauss[:128].copy()
    k = np.random.default_rng(2).integers(-6, 7, size=(128, 1)).astype(np.float32)
    W2 = (W * np.exp2(k)).astype(np.float32)
    a = oracle.encode(W, 4.0, tile_vectors=256, prob_bits=11, sample_vectors=1 << 20)
    b = oracle.encode(W2, 4.0, tile_vectors=256, prob_bits=11, sample_vectors=1 << 20)
    np.testing.assert_array_equal(a.fields, b.fields)
    np.testing.assert_array_equal(a.row_scales * np.exp2(k[:, 0]), b.row_scales)
    assert oracle.row_norm(np.zeros(16, np.float32)) == 1.0
    assert oracle.row_norm(np.full(16, -3.0, np.float32)) == 3.0


def test_zero_rows_and_determinism():
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((64, 256)) * 0.05).astype(np.float32)
    W[5] = 0
    W[17] = 0
    a = oracle.encode(W, 5.0, tile_vectors=64)
    b = oracle.encode(W, 5.0, tile_vectors=64)
    assert a.row_scales[5] == 0 and a.row_scales[17] == 0
    np.testing.assert_array_equal(a.payload, b.payload)
    np.testing.assert_array_equal(a.tile_index, b.tile_index)
    np.testing.assert_array_equal(a.freq_tables, b.freq_tables)
    out = oracle.decode_blob(a, oracle.FP32)
    assert np.all(out[5] == 0) and np.all(out[17] == 0)


def test_precision_escalation():
    # a full-tensor alphabet wider than 2^11 (an outlier row outside the sample) raises b (App. C.1)
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((512, 64)) * 0.02).astype(np.float32)
    W[:, 0] *= 1.0
    W[300, :] = 0.0
    W[300, 0] = 50.0                 # a row whose RMS is set by one huge value
    W[300, 1:] = rng.standard_normal(63).astype(np.float32) * 1e-4
    a = oracle.encode(W, 7.0, sample_vectors=64, seed=5)
    assert a.b >= 11
    _check_alphabets(a)
    np.testing.assert_array_equal(
        oracle.decode_fields(a.payload, a.tile_index, a.freq_tables, a.rows, a.cols), a.fields)


def _check_alphabets(bl):
    ft = bl.freq_tables
    desc = ft[48:48 + 8 * bl.ntab].view(np.int32).reshape(bl.ntab, 2)
    assert np.all(desc[:, 1] <= (1 << bl.b))
    return desc[:, 1].max()


def test_coarsening_at_maximum_precision():
    # rows the sample never sees carry an alphabet wider than 2^15 at the searched scale:
    # b climbs to 15 and the scale is then coarsened until the alphabets fit (App. C.1)
    rng = np.random.default_rng(6)
    W = (rng.standard_normal((256, 4096)) * 1e-3).astype(np.float32)
    hot = rng.choice(256, size=8, replace=False)
    for r in hot:
        W[r] = (rng.standard_normal(4096) * 1e-6).astype(np.float32)
        W[r, rng.integers(4096)] = 1.0      # |x| = 64 after the RMS normalisation
    assert not set(oracle.sample_rows(256, 4096, 16, seed=1)) & set(hot)
    a = oracle.encode(W, 14.0, sample_vectors=16, seed=1, prob_bits=12)
    assert a.b == 15
    amax = _check_alphabets(a)
    assert amax <= 1 << 15
    np.testing.assert_array_equal(
        oracle.decode_fields(a.payload, a.tile_index, a.freq_tables, a.rows, a.cols), a.fields)


# ------------------------------------------------------------------ per-row RDO (§3.5, App. C.2)

def _heterogeneous_rows(seed=1, rows=256, cols=512):
    """Rows with different tails and scales: the case where per-row resolutions differ."""
    rng = np.random.default_rng(seed)
    W = np.empty((rows, cols), np.float32)
    for r in range(rows):
        W[r] = rng.standard_t([2.5, 4, 8, 30][r % 4], cols) * 0.02 * np.exp(rng.normal(0, 0.5))
    return W


def _rel_l2(ob, W):
    dec = oracle.decode_blob(ob, oracle.FP32).reshape(W.shape)
    return float(np.linalg.norm(dec - W) / np.linalg.norm(W))


def test_rdo_candidate_ratios_are_nested_log_bisections():
    # §3.5: ratios in [0.70, 1.45], the first 1, each next one the log-scale midpoint of the
    # largest gap left (the two halves of [1, 1.45] tie; the lower one goes first)
    want = [1.0, 1.45 ** 0.5, 0.70 ** 0.5, 1.45 ** 0.25, 1.45 ** 0.75]
    np.testing.assert_allclose(oracle.rdo_ratios(5), want, rtol=1e-15)
    r20 = oracle.rdo_ratios(20)
    for k in range(1, 20):
        np.testing.assert_array_equal(oracle.rdo_ratios(k), r20[:k])  # nested
    assert np.all((r20 > 0.70) & (r20 < 1.45)) and len(set(r20)) == 20
    gaps = np.diff(np.log(np.sort(np.concatenate([[0.70, 1.45], r20]))))
    assert gaps.max() <= 2 * gaps.min() + 1e-12  # bisection keeps the log spacing within a factor 2


def test_rdo_off_and_one_candidate_leave_the_stream_unchanged():
    W = _heterogeneous_rows(seed=2, rows=64)
    a = oracle.encode(W, 4.0)
    for kw in (dict(rdo_candidates=1), dict(rdo_candidates=1, rdo_sweeps=3), dict(rdo_candidates=0)):
        b = oracle.encode(W, 4.0, **kw)
        for f in ("payload", "tile_index", "freq_tables", "row_scales"):
            np.testing.assert_array_equal(getattr(a, f), getattr(b, f))


@pytest.mark.parametrize("target", [2.0, 3.0, 5.0])
def test_rdo_lowers_distortion_within_the_budget(target):
    # the allocation keeps the baseline's storage budget and, with more resolutions per row,
    # reconstructs closer (the paper's Fig. 4 direction: 14.35 % -> 14.11 % at K = 5)
    W = _heterogeneous_rows(seed=3)
    base = oracle.encode(W, target)
    e0 = _rel_l2(base, W)
    k5 = oracle.encode(W, target, rdo_candidates=5)
    k9 = oracle.encode(W, target, rdo_candidates=9)
    assert k5.stored_bpp <= base.stored_bpp * 1.002 and k9.stored_bpp <= base.stored_bpp * 1.002
    e5, e9 = _rel_l2(k5, W), _rel_l2(k9, W)
    assert e5 < e0 and e9 <= e5 * 1.005, (e0, e5, e9)
    # the stored fields decode to themselves and every row scale is the refit of its own points
    y = oracle.decode_blob(k5, oracle.LATTICE).reshape(W.shape).astype(np.float64) / 2
    for r in range(0, W.shape[0], 37):
        assert k5.row_scales[r] == oracle.refit_row(W[r], y[r])


def test_rdo_second_sweep_keeps_the_budget():
    W = _heterogeneous_rows(seed=4)
    base = oracle.encode(W, 3.0)
    two = oracle.encode(W, 3.0, rdo_candidates=5, rdo_sweeps=2)
    assert two.stored_bpp <= base.stored_bpp * 1.002
    assert _rel_l2(two, W) < _rel_l2(base, W)
