"""The linear-layer oracle pinned to a brute-force triple loop (exact on integer values) and to the
identity, and its tolerance bound checked against float32 accumulation in two orders."""
import numpy as np

import oracle


def test_brute_force_and_identity():
    rng = np.random.default_rng(0)
    W = rng.integers(-50, 50, (7, 13)).astype(np.float32)
    x = rng.integers(-50, 50, (5, 13)).astype(np.float32)
    y = oracle.linear(W, x)
    want = np.zeros((5, 7))
    for t in range(5):
        for o in range(7):
            acc = 0.0
            for k in range(13):
                acc += float(x[t, k]) * float(W[o, k])
            want[t, o] = acc
    np.testing.assert_array_equal(y, want)  # integer values: every operation exact
    np.testing.assert_array_equal(oracle.linear(W, np.eye(13)), W.T)


def test_tolerance_covers_float32_accumulation():
    rng = np.random.default_rng(1)
    W = (rng.standard_normal((16, 3000)) * 0.02).astype(np.float32)
    x = rng.standard_normal((8, 3000)).astype(np.float32)
    ref = oracle.linear(W, x)
    tol = oracle.linear_tolerance(W, x, 2.0 ** -24)
    for order in (slice(None), slice(None, None, -1)):  # forward and backward sums in float32
        acc = np.zeros((8, 16), np.float32)
        for k in range(3000)[order]:
            acc += x[:, k:k + 1] * W[:, k][None, :]
        assert np.all(np.abs(acc.astype(np.float64) - ref) <= tol)
    assert np.all(tol > 0)
