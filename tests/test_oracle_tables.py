"""Direct pins of two encoder readings of the oracle.

Frequency normalisation (EntroPack paper §3.6, App. C.1: tables at precision b): hand-worked
counts -> frequencies (tests/golden/normalize_freqs_worked.txt), then the invariants any
normalisation must keep on random counts: the frequencies sum to 2^b, a symbol gets f > 0
exactly when it was observed, and the tables cost little over the empirical entropy.

Sampled rows (App. C.1: complete rows, shape-dependent seed): a partial Fisher-Yates draw
worked by hand from SplitMix64 outputs that are published for seed 0 (the generator started
one step later), and the distribution of full draws over many seeds, which is uniform over
the permutations only when the swap index is drawn from the right range.
"""
import os
from itertools import permutations

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "normalize_freqs_worked.txt")


def _worked():
    for line in open(GOLDEN):
        if not line.strip() or line.startswith("#"):
            continue
        b, counts, want, _why = (p.strip() for p in line.split("|"))
        yield int(b), [int(v) for v in counts.split()], [int(v) for v in want.split()]


def test_normalize_freqs_worked_examples():
    n = 0
    for b, counts, want in _worked():
        got = oracle.normalize_freqs(np.array(counts), b)
        assert [int(v) for v in got] == want, (b, counts, list(got), want)
        n += 1
    assert n == 14


def test_normalize_freqs_invariants_on_random_counts():
    rng = np.random.default_rng(11)
    for trial in range(300):
        b = int(rng.integers(4, 16))
        M = 1 << b
        A = int(rng.integers(1, min(M, 400) + 1))
        shape = rng.choice(["geometric", "flat", "sparse", "peaked"])
        if shape == "geometric":
            counts = rng.geometric(0.2, A) * (rng.random(A) < 0.9)
        elif shape == "flat":
            counts = rng.integers(0, 50, A)
        elif shape == "sparse":
            counts = (rng.random(A) < 0.05) * rng.integers(1, 5, A)
        else:
            counts = np.zeros(A, np.int64)
            counts[rng.integers(A)] = 10 ** 6
            counts += rng.random(A) < 0.3
        if counts.sum() == 0:
            counts[0] = 1
        f = oracle.normalize_freqs(counts, b).astype(np.int64)
        assert f.sum() == M, (trial, b, A)
        np.testing.assert_array_equal(f > 0, counts > 0)
        # coding cost under the normalised tables versus the empirical entropy: the rounding
        # loses little (a table built from wrong symbols or a transposed index would not)
        p = counts[counts > 0] / counts.sum()
        q = f[counts > 0] / M
        loss = float((p * np.log2(p / q)).sum())
        observed = int((counts > 0).sum())
        assert loss <= 0.05 + observed / M * 2.0, (trial, b, A, shape, loss)


GAMMA = 0x9E3779B97F4A7C15  # SplitMix64's increment: as a seed, the seed-0 stream one step on
SEED0 = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F, 0xF88BB8A8724C81EC, 0x1B39896A51A8749B]


def test_splitmix64_seed_zero_stream_and_its_shift():
    assert [int(v) for v in oracle.splitmix64(0, 5)] == SEED0
    assert [int(v) for v in oracle.splitmix64(GAMMA, 4)] == SEED0[1:]


def test_sample_rows_worked_example():
    """rows = 5, cols = 8 (one vector a row), a budget of 4 vectors -> 4 rows; seed GAMMA draws
    r = SEED0[1:].  By hand: perm = [0 1 2 3 4];
      i = 0: j = 0 + r0 mod 5 = 0 + 0 (7960286522194355700 ends in 00)  -> row 0, perm unchanged;
      i = 1: j = 1 + r1 mod 4 = 1 + 3 (487617019471545679: 79 mod 4 = 3) -> swap 1, 4: row 4;
      i = 2: j = 2 + r2 mod 3 = 2 + 1 (digit sum of 17909611376780542444 is 88) -> swap 2, 3: row 3;
      i = 3: j = 3 + r3 mod 2 = 3 + 1 (1961750202426094747 is odd) -> swap 3, 4: row 1."""
    assert [7960286522194355700 % 5, 487617019471545679 % 4, 17909611376780542444 % 3, 1961750202426094747 % 2] \
        == [0, 3, 1, 1]
    assert [int(v) for v in oracle.sample_rows(5, 8, 4, seed=GAMMA)] == [0, 4, 3, 1]


def test_sample_rows_draws_every_permutation_equally_often():
    """Full draws of 4 rows over 24,000 seeds: each of the 24 orders about 1,000 times.  A swap
    index drawn from [0, rows) or from [i + 1, rows) instead of [i, rows) skews this at once."""
    seen = {p: 0 for p in permutations(range(4))}
    n = 24000
    for seed in range(1, n + 1):
        seen[tuple(int(v) for v in oracle.sample_rows(4, 8, 4, seed=seed))] += 1
    exp = n / 24
    chi2 = sum((c - exp) ** 2 / exp for c in seen.values())
    assert min(seen.values()) > 0
    assert chi2 < 60.0, chi2  # 23 degrees of freedom: the 0.01 % tail starts near 57


def test_sample_rows_partial_draw_is_uniform_over_rows():
    """Partial draws (3 of 9 rows): every row is drawn with probability 1/3, every row first with
    probability 1/9."""
    n = 18000
    anywhere = np.zeros(9)
    first = np.zeros(9)
    for seed in range(1, n + 1):
        s = oracle.sample_rows(9, 8, 3, seed=seed)
        anywhere[s] += 1
        first[s[0]] += 1
    np.testing.assert_allclose(anywhere / n, 1 / 3, atol=0.02)
    np.testing.assert_allclose(first / n, 1 / 9, atol=0.015)
