"""Pins of the sampled-row selection (EntroPack paper App. C.1: complete rows,
shape-dependent seed, fixed through the search)."""
import numpy as np

import oracle


def test_splitmix64_published_outputs():
    # first outputs of Vigna's reference splitmix64 seeded with 0
    got = oracle.splitmix64(0, 3)
    assert [int(v) for v in got] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_sample_rows_count_distinct_deterministic():
    for rows, cols, sv in ((3840, 10240, 1 << 18), (256, 512, 1 << 18), (25600, 5120, 1 << 18), (1000, 64, 50)):
        s = oracle.sample_rows(rows, cols, sv)
        assert len(s) == min(rows, -(-sv // (cols // 8)))
        assert len(np.unique(s)) == len(s)
        assert s.min() >= 0 and s.max() < rows
        np.testing.assert_array_equal(s, oracle.sample_rows(rows, cols, sv))
    a = oracle.sample_rows(3840, 10240, 1 << 18)
    b = oracle.sample_rows(3840, 10248, 1 << 18)
    assert not np.array_equal(a[:10], b[:10])      # the seed depends on the shape
    assert not np.array_equal(a, oracle.sample_rows(3840, 10240, 1 << 18, seed=99))
