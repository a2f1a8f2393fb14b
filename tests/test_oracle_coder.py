"""Pins of the oracle's tiled interleaved rANS coder (EntroPack paper §3.6,
App. C.3): exact field recovery, terminal states, cursor landing, code length
close to the ideal length under the stored tables, and planted-fault detection.
"""
import numpy as np
import pytest

import oracle


def _random_fields(rng, nvec, spread=(3.0, 5.0)):
    y, c = oracle.quantize_e8(rng.normal(0, rng.uniform(*spread), (nvec, 8)) * rng.uniform(0.5, 2.0))
    return oracle.fields_of(y, c)


def _parse_tables(ft):
    ft = np.asarray(ft, np.uint8)
    b = int(ft[8:12].view(np.uint32)[0])
    ntab = int(ft[40:44].view(np.uint32)[0])
    desc = ft[48:48 + 8 * ntab].view(np.int32).reshape(ntab, 2)
    off = (48 + 8 * ntab + 15) // 16 * 16
    tabs = []
    for t in range(ntab):
        mn, A = int(desc[t, 0]), int(desc[t, 1])
        fr = ft[off:off + 2 * A].view(np.uint16).astype(np.int64)
        off += 2 * A
        tabs.append((mn, fr))
    return b, tabs


def _ideal_bits(fields, ft):
    b, tabs = _parse_tables(ft)
    bits = 0.0
    for k in range(9):
        for c in (0, 1):
            sel = fields[:, 0] == c if k else np.ones(len(fields), bool)
            t = 0 if k == 0 else 1 + 2 * (k - 1) + c
            mn, fr = tabs[t]
            vals = fields[sel, k] - mn
            bits += float(np.sum(b - np.log2(fr[vals])))
            if k == 0:
                break
    return bits


@pytest.mark.parametrize("b,V,nvec", [(9, 32, 32 * 7 + 5), (11, 33, 2000), (11, 512, 4096), (12, 100, 1003),
                                      (15, 1820, 5000), (10, 455, 455 * 3), (11, 1, 64)])
def test_round_trip_and_terminal_state(b, V, nvec):
    rng = np.random.default_rng(b * 1000 + V)
    f = _random_fields(rng, nvec)
    rows, cols = 1, 8 * nvec
    bl = oracle.encode_fields(f, rows, cols, np.ones(rows, np.float32), b, V)
    assert bl.ntiles == -(-nvec // V)
    # decode_fields checks internally that every lane ends at 2^15 and the cursor lands
    # exactly on the next tile's offset; it raises otherwise.
    g = oracle.decode_fields(bl.payload, bl.tile_index, bl.freq_tables, rows, cols)
    np.testing.assert_array_equal(g, f)
    # tiles decode independently: any tile range alone gives the same fields
    t0 = bl.ntiles // 2
    g2 = oracle.decode_fields(bl.payload, bl.tile_index, bl.freq_tables, rows, cols, t0, bl.ntiles)
    np.testing.assert_array_equal(g2, f[t0 * V:])
    # offsets are monotone, start at 0 and end at the payload size
    offs = bl.tile_index[0::33]
    assert offs[0] == 0 and offs[-1] == bl.payload.size and np.all(np.diff(offs.astype(np.int64)) >= 0)


def test_code_length_near_ideal():
    rng = np.random.default_rng(5)
    nvec = 40000
    f = _random_fields(rng, nvec, spread=(2.0, 8.0))
    for b, V in ((11, 1820), (12, 455), (9, 64)):
        bl = oracle.encode_fields(f, 1, 8 * nvec, np.ones(1, np.float32), b, V)
        ideal = _ideal_bits(f, bl.freq_tables)
        bits = 16.0 * bl.payload.size
        # the 32 terminal states of a tile hold up to 16 bits each of the message
        assert ideal - 512 * bl.ntiles - 64 <= bits <= ideal * 1.002 + 64, (b, V, bits, ideal)


def test_single_symbol_tables_consume_nothing():
    nvec = 3000
    f = np.zeros((nvec, 9), np.int32)      # every vector is the origin: all tables have A = 1, f = M
    bl = oracle.encode_fields(f, 1, 8 * nvec, np.ones(1, np.float32), 11, 512)
    assert bl.payload.size == 0
    assert np.all(bl.tile_index.reshape(-1)[:-1].reshape(-1, 33)[:, 1:] == 1 << 15)
    g = oracle.decode_fields(bl.payload, bl.tile_index, bl.freq_tables, 1, 8 * nvec)
    np.testing.assert_array_equal(g, f)


def test_full_alphabet_at_capacity():
    # a coordinate table whose alphabet is exactly 2^b: every symbol has f = 1
    b = 9
    M = 1 << b
    nvec = 4 * M
    rng = np.random.default_rng(6)
    z = np.zeros((nvec, 8), np.float64)
    z[:, 0] = np.tile(np.arange(M), 4) - M // 2
    z[:, 7] = z.sum(axis=1) % 2
    f = oracle.fields_of(z, np.zeros(nvec, np.int32))
    bl = oracle.encode_fields(f, 1, 8 * nvec, np.ones(1, np.float32), b, 96)
    _, tabs = _parse_tables(bl.freq_tables)
    assert tabs[1][1].size == M and np.all(tabs[1][1] == 1)
    g = oracle.decode_fields(bl.payload, bl.tile_index, bl.freq_tables, 1, 8 * nvec)
    np.testing.assert_array_equal(g, f)
    # one coordinate alphabet wider than 2^b is refused
    z[0, 0] = M
    z[:, 7] = z[:, :7].sum(axis=1) % 2
    f = oracle.fields_of(z, np.zeros(nvec, np.int32))
    with pytest.raises(ValueError):
        oracle.encode_fields(f, 1, 8 * nvec, np.ones(1, np.float32), b, 96)


def test_empty_coset_tables():
    rng = np.random.default_rng(7)
    nvec = 2000
    y, c = oracle.quantize_e8(rng.normal(0, 3, (nvec, 8)))
    z = np.rint(y - 0.5 * c[:, None])
    z[:, 7] += z.sum(axis=1) % 2
    f = oracle.fields_of(z, np.zeros(nvec, np.int32))
    bl = oracle.encode_fields(f, 1, 8 * nvec, np.ones(1, np.float32), 11, 300)
    _, tabs = _parse_tables(bl.freq_tables)
    assert all(tabs[1 + 2 * k + 1][1].size == 0 for k in range(8))   # c = 1 tables are empty
    g = oracle.decode_fields(bl.payload, bl.tile_index, bl.freq_tables, 1, 8 * nvec)
    np.testing.assert_array_equal(g, f)


def test_planted_faults_are_detected():
    rng = np.random.default_rng(8)
    nvec = 3000
    f = _random_fields(rng, nvec)
    bl = oracle.encode_fields(f, 1, 8 * nvec, np.ones(1, np.float32), 11, 512)
    args = (1, 8 * nvec)
    # a flipped payload word
    p = bl.payload.copy()
    p[len(p) // 2] ^= 0x5A5A
    with pytest.raises(ValueError):
        oracle.decode_fields(p, bl.tile_index, bl.freq_tables, *args)
    # a state below 2^15
    t = bl.tile_index.copy()
    t[1] = 5
    with pytest.raises(ValueError):
        oracle.decode_fields(bl.payload, t, bl.freq_tables, *args)
    # an offset past the payload
    t = bl.tile_index.copy()
    t[33] = t[-1] + 100
    with pytest.raises(ValueError):
        oracle.decode_fields(bl.payload, t, bl.freq_tables, *args)
    # frequencies that no longer sum to 2^b
    ft = bl.freq_tables.copy()
    ft[-2:] = 0
    with pytest.raises(ValueError):
        oracle.decode_fields(bl.payload, bl.tile_index, ft, *args)
    # b out of range
    ft = bl.freq_tables.copy()
    ft[8:12] = np.array([16], np.uint32).view(np.uint8)
    with pytest.raises(ValueError):
        oracle.decode_fields(bl.payload, bl.tile_index, ft, *args)
