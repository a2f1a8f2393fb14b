"""Pins of the tile layout and the stored-size accounting against the pages' own numbers."""
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    out = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            out.append([float(v) for v in line.split()])
    return out


def test_table5_tile_metadata_closed_form():
    nvec = 10240 * 3840 // 8
    for tgt, S, V, T, b, meta in _rows("table5_tile_metadata.txt"):
        assert oracle.default_tile_symbols(tgt) == S
        assert oracle.tile_vectors(int(S)) == V
        assert -(-nvec // int(V)) == T
        assert oracle.tile_metadata_bytes(int(T)) == meta
        # App. C.1: the starting b is 11 at or below 7 bpp, else 12
        assert (11 if tgt <= 7 else 12) == b


def test_tile_vectors_floor():
    # V = max(32, floor(S/9)) (App. C.3)
    assert oracle.tile_vectors(100) == 32
    assert oracle.tile_vectors(9 * 32) == 32
    assert oracle.tile_vectors(9 * 33 + 8) == 33


def test_stored_bytes_closed_form():
    rng = np.random.default_rng(1)
    W = (rng.standard_normal((96, 256)) * 0.02).astype(np.float32)
    bl = oracle.encode(W, 4.0, tile_vectors=100)
    ntab = 17
    tables = (48 + 8 * ntab + 15) // 16 * 16 + 2 * sum(
        int(v) for v in bl.freq_tables[48:48 + 8 * ntab].view(np.int32).reshape(ntab, 2)[:, 1])
    assert tables == bl.freq_tables.size
    expect = 2 * bl.payload.size + (bl.ntiles * 132 + 4) + tables + 4 * 96
    assert bl.stored_bytes == expect
    assert abs(bl.stored_bpp - 8 * expect / W.size) < 1e-12
    bl2 = oracle.encode(W, 4.0, tile_vectors=100, has_container_scales=True)
    assert bl2.stored_bytes - 2 * bl2.payload.size - bl2.freq_tables.size - (bl2.ntiles * 132 + 4) == 8 * 96
