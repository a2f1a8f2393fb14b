"""The library's CPU packer (ep_encode_tensor) against the oracle's encoder:
byte-identical stored representation for the same input and options, for any
thread count; and the oracle decodes the packer's output exactly."""
import numpy as np
import pytest

import oracle
import dit_weight_compression_ep_b200 as ep
from dit_weight_compression_ep_b200 import build, synth


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def _same(ob, lb):
    assert lb.b == ob.b and lb.V == ob.V and lb.ntiles == ob.ntiles
    assert lb.payload_words == ob.payload.size
    np.testing.assert_array_equal(lb.payload[:lb.payload_words], ob.payload)
    assert lb.payload.size % 8 == 0 and np.all(lb.payload[lb.payload_words:] == 0)
    np.testing.assert_array_equal(lb.tile_index, ob.tile_index)
    np.testing.assert_array_equal(lb.freq_tables, ob.freq_tables)
    np.testing.assert_array_equal(lb.row_scales.view(np.uint32), ob.row_scales.view(np.uint32))
    assert lb.stored_bytes == ob.stored_bytes
    assert lb.s == ob.s


def _mixed_rows(seed, rows=160, cols=512):
    """Rows with different tails and scales (where the per-row refinement changes choices)."""
    rng = np.random.default_rng(seed)
    W = np.empty((rows, cols), np.float32)
    for r in range(rows):
        W[r] = rng.standard_t([2.5, 4, 8, 30][r % 4], cols) * 0.02 * np.exp(rng.normal(0, 0.5))
    return W


CASES = [
    ("small fp32", lambda: synth.generate(synth.small_fp32()), 4.0, dict(prob_bits=12, tile_vectors=512)),
    ("t5 2bpp", lambda: (np.random.default_rng(1).standard_t(5, (300, 512)) * 0.02).astype(np.float32), 2.0, {}),
    ("gauss 3bpp", lambda: (np.random.default_rng(2).standard_normal((256, 1024)) * 0.02).astype(np.float32), 3.0,
     {}),
    ("gauss 6bpp", lambda: (np.random.default_rng(3).standard_normal((128, 2048)) * 0.02).astype(np.float32), 6.0,
     {}),
    ("t6 8bpp", lambda: (np.random.default_rng(4).standard_t(6, (256, 768)) * 0.02).astype(np.float32), 8.0, {}),
    ("tiny cols", lambda: (np.random.default_rng(5).standard_normal((500, 8)) * 0.1).astype(np.float32), 4.0, {}),
    ("one row", lambda: (np.random.default_rng(6).standard_normal((1, 4096)) * 0.1).astype(np.float32), 5.0,
     dict(tile_vectors=33)),
    ("container", lambda: synth.to_int8_container(
        (np.random.default_rng(7).standard_normal((64, 512)) * 0.02).astype(np.float32))[0], 5.0,
     dict(has_container_scales=True)),
    ("small sample", lambda: (np.random.default_rng(8).standard_normal((400, 256)) * 0.02).astype(np.float32), 4.0,
     dict(sample_vectors=500, seed=77, search_steps=9)),
    ("ragged 1001", lambda: (np.random.default_rng(12).standard_t(5, (90, 1001)) * 0.02).astype(np.float32), 4.0, {}),
    ("ragged 60", lambda: (np.random.default_rng(13).standard_normal((300, 60)) * 0.02).astype(np.float32), 6.0,
     dict(tile_vectors=50)),
    ("ragged 5", lambda: (np.random.default_rng(14).standard_normal((700, 5)) * 0.02).astype(np.float32), 3.0, {}),
    ("rdo ragged 517", lambda: _mixed_rows(15, cols=517), 3.0, dict(rdo_candidates=5)),
    ("rdo K=5", lambda: _mixed_rows(9), 3.0, dict(rdo_candidates=5)),
    ("rdo K=7 two sweeps 8bpp", lambda: _mixed_rows(10), 8.0, dict(rdo_candidates=7, rdo_sweeps=2)),
    ("rdo K=3 2bpp", lambda: _mixed_rows(11, rows=96), 2.0, dict(rdo_candidates=3)),
]


@pytest.mark.parametrize("name,make,bpp,kw", CASES, ids=[c[0] for c in CASES])
def test_packer_matches_oracle(name, make, bpp, kw):
    W = make()
    ob = oracle.encode(W, bpp, **kw)
    for threads in (1, 3, 0):
        lb = ep.encode_tensor(W, bpp, num_threads=threads, **kw)
        _same(ob, lb)


def test_packer_escalation_and_coarsening_match_oracle():
    rng = np.random.default_rng(6)
    W = (rng.standard_normal((256, 4096)) * 1e-3).astype(np.float32)
    hot = rng.choice(256, size=8, replace=False)
    for r in hot:
        W[r] = (rng.standard_normal(4096) * 1e-6).astype(np.float32)
        W[r, rng.integers(4096)] = 1.0
    kw = dict(sample_vectors=16, seed=1, prob_bits=12)
    ob = oracle.encode(W, 14.0, **kw)
    lb = ep.encode_tensor(W, 14.0, **kw)
    assert ob.b == 15
    _same(ob, lb)


def test_oracle_decodes_packer_output():
    W = synth.generate(synth.dit_attn_proj())[:512]
    lb = ep.encode_tensor(W, 5.0)
    f = oracle.decode_fields(lb.payload[:lb.payload_words], lb.tile_index, lb.freq_tables, lb.rows, lb.cols)
    assert f.shape == (lb.rows * lb.cols // 8, 9)
    out = oracle.decode(lb.payload[:lb.payload_words], lb.tile_index, lb.freq_tables, lb.row_scales, lb.rows,
                        lb.cols, oracle.FP32).reshape(W.shape)
    rel = np.linalg.norm(out - W) / np.linalg.norm(W)
    assert 0.0 < rel < 0.06
