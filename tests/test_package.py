"""Packages (a safetensors file and its JSON sidecar) round-trip the stored arrays exactly, read
back with plain safetensors, and report the package rate as 8 * sum(stored bytes) / sum(numel)."""
import json

import numpy as np
import pytest

import dit_weight_compression_ep_b200 as ep
from dit_weight_compression_ep_b200 import package, synth


@pytest.fixture(scope="module")
def blobs():
    from dit_weight_compression_ep_b200 import build

    build.build()
    rng = np.random.default_rng(5)
    W = (rng.standard_t(5, (40, 1001)) * 0.02).astype(np.float32)
    return {
        "dit_block0_qkv": ep.encode_tensor(synth.generate(synth.small_fp32()), 4.0),
        "ragged": ep.encode_tensor(W, 6.0, tile_vectors=100),
        "rdo": ep.encode_tensor(W, 3.0, rdo_candidates=3),
        "tiny": ep.encode_tensor(np.full((3, 5), 0.01, np.float32), 2.3),  # an empty payload
    }


def test_round_trip_and_sidecar(tmp_path, blobs):
    path = str(tmp_path / "model_4bpp.safetensors")
    side = package.save_package(path, blobs, extra={"note": "synthetic"})
    back = package.load_package(path)
    assert set(back) == set(blobs)
    for name, b in blobs.items():
        g = back[name]
        assert (g.rows, g.cols, g.b, g.V, g.ntiles, g.payload_words) == (b.rows, b.cols, b.b, b.V, b.ntiles,
                                                                        b.payload_words)
        np.testing.assert_array_equal(g.payload[:b.payload_words], b.payload[:b.payload_words])
        assert not g.payload[b.payload_words:].any() and g.payload.size % 8 == 0
        np.testing.assert_array_equal(g.tile_index, b.tile_index)
        np.testing.assert_array_equal(g.freq_tables, b.freq_tables)
        np.testing.assert_array_equal(g.row_scales.view(np.uint32), b.row_scales.view(np.uint32))
        assert (g.s, g.stored_bytes, g.stored_bpp) == (b.s, b.stored_bytes, b.stored_bpp)
    with open(tmp_path / "model_4bpp.json") as f:
        assert json.load(f) == json.loads(json.dumps(side))
    numel = sum(b.rows * b.cols for b in blobs.values())
    stored = sum(b.stored_bytes for b in blobs.values())
    assert side["bpp"] == pytest.approx(8.0 * stored / numel) and side["extra"] == {"note": "synthetic"}
    assert side["ratio_vs_bf16"] == pytest.approx(side["bpp"] / 16.0)


def test_plain_safetensors_reads_it(tmp_path, blobs):
    from safetensors.numpy import load_file

    path = str(tmp_path / "p.safetensors")
    package.save_package(path, blobs)
    t = load_file(path)
    assert t["ragged.tile_index"].dtype == np.uint32 and t["ragged.payload"].dtype == np.uint16
    assert t["ragged.freq_tables"].dtype == np.uint8 and t["ragged.row_scales"].dtype == np.float32
    np.testing.assert_array_equal(t["rdo.tile_index"], blobs["rdo"].tile_index)


def test_refusals(tmp_path, blobs):
    from safetensors.numpy import save_file

    with pytest.raises(ValueError):
        package.save_package(str(tmp_path / "x.safetensors"), {"a.b": blobs["tiny"]})
    other = str(tmp_path / "other.safetensors")
    save_file({"w": np.zeros(4, np.float32)}, other)
    with pytest.raises(ValueError):
        package.load_package(other)
