"""A package loaded straight to the GPU decodes to the oracle's values."""
import numpy as np
import pytest

import dit_weight_compression_ep_b200 as ep
from dit_weight_compression_ep_b200 import synth
from gpu_util import assert_parity, oracle_decode, to_raw

pytestmark = pytest.mark.gpu


def test_load_package_to_device_and_decode(tmp_path):
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dit_weight_compression_ep_b200 import build

    build.build()
    rng = np.random.default_rng(8)
    blobs = {"a": ep.encode_tensor(synth.generate(synth.small_fp32(seed=9)), 4.0),
             "b": ep.encode_tensor((rng.standard_normal((33, 1001)) * 0.02).astype(np.float32), 8.0)}
    path = str(tmp_path / "pkg.safetensors")
    ep.save_package(path, blobs)
    dev = ep.load_package_to_device(path)
    for name, blob in blobs.items():
        out = ep.decode_tensor(dev[name], ep.BF16)
        assert ep.decode_status() == 0
        assert_parity(to_raw(out), oracle_decode(blob, ep.BF16), ep.BF16, name)


def test_device_blob_round_trips_to_host():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    blob = ep.encode_tensor(synth.generate(synth.small_fp32(seed=10)), 5.0)
    back = ep.DeviceBlob(blob).to_host()
    np.testing.assert_array_equal(back.payload[:blob.payload_words], blob.payload[:blob.payload_words])
    np.testing.assert_array_equal(back.tile_index, blob.tile_index)
    assert (back.payload_words, back.s, back.stored_bytes) == (blob.payload_words, blob.s, blob.stored_bytes)
