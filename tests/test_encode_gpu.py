"""The GPU encoder (ep_encode_tensor_gpu) against the CPU packer, byte for byte: payload, tile
records, tables, row scales, the chosen scale and the stored rate.  The packer is itself
byte-identical to the oracle's encoder (test_packer.py), so this pins the GPU encoder to the
oracle; its streams then decode to the oracle's values."""
import numpy as np
import pytest

import dit_weight_compression_ep_b200 as ep
from dit_weight_compression_ep_b200 import synth
from gpu_util import assert_parity, oracle_decode, to_raw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dit_weight_compression_ep_b200 import build

    build.build()
    ep.lib()


def _same(W, bpp, **kw):
    import torch

    cpu = ep.encode_tensor(W, bpp, **kw)
    gpu = ep.encode_tensor_gpu(torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda(), bpp, **kw)
    assert (gpu.rows, gpu.cols, gpu.b, gpu.V, gpu.ntiles) == (cpu.rows, cpu.cols, cpu.b, cpu.V, cpu.ntiles)
    assert gpu.s == cpu.s
    np.testing.assert_array_equal(gpu.freq_tables, cpu.freq_tables)
    np.testing.assert_array_equal(gpu.row_scales.view(np.uint32), cpu.row_scales.view(np.uint32))
    np.testing.assert_array_equal(gpu.tile_index, cpu.tile_index)
    assert gpu.payload_words == cpu.payload_words
    np.testing.assert_array_equal(gpu.payload, cpu.payload)
    assert gpu.stored_bpp == cpu.stored_bpp
    return gpu


@pytest.mark.parametrize("bpp", [2.3, 3.0, 4.0, 5.0, 6.0, 8.0])
def test_small_matrix_every_rate(bpp):
    _same(synth.generate(synth.small_fp32()), bpp)


@pytest.mark.parametrize("rows,cols,V", [(3, 5, 2), (17, 1001, 100), (1, 8, 32), (300, 1, 33), (64, 1020, 1820),
                                         (40, 4097, 455)])
def test_shapes_and_ragged_widths(rows, cols, V):
    rng = np.random.default_rng(rows * 7 + cols)
    W = (rng.standard_t(5, (rows, cols)) * 0.02).astype(np.float32)
    _same(W, 4.0, tile_vectors=V)


@pytest.mark.parametrize("b", [9, 12, 13, 15])
def test_fixed_precisions_and_escalation(b):
    rng = np.random.default_rng(b)
    W = (rng.standard_normal((96, 1024)) * 0.02 * np.exp(rng.normal(0, 0.4, (96, 1)))).astype(np.float32)
    W[5, 7] = 3.0  # an outlier: wide alphabets (the b escalation or the coarsening path)
    _same(W, 7.5 if b >= 12 else 4.0, prob_bits=b, tile_vectors=100)


def test_zero_rows_signed_zeros_and_options():
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((64, 512)) * 0.05).astype(np.float32)
    W[3] = 0
    W[10] = -W[10]
    _same(W, 3.0, tile_vectors=64, seed=99, sample_vectors=1000, search_steps=9)
    vals, _ = synth.to_int8_container(synth.generate(synth.small_fp32(seed=5)))
    _same(vals, 5.0, has_container_scales=True)


def test_full_size_headline_and_decode():
    """The 3840x10240 headline at 4 bpp: the same blob, and its GPU decode equals the oracle on
    sampled tiles."""
    W = synth.generate(synth.headline())
    blob = _same(W, 4.0)
    out = to_raw(ep.decode_tensor(ep.DeviceBlob(blob), ep.BF16)).reshape(-1)
    assert ep.decode_status() == 0
    rng = np.random.default_rng(5)
    per = 8 * blob.V
    for t in sorted(set([0, blob.ntiles - 1] + list(rng.choice(blob.ntiles, 6, replace=False)))):
        lo, hi = t * per, min((t + 1) * per, blob.rows * blob.cols)
        assert_parity(out[lo:hi], oracle_decode(blob, ep.BF16, t, t + 1), ep.BF16, f"tile {t}")


@pytest.mark.parametrize("kind,bpp", [("qkv", 8.0), ("out", 2.3), ("down", 6.0)])
def test_dit_layers(kind, bpp):
    _same(synth.generate(synth.dit_stack_layer(1, kind)), bpp)


@pytest.mark.parametrize("K,sweeps,rows,cols", [(2, 1, 64, 512), (4, 2, 96, 1024), (5, 1, 17, 1001), (8, 3, 40, 256)])
def test_per_row_refinement(K, sweeps, rows, cols):
    """App. C.2 on the GPU: the packer's bytes for every candidate count and sweep count."""
    rng = np.random.default_rng(K * 10 + sweeps)
    W = np.empty((rows, cols), np.float32)
    for r in range(rows):
        W[r] = rng.standard_t([2.5, 4, 8, 30][r % 4], cols) * 0.02 * np.exp(rng.normal(0, 0.5))
    _same(W, 3.0, rdo_candidates=K, rdo_sweeps=sweeps, tile_vectors=200)


def test_per_row_refinement_full_size():
    _same(synth.generate(synth.headline()), 3.0, rdo_candidates=4)


@pytest.mark.parametrize("bpp", [2.0, 8.0])
def test_llm_prefill_shape_with_outliers(bpp):
    """25600x5120 (131 M weights) with 0.05 % outliers at 10 sigma: wide alphabets, b = 12 at
    8 bpp; the same blob as the packer."""
    _same(synth.generate(synth.llm_prefill(False)), bpp)


def test_host_pointer_is_refused_before_any_launch():
    """A host buffer passed as the weights: refused on the host (no kernel reads it)."""
    import ctypes as C

    W = np.zeros((16, 64), np.float32)
    o = ep._lib._Opts(0, 0, 0, 0, 0, 0, 0, 0, 0)
    out = C.POINTER(ep._lib._Blob)()
    rc = ep.lib().ep_encode_tensor_gpu(None, W.ctypes.data, 16, 64, 4.0, C.byref(o), C.byref(out))
    assert rc == ep._lib.STATUS_CODES["EP_EINVAL"]
    # the device still works
    import torch

    _same(np.ones((4, 16), np.float32) * 0.01, 4.0)
    torch.cuda.synchronize()


def _host_arrays(blob):
    """The stored arrays (payload words up to the final offset; the allocation padding is zero in both)."""
    return (blob.payload[:blob.payload_words], blob.tile_index, blob.freq_tables, blob.row_scales.view(np.uint32))


@pytest.mark.parametrize("rows,cols,bpp", [(256, 512, 4.0), (17, 1001, 8.0), (3, 5, 2.3)])
def test_device_output_equals_the_packer_and_decodes(rows, cols, bpp):
    """ep_encode_tensor_gpu_device: the packer's bytes, left on the GPU, decoded there to the
    oracle's values."""
    import torch

    rng = np.random.default_rng(rows + cols)
    W = (rng.standard_t(5, (rows, cols)) * 0.02).astype(np.float32)
    cpu = ep.encode_tensor(W, bpp)
    db = ep.encode_tensor_gpu_to_device(torch.from_numpy(W).cuda(), bpp)
    got = db.to_host()
    for a, b in zip(_host_arrays(got), _host_arrays(cpu)):
        np.testing.assert_array_equal(a, b)
    assert (got.s, got.stored_bpp, got.b, got.V, got.ntiles) == (cpu.s, cpu.stored_bpp, cpu.b, cpu.V, cpu.ntiles)
    out = ep.decode_tensor(db, ep.BF16)
    assert ep.decode_status() == 0
    assert_parity(to_raw(out), oracle_decode(cpu, ep.BF16), ep.BF16, "device blob")


@pytest.mark.parametrize("rows,cols", [(3840, 3840), (33, 101)])
def test_bf16_weights_encode_like_their_float32_values(rows, cols):
    """bfloat16 input is widened exactly: the bytes of the packer on the float32 values."""
    import torch

    W = torch.from_numpy(synth.generate(synth.dit_attn_proj())[:rows, :cols].copy()).to(torch.bfloat16).cuda()
    ref = ep.encode_tensor(W.float().cpu().numpy(), 5.0)
    got = ep.encode_tensor_gpu(W, 5.0)
    for a, b in zip(_host_arrays(got), _host_arrays(ref)):
        np.testing.assert_array_equal(a, b)
    assert got.s == ref.s
