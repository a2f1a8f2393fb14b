"""The GPU encoder against the ORACLE's encoder, byte for byte, on the same input.

EntroPack paper §3.1 (the encode pipeline: row normalisation, the sampled scale search of
§3.4 and App. C.1, E8 quantisation, the row-scale refit of §3.5, the 17 tables of §3.6 and
App. A.3, tiled rANS of App. C.3) and App. C.2 (the per-row refinement).  The GPU encoder
shares host code with the CPU packer, so comparing it with the packer alone would compare
the product with itself; here every stored array and the chosen scale come from
``oracle.encode`` instead: payload words, tile records, table header and frequencies, row
scales, the scale s and the stored byte count.  Inputs stay at sizes the oracle encodes in a
second or less (at most 1024 x 4096), and span every target rate, ragged widths, fixed and
escalated precisions up to b = 15 (the coarsening path), container scales, the per-row
refinement with several candidate and sweep counts, device-resident output, and bfloat16
input.
"""
import numpy as np
import pytest

import oracle
import dit_weight_compression_ep_b200 as ep
from dit_weight_compression_ep_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dit_weight_compression_ep_b200 import build

    build.build()
    ep.lib()


def _stored(blob):
    """The stored arrays of a library blob (payload words up to the final offset)."""
    return (blob.payload[:blob.payload_words], blob.tile_index, blob.freq_tables, blob.row_scales.view(np.uint32))


def _assert_oracle_bytes(got, ob, what):
    assert (got.rows, got.cols, got.b, got.V, got.ntiles) == (ob.rows, ob.cols, ob.b, ob.V, ob.ntiles), what
    assert got.s == ob.s, f"{what}: scale {got.s!r} vs oracle {ob.s!r}"
    names = ("payload", "tile_index", "freq_tables", "row_scales")
    want = (ob.payload, ob.tile_index, ob.freq_tables, ob.row_scales.view(np.uint32))
    for name, a, b in zip(names, _stored(got), want):
        assert a.shape == b.shape, f"{what}: {name} shape {a.shape} vs oracle {b.shape}"
        bad = np.nonzero(a != b)[0]
        assert bad.size == 0, f"{what}: {name} differs from the oracle at {bad.size} positions, first {bad[:5]}"
    assert got.stored_bytes == ob.stored_bytes, what


def _gpu_host(W, bpp, **kw):
    import torch

    return ep.encode_tensor_gpu(torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda(), bpp, **kw)


def _gpu_device(W, bpp, **kw):
    import torch

    return ep.encode_tensor_gpu_to_device(torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda(), bpp,
                                          **kw).to_host()


def _t5_rows(seed, rows, cols, sigma=0.5):
    rng = np.random.default_rng(seed)
    return (rng.standard_t(5, (rows, cols)) * 0.02 * np.exp(rng.normal(0, sigma, (rows, 1)))).astype(np.float32)


def _mixed_rows(seed, rows, cols):
    """Rows with different tails and scales, where the per-row refinement changes its choices."""
    rng = np.random.default_rng(seed)
    W = np.empty((rows, cols), np.float32)
    for r in range(rows):
        W[r] = rng.standard_t([2.5, 4, 8, 30][r % 4], cols) * 0.02 * np.exp(rng.normal(0, 0.5))
    return W


@pytest.mark.parametrize("bpp", [2.3, 3.0, 4.0, 5.0, 6.0, 8.0])
def test_every_rate_host_and_device_output(bpp):
    W = _t5_rows(int(bpp * 10), 256, 1024)
    ob = oracle.encode(W, bpp)
    _assert_oracle_bytes(_gpu_host(W, bpp), ob, f"{bpp} bpp, host blob")
    _assert_oracle_bytes(_gpu_device(W, bpp), ob, f"{bpp} bpp, device blob")


@pytest.mark.parametrize("rows,cols,V", [(17, 1001, 100), (300, 60, 50), (40, 4097, 455), (700, 5, 0), (1, 8, 32),
                                         (3, 5, 2)])
def test_ragged_widths_and_tiny_shapes(rows, cols, V):
    W = _t5_rows(rows + cols, rows, cols)
    ob = oracle.encode(W, 4.0, tile_vectors=V)
    _assert_oracle_bytes(_gpu_host(W, 4.0, tile_vectors=V), ob, f"{rows}x{cols} V={V}")


@pytest.mark.parametrize("b", [9, 11, 12, 13, 15])
def test_fixed_precision_escalation_and_coarsening(b):
    """A far outlier widens the alphabets: b rises from the given start (App. C.1), and at b = 15
    the scale is coarsened until the alphabets fit."""
    rng = np.random.default_rng(b)
    W = (rng.standard_normal((96, 1024)) * 0.02 * np.exp(rng.normal(0, 0.4, (96, 1)))).astype(np.float32)
    W[5, 7] = 3.0
    bpp = 7.5 if b >= 12 else 4.0
    ob = oracle.encode(W, bpp, prob_bits=b, tile_vectors=100)
    assert ob.b >= b
    _assert_oracle_bytes(_gpu_host(W, bpp, prob_bits=b, tile_vectors=100), ob, f"b={b}")


@pytest.mark.parametrize("bpp,b_end", [(9.0, 14), (10.0, 15)])
def test_escalation_from_12(bpp, b_end):
    """One far outlier per 32768-wide row: the full-tensor alphabets outgrow 2^b, so the search
    escalates b from 12 to 14 (9 bpp) and to 15 (10 bpp)."""
    rng = np.random.default_rng(21)
    W = (rng.standard_normal((32, 32768)) * 0.01).astype(np.float32)
    W[np.arange(32), rng.integers(0, 32768, 32)] = rng.choice([-1.0, 1.0], 32) * 4.0
    kw = dict(prob_bits=12, tile_vectors=455)
    ob = oracle.encode(W, bpp, **kw)
    assert ob.b == b_end
    _assert_oracle_bytes(_gpu_host(W, bpp, **kw), ob, f"escalation to {b_end}")
    _assert_oracle_bytes(_gpu_device(W, bpp, **kw), ob, f"escalation to {b_end}, device blob")


def test_coarsening_at_b15():
    """Rows the sample never sees carry an alphabet wider than 2^15 at the searched scale: b
    climbs to 15 and the scale is coarsened until the alphabets fit (App. C.1)."""
    rng = np.random.default_rng(6)
    W = (rng.standard_normal((256, 4096)) * 1e-3).astype(np.float32)
    for r in rng.choice(256, size=8, replace=False):
        W[r] = (rng.standard_normal(4096) * 1e-6).astype(np.float32)
        W[r, rng.integers(4096)] = 1.0
    kw = dict(sample_vectors=16, seed=1, prob_bits=12)
    ob = oracle.encode(W, 14.0, **kw)
    assert ob.b == 15
    _assert_oracle_bytes(_gpu_host(W, 14.0, **kw), ob, "coarsening")
    _assert_oracle_bytes(_gpu_device(W, 14.0, **kw), ob, "coarsening, device blob")


@pytest.mark.parametrize("kind", ["int8", "e4m3", "uint8"])
def test_container_values_and_scales(kind):
    src = _t5_rows(31, 192, 1024, sigma=0.3)
    if kind == "int8":
        vals, _ = synth.to_int8_container(src)
    elif kind == "e4m3":
        vals, _ = synth.to_e4m3_container(src)
    else:
        vals, _ = synth.to_uint8_container(src)
    cs = kind != "uint8"
    ob = oracle.encode(vals, 5.0, has_container_scales=cs)
    _assert_oracle_bytes(_gpu_host(vals, 5.0, has_container_scales=cs), ob, kind)


def test_zero_rows_signed_zeros_and_search_options():
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((64, 512)) * 0.05).astype(np.float32)
    W[3] = 0
    W[10] = -W[10]
    W[20] = -0.0
    kw = dict(tile_vectors=64, seed=99, sample_vectors=1000, search_steps=9)
    _assert_oracle_bytes(_gpu_host(W, 3.0, **kw), oracle.encode(W, 3.0, **kw), "options")


@pytest.mark.parametrize("K,sweeps,bpp,rows,cols", [(3, 2, 3.0, 160, 512), (5, 1, 3.0, 90, 1001),
                                                    (4, 2, 8.0, 128, 768), (9, 3, 2.3, 64, 1024)])
def test_per_row_refinement(K, sweeps, bpp, rows, cols):
    """App. C.2 on the GPU (candidates, sweeps, the lambda bisection and the rebuilt tables)
    against the oracle's refinement."""
    W = _mixed_rows(K * 100 + sweeps, rows, cols)
    kw = dict(rdo_candidates=K, rdo_sweeps=sweeps, tile_vectors=200)
    ob = oracle.encode(W, bpp, **kw)
    _assert_oracle_bytes(_gpu_host(W, bpp, **kw), ob, f"RDO K={K} sweeps={sweeps}")
    _assert_oracle_bytes(_gpu_device(W, bpp, **kw), ob, f"RDO K={K} sweeps={sweeps}, device blob")


def test_largest_oracle_case_1024x4096():
    W = _t5_rows(77, 1024, 4096)
    ob = oracle.encode(W, 4.0)
    _assert_oracle_bytes(_gpu_host(W, 4.0), ob, "1024x4096")
    _assert_oracle_bytes(_gpu_device(W, 4.0), ob, "1024x4096, device blob")


@pytest.mark.parametrize("rows,cols,bpp", [(512, 2048, 5.0), (33, 101, 4.0)])
def test_bfloat16_input(rows, cols, bpp):
    """bfloat16 weights on the GPU are widened exactly; the oracle encodes the widened values."""
    import torch

    W = torch.from_numpy(_t5_rows(rows, rows, cols)).to(torch.bfloat16).cuda()
    ob = oracle.encode(W.float().cpu().numpy(), bpp)
    _assert_oracle_bytes(ep.encode_tensor_gpu(W, bpp), ob, "bf16 in, host blob")
    _assert_oracle_bytes(ep.encode_tensor_gpu_to_device(W, bpp).to_host(), ob, "bf16 in, device blob")
