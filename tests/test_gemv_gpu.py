"""ep_decode_gemv: a linear layer on a few tokens whose weight is decoded inside the product
(EntroPack paper §4.3 and Fig. 5: the weight is reconstructed on demand for the matmul).

The reference is the oracle's float64 product of its own BF16 decode of the weight
(`oracle.linear`) with the BF16 activations widened exactly, and the tolerance is the oracle's
float32-accumulation bound (`oracle.linear_tolerance`, gamma_K sum|x w|: any order of float32
additions, the atomic adds included) with no output rounding beyond float32.  Cases: every token count (1, 2, 4, 8), the
packed (b = 11), two-level (b = 12) and bucketed (b = 13) tables, widths whose rows do not end
on a round of 32 vectors, per-call and prepared tables, several tiles per row and several rows
per tile, and the 3840x10240 headline on sampled rows.
"""
import numpy as np
import pytest

import oracle
import dit_weight_compression_ep_b200 as ep
from dit_weight_compression_ep_b200 import synth
from gpu_util import oracle_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dit_weight_compression_ep_b200 import build

    build.build()


def _x(ntok, cols, seed):
    import torch

    g = torch.Generator(device="cpu").manual_seed(seed)
    return (torch.randn(ntok, cols, generator=g) * 0.5).to(torch.bfloat16).cuda()


def _bf16_weights(blob, t0=0, t1=None):
    """The oracle's BF16 decode (written from the format definition), widened to float64."""
    bits = np.asarray(oracle_decode(blob, ep.BF16, t0, t1), np.uint16).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


def _check(blob, x, y, rows_sel=None):
    """y against the oracle's product on the whole matrix, or on the rows rows_sel."""
    xs = x.cpu().float().numpy().astype(np.float64)  # BF16 widens to float64 exactly
    got = y.cpu().numpy().astype(np.float64)
    if rows_sel is None:
        W = _bf16_weights(blob).reshape(blob.rows, blob.cols)
        want, tol = oracle.linear(W, xs), oracle.linear_tolerance(W, xs, 0.0)
        bad = np.abs(got - want) > tol
        assert not bad.any(), f"{bad.sum()} of {bad.size} outside the bound; worst {np.abs(got - want)[bad].max()}"
        return
    per = 8 * blob.V
    for r in rows_sel:
        e0, e1 = r * blob.cols, (r + 1) * blob.cols
        t0, t1 = e0 // per, (e1 - 1) // per + 1
        flat = _bf16_weights(blob, t0, t1)
        w = flat[e0 - t0 * per:e1 - t0 * per][None, :]
        want, tol = oracle.linear(w, xs), oracle.linear_tolerance(w, xs, 0.0)
        assert np.all(np.abs(got[:, [r]] - want) <= tol), f"row {r}"


@pytest.mark.parametrize("ntok", [1, 2, 4, 8])
def test_every_token_count_small_matrix(ntok):
    blob = ep.encode_tensor(synth.generate(synth.small_fp32()), 4.0, prob_bits=11, tile_vectors=100)
    db = ep.DeviceBlob(blob)
    x = _x(ntok, blob.cols, ntok)
    y = ep.decode_gemv(db, x)
    assert ep.decode_status() == 0
    _check(blob, x, y)
    y2 = ep.decode_gemv(db, x, lut=ep.prepare_lut(db))
    assert ep.decode_status() == 0
    _check(blob, x, y2)


@pytest.mark.parametrize("rows,cols,bpp,b,V", [(300, 1000, 4.0, 11, 455), (96, 4096, 8.0, 12, 455),
                                               (64, 2048, 7.5, 13, 100), (1024, 4096, 3.0, 11, 1820),
                                               (17, 8, 5.0, 11, 32)])
def test_table_formats_and_shapes(rows, cols, bpp, b, V):
    rng = np.random.default_rng(rows + cols)
    W = (rng.standard_t(5, (rows, cols)) * 0.02 * np.exp(rng.normal(0, 0.4, (rows, 1)))).astype(np.float32)
    if b >= 12:
        W[3, 5] = 1.5  # a wide alphabet
    blob = ep.encode_tensor(W, bpp, prob_bits=b, tile_vectors=V)
    db = ep.DeviceBlob(blob)
    for ntok in (1, 8):
        x = _x(ntok, cols, rows * ntok)
        y = ep.decode_gemv(db, x)
        assert ep.decode_status() == 0
        _check(blob, x, y)


def test_headline_sampled_rows_prepared_table():
    blob = ep.encode_tensor(synth.generate(synth.headline()), 4.0)
    db = ep.DeviceBlob(blob)
    lut = ep.prepare_lut(db)
    x = _x(4, blob.cols, 7)
    y = ep.decode_gemv(db, x, lut=lut)
    assert ep.decode_status() == 0
    rng = np.random.default_rng(3)
    _check(blob, x, y, rows_sel=sorted(set([0, blob.rows - 1] + [int(r) for r in rng.choice(blob.rows, 10)])))


def test_refusals_on_the_host():
    import torch

    blob = ep.encode_tensor(synth.generate(synth.small_fp32()), 4.0)
    db = ep.DeviceBlob(blob)
    with pytest.raises(ep.EntroPackError):
        ep.decode_gemv(db, _x(3, blob.cols, 1))  # 3 tokens
    odd = ep.encode_tensor(np.ones((8, 12), np.float32) * 0.01, 4.0)
    with pytest.raises(ep.EntroPackError):
        ep.decode_gemv(ep.DeviceBlob(odd), torch.zeros((1, 12), dtype=torch.bfloat16, device="cuda"))  # width % 8
    with pytest.raises(ValueError):
        ep.decode_gemv(db, torch.zeros((1, blob.cols), dtype=torch.float32, device="cuda"))


def test_compressed_linear_matvec_with_bias():
    import torch

    blob = ep.encode_tensor(synth.generate(synth.small_fp32()), 4.0)
    db = ep.DeviceBlob(blob)
    bias = torch.linspace(-1, 1, blob.rows, device="cuda")
    lin = ep.CompressedLinear(db, "bf16", bias=bias)
    x = _x(2, blob.cols, 11)
    y = lin.matvec(x)
    assert ep.decode_status() == 0
    W = _bf16_weights(blob).reshape(blob.rows, blob.cols)
    xs = x.cpu().float().numpy().astype(np.float64)
    b = bias.cpu().numpy().astype(np.float64)
    want = oracle.linear(W, xs) + b
    # the product's bound, plus one float32 rounding of the bias add
    tol = oracle.linear_tolerance(W, xs, 0.0) + np.abs(want) * 2.0 ** -23
    assert np.all(np.abs(y.cpu().numpy().astype(np.float64) - want) <= tol)
    with pytest.raises(ValueError):
        lin.matvec(_x(3, blob.cols, 1))


@pytest.mark.parametrize("seed", range(6))
def test_random_shapes_rates_and_token_counts(seed):
    """Seeded random widths (multiples of 8), heights, rates, tile sizes and token counts, per-call
    and prepared tables, against the oracle's product."""
    rng = np.random.default_rng(900 + seed)
    rows, cols = int(rng.integers(1, 400)), 8 * int(rng.integers(1, 300))
    bpp = float(rng.choice([2.3, 3.0, 4.0, 5.0, 6.0, 8.0]))
    V = int(rng.choice([32, 33, 100, 455, 910]))
    W = (rng.standard_t(6, (rows, cols)) * 0.02 * np.exp(rng.normal(0, 0.3, (rows, 1)))).astype(np.float32)
    blob = ep.encode_tensor(W, bpp, tile_vectors=V)
    db = ep.DeviceBlob(blob)
    ntok = int(rng.choice(ep.GEMV_TOKENS))
    x = _x(ntok, cols, 1000 + seed)
    lut = ep.prepare_lut(db) if seed % 2 else None
    y = ep.decode_gemv(db, x, lut=lut)
    assert ep.decode_status() == 0
    _check(blob, x, y)
