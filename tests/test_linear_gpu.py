"""CompressedLinear: a linear layer whose weight is decoded by the library before each product.
Each route's output equals, bit for bit, the same library GEMM run on the weight the oracle
decodes (the decoded weight is bit-exact and the GEMM sees the same operands)."""
import numpy as np
import pytest

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
    ep.lib()
    ep.decode_status()


def _oracle_weight(blob, dt, torch_dtype):
    import torch

    raw = np.ascontiguousarray(oracle_decode(blob, dt)).reshape(blob.rows, blob.cols)
    t = torch.from_numpy(raw.view(np.int16 if raw.itemsize == 2 else np.int8).copy()).cuda()
    return t.view(torch_dtype)


def test_bf16_route():
    import torch

    W = synth.generate(synth.small_fp32(seed=3))  # 256 x 512
    blob = ep.encode_tensor(W, 4.0)
    lin = ep.CompressedLinear(ep.DeviceBlob(blob), "bf16")
    x = (torch.randn(64, 512, device="cuda") * 0.5).to(torch.bfloat16)
    bias = torch.randn(256, device="cuda").to(torch.bfloat16)
    y = lin(x)
    ref = torch.matmul(x, _oracle_weight(blob, ep.BF16, torch.bfloat16).t())
    assert ep.decode_status() == 0
    assert torch.equal(y, ref)
    lin.bias = bias
    assert torch.equal(lin(x), ref + bias)


def test_fp8_and_int8_routes():
    import torch

    W = synth.generate(synth.small_fp32(seed=4))
    x = torch.randn(64, 512, device="cuda") * 0.5
    xs = (torch.rand(64, 1, device="cuda") + 0.5)
    vals, wsc = synth.to_e4m3_container(W)
    blob = ep.encode_tensor(vals, 5.0, has_container_scales=True)
    lin = ep.CompressedLinear(ep.DeviceBlob(blob), "fp8", weight_scales=wsc)
    x8 = x.clamp(-448, 448).to(torch.float8_e4m3fn)
    ws = torch.from_numpy(wsc).cuda().view(1, -1)
    ref = torch._scaled_mm(x8, _oracle_weight(blob, ep.FP8_E4M3, torch.float8_e4m3fn).t(), scale_a=xs, scale_b=ws,
                           out_dtype=torch.bfloat16)
    assert torch.equal(lin(x8, xs), ref)
    vali, wsci = synth.to_int8_container(W)
    blobi = ep.encode_tensor(vali, 5.0, has_container_scales=True)
    lini = ep.CompressedLinear(ep.DeviceBlob(blobi), "int8", weight_scales=wsci)
    xi = x.mul(20).round().clamp(-127, 127).to(torch.int8)
    wsi = torch.from_numpy(wsci).cuda().view(1, -1)
    refi = (torch._int_mm(xi, _oracle_weight(blobi, ep.INT8, torch.int8).t()).float() * xs * wsi).to(torch.bfloat16)
    assert torch.equal(lini(xi, xs), refi)
    assert ep.decode_status() == 0


def test_layers_sharing_one_scratch():
    import torch

    blobs = [ep.encode_tensor(synth.generate(synth.small_fp32(seed=s)), 4.0) for s in (5, 6)]
    scratch = torch.empty(256 * 512, dtype=torch.bfloat16, device="cuda")
    lins = [ep.CompressedLinear(ep.DeviceBlob(b), "bf16", scratch=scratch) for b in blobs]
    x = (torch.randn(32, 512, device="cuda") * 0.5).to(torch.bfloat16)
    for b, lin in zip(blobs, lins):
        assert torch.equal(lin(x), torch.matmul(x, _oracle_weight(b, ep.BF16, torch.bfloat16).t()))
    with pytest.raises(ValueError):
        ep.CompressedLinear(ep.DeviceBlob(blobs[0]), "fp8")  # no container scales
    with pytest.raises(ValueError):
        ep.CompressedLinear(ep.DeviceBlob(blobs[0]), "bf16", scratch=torch.empty(10, dtype=torch.bfloat16,
                                                                                  device="cuda"))


def test_group_decode_then_calls():
    """A LinearGroup decodes its layers' weights in one batch launch; the calls with decode=False
    give the same bits as calls that decode one layer at a time."""
    import torch

    blobs = [ep.encode_tensor(synth.generate(synth.small_fp32(seed=s)), bpp) for s, bpp in ((7, 3.0), (8, 5.0),
                                                                                               (9, 8.0))]
    lins = [ep.CompressedLinear(ep.DeviceBlob(b), "bf16") for b in blobs]
    group = ep.LinearGroup(lins)
    x = (torch.randn(48, 512, device="cuda") * 0.5).to(torch.bfloat16)
    for lin in lins:
        lin.scratch.zero_()
    group.run()
    got = [lin(x, decode=False) for lin in lins]
    want = [torch.matmul(x, _oracle_weight(b, ep.BF16, torch.bfloat16).t()) for b in blobs]
    assert ep.decode_status() == 0
    for g, w in zip(got, want):
        assert torch.equal(g, w)
    with pytest.raises(ValueError):
        ep.LinearGroup([lins[0], lins[0]])  # one scratch twice
    # two views of one buffer at different offsets that overlap by a few elements
    n = blobs[0].rows * blobs[0].cols
    buf = torch.empty(2 * n - 16, dtype=torch.bfloat16, device="cuda")
    a = ep.CompressedLinear(ep.DeviceBlob(blobs[0]), "bf16", scratch=buf[:n])
    b = ep.CompressedLinear(ep.DeviceBlob(blobs[1]), "bf16", scratch=buf[n - 16:])
    with pytest.raises(ValueError):
        ep.LinearGroup([a, b])
    ep.LinearGroup([a, ep.CompressedLinear(ep.DeviceBlob(blobs[1]), "bf16")])  # disjoint: accepted


def test_bf16_route_within_the_fp64_oracle_bound():
    """The bf16 route against the float64 product of the oracle's decoded weight, within the bound
    for float32 accumulation in any order plus the bf16 output rounding."""
    import torch

    import oracle

    W = synth.generate(synth.headline())[:256, :2048].copy()
    blob = ep.encode_tensor(W, 4.0)
    lin = ep.CompressedLinear(ep.DeviceBlob(blob), "bf16")
    x = (torch.randn(64, 2048, device="cuda") * 0.5).to(torch.bfloat16)
    # the bound assumes float32 accumulation: no reduced-precision split-K reductions
    keep = torch.backends.cuda.matmul.allow_bf16_reduced_precision_reduction
    torch.backends.cuda.matmul.allow_bf16_reduced_precision_reduction = False
    try:
        y = lin(x).float().cpu().numpy().astype(np.float64)
    finally:
        torch.backends.cuda.matmul.allow_bf16_reduced_precision_reduction = keep
    # the oracle's own bf16 decode (its conversion is written from the format definition)
    Wbits = oracle.decode_blob(blob, oracle.BF16).astype(np.uint32) << 16
    Wb = Wbits.view(np.float32).astype(np.float64)
    xb = x.float().cpu().numpy()
    ref = oracle.linear(Wb, xb)
    tol = oracle.linear_tolerance(Wb, xb, 2.0 ** -8)
    # the decoder may differ from the oracle by one bf16 unit in the last place per weight
    # (the pages' tolerance for float outputs): sum_k |x_k| ulp(W_jk) more
    ulp = np.ldexp(1.0, np.frexp(np.abs(Wb))[1] - 8)
    tol = tol + np.abs(xb.astype(np.float64)) @ ulp.T
    assert np.all(np.abs(y - ref) <= tol)
