"""A linear layer whose weight is stored compressed on the GPU (EntroPack paper §4.3, Fig. 5: the
weight is reconstructed before the matrix product).

Each call decodes the weight into a scratch buffer with the library's decoder (the lookup table is
prepared once, when the layer is built) and multiplies with the library GEMM through torch:

- "bf16": y = x W^T, W decoded to bf16 (torch.matmul);
- "fp8": W decoded to its FP8-e4m3 container values, y = (x8 W8^T) scaled by the per-token
  activation scales and the weight's per-row container scales (torch._scaled_mm);
- "int8": W decoded to its INT8 container values, y = (x8 W8^T as int32) times the same two
  scales (torch._int_mm).

Layers that run one after another can share one scratch buffer (pass the same tensor).

For a few tokens, `matvec` multiplies inside the decode instead (ep_decode_gemv): the weights,
rounded to BF16 as the bf16 route's are, go straight into float32 multiply-adds with the BF16
activations and are never written; on B200 that is the faster route up to 2 tokens and even
at 4."""
from __future__ import annotations

from ._lib import (BF16, FP8_E4M3, GEMV_TOKENS, INT8, DecodeBatch, DeviceBlob, _torch_dtype, decode_gemv,
                   decode_tensor_prepared, prepare_lut)

ROUTES = {"bf16": BF16, "fp8": FP8_E4M3, "int8": INT8}


class CompressedLinear:
    """y = x W^T (+ bias) with W [out_features, in_features] held as a DeviceBlob."""

    def __init__(self, weight: DeviceBlob, route: str = "bf16", weight_scales=None, bias=None, scratch=None):
        import torch

        if route not in ROUTES:
            raise ValueError(f"route must be one of {sorted(ROUTES)}")
        self.weight, self.route, self.bias = weight, route, bias
        self.dtype = ROUTES[route]
        self.out_features, self.in_features = weight.rows, weight.cols
        dev = weight.payload.device
        if route != "bf16":
            if weight_scales is None:
                raise ValueError("the fp8 and int8 routes need the weight's per-row container scales")
            self.wscale = torch.as_tensor(weight_scales, dtype=torch.float32, device=dev).reshape(1, -1)
            if self.wscale.shape[1] != self.out_features:
                raise ValueError("one container scale per weight row")
        self.lut = prepare_lut(weight)
        need = (self.out_features, self.in_features)
        tdt = _torch_dtype(self.dtype)
        if scratch is None:
            scratch = torch.empty(need, dtype=tdt, device=dev)
        if scratch.dtype != tdt or scratch.numel() < self.out_features * self.in_features or not scratch.is_contiguous():
            raise ValueError("scratch must be a contiguous buffer of the route's dtype, large enough for the weight")
        self.scratch = scratch.reshape(-1)[: self.out_features * self.in_features].view(need)

    def decoded_weight(self, stream=None):
        """Decode the weight into the scratch buffer (on `stream`, default torch's current stream)."""
        return decode_tensor_prepared(self.weight, self.lut, self.dtype, out=self.scratch, stream=stream)

    def __call__(self, x, x_scale=None, decode: bool = True):
        """x: [tokens, in_features]; bf16 for the bf16 route, float8_e4m3fn (fp8) or int8 (int8) with
        x_scale [tokens, 1] float32 for the others.  Returns bf16 [tokens, out_features].
        decode=False multiplies by the scratch as it stands (a LinearGroup decoded it)."""
        import torch

        W = self.decoded_weight() if decode else self.scratch
        if self.route == "bf16":
            y = torch.matmul(x, W.t())
        else:
            if x_scale is None:
                raise ValueError("the fp8 and int8 routes need per-token activation scales")
            if self.route == "fp8":
                y = torch._scaled_mm(x, W.t(), scale_a=x_scale, scale_b=self.wscale, out_dtype=torch.bfloat16)
            else:
                y = (torch._int_mm(x, W.t()).float() * x_scale * self.wscale).to(torch.bfloat16)
        if self.bias is not None:
            y = y + self.bias
        return y

    def matvec(self, x, out=None):
        """y = x W^T (+ bias) with the product taken inside the decode (ep_decode_gemv): x bf16
        [tokens, in_features] with tokens in GEMV_TOKENS, W the decoded weight in BF16 (whatever
        the route), float32 accumulation.  Returns float32 [tokens, out_features] (into `out` if
        given)."""
        if x.dim() != 2 or x.shape[0] not in GEMV_TOKENS:
            raise ValueError(f"matvec takes {GEMV_TOKENS} tokens")
        y = decode_gemv(self.weight, x, lut=self.lut, y=out)
        if self.bias is not None:
            y.add_(self.bias)
        return y


class LinearGroup:
    """Several CompressedLinear layers whose weights are decoded together in one launch
    (ep_decode_batch: the SMs shared out among the weights), e.g. the linear layers of one
    transformer block before the block runs.  The layers need non-overlapping scratch buffers and one
    route dtype; call the layers with decode=False after run()."""

    def __init__(self, layers):
        layers = list(layers)
        if not layers:
            raise ValueError("an empty group")
        if len({lay.dtype for lay in layers}) != 1:
            raise ValueError("the layers of a group share one route dtype")
        # the batch writes every weight at once: the scratch byte ranges must not overlap
        spans = sorted((lay.scratch.data_ptr(), lay.scratch.data_ptr() + lay.scratch.numel() * lay.scratch.element_size())
                       for lay in layers)
        if any(nxt[0] < cur[1] for cur, nxt in zip(spans, spans[1:])):
            raise ValueError("the layers of a group need scratch buffers that do not overlap")
        self.layers = layers
        self.batch = DecodeBatch([(lay.weight, lay.lut, lay.scratch) for lay in layers], layers[0].dtype)

    def run(self, stream=None):
        """Decode every layer's weight into its scratch (one launch on `stream`)."""
        self.batch.run(stream=stream)
