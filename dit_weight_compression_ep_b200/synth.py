"""Seeded synthetic weight matrices shaped like DiT and LLM linear layers.

This module only draws random numbers and casts containers; it holds none of the
codec's arithmetic, so both the library's tests and the oracle's tests may use it.

Every tensor is generated in blocks of ``BLOCK_ROWS`` rows; block i draws from
``numpy.random.default_rng([seed, i])`` (PCG64) in this order:
  1. the base values (Student-t(nu) or Normal), times ``base_std``;
  2. outliers: ``round(p * n_block)`` distinct positions set to +-k*base_std
     (random sign), before any row scaling;
  3. the per-row lognormal scales exp(N(0, sigma^2)) of the block's rows.
The result is cast to the container (fp32 / bf16 round-to-nearest-even).
The real layers the pages measure on are not available; these stand in with the
same shapes and the distributions the workload descriptions name.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

BLOCK_ROWS = 256


@dataclass(frozen=True)
class WeightSpec:
    rows: int
    cols: int
    dist: str = "normal"        # "normal" or "t"
    nu: float = 5.0             # Student-t degrees of freedom
    base_std: float = 0.02
    outlier_frac: float = 0.0
    outlier_k: float = 8.0
    row_lognormal: float = 0.0  # sigma of the per-row lognormal scale (0: none)
    seed: int = 0
    container: str = "fp32"     # "fp32" or "bf16"


def _block(spec: WeightSpec, i: int, r0: int, r1: int) -> np.ndarray:
    rng = np.random.default_rng([spec.seed, i])
    shape = (r1 - r0, spec.cols)
    if spec.dist == "t":
        base = rng.standard_t(spec.nu, size=shape)
    else:
        base = rng.standard_normal(size=shape)
    base *= spec.base_std
    if spec.outlier_frac > 0:
        n = base.size
        k = int(round(spec.outlier_frac * n))
        if k:
            pos = rng.choice(n, size=k, replace=False)
            sign = rng.choice(np.array([-1.0, 1.0]), size=k)
            base.reshape(-1)[pos] = sign * spec.outlier_k * spec.base_std
    if spec.row_lognormal > 0:
        base *= np.exp(rng.normal(0.0, spec.row_lognormal, size=(shape[0], 1)))
    return base.astype(np.float32)


def generate(spec: WeightSpec) -> np.ndarray:
    """Return the weight matrix as float32 values of its container."""
    out = np.empty((spec.rows, spec.cols), np.float32)
    for i, r0 in enumerate(range(0, spec.rows, BLOCK_ROWS)):
        r1 = min(spec.rows, r0 + BLOCK_ROWS)
        out[r0:r1] = _block(spec, i, r0, r1)
    if spec.container == "bf16":
        out = to_bf16_values(out)
    return out


def to_bf16_values(a: np.ndarray) -> np.ndarray:
    import torch

    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def to_e4m3_container(a: np.ndarray):
    """Per-row scaled FP8-e4m3 container: scale = amax/448; returns (code values as fp32, scales)."""
    import torch

    a = np.ascontiguousarray(a, np.float32)
    amax = np.abs(a).max(axis=1)
    scale = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    q = torch.from_numpy(a / scale[:, None]).clamp_(-448.0, 448.0).to(torch.float8_e4m3fn)
    return q.to(torch.float32).numpy(), scale


def to_uint8_container(a: np.ndarray):
    """Per-tensor UINT8 container with offset 128: scale = amax/127, code = nearest + 128, clamped
    to [0, 255].  Returns (the codes minus the offset as fp32 -- what the codec codes --, scale)."""
    a = np.ascontiguousarray(a, np.float32)
    amax = float(np.abs(a).max())
    scale = np.float32(amax / 127.0) if amax > 0 else np.float32(1.0)
    q = np.clip(np.rint(a / scale) + 128, 0, 255)
    return (q - 128).astype(np.float32), scale


def to_int8_container(a: np.ndarray):
    """Per-channel (row) symmetric INT8 container: scale = amax/127, nearest, clamp +-127."""
    a = np.ascontiguousarray(a, np.float32)
    amax = np.abs(a).max(axis=1)
    scale = np.where(amax > 0, amax / np.float32(127.0), np.float32(1.0)).astype(np.float32)
    q = np.clip(np.rint(a / scale[:, None]), -127, 127).astype(np.float32)
    return q, scale


# ---- the workloads -------------------------------------------------------

def small_fp32(seed: int = 0) -> WeightSpec:
    """256x512 fp32, Student-t(5)*0.02 times row lognormal(0.5)."""
    return WeightSpec(256, 512, "t", 5.0, 0.02, 0.0, 0.0, 0.5, seed, "fp32")


def dit_attn_proj(seed: int = 2) -> WeightSpec:
    """3840x3840 bf16, N(0, 0.02^2), 0.1% outliers at 8 sigma, row lognormal(0.3)."""
    return WeightSpec(3840, 3840, "normal", 5.0, 0.02, 0.001, 8.0, 0.3, seed, "bf16")


DIT_KINDS = {  # kind -> (rows = out features, cols = in features)
    "qkv": (11520, 3840),
    "out": (3840, 3840),
    "gate": (10240, 3840),
    "up": (10240, 3840),
    "down": (3840, 10240),
}
DIT_BPP_CHOICES = (2.3, 3.0, 4.0, 6.0, 8.0)


def dit_stack_layer(block: int, kind: str) -> WeightSpec:
    """One layer of the 30-block DiT linear stack: bf16, Student-t(6)*0.02."""
    rows, cols = DIT_KINDS[kind]
    k = list(DIT_KINDS).index(kind)
    return WeightSpec(rows, cols, "t", 6.0, 0.02, 0.0, 0.0, 0.0, 1000 * block + k, "bf16")


def dit_stack_bpp(nblocks: int = 30, seed: int = 3):
    """Per-layer target bpp drawn uniformly from {2.3, 3, 4, 6, 8}: {(block, kind): bpp}."""
    rng = np.random.default_rng(seed)
    out = {}
    for b in range(nblocks):
        for kind in DIT_KINDS:
            out[(b, kind)] = float(DIT_BPP_CHOICES[int(rng.integers(len(DIT_BPP_CHOICES)))])
    return out


def lowp_source(seed: int = 4) -> WeightSpec:
    """3840x10240 fp32 source of the FP8 / INT8 containers: t(6)*0.02 times row lognormal(0.3)."""
    return WeightSpec(3840, 10240, "t", 6.0, 0.02, 0.0, 0.0, 0.3, seed, "fp32")


def llm_prefill(wide: bool, seed: int | None = None) -> WeightSpec:
    """5120x25600 (wide) or 25600x5120 bf16, N(0, 0.015^2), 0.05% at 10 sigma, row lognormal(0.5)."""
    rows, cols = (5120, 25600) if wide else (25600, 5120)
    s = seed if seed is not None else (5 if wide else 6)
    return WeightSpec(rows, cols, "normal", 5.0, 0.015, 0.0005, 10.0, 0.5, s, "bf16")


def headline(seed: int = 7) -> WeightSpec:
    """3840x10240 bf16, Student-t(6)*0.02: the DiT FFN down-projection shape."""
    return WeightSpec(3840, 10240, "t", 6.0, 0.02, 0.0, 0.0, 0.0, seed, "bf16")
