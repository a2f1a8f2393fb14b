"""EntroPack fused GPU weight reconstruction for B200 (sm_100a).

The library is ``libentropack.so`` (C ABI, ``include/entropack.h``): a CPU packer
``ep_encode_tensor`` and the stream-ordered GPU decoder ``ep_decode_tensor``.
This package is a thin ctypes binding over it; nothing here computes the codec.
Importing the package does not load the library; the first call does, and it
raises if the library has not been built.
"""
from ._lib import (BF16, FP16, FP8_E4M3, INT8, FP32, LATTICE_I32, UINT8, Blob, DeviceBlob, EntroPackError,  # noqa: F401
                   GEMV_TOKENS, LUT_BYTES, DecodeBatch, batch_apportion, check_status, decode_status, decode_tensor,
                   decode_tensor_noalloc, decode_tensor_prepared, decode_gemv, encode_tensor, encode_tensor_gpu,
                   encode_tensor_gpu_to_device, lib, prepare_lut)
from .linear import CompressedLinear, LinearGroup  # noqa: F401,E402
from .package import load_package, load_package_to_device, save_package  # noqa: F401,E402
