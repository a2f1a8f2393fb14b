"""ctypes binding of libentropack.so (the C ABI of include/entropack.h).

Argument marshalling only: every step of the codec runs inside the library (the
packer on the host, the decoder in its sm_100a kernel).  PyTorch provides device
memory and streams.  There is no fallback: if the library has not been built the
first call raises.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SO_PATH = os.path.join(_HERE, "libentropack.so")

# ep_dtype
BF16, FP16, FP8_E4M3, INT8, FP32, LATTICE_I32, UINT8 = 0, 1, 2, 3, 4, 5, 6
DTYPE_NAMES = {"bf16": BF16, "fp16": FP16, "e4m3": FP8_E4M3, "fp8_e4m3": FP8_E4M3, "int8": INT8, "fp32": FP32,
               "lattice": LATTICE_I32, "uint8": UINT8}
OUT_BYTES = {BF16: 2, FP16: 2, FP8_E4M3: 1, INT8: 1, FP32: 4, LATTICE_I32: 4, UINT8: 1}

# ep_status
STATUS = {0: "EP_OK", 1: "EP_EINVAL", 2: "EP_EUNSUPPORTED", 3: "EP_EALPHABET", 4: "EP_ECUDA", 5: "EP_ECORRUPT",
          6: "EP_ENOMEM"}
STATUS_CODES = {v: k for k, v in STATUS.items()}


class EntroPackError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)}")
        self.code = code


class _Opts(C.Structure):
    _fields_ = [
        ("prob_bits", C.c_int),
        ("tile_vectors", C.c_int),
        ("sample_vectors", C.c_int64),
        ("search_steps", C.c_int),
        ("seed", C.c_uint64),
        ("has_container_scales", C.c_int),
        ("num_threads", C.c_int),
        ("rdo_candidates", C.c_int),
        ("rdo_sweeps", C.c_int),
    ]


class _BatchItem(C.Structure):
    _fields_ = [
        ("tiles", C.c_void_p),
        ("tile_index", C.c_void_p),
        ("freq_tables", C.c_void_p),
        ("row_scales", C.c_void_p),
        ("lut", C.c_void_p),
        ("rows", C.c_int64),
        ("cols", C.c_int64),
        ("ntiles", C.c_int64),
        ("tile_vectors", C.c_int64),
        ("prob_bits", C.c_int),
        ("out", C.c_void_p),
    ]


class _DevBlob(C.Structure):
    _fields_ = [
        ("rows", C.c_int64),
        ("cols", C.c_int64),
        ("b", C.c_int),
        ("V", C.c_int),
        ("ntiles", C.c_int),
        ("payload_words", C.c_uint64),
        ("payload_alloc_words", C.c_size_t),
        ("freq_bytes", C.c_size_t),
        ("payload", C.c_void_p),
        ("tile_index", C.c_void_p),
        ("freq_tables", C.c_void_p),
        ("row_scales", C.c_void_p),
        ("s", C.c_double),
        ("stored_bpp", C.c_double),
        ("stored_bytes", C.c_int64),
    ]


class _Blob(C.Structure):
    _fields_ = [
        ("rows", C.c_int64),
        ("cols", C.c_int64),
        ("b", C.c_int),
        ("V", C.c_int),
        ("J", C.c_int),
        ("ntiles", C.c_int),
        ("payload", C.POINTER(C.c_uint16)),
        ("payload_words", C.c_size_t),
        ("payload_alloc_words", C.c_size_t),
        ("tile_index", C.POINTER(C.c_uint32)),
        ("freq_tables", C.POINTER(C.c_uint8)),
        ("freq_bytes", C.c_size_t),
        ("row_scales", C.POINTER(C.c_float)),
        ("s", C.c_double),
        ("stored_bpp", C.c_double),
        ("stored_bytes", C.c_int64),
    ]


_lib = None


def lib() -> C.CDLL:
    """Load libentropack.so; raise if it is missing (no fallback path exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(SO_PATH):
            raise RuntimeError(f"{SO_PATH} is not built; run `python -m dit_weight_compression_ep_b200.build`")
        L = C.CDLL(SO_PATH)
        P = C.c_void_p
        L.ep_encode_tensor.argtypes = [P, C.c_int64, C.c_int64, C.c_double, C.POINTER(_Opts),
                                       C.POINTER(C.POINTER(_Blob))]
        L.ep_encode_tensor.restype = C.c_int
        L.ep_encode_tensor_gpu.argtypes = [P, P, C.c_int64, C.c_int64, C.c_double, C.POINTER(_Opts),
                                           C.POINTER(C.POINTER(_Blob))]
        L.ep_encode_tensor_gpu.restype = C.c_int
        L.ep_encode_tensor_gpu_device.argtypes = [P, P, C.c_int, C.c_int64, C.c_int64, C.c_double,
                                                  C.POINTER(_Opts), C.POINTER(_DevBlob)]
        L.ep_encode_tensor_gpu_device.restype = C.c_int
        L.ep_free_device_blob.argtypes = [C.POINTER(_DevBlob)]
        L.ep_free_device_blob.restype = None
        L.ep_free_blob.argtypes = [C.POINTER(_Blob)]
        L.ep_free_blob.restype = None
        L.ep_decode_tensor.argtypes = [P, P, P, P, P, C.c_int64, C.c_int64, C.c_int, P]
        L.ep_decode_tensor.restype = C.c_int
        L.ep_decode_tensor_noalloc.argtypes = [P, P, P, P, P, C.c_int64, C.c_int64, C.c_int, P]
        L.ep_decode_tensor_noalloc.restype = C.c_int
        L.ep_decode_prepare.argtypes = [P, P, C.c_int64, C.c_int64, P, C.c_size_t]
        L.ep_decode_prepare.restype = C.c_int
        L.ep_decode_tensor_prepared.argtypes = [P, P, P, P, P, P, C.c_size_t, C.c_int64, C.c_int64, C.c_int, P]
        L.ep_decode_tensor_prepared.restype = C.c_int
        L.ep_decode_gemv.argtypes = [P, P, P, P, P, P, C.c_size_t, C.c_int64, C.c_int64, P, C.c_int, P]
        L.ep_decode_gemv.restype = C.c_int
        L.ep_batch_create.argtypes = [C.POINTER(_BatchItem), C.c_int, C.c_int, C.POINTER(C.c_void_p)]
        L.ep_batch_create.restype = C.c_int
        L.ep_batch_create_on.argtypes = [C.POINTER(_BatchItem), C.c_int, C.c_int, C.c_int, C.POINTER(C.c_void_p)]
        L.ep_batch_create_on.restype = C.c_int
        L.ep_decode_batch.argtypes = [P, P]
        L.ep_decode_batch.restype = C.c_int
        L.ep_batch_free.argtypes = [P]
        L.ep_batch_free.restype = None
        L.ep_batch_apportion.argtypes = [C.c_int, C.POINTER(C.c_int64), C.POINTER(C.c_int64), C.POINTER(C.c_int),
                                         C.c_int, C.POINTER(C.c_int)]
        L.ep_batch_apportion.restype = C.c_int
        L.ep_decode_status.argtypes = [P]
        L.ep_decode_status.restype = C.c_int
        L.ep_status_string.argtypes = [C.c_int]
        L.ep_status_string.restype = C.c_char_p
        _lib = L
    return _lib


EXPORTED = ("ep_encode_tensor", "ep_encode_tensor_gpu", "ep_encode_tensor_gpu_device", "ep_free_device_blob",
            "ep_free_blob", "ep_decode_tensor", "ep_decode_tensor_noalloc", "ep_decode_prepare",
            "ep_decode_tensor_prepared", "ep_decode_gemv", "ep_batch_create", "ep_batch_create_on",
            "ep_decode_batch", "ep_batch_free", "ep_batch_apportion", "ep_decode_status", "ep_status_string")

LUT_BYTES = 131104  # EP_LUT_BYTES: a prepared decode table


@dataclass
class Blob:
    """Host copy of a compressed tensor (the packer's output)."""

    rows: int
    cols: int
    b: int
    V: int
    ntiles: int
    payload: np.ndarray       # uint16, padded with zero words to a multiple of 8
    payload_words: int        # stored words (the final offset)
    tile_index: np.ndarray    # uint32 [33*T + 1]
    freq_tables: np.ndarray   # uint8
    row_scales: np.ndarray    # float32 [rows]
    s: float = 0.0
    stored_bpp: float = 0.0
    stored_bytes: int = 0

    @property
    def numel(self) -> int:
        return self.rows * self.cols

    def stored_device_bytes(self) -> int:
        """Bytes the decoder reads: payload + tile index + tables + row scales."""
        return 2 * self.payload_words + 4 * self.tile_index.size + self.freq_tables.size + 4 * self.rows

    @staticmethod
    def from_arrays(payload, tile_index, freq_tables, row_scales, rows: int, cols: int) -> "Blob":
        """Wrap stored arrays produced elsewhere (e.g. read from a file)."""
        payload = np.asarray(payload, np.uint16).reshape(-1)
        words = payload.size
        pad = (-words) % 8
        padded = np.concatenate([payload, np.zeros(pad, np.uint16)]) if pad else payload.copy()
        ft = np.ascontiguousarray(freq_tables, np.uint8)
        h = ft[:24].view(np.uint32)
        return Blob(rows, cols, int(h[2]), int(h[3]), int(h[5]), padded, words,
                    np.ascontiguousarray(tile_index, np.uint32), ft, np.ascontiguousarray(row_scales, np.float32))


def encode_tensor(W: np.ndarray, target_bpp: float, *, prob_bits: int = 0, tile_vectors: int = 0,
                  sample_vectors: int = 0, search_steps: int = 0, seed: int = 0,
                  has_container_scales: bool = False, num_threads: int = 0, rdo_candidates: int = 0,
                  rdo_sweeps: int = 0) -> Blob:
    """Compress a host float32 matrix with the library's CPU packer (ep_encode_tensor);
    rdo_candidates > 1 turns on the per-row refinement (App. C.2)."""
    W = np.ascontiguousarray(W, np.float32)
    if W.ndim != 2:
        raise ValueError("W must be 2-D")
    o = _Opts(prob_bits, tile_vectors, sample_vectors, search_steps, seed, int(has_container_scales), num_threads,
              int(rdo_candidates), int(rdo_sweeps))
    out = C.POINTER(_Blob)()
    rc = lib().ep_encode_tensor(W.ctypes.data, W.shape[0], W.shape[1], float(target_bpp), C.byref(o), C.byref(out))
    if rc:
        raise EntroPackError(rc, "ep_encode_tensor")
    return _take_blob(out)


def encode_tensor_gpu(W, target_bpp: float, *, prob_bits: int = 0, tile_vectors: int = 0, sample_vectors: int = 0,
                      search_steps: int = 0, seed: int = 0, has_container_scales: bool = False,
                      rdo_candidates: int = 0, rdo_sweeps: int = 0, stream=None) -> Blob:
    """Compress a float32 or bfloat16 CUDA matrix on the GPU into a host Blob: the same bytes as
    encode_tensor on the float32 values (ep_encode_tensor_gpu; bfloat16 goes through
    ep_encode_tensor_gpu_device and a copy back).  Launched on `stream` (default torch's current
    stream).  rdo_candidates > 1 runs the per-row refinement (App. C.2) on the GPU as well."""
    import torch

    if not (isinstance(W, torch.Tensor) and W.is_cuda and W.dtype in (torch.float32, torch.bfloat16) and W.dim() == 2):
        raise ValueError("W must be a 2-D float32 or bfloat16 CUDA tensor")
    if W.dtype == torch.bfloat16:
        db = encode_tensor_gpu_to_device(W, target_bpp, prob_bits=prob_bits, tile_vectors=tile_vectors,
                                         sample_vectors=sample_vectors, search_steps=search_steps, seed=seed,
                                         has_container_scales=has_container_scales, rdo_candidates=rdo_candidates,
                                         rdo_sweeps=rdo_sweeps, stream=stream)
        return db.to_host()
    W = W.contiguous()
    o = _Opts(prob_bits, tile_vectors, sample_vectors, search_steps, seed, int(has_container_scales), 0,
              int(rdo_candidates), int(rdo_sweeps))
    st = stream if stream is not None else torch.cuda.current_stream(W.device)
    out = C.POINTER(_Blob)()
    rc = lib().ep_encode_tensor_gpu(C.c_void_p(st.cuda_stream), W.data_ptr(), W.shape[0], W.shape[1],
                                    float(target_bpp), C.byref(o), C.byref(out))
    if rc:
        raise EntroPackError(rc, "ep_encode_tensor_gpu")
    return _take_blob(out)


def encode_tensor_gpu_to_device(W, target_bpp: float, *, prob_bits: int = 0, tile_vectors: int = 0,
                                sample_vectors: int = 0, search_steps: int = 0, seed: int = 0,
                                has_container_scales: bool = False, rdo_candidates: int = 0, rdo_sweeps: int = 0,
                                stream=None) -> "DeviceBlob":
    """Compress a float32 or bfloat16 CUDA matrix with ep_encode_tensor_gpu_device and keep the result on
    the GPU: a DeviceBlob ready for the decoders (its arrays are copied into torch-owned tensors and
    the library's buffers freed)."""
    import torch

    if not (isinstance(W, torch.Tensor) and W.is_cuda and W.dtype in (torch.float32, torch.bfloat16) and W.dim() == 2):
        raise ValueError("W must be a 2-D float32 or bfloat16 CUDA tensor")
    W = W.contiguous()
    o = _Opts(prob_bits, tile_vectors, sample_vectors, search_steps, seed, int(has_container_scales), 0,
              int(rdo_candidates), int(rdo_sweeps))
    st = stream if stream is not None else torch.cuda.current_stream(W.device)
    d = _DevBlob()
    rc = lib().ep_encode_tensor_gpu_device(C.c_void_p(st.cuda_stream), W.data_ptr(), int(W.dtype == torch.bfloat16),
                                           W.shape[0], W.shape[1], float(target_bpp), C.byref(o), C.byref(d))
    if rc:
        raise EntroPackError(rc, "ep_encode_tensor_gpu_device")
    try:
        def take(ptr, n, typestr, dtype):
            if n == 0:
                return torch.empty(0, dtype=dtype, device=W.device)
            view = torch.as_tensor(_CudaMem(ptr, n, typestr), device=W.device)
            return view.clone()  # a copy the caching allocator owns; the library's buffer is freed below

        T = d.ntiles
        db = DeviceBlob.__new__(DeviceBlob)
        db.rows, db.cols, db.b, db.V, db.ntiles = d.rows, d.cols, d.b, d.V, T
        db.payload = take(d.payload, max(int(d.payload_alloc_words), 8), "<i2", torch.int16)
        db.tile_index = take(d.tile_index, 33 * T + 1, "<i4", torch.int32)
        db.freq_tables = take(d.freq_tables, int(d.freq_bytes), "|u1", torch.uint8)
        db.row_scales = take(d.row_scales, int(d.rows), "<f4", torch.float32)
        db.read_bytes = 2 * int(d.payload_words) + 4 * (33 * T + 1) + int(d.freq_bytes) + 4 * int(d.rows)
        db.payload_words, db.s, db.stored_bpp, db.stored_bytes = int(d.payload_words), d.s, d.stored_bpp, \
            int(d.stored_bytes)
        st.synchronize()
        return db
    finally:
        lib().ep_free_device_blob(C.byref(d))


class _CudaMem:
    """A device buffer of the library, seen through the CUDA array interface (no copy)."""

    def __init__(self, ptr: int, n: int, typestr: str):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": typestr, "data": (int(ptr), False),
                                         "version": 3, "strides": None}


def _take_blob(out) -> Blob:
    """Copy a library blob into numpy arrays and free it."""
    try:
        b = out.contents
        T = b.ntiles
        payload = np.ctypeslib.as_array(b.payload, shape=(b.payload_alloc_words,)).copy() if b.payload_alloc_words \
            else np.zeros(0, np.uint16)
        tix = np.ctypeslib.as_array(b.tile_index, shape=(33 * T + 1,)).copy()
        ft = np.ctypeslib.as_array(b.freq_tables, shape=(b.freq_bytes,)).copy()
        rs = np.ctypeslib.as_array(b.row_scales, shape=(b.rows,)).copy()
        return Blob(b.rows, b.cols, b.b, b.V, T, payload, int(b.payload_words), tix, ft, rs, b.s, b.stored_bpp,
                    int(b.stored_bytes))
    finally:
        lib().ep_free_blob(out)


class DeviceBlob:
    """A compressed tensor resident in GPU memory (torch tensors own the buffers)."""

    def __init__(self, blob: Blob, device="cuda"):
        import torch

        self.rows, self.cols, self.b, self.V, self.ntiles = blob.rows, blob.cols, blob.b, blob.V, blob.ntiles
        pay = blob.payload if blob.payload.size else np.zeros(8, np.uint16)
        self.payload = torch.from_numpy(pay.view(np.int16)).to(device)
        self.tile_index = torch.from_numpy(blob.tile_index.view(np.int32)).to(device)
        self.freq_tables = torch.from_numpy(blob.freq_tables).to(device)
        self.row_scales = torch.from_numpy(blob.row_scales).to(device)
        self.read_bytes = blob.stored_device_bytes()
        self.payload_words, self.s = int(blob.payload_words), blob.s
        self.stored_bpp, self.stored_bytes = blob.stored_bpp, blob.stored_bytes


def _device_blob_to_host(self) -> Blob:
    """The arrays of a GPU-encoded DeviceBlob copied into a host Blob (same bytes)."""
    import torch

    pay = self.payload.cpu().numpy().view(np.uint16)
    return Blob(self.rows, self.cols, self.b, self.V, self.ntiles, pay, self.payload_words,
                self.tile_index.cpu().numpy().view(np.uint32), self.freq_tables.cpu().numpy(),
                self.row_scales.cpu().numpy(), self.s, self.stored_bpp, self.stored_bytes)


DeviceBlob.to_host = _device_blob_to_host


def _torch_dtype(dt: int):
    import torch

    return {BF16: torch.bfloat16, FP16: torch.float16, FP8_E4M3: torch.float8_e4m3fn, INT8: torch.int8,
            FP32: torch.float32, LATTICE_I32: torch.int32, UINT8: torch.uint8}[dt]


def _output(db: DeviceBlob, out_dtype: int, out, shape=None):
    """`out`, or a new tensor, for a decode of db into out_dtype; a given buffer must be a
    contiguous CUDA tensor of the output dtype on db's device, large enough for the result (the
    C ABI takes a bare pointer and cannot check its extent)."""
    import torch

    shape = shape or (db.rows, db.cols)
    tdt = _torch_dtype(out_dtype) if isinstance(out_dtype, int) else out_dtype
    if out is None:
        return torch.empty(shape, dtype=tdt, device=db.payload.device)
    n = 1
    for d in shape:
        n *= int(d)
    if not (isinstance(out, torch.Tensor) and out.is_cuda and out.dtype == tdt and out.is_contiguous()
            and out.device == db.payload.device and out.numel() >= n):
        raise ValueError(f"out must be a contiguous {tdt} CUDA tensor on {db.payload.device} with at least {n} elements")
    return out


def decode_tensor(db: DeviceBlob, out_dtype: int = BF16, out=None, stream=None):
    """Launch ep_decode_tensor on `stream` (default: torch's current stream); returns `out`."""
    import torch

    out = _output(db, out_dtype, out)
    st = stream if stream is not None else torch.cuda.current_stream(db.payload.device)
    rc = lib().ep_decode_tensor(C.c_void_p(st.cuda_stream), db.payload.data_ptr(), db.tile_index.data_ptr(),
                                db.freq_tables.data_ptr(), db.row_scales.data_ptr(), db.rows, db.cols,
                                int(out_dtype), out.data_ptr())
    if rc:
        raise EntroPackError(rc, "ep_decode_tensor")
    return out


def decode_tensor_noalloc(db: DeviceBlob, out_dtype: int = BF16, out=None, stream=None):
    """ep_decode_tensor_noalloc: the same decode with the library's fixed device scratch array
    (no device allocation by the library); calls that overlap on the GPU must be ordered by the caller."""
    import torch

    out = _output(db, out_dtype, out)
    st = stream if stream is not None else torch.cuda.current_stream(db.payload.device)
    rc = lib().ep_decode_tensor_noalloc(C.c_void_p(st.cuda_stream), db.payload.data_ptr(), db.tile_index.data_ptr(),
                                        db.freq_tables.data_ptr(), db.row_scales.data_ptr(), db.rows, db.cols,
                                        int(out_dtype), out.data_ptr())
    if rc:
        raise EntroPackError(rc, "ep_decode_tensor_noalloc")
    return out


def _check_lut(db: DeviceBlob, lut):
    """A prepared-table buffer: a contiguous CUDA tensor on db's device (its size the C ABI checks)."""
    import torch

    if not (isinstance(lut, torch.Tensor) and lut.is_cuda and lut.is_contiguous() and lut.device == db.payload.device):
        raise ValueError(f"the table buffer must be a contiguous CUDA tensor on {db.payload.device}")


def prepare_lut(db: DeviceBlob, lut=None, stream=None):
    """ep_decode_prepare: build the tensor's decode lookup table once into a LUT_BYTES uint8
    device buffer (allocated here when `lut` is None); returns the buffer."""
    import torch

    if lut is None:
        lut = torch.empty(LUT_BYTES, dtype=torch.uint8, device=db.payload.device)
    _check_lut(db, lut)
    st = stream if stream is not None else torch.cuda.current_stream(db.payload.device)
    rc = lib().ep_decode_prepare(C.c_void_p(st.cuda_stream), db.freq_tables.data_ptr(), db.rows, db.cols,
                                 lut.data_ptr(), lut.numel() * lut.element_size())
    if rc:
        raise EntroPackError(rc, "ep_decode_prepare")
    return lut


def decode_tensor_prepared(db: DeviceBlob, lut, out_dtype: int = BF16, out=None, stream=None):
    """ep_decode_tensor_prepared: the decode with a table prepare_lut built from this tensor."""
    import torch

    _check_lut(db, lut)
    out = _output(db, out_dtype, out)
    st = stream if stream is not None else torch.cuda.current_stream(db.payload.device)
    rc = lib().ep_decode_tensor_prepared(C.c_void_p(st.cuda_stream), db.payload.data_ptr(),
                                         db.tile_index.data_ptr(), db.freq_tables.data_ptr(),
                                         db.row_scales.data_ptr(), lut.data_ptr(), lut.numel() * lut.element_size(),
                                         db.rows, db.cols, int(out_dtype), out.data_ptr())
    if rc:
        raise EntroPackError(rc, "ep_decode_tensor_prepared")
    return out


GEMV_TOKENS = (1, 2, 4, 8)


def decode_gemv(db: DeviceBlob, x, lut=None, y=None, stream=None):
    """ep_decode_gemv: y = x W^T with W the tensor's decoded weight in BF16, computed inside the
    decode (x: bfloat16 CUDA tensor [ntok, cols], ntok in GEMV_TOKENS; lut: a prepare_lut table or
    None).  Returns y, float32 [ntok, rows]."""
    import torch

    if not (isinstance(x, torch.Tensor) and x.is_cuda and x.dtype == torch.bfloat16 and x.dim() == 2
            and x.shape[1] == db.cols and x.device == db.payload.device):
        raise ValueError("x must be a bfloat16 CUDA tensor [tokens, cols] on the blob's device")
    x = x.contiguous()
    if lut is not None:
        _check_lut(db, lut)
    y = _output(db, torch.float32, y, (x.shape[0], db.rows))
    st = stream if stream is not None else torch.cuda.current_stream(db.payload.device)
    rc = lib().ep_decode_gemv(C.c_void_p(st.cuda_stream), db.payload.data_ptr(), db.tile_index.data_ptr(),
                              db.freq_tables.data_ptr(), db.row_scales.data_ptr(),
                              lut.data_ptr() if lut is not None else None,
                              lut.numel() * lut.element_size() if lut is not None else 0, db.rows, db.cols,
                              x.data_ptr(), int(x.shape[0]), y.data_ptr())
    if rc:
        raise EntroPackError(rc, "ep_decode_gemv")
    return y


def batch_apportion(ntiles, tile_vectors, prob_bits, num_ctas: int):
    """ep_batch_apportion (host only): SMs per tensor when a batch shares num_ctas of them out."""
    n = len(ntiles)
    counts = (C.c_int * max(n, 1))()
    rc = lib().ep_batch_apportion(n, (C.c_int64 * max(n, 1))(*ntiles), (C.c_int64 * max(n, 1))(*tile_vectors),
                                  (C.c_int * max(n, 1))(*prob_bits), num_ctas, counts)
    if rc:
        raise EntroPackError(rc, "ep_batch_apportion")
    return list(counts)[:n]


class DecodeBatch:
    """ep_batch_create / ep_decode_batch: decode several tensors in one launch.

    items: (DeviceBlob, prepared table, output tensor or None) triples; the outputs are allocated
    here when None.  The blobs, tables and outputs are kept alive with the handle.  num_ctas:
    the SMs the launch uses (ep_batch_create_on), None for all of them."""

    def __init__(self, items, out_dtype: int = BF16, num_ctas=None):
        import torch

        self.out_dtype = out_dtype
        self.items = []
        arr = (_BatchItem * len(items))()
        for k, (db, lut, out) in enumerate(items):
            _check_lut(db, lut)
            out = _output(db, out_dtype, out)
            self.items.append((db, lut, out))
            arr[k] = _BatchItem(db.payload.data_ptr(), db.tile_index.data_ptr(), db.freq_tables.data_ptr(),
                                db.row_scales.data_ptr(), lut.data_ptr(), db.rows, db.cols, db.ntiles, db.V, db.b,
                                out.data_ptr())
        h = C.c_void_p()
        if num_ctas is None:
            rc = lib().ep_batch_create(arr, len(items), int(out_dtype), C.byref(h))
        else:
            rc = lib().ep_batch_create_on(arr, len(items), int(out_dtype), int(num_ctas), C.byref(h))
        if rc:
            raise EntroPackError(rc, "ep_batch_create")
        self._h = h

    @property
    def outputs(self):
        return [o for _, _, o in self.items]

    def run(self, stream=None):
        import torch

        st = stream if stream is not None else torch.cuda.current_stream(self.items[0][0].payload.device)
        rc = lib().ep_decode_batch(C.c_void_p(st.cuda_stream), self._h)
        if rc:
            raise EntroPackError(rc, "ep_decode_batch")
        return self.outputs

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            lib().ep_batch_free(h)
            self._h = None


def decode_status(stream=None) -> int:
    """Synchronise the stream and read (and clear) the device status word; returns the ep_status code."""
    import torch

    st = stream if stream is not None else torch.cuda.current_stream()
    return int(lib().ep_decode_status(C.c_void_p(st.cuda_stream)))


def check_status(stream=None) -> None:
    rc = decode_status(stream)
    if rc:
        raise EntroPackError(rc, "decode")
