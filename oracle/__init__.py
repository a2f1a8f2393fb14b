"""Plain CPU oracle of the EntroPack codec (TEST INFRASTRUCTURE).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The codec's arithmetic lives in
``ep_oracle.c`` (plain C, double precision, no threads, no SIMD); this module
builds it and marshals numpy arrays through ctypes.  The one function written
here is ``linear`` (with ``linear_tolerance``): the float64 product of a decoded
weight, which is the reference for a linear layer (pinned in
``tests/test_oracle_linear.py``).  It shares nothing with the library in
``dit_weight_compression_ep_b200``.

Each C function cites the passage of the EntroPack paper it follows; the header
comment of ``ep_oracle.c`` lists which functions are pinned by tests and which
readings are "parity unpinned".
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ep_oracle.c")
_SO = os.path.join(_HERE, "libep_oracle.so")

# dtype codes of the oracle's decoder
BF16, FP16, E4M3, INT8, FP32, LATTICE, UINT8 = 0, 1, 2, 3, 4, 5, 6
_NP_OUT = {BF16: np.uint16, FP16: np.uint16, E4M3: np.uint8, INT8: np.int8, FP32: np.float32, LATTICE: np.int32,
           UINT8: np.uint8}


def build(force: bool = False) -> str:
    """Compile ep_oracle.c into libep_oracle.so (gcc, strict IEEE: no contraction, no fast-math)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "ep_oracle.h"))
    ):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
             "-Wall", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _SO)
    return _SO


class _Opts(C.Structure):
    _fields_ = [
        ("target_bpp", C.c_double),
        ("prob_bits", C.c_int),
        ("tile_vectors", C.c_int),
        ("sample_vectors", C.c_int64),
        ("search_steps", C.c_int),
        ("seed", C.c_uint64),
        ("has_container_scales", C.c_int),
        ("direct_z8", C.c_int),
        ("pooled", C.c_int),
        ("rdo_candidates", C.c_int),
        ("rdo_sweeps", C.c_int),
    ]


_lib = None


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(_SO)
        P = C.c_void_p
        I64 = C.c_int64
        L.epo_splitmix64.argtypes = [C.c_uint64, I64, P]
        L.epo_shape_seed.argtypes = [I64, I64]
        L.epo_shape_seed.restype = C.c_uint64
        L.epo_sample_rows.argtypes = [I64, I64, I64, C.c_uint64, P]
        L.epo_sample_rows.restype = I64
        L.epo_row_norm.argtypes = [P, I64]
        L.epo_row_norm.restype = C.c_double
        L.epo_quantize_e8_batch.argtypes = [P, I64, P, P]
        L.epo_fields_batch.argtypes = [P, P, I64, C.c_int, P]
        L.epo_points_batch.argtypes = [P, I64, C.c_int, P]
        L.epo_normalize_freqs.argtypes = [P, C.c_uint32, C.c_uint64, C.c_uint32, P]
        L.epo_default_tile_symbols.argtypes = [C.c_double]
        L.epo_default_tile_symbols.restype = I64
        L.epo_tile_vectors.argtypes = [I64]
        L.epo_tile_vectors.restype = I64
        L.epo_tile_metadata_bytes.argtypes = [I64]
        L.epo_tile_metadata_bytes.restype = I64
        L.epo_refit_row.argtypes = [P, P, I64]
        L.epo_refit_row.restype = C.c_float
        L.epo_encode.argtypes = [P, I64, I64, C.POINTER(_Opts), C.POINTER(P)]
        L.epo_rdo_ratios.argtypes = [C.c_int, P]
        L.epo_encode.restype = C.c_int
        L.epo_encode_fields.argtypes = [P, I64, I64, P, C.c_int, C.c_int, C.c_int, C.POINTER(P)]
        L.epo_encode_fields.restype = C.c_int
        L.epo_estimate_rate.argtypes = [P, I64, I64, C.POINTER(_Opts), C.c_double, C.c_int]
        L.epo_estimate_rate.restype = C.c_double
        L.epo_free.argtypes = [P]
        L.epo_blob_info.argtypes = [P, P, P]
        L.epo_blob_copy.argtypes = [P, P, P, P, P, P]
        L.epo_convert.argtypes = [P, I64, C.c_int, P]
        L.epo_decode_fields.argtypes = [P, P, P, I64, I64, I64, I64, P]
        L.epo_decode_fields.restype = C.c_int
        L.epo_decode.argtypes = [P, P, P, P, I64, I64, C.c_int, I64, I64, P]
        L.epo_decode.restype = C.c_int
        _lib = L
    return _lib


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


@dataclass
class Blob:
    """The stored representation (§3.6 "Stored representation") as numpy arrays."""

    rows: int
    cols: int
    nvec: int
    b: int
    V: int
    ntiles: int
    ntab: int
    flags: int
    s: float
    stored_bpp: float
    stored_bytes: int
    payload: np.ndarray      # uint16 words, all tiles concatenated
    tile_index: np.ndarray   # uint32, per tile [offset, 32 states], then the final offset
    freq_tables: np.ndarray  # uint8, self-describing table header + u16 frequencies
    row_scales: np.ndarray   # float32, one per row
    fields: np.ndarray       # int32 [nvec, 9]: the encoder's fields (c, z1..z7, m)
    extra: dict = field(default_factory=dict)


def _blob_from_handle(h: int) -> Blob:
    L = lib()
    ints = np.zeros(11, np.int64)
    dbls = np.zeros(3, np.float64)
    L.epo_blob_info(h, _p(ints), _p(dbls))
    rows, cols, nvec, b, V, ntiles, pw, fb, sb, ntab, flags = (int(v) for v in ints)
    payload = np.zeros(max(pw, 1), np.uint16)[:pw]
    tix = np.zeros(33 * ntiles + 1, np.uint32)
    ft = np.zeros(fb, np.uint8)
    rs = np.zeros(rows, np.float32)
    fl = np.zeros((nvec, 9), np.int32)
    L.epo_blob_copy(h, _p(np.ascontiguousarray(payload)) if pw else None, _p(tix), _p(ft), _p(rs), _p(fl))
    L.epo_free(h)
    return Blob(rows, cols, nvec, b, V, ntiles, ntab, flags, float(dbls[0]), float(dbls[1]), sb,
                payload, tix, ft, rs, fl)


def encode(W: np.ndarray, target_bpp: float, *, prob_bits: int = 0, tile_vectors: int = 0,
           sample_vectors: int = 0, search_steps: int = 0, seed: int = 0,
           has_container_scales: bool = False, direct_z8: bool = False, pooled: bool = False,
           rdo_candidates: int = 0, rdo_sweeps: int = 0) -> Blob:
    """Full encoder (§3.1): normalise, search s, quantise, refit, optional per-row RDO (§3.5,
    App. C.2), tables, tiled rANS."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    rows, cols = W.shape
    o = _Opts(target_bpp, prob_bits, tile_vectors, sample_vectors, search_steps, seed,
              int(has_container_scales), int(direct_z8), int(pooled), int(rdo_candidates), int(rdo_sweeps))
    h = C.c_void_p()
    rc = lib().epo_encode(_p(W), rows, cols, C.byref(o), C.byref(h))
    if rc:
        raise ValueError(f"oracle encode failed ({rc})")
    return _blob_from_handle(h.value)


def encode_fields(fields: np.ndarray, rows: int, cols: int, row_scales: np.ndarray, b: int, V: int,
                  flags: int = 0) -> Blob:
    """Entropy-code given fields (the coder alone, for tests)."""
    fields = np.ascontiguousarray(fields, dtype=np.int32)
    row_scales = np.ascontiguousarray(row_scales, dtype=np.float32)
    h = C.c_void_p()
    rc = lib().epo_encode_fields(_p(fields), rows, cols, _p(row_scales), b, V, flags, C.byref(h))
    if rc:
        raise ValueError(f"oracle encode_fields failed ({rc})")
    return _blob_from_handle(h.value)


def estimate_rate(W: np.ndarray, target_bpp: float, s: float, b: int, **kw) -> float:
    W = np.ascontiguousarray(W, dtype=np.float32)
    o = _Opts(target_bpp, kw.get("prob_bits", 0), kw.get("tile_vectors", 0), kw.get("sample_vectors", 0),
              kw.get("search_steps", 0), kw.get("seed", 0), int(kw.get("has_container_scales", False)),
              int(kw.get("direct_z8", False)), int(kw.get("pooled", False)))
    return float(lib().epo_estimate_rate(_p(W), W.shape[0], W.shape[1], C.byref(o), s, b))


def _bufs(payload, tile_index, freq_tables):
    payload = np.ascontiguousarray(payload, dtype=np.uint16)
    if payload.size == 0:
        payload = np.zeros(1, np.uint16)
    return payload, np.ascontiguousarray(tile_index, dtype=np.uint32), np.ascontiguousarray(freq_tables, np.uint8)


def decode_fields(payload, tile_index, freq_tables, rows: int, cols: int, t0: int = 0, t1: int | None = None,
                  V: int | None = None) -> np.ndarray:
    """Decode the (c, z1..z7, m) fields of tiles [t0, t1)."""
    payload, tile_index, freq_tables = _bufs(payload, tile_index, freq_tables)
    ntiles = (tile_index.size - 1) // 33
    t1 = ntiles if t1 is None else t1
    V = int(freq_tables[12:16].view(np.uint32)[0]) if V is None else V
    nvec = rows * -(-cols // 8)
    nv = min(t1 * V, nvec) - t0 * V
    out = np.zeros((max(nv, 0), 9), np.int32)
    rc = lib().epo_decode_fields(_p(payload), _p(tile_index), _p(freq_tables), rows, cols, t0, t1,
                                 _p(out) if out.size else None)
    if rc:
        raise ValueError(f"oracle decode failed ({rc})")
    return out


def decode(payload, tile_index, freq_tables, row_scales, rows: int, cols: int, dtype: int,
           t0: int = 0, t1: int | None = None) -> np.ndarray:
    """Decode tiles [t0, t1) to dtype; returns the tiles' weights flat: the contiguous range of
    the row-major matrix their vectors cover (8 per vector, fewer at a padded row end)."""
    payload, tile_index, freq_tables = _bufs(payload, tile_index, freq_tables)
    row_scales = np.ascontiguousarray(row_scales, dtype=np.float32)
    ntiles = (tile_index.size - 1) // 33
    t1 = ntiles if t1 is None else t1
    V = int(freq_tables[12:16].view(np.uint32)[0])
    nq = -(-cols // 8)  # vectors per row: rows are padded to whole vectors
    nvec = rows * nq
    v0, v1 = t0 * V, min(t1 * V, nvec)
    elem = lambda v: (v // nq) * cols + 8 * (v % nq) if v < nvec else rows * cols  # noqa: E731
    out = np.zeros(max(elem(v1) - elem(v0), 0) if v1 > v0 else 0, _NP_OUT[dtype])
    rc = lib().epo_decode(_p(payload), _p(tile_index), _p(freq_tables), _p(row_scales), rows, cols, dtype,
                          t0, t1, _p(out) if out.size else None)
    if rc:
        raise ValueError(f"oracle decode failed ({rc})")
    return out


def decode_blob(bl: Blob, dtype: int) -> np.ndarray:
    return decode(bl.payload, bl.tile_index, bl.freq_tables, bl.row_scales, bl.rows, bl.cols, dtype).reshape(
        bl.rows, bl.cols)


# ---- small pieces, exposed for the pin tests ----

def splitmix64(seed: int, n: int) -> np.ndarray:
    out = np.zeros(n, np.uint64)
    lib().epo_splitmix64(seed, n, _p(out))
    return out


def sample_rows(rows: int, cols: int, sample_vectors: int, seed: int = 0) -> np.ndarray:
    out = np.zeros(rows, np.int64)
    n = lib().epo_sample_rows(rows, cols, sample_vectors, seed, _p(out))
    return out[:n]


def row_norm(w: np.ndarray) -> float:
    w = np.ascontiguousarray(w, dtype=np.float32)
    return float(lib().epo_row_norm(_p(w), w.size))


def quantize_e8(u: np.ndarray):
    """Nearest E8 points of u [n, 8] (float64); returns (y [n, 8], c [n])."""
    u = np.ascontiguousarray(u, dtype=np.float64).reshape(-1, 8)
    y = np.zeros_like(u)
    c = np.zeros(u.shape[0], np.int32)
    lib().epo_quantize_e8_batch(_p(u), u.shape[0], _p(y), _p(c))
    return y, c


def fields_of(y: np.ndarray, c: np.ndarray, direct_z8: bool = False) -> np.ndarray:
    y = np.ascontiguousarray(y, dtype=np.float64).reshape(-1, 8)
    c = np.ascontiguousarray(c, dtype=np.int32)
    f = np.zeros((y.shape[0], 9), np.int32)
    lib().epo_fields_batch(_p(y), _p(c), y.shape[0], int(direct_z8), _p(f))
    return f


def rdo_ratios(K: int) -> np.ndarray:
    """The K nested candidate ratios of the per-row refinement (App. C.2)."""
    out = np.zeros(K, np.float64)
    lib().epo_rdo_ratios(int(K), _p(out))
    return out


def points_of(fields: np.ndarray, direct_z8: bool = False) -> np.ndarray:
    """Inverse field map; returns 2y as int32 [n, 8]."""
    fields = np.ascontiguousarray(fields, dtype=np.int32).reshape(-1, 9)
    y2 = np.zeros((fields.shape[0], 8), np.int32)
    lib().epo_points_batch(_p(fields), fields.shape[0], int(direct_z8), _p(y2))
    return y2


def normalize_freqs(count: np.ndarray, b: int) -> np.ndarray:
    count = np.ascontiguousarray(count, dtype=np.uint64)
    f = np.zeros(count.size, np.uint32)
    lib().epo_normalize_freqs(_p(count), count.size, int(count.sum()), 1 << b, _p(f))
    return f


def default_tile_symbols(target_bpp: float) -> int:
    return int(lib().epo_default_tile_symbols(target_bpp))


def tile_vectors(S: int) -> int:
    return int(lib().epo_tile_vectors(S))


def tile_metadata_bytes(ntiles: int) -> int:
    return int(lib().epo_tile_metadata_bytes(ntiles))


def refit_row(w: np.ndarray, y: np.ndarray) -> float:
    w = np.ascontiguousarray(w, dtype=np.float32)
    y = np.ascontiguousarray(y, dtype=np.float64)
    return float(lib().epo_refit_row(_p(w), _p(y), w.size))


def convert(x: np.ndarray, dtype: int) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.zeros(x.size, _NP_OUT[dtype])
    lib().epo_convert(_p(x), x.size, dtype, _p(out))
    return out


def linear(W: np.ndarray, x: np.ndarray) -> np.ndarray:
    """A linear layer's output y = x W^T in float64, from the weight's decoded values ([paper] §4.3,
    Fig. 5: the weight is reconstructed, then multiplied).  The reference for decode-then-GEMM and
    for a GEMM that decodes its weight operand itself; the matrix product is the library's, on
    float64 copies of the inputs."""
    return np.asarray(x, np.float64) @ np.asarray(W, np.float64).T


def linear_tolerance(W: np.ndarray, x: np.ndarray, out_unit: float) -> np.ndarray:
    """Per-element bound on |y_gemm - y| for a GEMM that forms exact products and accumulates in
    float32 in any order, then rounds to an output format of unit roundoff out_unit: the standard
    dot-product bound gamma_K sum|x_k w_k| (gamma_K = K u / (1 - K u), u = 2^-24, K the inner
    dimension), plus out_unit |y| for the final rounding."""
    K = np.asarray(W).shape[1]
    u = 2.0 ** -24
    gamma = K * u / (1.0 - K * u)
    absdot = np.abs(np.asarray(x, np.float64)) @ np.abs(np.asarray(W, np.float64)).T
    return gamma * absdot * (1.0 + out_unit) + out_unit * np.abs(linear(W, x))
