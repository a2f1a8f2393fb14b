"""Helpers shared by the GPU parity tests (no codec arithmetic here)."""
import numpy as np

import oracle
import dit_weight_compression_ep_b200 as ep

ORACLE_DT = {ep.BF16: oracle.BF16, ep.FP16: oracle.FP16, ep.FP8_E4M3: oracle.E4M3, ep.INT8: oracle.INT8,
             ep.FP32: oracle.FP32, ep.LATTICE_I32: oracle.LATTICE, ep.UINT8: oracle.UINT8}
RAW = {ep.BF16: np.uint16, ep.FP16: np.uint16, ep.FP8_E4M3: np.uint8, ep.INT8: np.uint8, ep.FP32: np.uint32,
       ep.LATTICE_I32: np.uint32, ep.UINT8: np.uint8}


def to_raw(t):
    """torch tensor -> numpy array of its raw bits."""
    import torch

    a = t.detach().cpu().contiguous()
    if a.dtype in (torch.bfloat16, torch.float16):
        return a.view(torch.int16).numpy().view(np.uint16)
    if a.dtype in (torch.float8_e4m3fn, torch.int8, torch.uint8):
        return a.view(torch.uint8).numpy()
    return a.view(torch.int32).numpy().view(np.uint32)


def ulp_diff(a, b, dt):
    """Distance in units in the last place between two raw bit arrays of a float format."""
    def key(x, bits):
        x = x.astype(np.int64)
        sign = x >> (bits - 1)
        mag = x & ((1 << (bits - 1)) - 1)
        return np.where(sign == 1, -mag, mag)

    bits = {ep.BF16: 16, ep.FP16: 16, ep.FP8_E4M3: 8, ep.FP32: 32}[dt]
    return np.abs(key(a, bits) - key(b, bits))


def assert_parity(got_raw, want, dt, what=""):
    """Bit-exact comparison (the design reaches exact equality; the spec's tolerance is <= 1 ulp
    for floating outputs, exact for lattice coordinates and INT8)."""
    want_raw = np.ascontiguousarray(want).reshape(-1).view(RAW[dt])
    got_raw = np.ascontiguousarray(got_raw).reshape(-1)
    assert got_raw.shape == want_raw.shape, (got_raw.shape, want_raw.shape)
    bad = np.nonzero(got_raw != want_raw)[0]
    if bad.size:
        msg = f"{what}: {bad.size} of {got_raw.size} differ; first at {bad[:5]}: got {got_raw[bad[:5]]} want " \
              f"{want_raw[bad[:5]]}"
        if dt in (ep.BF16, ep.FP16, ep.FP8_E4M3, ep.FP32):
            msg += f"; max ulp {ulp_diff(got_raw[bad], want_raw[bad], dt).max()}"
        raise AssertionError(msg)


def oracle_decode(blob, dt, t0=0, t1=None):
    """Oracle decode of the stored arrays of a library or oracle blob."""
    words = getattr(blob, "payload_words", None)
    payload = blob.payload[:words] if words is not None else blob.payload
    return oracle.decode(payload, blob.tile_index, blob.freq_tables, blob.row_scales, blob.rows, blob.cols,
                         ORACLE_DT[dt], t0, t1)


def as_lib_blob(ob):
    """An oracle blob as the library's Blob (stored arrays only)."""
    return ep.Blob.from_arrays(ob.payload, ob.tile_index, ob.freq_tables, ob.row_scales, ob.rows, ob.cols)
