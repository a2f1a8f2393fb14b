"""The decode entry point that allocates nothing (ep_decode_tensor_noalloc).

Callers that cannot allocate device memory -- code whose memory belongs to
another allocator, code that must not take cudaMalloc's implicit device
synchronisation, code running where allocation is not permitted -- use this
entry point; its scratch lives in a fixed device array inside the library.
This file is collected last so that a run stopping at the first failure has run
every other test before it.  It must pass alone in a fresh process too.
"""
import ctypes as C

import numpy as np
import pytest

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


def _raw(t):
    import torch

    return t.view(torch.int16).cpu().numpy() if t.dtype == torch.bfloat16 else t.view(torch.int32).cpu().numpy()


@pytest.mark.parametrize("which", ["small fp32 (bucketed table, b = 12)", "3840x10240 at 4 bpp (packed table)"])
def test_noalloc_matches_decode_tensor_on_two_calls(which):
    import torch

    if which.startswith("small"):
        blob = ep.encode_tensor(synth.generate(synth.small_fp32()), 4.0, prob_bits=12, tile_vectors=512)
    else:
        blob = ep.encode_tensor(synth.generate(synth.headline()), 4.0)
    db = ep.DeviceBlob(blob)
    ep.decode_status()  # start from a clear status word
    for dt in (ep.BF16, ep.LATTICE_I32):
        ref = ep.decode_tensor(db, dt)
        assert ep.decode_status() == 0
        want = _raw(ref)
        for call in range(2):  # two calls in a row share (and reuse) the fixed scratch array
            out = torch.full_like(ref, 0) if dt == ep.LATTICE_I32 else torch.zeros_like(ref)
            st = torch.cuda.current_stream()
            rc = ep.lib().ep_decode_tensor_noalloc(C.c_void_p(st.cuda_stream), db.payload.data_ptr(),
                                                   db.tile_index.data_ptr(), db.freq_tables.data_ptr(),
                                                   db.row_scales.data_ptr(), db.rows, db.cols, dt, out.data_ptr())
            assert rc == 0, rc
            assert ep.decode_status() == 0
            # the tests' tolerance: bit-exact against the existing entry point
            np.testing.assert_array_equal(_raw(out), want, err_msg=f"{which} dtype {dt} call {call}")
        # the package's Python wrapper of the same entry point (argument order and types)
        got = ep.decode_tensor_noalloc(db, dt)
        assert ep.decode_status() == 0
        np.testing.assert_array_equal(_raw(got), want, err_msg=f"{which} dtype {dt} through the wrapper")


def test_noalloc_rejects_bad_sizes_on_host():
    good = C.c_void_p(0x10000)
    EINVAL = ep._lib.STATUS_CODES["EP_EINVAL"]
    L = ep.lib()
    assert L.ep_decode_tensor_noalloc(None, good, good, good, good, 1 << 31, 64, ep.BF16, good) == EINVAL
    assert L.ep_decode_tensor_noalloc(None, good, good, good, good, 0, 64, ep.BF16, good) == EINVAL
