"""The C ABI library loads on a host without a GPU, exports every entry point
include/*.h declares, and rejects bad arguments on the host before any CUDA call."""
import ctypes as C
import glob
import os
import re

import numpy as np
import pytest

import dit_weight_compression_ep_b200 as ep
from dit_weight_compression_ep_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ep.lib()


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        for m in re.finditer(r"\b(ep_[a-z0-9_]+)\s*\(", src):
            names.add(m.group(1))
    return names


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert {"ep_encode_tensor", "ep_free_blob", "ep_decode_tensor", "ep_decode_status", "ep_status_string"} <= names
    for n in sorted(names):
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code in range(7):
        assert lib.ep_status_string(code)


def test_decode_rejects_bad_arguments_on_host(lib):
    good = C.c_void_p(0x10000)
    args = [None, good, good, good, good, 64, 64, ep.BF16, good]
    EINVAL, EUNSUP = ep._lib.STATUS_CODES["EP_EINVAL"], ep._lib.STATUS_CODES["EP_EUNSUPPORTED"]
    for i in (1, 2, 3, 4, 8):  # null buffers
        a = list(args)
        a[i] = None
        assert lib.ep_decode_tensor(*a) == EINVAL
    a = list(args)
    a[6] = -8                   # cols <= 0
    assert lib.ep_decode_tensor(*a) == EINVAL
    for dt in (7, 9, -1):       # unknown dtypes (EP_UINT8 = 6 is the last one)
        a = list(args)
        a[7] = dt
        assert lib.ep_decode_tensor(*a) == EUNSUP
    a = list(args)
    a[5] = 0                    # rows <= 0
    assert lib.ep_decode_tensor(*a) == EINVAL
    a = list(args)
    a[1] = C.c_void_p(0x10008)  # payload not 16-byte aligned
    assert lib.ep_decode_tensor(*a) == EINVAL
    a = list(args)
    a[8] = C.c_void_p(0x10004)  # output not 16-byte aligned
    assert lib.ep_decode_tensor(*a) == EINVAL


def test_prepared_decode_rejects_bad_arguments_on_host(lib):
    """Every case below is refused by the host checks, before any CUDA call."""
    good = C.c_void_p(0x10000)
    EINVAL, EUNSUP = ep._lib.STATUS_CODES["EP_EINVAL"], ep._lib.STATUS_CODES["EP_EUNSUPPORTED"]
    n = ep.LUT_BYTES
    prep = [None, good, 64, 64, good, n]
    for i, bad in ((1, None), (4, None), (4, C.c_void_p(0x10008)), (1, C.c_void_p(0x10004)), (5, n - 1), (5, 0),
                   (2, 0), (3, -8)):
        a = list(prep)
        a[i] = bad
        assert lib.ep_decode_prepare(*a) == EINVAL, (i, bad)
    dec = [None, good, good, good, good, good, n, 64, 64, ep.BF16, good]
    for i, bad in ((1, None), (2, None), (3, None), (4, None), (5, None), (10, None), (5, C.c_void_p(0x10008)),
                   (6, n - 1), (7, 0), (8, -8), (10, C.c_void_p(0x10004)), (1, C.c_void_p(0x10008))):
        a = list(dec)
        a[i] = bad
        assert lib.ep_decode_tensor_prepared(*a) == EINVAL, (i, bad)
    a = list(dec)
    a[9] = 7
    assert lib.ep_decode_tensor_prepared(*a) == EUNSUP


def test_lut_bytes_matches_the_header():
    src = open(os.path.join(ROOT, "include", "entropack.h")).read()
    m = re.search(r"#define\s+EP_LUT_BYTES\s+(\d+)", src)
    assert m and int(m.group(1)) == ep.LUT_BYTES == 128 * 1024 + 32


def test_encode_rejects_bad_arguments(lib):
    W = np.zeros((4, 16), np.float32)
    assert ep.encode_tensor(np.ones((4, 12), np.float32), 4.0).cols == 12  # rows padded to whole vectors
    with pytest.raises(ep.EntroPackError):
        ep.encode_tensor(np.zeros((0, 16), np.float32), 4.0)      # no rows
    with pytest.raises(ep.EntroPackError):
        ep.encode_tensor(W, 0.0)
    with pytest.raises(ep.EntroPackError):
        ep.encode_tensor(W, 4.0, prob_bits=16)
    with pytest.raises(ep.EntroPackError):
        ep.encode_tensor(W, 4.0, prob_bits=8)


def test_gpu_encoder_refuses_bad_arguments_on_host(lib):
    """Every case is refused before any CUDA call (a fake device pointer never reaches a kernel)."""
    EINVAL, EUNSUP = ep._lib.STATUS_CODES["EP_EINVAL"], ep._lib.STATUS_CODES["EP_EUNSUPPORTED"]
    good = C.c_void_p(0x10000)
    out = C.POINTER(ep._lib._Blob)()

    def call(W=good, rows=64, cols=64, bpp=4.0, **kw):
        o = ep._lib._Opts(kw.get("prob_bits", 0), 0, 0, 0, 0, 0, 0, kw.get("rdo", 0), 0)
        return lib.ep_encode_tensor_gpu(None, W, rows, cols, bpp, C.byref(o), C.byref(out))

    assert call(W=None) == EINVAL
    assert call(rows=0) == EINVAL
    assert call(cols=-1) == EINVAL
    assert call(bpp=0.0) == EINVAL
    assert call(W=C.c_void_p(0x10002)) == EINVAL      # not 4-byte aligned
    assert call(prob_bits=16) == EINVAL
    assert call(prob_bits=8) == EINVAL
    assert call(rows=1 << 20, cols=1 << 14) == EINVAL  # 2^31 vectors


def test_gpu_device_encoder_refuses_bad_arguments_on_host(lib):
    EINVAL, EUNSUP = ep._lib.STATUS_CODES["EP_EINVAL"], ep._lib.STATUS_CODES["EP_EUNSUPPORTED"]
    good = C.c_void_p(0x10000)
    d = ep._lib._DevBlob()

    def call(W=good, bf16=0, rows=64, cols=64, bpp=4.0, rdo=0, out=True):
        o = ep._lib._Opts(0, 0, 0, 0, 0, 0, 0, rdo, 0)
        return lib.ep_encode_tensor_gpu_device(None, W, bf16, rows, cols, bpp, C.byref(o), C.byref(d) if out else None)

    assert call(W=None) == EINVAL
    assert call(out=False) == EINVAL
    assert call(W=C.c_void_p(0x10002)) == EINVAL           # float32 needs 4-byte alignment
    assert call(W=C.c_void_p(0x10001), bf16=1) == EINVAL   # bfloat16 needs 2
    assert call(rows=0) == EINVAL
    assert call(bpp=-1.0) == EINVAL
    assert call(bf16=1, rows=1 << 20, cols=1 << 14) == EINVAL
    assert not d.payload and not d.tile_index
    lib.ep_free_device_blob(None)
    lib.ep_free_device_blob(C.byref(d))


def test_a_c_program_links_and_calls_the_library(tmp_path, lib):
    """A plain C99 program links against libentropack.so and calls it through the header: status
    strings and calls the host refuses before any CUDA work (safe on any machine)."""
    import shutil
    import subprocess

    from dit_weight_compression_ep_b200 import build as b

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use.c"
    src.write_text(r"""
#include <stdio.h>
#include <string.h>
#include "entropack.h"
int main(void) {
    if (strcmp(ep_status_string(EP_OK), "ok") != 0) return 1;
    if (ep_decode_tensor(NULL, NULL, NULL, NULL, NULL, 64, 64, EP_BF16, NULL) != EP_EINVAL) return 2;
    if (ep_decode_prepare(NULL, NULL, 64, 64, NULL, EP_LUT_BYTES) != EP_EINVAL) return 3;
    ep_blob* out = NULL;
    if (ep_encode_tensor(NULL, 4, 4, 4.0, NULL, &out) != EP_EINVAL || out != NULL) return 4;
    int64_t T = 10, V = 100; int bb = 11, counts[1];
    if (ep_batch_apportion(1, &T, &V, &bb, 148, counts) != EP_OK || counts[0] != 10) return 5;
    ep_free_blob(NULL);
    printf("c ok\n");
    return 0;
}
""")
    exe = tmp_path / "use"
    libdir = os.path.dirname(b.SO)
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-l:" + os.path.basename(b.SO), "-Wl,-rpath," + libdir], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "c ok", (r.returncode, r.stdout, r.stderr)


def test_header_compiles_as_c99(tmp_path):
    """include/entropack.h is a C header: every declaration compiles as strict C99."""
    import shutil
    import subprocess

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "h.c"
    src.write_text('#include "entropack.h"\n'
                   "int main(void) { ep_device_blob d = {0}; ep_batch_item it = {0}; ep_encode_opts o = {0};\n"
                   "  (void)d; (void)it; (void)o; return (int)EP_LUT_BYTES - 131104; }\n")
    exe = tmp_path / "h"
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe)], check=True)
    assert subprocess.run([str(exe)]).returncode == 0
