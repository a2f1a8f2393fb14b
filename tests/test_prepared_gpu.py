"""GPU parity of the prepared-table decode: ep_decode_prepare builds a tensor's decode lookup
table once, ep_decode_tensor_prepared decodes with it (no per-call table build, no grid
barrier).  Expected values come only from the oracle's decoder; the comparison is bit-exact,
over every LUT format the decoder picks from the table header (packed entries with and
without the stored-f bit, the two-level table at b <= 12, the bucketed table at b >= 13 or with
wide alphabets), ragged widths, and the table/tensor mismatches the trailer must catch.
"""
import numpy as np
import pytest

import oracle
import dit_weight_compression_ep_b200 as ep
from dit_weight_compression_ep_b200 import synth
from gpu_util import as_lib_blob, assert_parity, oracle_decode, to_raw

pytestmark = pytest.mark.gpu

ECORRUPT = ep._lib.STATUS_CODES["EP_ECORRUPT"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dit_weight_compression_ep_b200 import build

    build.build()
    ep.lib()
    ep.decode_status()  # clear the status word


def _prepared(blob, dts, what):
    db = ep.DeviceBlob(blob)
    lut = ep.prepare_lut(db)
    assert ep.decode_status() == 0
    for dt in dts:
        got = to_raw(ep.decode_tensor_prepared(db, lut, dt))
        assert ep.decode_status() == 0
        assert_parity(got, oracle_decode(blob, dt), dt, f"{what} dt={dt}")


@pytest.mark.parametrize("b,bpp", [(9, 3.0), (10, 4.0), (11, 4.0), (11, 6.0), (12, 7.5), (13, 7.5), (15, 7.5)])
def test_every_precision(b, bpp):
    rng = np.random.default_rng(7 * b)
    W = (rng.standard_t(5, (96, 1024)) * 0.02 * np.exp(rng.normal(0, 0.4, (96, 1)))).astype(np.float32)
    ob = oracle.encode(W, bpp, prob_bits=b, tile_vectors=100)
    assert ob.b == b
    _prepared(as_lib_blob(ob), [ep.BF16, ep.FP8_E4M3, ep.INT8, ep.UINT8, ep.FP32, ep.LATTICE_I32], f"b={b}")


@pytest.mark.parametrize("lo,hi,p", [(12.0, 40.0, 0.01), (20.0, 60.0, 0.02)])
def test_two_level_and_bucketed_tables_at_8bpp(lo, hi, p):
    """b = 12 with sparse, widely spaced outliers: the two-level table with its bounded walk,
    and with larger alphabets the bucketed table."""
    rng = np.random.default_rng(5)
    W = rng.standard_normal((512, 1024)).astype(np.float32)
    mask = rng.random(W.shape) < p
    W[mask] = (rng.choice([-1, 1], mask.sum()) * rng.uniform(lo, hi, mask.sum())).astype(np.float32)
    blob = ep.encode_tensor(W, 8.0)
    assert blob.b == 12
    _prepared(blob, [ep.BF16, ep.LATTICE_I32], f"outliers {lo}-{hi}")


def test_one_coset_and_full_alphabet():
    b = 9
    M = 1 << b
    nvec = 6 * M
    z = np.zeros((nvec, 8))
    z[:, 0] = np.tile(np.arange(M), 6) - M // 2
    z[:, 1:7] = np.random.default_rng(1).integers(-3, 4, (nvec, 6))
    z[:, 7] = z[:, :7].sum(axis=1) % 2
    f = oracle.fields_of(z, np.zeros(nvec, np.int32))
    rows, cols = 12, 8 * nvec // 12
    ob = oracle.encode_fields(f, rows, cols, np.linspace(0.01, 0.1, rows).astype(np.float32), b, 200)
    _prepared(as_lib_blob(ob), [ep.BF16, ep.LATTICE_I32], "one coset")


@pytest.mark.parametrize("rows,cols,V", [(3, 5, 2), (17, 1001, 100), (64, 1020, 1820), (1, 8, 32)])
def test_shapes_and_ragged_widths(rows, cols, V):
    rng = np.random.default_rng(rows + cols)
    W = (rng.standard_t(5, (rows, cols)) * 0.02).astype(np.float32)
    ob = oracle.encode(W, 5.0, tile_vectors=V)
    _prepared(as_lib_blob(ob), [ep.BF16, ep.FP32, ep.INT8], f"{rows}x{cols}")


def test_one_table_shared_by_two_streams():
    """The prepared table is only read: two streams decode with it at the same time."""
    import torch

    blob = ep.encode_tensor(synth.generate(synth.small_fp32(seed=21)), 4.0, tile_vectors=64)
    db = ep.DeviceBlob(blob)
    lut = ep.prepare_lut(db)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    for k in range(6):
        s = (s1, s2)[k % 2]
        with torch.cuda.stream(s):
            outs.append(ep.decode_tensor_prepared(db, lut, ep.BF16, stream=s))
    torch.cuda.synchronize()
    assert ep.decode_status() == 0
    want = oracle_decode(blob, ep.BF16)
    for o in outs:
        assert_parity(to_raw(o), want, ep.BF16, "two streams")


def test_graph_capture_and_replay():
    import torch

    b1 = ep.encode_tensor(synth.generate(synth.small_fp32(seed=22)), 4.0)
    b2 = ep.encode_tensor(synth.generate(synth.small_fp32(seed=23)), 8.0, tile_vectors=100)
    d1, d2 = ep.DeviceBlob(b1), ep.DeviceBlob(b2)
    l1, l2 = ep.prepare_lut(d1), ep.prepare_lut(d2)
    o1 = ep.decode_tensor_prepared(d1, l1, ep.BF16)
    o2 = ep.decode_tensor_prepared(d2, l2, ep.FP16)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        ep.decode_tensor_prepared(d1, l1, ep.BF16, out=o1, stream=s)
        ep.decode_tensor_prepared(d2, l2, ep.FP16, out=o2, stream=s)
    o1.zero_()
    o2.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert ep.decode_status() == 0
    assert_parity(to_raw(o1), oracle_decode(b1, ep.BF16), ep.BF16, "graph 1")
    assert_parity(to_raw(o2), oracle_decode(b2, ep.FP16), ep.FP16, "graph 2")
    del g


def test_table_of_another_layout_is_refused():
    """A table prepared for another header (here another b), or a buffer ep_decode_prepare never
    wrote, raises EP_ECORRUPT and leaves the output untouched."""
    import torch

    rng = np.random.default_rng(31)
    W = (rng.standard_normal((64, 512)) * 0.02).astype(np.float32)
    a = ep.DeviceBlob(ep.encode_tensor(W, 4.0, prob_bits=11, tile_vectors=64))
    b = ep.DeviceBlob(ep.encode_tensor(W, 4.0, prob_bits=10, tile_vectors=64))
    lut_a = ep.prepare_lut(a)
    assert ep.decode_status() == 0
    blank = torch.zeros(ep.LUT_BYTES, dtype=torch.uint8, device="cuda")
    for lut in (lut_a, blank):
        out = torch.full((64, 512), 7.0, dtype=torch.bfloat16, device="cuda")
        ep.decode_tensor_prepared(b, lut, ep.BF16, out=out)
        assert ep.decode_status() == ECORRUPT
        assert bool((out == 7.0).all())
    # the device stays usable and the right table still decodes exactly
    got = to_raw(ep.decode_tensor_prepared(b, ep.prepare_lut(b), ep.BF16))
    assert ep.decode_status() == 0
    blob_b = ep.encode_tensor(W, 4.0, prob_bits=10, tile_vectors=64)
    assert_parity(got, oracle_decode(blob_b, ep.BF16), ep.BF16, "after refusal")


def test_bad_tables_and_corrupt_payload_raise_status():
    rng = np.random.default_rng(9)
    W = (rng.standard_normal((128, 1024)) * 0.02).astype(np.float32)
    good = ep.encode_tensor(W, 4.0, tile_vectors=200)
    ft = good.freq_tables.copy()
    ft[-2:] = np.array([ft[-2:].view(np.uint16)[0] + 1], np.uint16).view(np.uint8)  # a table sums past 2^b
    bad = ep.Blob(good.rows, good.cols, good.b, good.V, good.ntiles, good.payload, good.payload_words,
                  good.tile_index, ft, good.row_scales)
    db = ep.DeviceBlob(bad)
    lut = ep.prepare_lut(db)
    assert ep.decode_status() == ECORRUPT      # the preparation reports the table
    ep.decode_tensor_prepared(db, lut, ep.BF16)
    assert ep.decode_status() == ECORRUPT      # and so does every decode with it
    p = good.payload.copy()
    p[good.payload_words // 2] ^= 0x1234
    corrupt = ep.Blob(good.rows, good.cols, good.b, good.V, good.ntiles, p, good.payload_words,
                      good.tile_index, good.freq_tables, good.row_scales)
    dc = ep.DeviceBlob(corrupt)
    ep.decode_tensor_prepared(dc, ep.prepare_lut(dc), ep.BF16)
    assert ep.decode_status() == ECORRUPT
    dg = ep.DeviceBlob(good)
    got = to_raw(ep.decode_tensor_prepared(dg, ep.prepare_lut(dg), ep.BF16))
    assert ep.decode_status() == 0
    assert_parity(got, oracle_decode(good, ep.BF16), ep.BF16, "good after corrupt")


def test_headline_3840x10240_prepared_equals_oracle_samples():
    """Full size: the prepared decode equals the per-call decode everywhere, and the oracle on a
    seeded sample of tiles (plus the first and the last)."""
    W = synth.generate(synth.headline())
    blob = ep.encode_tensor(W, 4.0)
    db = ep.DeviceBlob(blob)
    lut = ep.prepare_lut(db)
    got = to_raw(ep.decode_tensor_prepared(db, lut, ep.BF16)).reshape(-1)
    ref = to_raw(ep.decode_tensor(db, ep.BF16)).reshape(-1)
    assert ep.decode_status() == 0
    np.testing.assert_array_equal(got, ref)
    rng = np.random.default_rng(777)
    per = 8 * blob.V
    for t in sorted(set([0, blob.ntiles - 1] + list(rng.choice(blob.ntiles, 12, replace=False)))):
        lo, hi = t * per, min((t + 1) * per, blob.rows * blob.cols)
        assert_parity(got[lo:hi], oracle_decode(blob, ep.BF16, t, t + 1), ep.BF16, f"tile {t}")
