"""GPU parity: ep_decode_tensor (through the C ABI) against the CPU oracle.

Inputs are seeded synthetic tensors; streams come from the oracle's encoder for
the small cases and from the library's packer (byte-identical to the oracle's
encoder, see test_packer.py) for the full-size workloads.  Expected values come
only from the oracle's decoder.  The comparison is bit-exact for every output
type (the spec allows 1 ulp for floating outputs; the single-rounding FFMA design
reaches exact equality).
"""
import numpy as np
import pytest

import oracle
import dit_weight_compression_ep_b200 as ep
from dit_weight_compression_ep_b200 import synth
from gpu_util import as_lib_blob, assert_parity, oracle_decode, to_raw

pytestmark = pytest.mark.gpu

ALL_DT = [ep.BF16, ep.FP16, ep.FP8_E4M3, ep.INT8, ep.FP32, ep.LATTICE_I32, ep.UINT8]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dit_weight_compression_ep_b200 import build

    build.build()
    ep.lib()
    ep.decode_status()  # clear the status word


def _gpu(blob, dt, stream=None):
    db = ep.DeviceBlob(blob)
    out = ep.decode_tensor(db, dt, stream=stream)
    rc = ep.decode_status(stream)
    assert rc == 0, f"device status {rc}"
    return to_raw(out)


def _check(blob, dts=ALL_DT, what=""):
    for dt in dts:
        assert_parity(_gpu(blob, dt), oracle_decode(blob, dt), dt, f"{what} dt={dt}")


# ---------------------------------------------------------------- small cases

def test_small_fp32_all_dtypes():
    W = synth.generate(synth.small_fp32())
    ob = oracle.encode(W, 4.0, prob_bits=12, tile_vectors=512)
    assert ob.ntiles == 32 and ob.b == 12
    _check(as_lib_blob(ob), what="256x512 fp32")


@pytest.mark.parametrize("b", [9, 10, 11, 12, 13, 15])
@pytest.mark.parametrize("V", [32, 33, 100, 455])
def test_precisions_and_tile_sizes(b, V):
    rng = np.random.default_rng(100 * b + V)
    W = (rng.standard_normal((96, 1024)) * 0.02 * np.exp(rng.normal(0, 0.4, (96, 1)))).astype(np.float32)
    ob = oracle.encode(W, 4.0 if b <= 11 else 7.5, prob_bits=b, tile_vectors=V)
    assert ob.b == b
    _check(as_lib_blob(ob), [ep.BF16, ep.INT8, ep.LATTICE_I32, ep.UINT8], f"b={b} V={V}")


@pytest.mark.parametrize("rows,cols,V", [(1, 8, 32), (1, 256, 1), (3, 64, 32), (5, 24, 7), (17, 8, 50),
                                         (40, 2048, 1820), (7, 4096, 3640)])
def test_shapes(rows, cols, V):
    rng = np.random.default_rng(rows * cols + V)
    W = (rng.standard_t(5, (rows, cols)) * 0.02).astype(np.float32)
    ob = oracle.encode(W, 5.0, tile_vectors=V)
    _check(as_lib_blob(ob), [ep.BF16, ep.FP32, ep.LATTICE_I32], f"{rows}x{cols} V={V}")


@pytest.mark.parametrize("rows,cols,V", [(3, 5, 2), (40, 60, 32), (17, 1001, 100), (9, 4097, 455), (300, 1, 33),
                                         (64, 1020, 1820)])
def test_widths_not_a_multiple_of_8(rows, cols, V):
    """Rows padded to whole vectors: the decoder writes the real entries element by element."""
    rng = np.random.default_rng(rows * cols + V)
    W = (rng.standard_t(5, (rows, cols)) * 0.02).astype(np.float32)
    ob = oracle.encode(W, 5.0, tile_vectors=V)
    _check(as_lib_blob(ob), ALL_DT, f"{rows}x{cols} V={V}")


def test_one_coset_and_wide_alphabet():
    # every vector in D8 (the c = 1 tables are empty) and a coordinate alphabet of exactly 2^b
    b = 9
    M = 1 << b
    nvec = 6 * M
    z = np.zeros((nvec, 8))
    z[:, 0] = np.tile(np.arange(M), 6) - M // 2
    z[:, 1:7] = np.random.default_rng(1).integers(-3, 4, (nvec, 6))
    z[:, 7] = z[:, :7].sum(axis=1) % 2
    f = oracle.fields_of(z, np.zeros(nvec, np.int32))
    rows, cols = 12, 8 * nvec // 12
    rs = np.linspace(0.01, 0.1, rows).astype(np.float32)
    ob = oracle.encode_fields(f, rows, cols, rs, b, 200)
    _check(as_lib_blob(ob), ALL_DT, "one coset, A = 2^b")


def test_rdo_stream():
    """A stream from the per-row refinement (App. C.2): rows at different resolutions, same decoder."""
    rng = np.random.default_rng(14)
    W = np.empty((128, 512), np.float32)
    for r in range(128):
        W[r] = rng.standard_t([2.5, 4, 8, 30][r % 4], 512) * 0.02 * np.exp(rng.normal(0, 0.5))
    ob = oracle.encode(W, 3.0, rdo_candidates=5, tile_vectors=200)
    _check(as_lib_blob(ob), [ep.BF16, ep.FP32, ep.LATTICE_I32], "rdo K=5")


def test_zero_rows_and_signed_zeros():
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((64, 512)) * 0.05).astype(np.float32)
    W[3] = 0
    W[10] = -W[10]
    ob = oracle.encode(W, 3.0, tile_vectors=64)
    _check(as_lib_blob(ob), ALL_DT, "zero rows")


def test_tiny_and_negative_scales():
    # rows whose reconstruction scale is subnormal, zero or negative take the exact slow path
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((32, 256)) * 0.05).astype(np.float32)
    ob = oracle.encode(W, 4.0, tile_vectors=64)
    rs = ob.row_scales.copy()
    rs[0] = np.float32(1e-39)
    rs[1] = np.float32(-3e-38)
    rs[2] = np.float32(0.0)
    rs[3] = np.float32(-0.5)
    rs[4] = np.float32(2.0 ** -125)
    blob = ep.Blob.from_arrays(ob.payload, ob.tile_index, ob.freq_tables, rs, ob.rows, ob.cols)
    _check(blob, ALL_DT, "tiny scales")


def test_two_tensors_on_two_streams_at_once():
    """Two tensors decoded over and over on two streams with no ordering between the streams:
    per call (the library orders its per-call decodes through its workspace) and with
    prepared tables (no shared state: the launches may overlap on the GPU).  Every output
    equals the oracle."""
    import torch

    blobs = [ep.encode_tensor(synth.generate(synth.headline())[:1024, :4096].copy(), 4.0),
             ep.encode_tensor(synth.generate(synth.dit_attn_proj())[:2048, :2048].copy(), 8.0)]
    dbs = [ep.DeviceBlob(b) for b in blobs]
    outs = [torch.zeros((b.rows, b.cols), dtype=torch.bfloat16, device="cuda") for b in blobs]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    torch.cuda.synchronize()
    ep.decode_status()
    for _ in range(6):
        for db, out, st in zip(dbs, outs, streams):
            ep.decode_tensor(db, ep.BF16, out=out, stream=st)
    torch.cuda.synchronize()
    assert ep.decode_status() == 0
    for b, out in zip(blobs, outs):
        assert_parity(to_raw(out), oracle_decode(b, ep.BF16), ep.BF16, "two streams, per call")
    luts = [ep.prepare_lut(db) for db in dbs]
    pouts = [torch.zeros_like(o) for o in outs]
    torch.cuda.synchronize()
    for _ in range(6):
        for db, lut, out, st in zip(dbs, luts, pouts, streams):
            ep.decode_tensor_prepared(db, lut, ep.BF16, out=out, stream=st)
    torch.cuda.synchronize()
    assert ep.decode_status() == 0
    for b, out in zip(blobs, pouts):
        assert_parity(to_raw(out), oracle_decode(b, ep.BF16), ep.BF16, "two streams, prepared")


def test_repeat_on_side_stream():
    import torch

    W = synth.generate(synth.small_fp32(seed=11))
    blob = ep.encode_tensor(W, 4.0)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        a = _gpu(blob, ep.BF16, stream=s)
        b = _gpu(blob, ep.BF16, stream=s)
    np.testing.assert_array_equal(a, b)
    assert_parity(a, oracle_decode(blob, ep.BF16), ep.BF16, "side stream")


def test_cuda_graph_capture_and_replay():
    """Two decodes of different streams captured in one CUDA graph (the library's first call on
    the device happens before the capture) and replayed: the same bits as the oracle."""
    import torch

    b1 = ep.encode_tensor(synth.generate(synth.small_fp32(seed=12)), 4.0)
    b2 = ep.encode_tensor(synth.generate(synth.small_fp32(seed=13)), 6.0, tile_vectors=100)
    d1, d2 = ep.DeviceBlob(b1), ep.DeviceBlob(b2)
    o1 = ep.decode_tensor(d1, ep.BF16)
    o2 = ep.decode_tensor(d2, ep.FP16)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ep.decode_tensor(d1, ep.BF16, out=o1)
        ep.decode_tensor(d2, ep.FP16, out=o2)
    o1.zero_()
    o2.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert ep.decode_status() == 0
    assert_parity(to_raw(o1).reshape(-1), oracle_decode(b1, ep.BF16), ep.BF16, "graph 1")
    assert_parity(to_raw(o2).reshape(-1), oracle_decode(b2, ep.FP16), ep.FP16, "graph 2")
    del g


# ------------------------------------------------------------ corrupt streams

def _status_of(blob):
    db = ep.DeviceBlob(blob)
    ep.decode_tensor(db, ep.BF16)
    return ep.decode_status()


def test_corruption_sets_status_without_fault():
    rng = np.random.default_rng(9)
    W = (rng.standard_normal((128, 1024)) * 0.02).astype(np.float32)
    good = ep.encode_tensor(W, 4.0, tile_vectors=200)
    assert _status_of(good) == 0

    def variant(**kw):
        d = dict(payload=good.payload.copy(), tile_index=good.tile_index.copy(),
                 freq_tables=good.freq_tables.copy(), row_scales=good.row_scales.copy())
        d.update(kw)
        b = ep.Blob(good.rows, good.cols, good.b, good.V, good.ntiles, d["payload"], good.payload_words,
                    d["tile_index"], d["freq_tables"], d["row_scales"])
        return b

    p = good.payload.copy()
    p[good.payload_words // 2] ^= 0x1234
    assert _status_of(variant(payload=p)) == ep._lib.STATUS_CODES["EP_ECORRUPT"]
    t = good.tile_index.copy()
    t[1 + 33 * 3] = 7                       # a state below 2^15
    assert _status_of(variant(tile_index=t)) == ep._lib.STATUS_CODES["EP_ECORRUPT"]
    t = good.tile_index.copy()
    t[33 * 2] = t[33 * 3] + 5               # offsets out of order
    assert _status_of(variant(tile_index=t)) == ep._lib.STATUS_CODES["EP_ECORRUPT"]
    t = good.tile_index.copy()
    t[33 * 4] = 0                           # a truncated tile
    assert _status_of(variant(tile_index=t)) == ep._lib.STATUS_CODES["EP_ECORRUPT"]
    ft = good.freq_tables.copy()
    ft[0] ^= 0xFF                           # bad magic
    assert _status_of(variant(freq_tables=ft)) == ep._lib.STATUS_CODES["EP_ECORRUPT"]
    ft = good.freq_tables.copy()
    ft[8:12] = np.array([16], np.uint32).view(np.uint8)   # b > 15
    assert _status_of(variant(freq_tables=ft)) == ep._lib.STATUS_CODES["EP_ECORRUPT"]
    ft = good.freq_tables.copy()
    ft[-2:] = np.array([ft[-2:].view(np.uint16)[0] + 1], np.uint16).view(np.uint8)  # sum != 2^b
    assert _status_of(variant(freq_tables=ft)) == ep._lib.STATUS_CODES["EP_ECORRUPT"]
    ft = good.freq_tables.copy()
    ft[44:48] = np.array([1], np.uint32).view(np.uint8)   # an ablation variant the GPU does not decode
    assert _status_of(variant(freq_tables=ft)) == ep._lib.STATUS_CODES["EP_EUNSUPPORTED"]
    # the device stays usable: a good stream still decodes exactly
    assert _status_of(good) == 0
    assert_parity(_gpu(good, ep.BF16), oracle_decode(good, ep.BF16), ep.BF16, "after corruption")


# ---------------------------------------------------- full-size workloads

def _full_check(blob, dts, what, sample_tiles=None):
    """Full oracle decode, or (sample_tiles) a seeded sample of tiles + first/last."""
    db = ep.DeviceBlob(blob)
    for dt in dts:
        out = ep.decode_tensor(db, dt)
        assert ep.decode_status() == 0
        got = to_raw(out).reshape(-1)
        if sample_tiles is None:
            assert_parity(got, oracle_decode(blob, dt), dt, what)
        else:
            rng = np.random.default_rng(12345)
            tiles = sorted(set([0, blob.ntiles - 1] + list(rng.choice(blob.ntiles, sample_tiles, replace=False))))
            per = 8 * blob.V
            for t in tiles:
                lo = t * per
                hi = min(lo + per, blob.rows * blob.cols)
                assert_parity(got[lo:hi], oracle_decode(blob, dt, t, t + 1), dt, f"{what} tile {t}")
        del out


def _slot_pairs_past_15(blob):
    """Host-side look at the stored tables: (b, slot pairs whose odd slot's symbol lies 15 or
    more symbols past the even slot's, records the two-level LUT would need)."""
    ft = blob.freq_tables
    b = int(ft[:48].view(np.uint32)[2])
    d = ft[48:48 + 17 * 8].view(np.int32).reshape(17, 2)
    fq = ft[192:].view(np.uint16).astype(np.int64)
    A = d[:, 1].astype(np.int64)
    off = np.concatenate([[0], np.cumsum(A)[:-1]])
    far, nrec = 0, 1
    for t in range(1, 17):
        cum = np.concatenate([[0], np.cumsum(fq[off[t]:off[t] + A[t]])])
        nrec += int(A[t]) + 1
        own = np.searchsorted(cum[:A[t]], np.arange(1 << b), side="right") - 1
        far += int(np.sum(own[1::2] - own[0::2] >= 15))
    return b, far, nrec


@pytest.mark.parametrize("lo,hi,p,two", [(12.0, 40.0, 0.01, True), (20.0, 60.0, 0.02, False)])
def test_sparse_outlier_alphabets_at_8bpp(lo, hi, p, two):
    """b = 12 with sparse, widely spaced outliers: many slot pairs whose odd slot's symbol is 15
    or more symbols on (the two-level LUT's bounded walk), and, with larger alphabets, the
    bucketed LUT.  Bit-exact against the oracle."""
    rng = np.random.default_rng(5)
    W = rng.standard_normal((512, 1024)).astype(np.float32)
    mask = rng.random(W.shape) < p
    W[mask] = (rng.choice([-1, 1], mask.sum()) * rng.uniform(lo, hi, mask.sum())).astype(np.float32)
    blob = ep.encode_tensor(W, 8.0)
    b, far, nrec = _slot_pairs_past_15(blob)
    assert b == 12 and far > 50
    assert (nrec <= 32768) == two  # the header rule that picks the two-level LUT
    _full_check(blob, [ep.BF16, ep.LATTICE_I32], f"sparse outliers {lo}-{hi}")


def test_headline_3840x10240_bf16_4bpp():
    W = synth.generate(synth.headline())
    blob = ep.encode_tensor(W, 4.0)
    assert blob.b == 11 and blob.V == 1820 and blob.ntiles == 2701
    _full_check(blob, [ep.BF16, ep.FP16], "headline")
    # property at full size: every decoded point lies in E8
    import torch

    y2 = ep.decode_tensor(ep.DeviceBlob(blob), ep.LATTICE_I32).view(-1, 8).to(torch.int64)
    par = y2 & 1
    assert bool((par == par[:, :1]).all()) and bool(((y2.sum(dim=1) // 2) % 2 == 0).all())


def test_dit_attention_projection_5bpp():
    W = synth.generate(synth.dit_attn_proj())
    blob = ep.encode_tensor(W, 5.0)
    _full_check(blob, [ep.BF16, ep.FP16], "attn proj")


def test_fp8_and_int8_containers_5bpp():
    src = synth.generate(synth.lowp_source())
    for kind in ("e4m3", "int8"):
        vals, scales = synth.to_e4m3_container(src) if kind == "e4m3" else synth.to_int8_container(src)
        blob = ep.encode_tensor(vals, 5.0, has_container_scales=True)
        assert abs(blob.stored_bpp / 5.0 - 1) < 0.03
        dt = ep.FP8_E4M3 if kind == "e4m3" else ep.INT8
        _full_check(blob, [dt], kind)


def test_uint8_container_5bpp():
    """UINT8 container (per-tensor scale, offset 128): the codec codes the codes minus 128 and
    the decoder adds it back; bit-exact against the oracle, and the round trip stays close."""
    src = synth.generate(synth.lowp_source())
    vals, _ = synth.to_uint8_container(src)
    blob = ep.encode_tensor(vals, 5.0)
    assert abs(blob.stored_bpp / 5.0 - 1) < 0.03
    _full_check(blob, [ep.UINT8], "uint8")
    import torch

    out = ep.decode_tensor(ep.DeviceBlob(blob), ep.UINT8).cpu().numpy().astype(np.float64) - 128.0
    rel = np.linalg.norm(out - vals) / np.linalg.norm(vals)
    assert rel < 0.1, rel


@pytest.mark.parametrize("wide", [True, False])
def test_llm_prefill_sweep_sampled(wide):
    W = synth.generate(synth.llm_prefill(wide))
    prev = None
    for bpp in (2, 3, 4, 5, 6, 7, 8):
        blob = ep.encode_tensor(W, float(bpp))
        assert abs(blob.stored_bpp / bpp - 1) < 0.03
        _full_check(blob, [ep.BF16], f"llm {wide} {bpp}", sample_tiles=24)
        import torch

        out = ep.decode_tensor(ep.DeviceBlob(blob), ep.FP32)
        Wt = torch.from_numpy(W).cuda()
        rel = float(torch.linalg.vector_norm(out - Wt) / torch.linalg.vector_norm(Wt))
        if prev is not None:
            assert rel < prev
        prev = rel
        del out, Wt


def test_dit_stack_layers_sampled():
    alloc = synth.dit_stack_bpp()
    for kind in synth.DIT_KINDS:
        blk = 7
        W = synth.generate(synth.dit_stack_layer(blk, kind))
        blob = ep.encode_tensor(W, alloc[(blk, kind)])
        _full_check(blob, [ep.BF16], f"dit {kind}", sample_tiles=16)


def test_binding_refuses_outputs_it_cannot_fill():
    """The C ABI takes bare output pointers; the binding checks a given buffer's device, dtype,
    layout and extent before passing it on (no launch happens on a refusal)."""
    import torch

    blob = ep.encode_tensor(synth.generate(synth.small_fp32(seed=3)), 4.0)
    db = ep.DeviceBlob(blob)
    lut = ep.prepare_lut(db)
    small = torch.empty((blob.rows, blob.cols - 8), dtype=torch.bfloat16, device="cuda")
    host = torch.empty((blob.rows, blob.cols), dtype=torch.bfloat16)
    wrong = torch.empty((blob.rows, blob.cols), dtype=torch.float16, device="cuda")
    strided = torch.empty((blob.cols, blob.rows), dtype=torch.bfloat16, device="cuda").t()
    for out in (small, host, wrong, strided):
        with pytest.raises(ValueError):
            ep.decode_tensor(db, ep.BF16, out=out)
        with pytest.raises(ValueError):
            ep.decode_tensor_prepared(db, lut, ep.BF16, out=out)
        with pytest.raises(ValueError):
            ep.decode_tensor_noalloc(db, ep.BF16, out=out)
    with pytest.raises(ValueError):
        ep.decode_tensor_prepared(db, lut.cpu(), ep.BF16)
    x = torch.zeros((2, blob.cols), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        ep.decode_gemv(db, x, y=torch.empty((1, blob.rows), device="cuda"))
    assert ep.decode_status() == 0
    # a larger contiguous buffer of the right dtype is accepted (the result fills its head)
    big = torch.empty((blob.rows + 3, blob.cols), dtype=torch.bfloat16, device="cuda")
    ep.decode_tensor(db, ep.BF16, out=big)
    assert ep.decode_status() == 0
    assert np.array_equal(to_raw(big).reshape(-1)[: blob.rows * blob.cols], oracle_decode(blob, ep.BF16))


@pytest.mark.parametrize("zero_first_column,bpp", [(False, 4.0), (False, 6.6), (True, 6.6), (True, 4.0)])
@pytest.mark.parametrize("dt", [ep.BF16, ep.LATTICE_I32])
def test_packed_table_field_widths(zero_first_column, bpp, dt):
    """Both packed-entry layouts at b = 11: f in b + 1 bits (coordinate alphabets within +-256, at
    4 bpp) and f - 1 in b bits (wider alphabets, at 6.6 bpp), each with and without a
    single-symbol coordinate table (every vector's first coordinate zero, so coset 0's z1 table
    holds only 0, f = 2^b).  Bit-exact against the oracle."""
    rng = np.random.default_rng(41)
    W = (rng.standard_t(6, (256, 1024)) * 0.02).astype(np.float32)
    if zero_first_column:
        W[:, ::8] = 0.0
    blob = ep.encode_tensor(W, bpp)
    assert blob.b == 11
    db = ep.DeviceBlob(blob)
    for got in (ep.decode_tensor(db, dt), ep.decode_tensor_prepared(db, ep.prepare_lut(db), dt)):
        assert ep.decode_status() == 0
        assert_parity(to_raw(got), oracle_decode(blob, dt), dt, f"bpp {bpp}, zeroed column {zero_first_column}")
