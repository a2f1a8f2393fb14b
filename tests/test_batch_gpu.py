"""GPU parity of the batched decode (ep_batch_create / ep_decode_batch): several tensors in one
launch, each SM decoding a share of one tensor's tiles with that tensor's prepared table.
Expected values come only from the oracle's decoder (full decodes for the small tensors,
seeded tile samples at full size); the comparison is bit-exact."""
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
    ep.decode_status()


def _mixed_blobs():
    """Tensors that take every LUT format and shape path: packed b = 9..11, the two-level table
    (b = 12), the bucketed one (b = 13), a ragged width, a one-tile tensor."""
    rng = np.random.default_rng(41)
    out = []
    for rows, cols, bpp, b, V in [(96, 1024, 3.0, 9, 100), (64, 512, 4.0, 11, 64), (128, 768, 7.5, 12, 50),
                                  (80, 1024, 7.5, 13, 128), (17, 1001, 5.0, 0, 100), (4, 64, 4.0, 0, 32),
                                  (256, 512, 2.3, 0, 0)]:
        W = (rng.standard_t(5, (rows, cols)) * 0.02 * np.exp(rng.normal(0, 0.4, (rows, 1)))).astype(np.float32)
        out.append(as_lib_blob(oracle.encode(W, bpp, prob_bits=b, tile_vectors=V)))
    return out


@pytest.mark.parametrize("dt", [ep.BF16, ep.FP16, ep.FP8_E4M3, ep.INT8, ep.UINT8, ep.FP32, ep.LATTICE_I32])
def test_mixed_batch_every_dtype(dt):
    blobs = _mixed_blobs()
    dbs = [ep.DeviceBlob(b) for b in blobs]
    batch = ep.DecodeBatch([(db, ep.prepare_lut(db), None) for db in dbs], dt)
    outs = batch.run()
    assert ep.decode_status() == 0
    for k, (blob, o) in enumerate(zip(blobs, outs)):
        assert_parity(to_raw(o), oracle_decode(blob, dt), dt, f"item {k} dt={dt}")


def test_single_item_batch_equals_oracle():
    blob = ep.encode_tensor(synth.generate(synth.small_fp32(seed=31)), 4.0)
    db = ep.DeviceBlob(blob)
    (o,) = ep.DecodeBatch([(db, ep.prepare_lut(db), None)], ep.BF16).run()
    assert ep.decode_status() == 0
    assert_parity(to_raw(o), oracle_decode(blob, ep.BF16), ep.BF16, "one item")


def test_batch_graph_replay_and_repeat():
    import torch

    blobs = _mixed_blobs()[:4]
    dbs = [ep.DeviceBlob(b) for b in blobs]
    batch = ep.DecodeBatch([(db, ep.prepare_lut(db), None) for db in dbs], ep.BF16)
    batch.run()
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        batch.run(stream=s)
    for o in batch.outputs:
        o.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert ep.decode_status() == 0
    for blob, o in zip(blobs, batch.outputs):
        assert_parity(to_raw(o), oracle_decode(blob, ep.BF16), ep.BF16, "graph")
    del g


def test_wrong_table_in_a_batch_is_refused_and_the_rest_decodes():
    import torch

    blobs = _mixed_blobs()[:3]
    dbs = [ep.DeviceBlob(b) for b in blobs]
    luts = [ep.prepare_lut(db) for db in dbs]
    outs = [torch.full((b.rows, b.cols), 3.0, dtype=torch.bfloat16, device="cuda") for b in blobs]
    # item 1 gets item 0's table (another b): refused, its output untouched
    batch = ep.DecodeBatch([(dbs[0], luts[0], outs[0]), (dbs[1], luts[0], outs[1]), (dbs[2], luts[2], outs[2])],
                           ep.BF16)
    batch.run()
    assert ep.decode_status() == ECORRUPT
    assert bool((outs[1] == 3.0).all())
    for k in (0, 2):
        assert_parity(to_raw(outs[k]), oracle_decode(blobs[k], ep.BF16), ep.BF16, f"item {k}")


def test_dit_block_at_mixed_rates_full_size():
    """One block of the DiT stack (qkv, out, gate, up, down) at the rates of the stack's first
    block, decoded in one launch: equal to each tensor's own decode everywhere, and to the oracle
    on a seeded sample of tiles of every tensor."""
    alloc = synth.dit_stack_bpp()
    kinds = ["qkv", "out", "gate", "up", "down"]
    bpps = [alloc[(0, k)] for k in kinds]
    blobs = [ep.encode_tensor(synth.generate(synth.dit_stack_layer(0, k)), float(bp)) for k, bp in zip(kinds, bpps)]
    dbs = [ep.DeviceBlob(b) for b in blobs]
    outs = ep.DecodeBatch([(db, ep.prepare_lut(db), None) for db in dbs], ep.BF16).run()
    assert ep.decode_status() == 0
    rng = np.random.default_rng(99)
    for k, (blob, db, o) in enumerate(zip(blobs, dbs, outs)):
        got = to_raw(o).reshape(-1)
        ref = to_raw(ep.decode_tensor(db, ep.BF16)).reshape(-1)
        np.testing.assert_array_equal(got, ref)
        per = 8 * blob.V
        for t in sorted(set([0, blob.ntiles - 1] + list(rng.choice(blob.ntiles, 4, replace=False)))):
            lo, hi = t * per, min((t + 1) * per, blob.rows * blob.cols)
            assert_parity(got[lo:hi], oracle_decode(blob, ep.BF16, t, t + 1), ep.BF16, f"{kinds[k]} tile {t}")
    assert ep.decode_status() == 0


def test_one_tensor_per_sm_and_the_limit():
    """As many tensors as SMs (each on one SM), then one more: refused on the host."""
    import torch

    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    rng = np.random.default_rng(77)
    blobs = []
    for k in range(nsm):
        rows, cols = int(rng.integers(1, 40)), 8 * int(rng.integers(1, 64))
        W = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
        blobs.append(ep.encode_tensor(W, float(rng.choice([2.5, 4.0, 8.0])), tile_vectors=int(rng.integers(8, 200))))
    dbs = [ep.DeviceBlob(b) for b in blobs]
    items = [(db, ep.prepare_lut(db), None) for db in dbs]
    outs = ep.DecodeBatch(items, ep.BF16).run()
    assert ep.decode_status() == 0
    for k, (blob, o) in enumerate(zip(blobs, outs)):
        assert_parity(to_raw(o), oracle_decode(blob, ep.BF16), ep.BF16, f"item {k}")
    with pytest.raises(ep.EntroPackError):
        ep.DecodeBatch(items + items[:1], ep.BF16)


@pytest.mark.parametrize("num_ctas", [7, 8, 23, 100])
def test_batch_on_part_of_the_gpu(num_ctas):
    """ep_batch_create_on: the mixed batch on a few SMs (several tiles per warp, several tensors
    sharing few CTAs) decodes exactly as on all of them."""
    blobs = _mixed_blobs()
    dbs = [ep.DeviceBlob(b) for b in blobs]
    outs = ep.DecodeBatch([(db, ep.prepare_lut(db), None) for db in dbs], ep.BF16, num_ctas=num_ctas).run()
    assert ep.decode_status() == 0
    for k, (blob, o) in enumerate(zip(blobs, outs)):
        assert_parity(to_raw(o), oracle_decode(blob, ep.BF16), ep.BF16, f"item {k} on {num_ctas} CTAs")


def test_headline_on_one_sm_sampled_tiles():
    """The 2,701-tile headline tensor on a single CTA: every warp walks about 113 tiles."""
    blob = ep.encode_tensor(synth.generate(synth.headline()), 4.0)
    db = ep.DeviceBlob(blob)
    (o,) = ep.DecodeBatch([(db, ep.prepare_lut(db), None)], ep.BF16, num_ctas=1).run()
    assert ep.decode_status() == 0
    got = to_raw(o).reshape(-1)
    per = 8 * blob.V
    rng = np.random.default_rng(5)
    for t in sorted(set([0, 1, 24, blob.ntiles - 1] + list(rng.choice(blob.ntiles, 6, replace=False)))):
        lo, hi = t * per, min((t + 1) * per, blob.rows * blob.cols)
        assert_parity(got[lo:hi], oracle_decode(blob, ep.BF16, t, t + 1), ep.BF16, f"tile {t}")


def test_batch_cta_count_refusals():
    import torch

    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    blobs = _mixed_blobs()
    dbs = [ep.DeviceBlob(b) for b in blobs]
    items = [(db, ep.prepare_lut(db), None) for db in dbs]
    for bad in (nsm + 1, len(items) - 1, -1):
        with pytest.raises(ep.EntroPackError):
            ep.DecodeBatch(items, ep.BF16, num_ctas=bad)
    ep.DecodeBatch(items, ep.BF16, num_ctas=len(items)).run()  # one CTA per tensor is allowed
    assert ep.decode_status() == 0
