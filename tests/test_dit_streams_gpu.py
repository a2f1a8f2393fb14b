"""Every (layer kind, rate) stream of the 30-block DiT linear stack, decoded on the GPU and
checked against the oracle.

The stack has five layer kinds (qkv 11520x3840, out 3840x3840, gate and up 10240x3840, down
3840x10240) and each layer's rate is drawn from {2.3, 3, 4, 6, 8} bpp, so 25 (kind, rate)
pairs occur; each pair is taken at the first block where the allocation gives it.  The pairs
span every tile size of the pages' table of tile sizes (V = 3640, 1820, 910, 455), b = 11
and b = 12 (App. C.1), and every LUT format those streams select.  Each stream is decoded
per call and again inside a batch (one batch per rate, the five kinds together, prepared
tables), and the first tile, the last tile and eight seeded tiles of each are compared bit
for bit with the oracle's decode of the same tiles.

The layers are generated and packed on the host by spawned worker processes (numpy and the
CPU packer only; no CUDA there), so the GPU process does only the decodes.
"""
import concurrent.futures as cf
import multiprocessing as mp
import os

import numpy as np
import pytest

import dit_weight_compression_ep_b200 as ep
from dit_weight_compression_ep_b200 import synth
from gpu_util import assert_parity, oracle_decode, to_raw

pytestmark = pytest.mark.gpu

KINDS = list(synth.DIT_KINDS)
RATES = list(synth.DIT_BPP_CHOICES)


def _pairs():
    """(kind, rate) -> the first block whose allocation gives that rate to that kind."""
    first = {}
    for (blk, kind), bpp in sorted(synth.dit_stack_bpp().items()):
        first.setdefault((kind, bpp), blk)
    return first


def _pack(job):
    """Worker: generate one layer and pack it with the CPU packer (host only)."""
    kind, bpp, blk = job
    W = synth.generate(synth.dit_stack_layer(blk, kind))
    return kind, bpp, blk, ep.encode_tensor(W, bpp, num_threads=2)


@pytest.fixture(scope="module")
def streams():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dit_weight_compression_ep_b200 import build

    build.build()
    first = _pairs()
    assert len(first) == 25, sorted(first)
    jobs = [(k, r, first[(k, r)]) for r in RATES for k in KINDS]
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with cf.ProcessPoolExecutor(workers, mp_context=mp.get_context("spawn")) as pool:
        packed = list(pool.map(_pack, jobs))
    return {(k, r): (blk, blob) for k, r, blk, blob in packed}


def _tiles(blob, seed):
    rng = np.random.default_rng(seed)
    return sorted(set([0, blob.ntiles - 1] + [int(t) for t in rng.choice(blob.ntiles, 8, replace=False)]))


def _check(out, blob, what, seed):
    got = to_raw(out).reshape(-1)
    per = 8 * blob.V
    for t in _tiles(blob, seed):
        lo, hi = t * per, min((t + 1) * per, blob.rows * blob.cols)
        assert_parity(got[lo:hi], oracle_decode(blob, ep.BF16, t, t + 1), ep.BF16, f"{what} tile {t}")


def test_all_25_streams_cover_the_formats(streams):
    Vs = {blob.V for _, blob in streams.values()}
    bs = {blob.b for _, blob in streams.values()}
    assert Vs == {3640, 1820, 910, 455}, Vs
    assert bs == {11, 12}, bs
    for (kind, bpp), (_, blob) in streams.items():
        assert abs(blob.stored_bpp / bpp - 1) < 0.03, (kind, bpp, blob.stored_bpp)


@pytest.mark.parametrize("bpp", RATES)
def test_per_call_decode(streams, bpp):
    for kind in KINDS:
        blk, blob = streams[(kind, bpp)]
        out = ep.decode_tensor(ep.DeviceBlob(blob), ep.BF16)
        assert ep.decode_status() == 0
        _check(out, blob, f"block {blk} {kind} {bpp} bpp, per call", seed=10 * KINDS.index(kind) + RATES.index(bpp))
        del out


@pytest.mark.parametrize("bpp", RATES)
def test_batched_decode(streams, bpp):
    items = []
    for kind in KINDS:
        db = ep.DeviceBlob(streams[(kind, bpp)][1])
        items.append((db, ep.prepare_lut(db), None))
    outs = ep.DecodeBatch(items, ep.BF16).run()
    assert ep.decode_status() == 0
    for kind, out in zip(KINDS, outs):
        blk, blob = streams[(kind, bpp)]
        _check(out, blob, f"block {blk} {kind} {bpp} bpp, batched", seed=10 * KINDS.index(kind) + RATES.index(bpp))
