"""Seeded random cases across every path at once: for each case (random shape, ragged widths
included, rate, precision, tile size, output type) the GPU encoder gives the packer's bytes, and
the per-call, prepared-table and batched decodes (every case in one batch launch) give the
oracle's values bit for bit."""
import numpy as np
import pytest

import dit_weight_compression_ep_b200 as ep
from gpu_util import assert_parity, oracle_decode, to_raw

pytestmark = pytest.mark.gpu

DTS = [ep.BF16, ep.FP16, ep.FP8_E4M3, ep.INT8, ep.UINT8, ep.FP32, ep.LATTICE_I32]


def _cases(seed: int, n: int):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        rows = int(rng.integers(1, 80))
        cols = int(rng.integers(1, 700))
        bpp = float(rng.choice([2.0, 2.5, 3.3, 4.0, 5.5, 7.0, 8.0]))
        b = int(rng.choice([0, 0, 9, 10, 11, 12, 13]))
        V = int(rng.choice([0, 7, 32, 100, 455]))
        dist = rng.integers(3)
        if dist == 0:
            W = rng.standard_normal((rows, cols)) * 0.02
        elif dist == 1:
            W = rng.standard_t(4, (rows, cols)) * 0.02 * np.exp(rng.normal(0, 0.5, (rows, 1)))
        else:
            W = rng.standard_normal((rows, cols)) * 0.01
            W[rng.random(W.shape) < 0.01] *= 40.0  # sparse outliers
        out.append((W.astype(np.float32), bpp, b, V, DTS[i % len(DTS)]))
    return out


@pytest.mark.parametrize("seed", [1, 2, 3, 4])
def test_random_cases_every_path(seed):
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dit_weight_compression_ep_b200 import build

    build.build()
    cases = _cases(seed, 25)
    blobs, dbs, luts = [], [], []
    for W, bpp, b, V, dt in cases:
        blob = ep.encode_tensor(W, bpp, prob_bits=b, tile_vectors=V)
        g = ep.encode_tensor_gpu(torch.from_numpy(W).cuda(), bpp, prob_bits=b, tile_vectors=V)
        np.testing.assert_array_equal(g.payload[:g.payload_words], blob.payload[:blob.payload_words])
        np.testing.assert_array_equal(g.tile_index, blob.tile_index)
        np.testing.assert_array_equal(g.freq_tables, blob.freq_tables)
        np.testing.assert_array_equal(g.row_scales.view(np.uint32), blob.row_scales.view(np.uint32))
        blobs.append(blob)
        db = ep.DeviceBlob(blob)
        dbs.append(db)
        luts.append(ep.prepare_lut(db))
    for (W, bpp, b, V, dt), blob, db, lut in zip(cases, blobs, dbs, luts):
        want = oracle_decode(blob, dt)
        what = f"{W.shape} bpp={bpp} b={blob.b} V={blob.V} dt={dt}"
        assert_parity(to_raw(ep.decode_tensor(db, dt)), want, dt, "per call " + what)
        assert_parity(to_raw(ep.decode_tensor_prepared(db, lut, dt)), want, dt, "prepared " + what)
    assert ep.decode_status() == 0
    # one batch per output type over the cases of that type
    for dt in DTS:
        idx = [i for i, c in enumerate(cases) if c[4] == dt]
        outs = ep.DecodeBatch([(dbs[i], luts[i], None) for i in idx], dt).run()
        assert ep.decode_status() == 0
        for i, o in zip(idx, outs):
            assert_parity(to_raw(o), oracle_decode(blobs[i], dt), dt, f"batch case {i}")
