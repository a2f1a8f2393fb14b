"""Host logic of the batched decode (no GPU): the share-out of SMs among a batch's tensors
(ep_batch_apportion) and the argument checks of ep_batch_create / ep_decode_batch, which
refuse bad arguments before any CUDA call."""
import ctypes as C

import pytest

import dit_weight_compression_ep_b200 as ep
from dit_weight_compression_ep_b200 import build

EINVAL = ep._lib.STATUS_CODES["EP_EINVAL"]
EUNSUP = ep._lib.STATUS_CODES["EP_EUNSUPPORTED"]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ep.lib()


def test_one_tensor_takes_every_sm_it_can_use():
    assert ep.batch_apportion([2701], [1820], [11], 148) == [148]
    assert ep.batch_apportion([40], [1820], [11], 148) == [40]  # never more SMs than tiles
    assert ep.batch_apportion([1], [32], [11], 148) == [1]


@pytest.mark.parametrize("n", [2, 3, 5, 8])
def test_equal_tensors_get_equal_shares(n):
    c = ep.batch_apportion([2701] * n, [1820] * n, [11] * n, 148)
    assert sum(c) == 148 and max(c) - min(c) <= 1


def test_shares_are_bounded_and_grow_with_work():
    T = [3038, 1013, 2701, 2701, 2701]
    c = ep.batch_apportion(T, [1820] * 5, [11] * 5, 148)
    assert sum(c) == 148 and all(1 <= ck <= tk for ck, tk in zip(c, T))
    assert c[0] > c[2] > c[1]                      # more tiles of the same length, more SMs
    # the same tile count with twice as long tiles is twice the work
    a, b = ep.batch_apportion([1000, 1000], [1820, 3640], [11, 11], 148)
    assert b > a
    # b >= 12 costs more per symbol (two-level or bucketed table)
    a, b = ep.batch_apportion([2000, 2000], [910, 910], [11, 12], 148)
    assert b > a


def test_many_tiny_tensors_leave_sms_idle():
    c = ep.batch_apportion([2, 3, 1], [64, 64, 64], [11, 11, 11], 148)
    assert c == [2, 3, 1]


def test_apportion_refuses_bad_arguments():
    lib = ep.lib()
    one = (C.c_int64 * 1)(1)
    b = (C.c_int * 1)(11)
    out = (C.c_int * 4)()
    assert lib.ep_batch_apportion(0, one, one, b, 148, out) == EINVAL     # no tensor
    assert lib.ep_batch_apportion(2, (C.c_int64 * 2)(1, 1), (C.c_int64 * 2)(1, 1), (C.c_int * 2)(11, 11), 1,
                                  out) == EINVAL                          # more tensors than SMs
    assert lib.ep_batch_apportion(1, (C.c_int64 * 1)(0), one, b, 148, out) == EINVAL  # a tensor with no tile
    assert lib.ep_batch_apportion(1, one, one, b, 148, None) == EINVAL


def _item(**kw):
    good = 0x10000
    d = dict(tiles=good, tile_index=good, freq_tables=good, row_scales=good, lut=good, rows=64, cols=64, ntiles=1,
             tile_vectors=512, prob_bits=11, out=good)
    d.update(kw)
    return ep._lib._BatchItem(**d)


@pytest.mark.parametrize("bad", [dict(tiles=None), dict(lut=None), dict(out=None), dict(lut=0x10008),
                                 dict(tiles=0x10008), dict(out=0x10004), dict(rows=0), dict(cols=-8),
                                 dict(ntiles=0), dict(tile_vectors=0),
                                 dict(rows=1 << 31), dict(rows=1, cols=1 << 34),
                                 dict(rows=1 << 20, cols=1 << 20),   # 2^37 vectors
                                 dict(rows=1 << 40, cols=1 << 40)])  # a product that would overflow
def test_batch_create_refuses_bad_items_on_host(bad):
    lib = ep.lib()
    arr = (ep._lib._BatchItem * 2)(_item(), _item(**bad))
    h = C.c_void_p()
    assert lib.ep_batch_create(arr, 2, ep.BF16, C.byref(h)) == EINVAL
    assert not h.value


def test_batch_create_and_launch_refuse_bad_arguments():
    lib = ep.lib()
    arr = (ep._lib._BatchItem * 1)(_item())
    h = C.c_void_p()
    assert lib.ep_batch_create(None, 1, ep.BF16, C.byref(h)) == EINVAL
    assert lib.ep_batch_create(arr, 0, ep.BF16, C.byref(h)) == EINVAL
    assert lib.ep_batch_create(arr, 1, ep.BF16, None) == EINVAL
    assert lib.ep_batch_create(arr, 1, 7, C.byref(h)) == EUNSUP
    assert lib.ep_decode_batch(None, None) == EINVAL
    lib.ep_batch_free(None)


def test_share_out_properties_random():
    """Random batches: every tensor gets 1..T SMs; together they use all SMs unless the tensors have
    fewer tiles than that; the share-out is deterministic.  (It may depend on the tensors' order
    where the cost model ties, e.g. tensors of one tile per warp, where more SMs change nothing.)"""
    from hypothesis import given, settings
    from hypothesis import strategies as st

    tensor = st.tuples(st.integers(1, 20000), st.sampled_from([32, 455, 910, 1820, 3640]),
                       st.sampled_from([9, 10, 11, 12, 13]))

    @settings(max_examples=200, deadline=None, derandomize=True)
    @given(st.lists(tensor, min_size=1, max_size=40), st.integers(40, 160))
    def check(ts, G):
        T = [t[0] for t in ts]
        V = [t[1] for t in ts]
        b = [t[2] for t in ts]
        c = ep.batch_apportion(T, V, b, G)
        assert all(1 <= ci <= ti for ci, ti in zip(c, T))
        assert sum(c) == min(G, sum(T))
        assert c == ep.batch_apportion(T, V, b, G)

    check()
