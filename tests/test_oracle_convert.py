"""Pins of the oracle's output conversions against the library conversions of
PyTorch's CPU backend (round to nearest even), plus the saturating FP8, the
symmetric INT8 and the offset UINT8 readings checked on their own edge cases."""
import numpy as np
import torch

import oracle


def _samples():
    rng = np.random.default_rng(21)
    bits = rng.integers(0, 2**32, size=400000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    extra = np.array([0.0, -0.0, 1.0, -1.0, 65504.0, 65519.99, 65520.0, 65536.0, 6.1e-5, 5.96e-8, 2.98e-8,
                      3.0e-8, 1e-40, -1e-40, 3.4e38, 448.0, 464.0, 480.0, 0.001953125, 0.0009765625,
                      0.0029296875, 1.0 + 2**-8, 1.0 + 3 * 2**-8, 1.0 + 2**-11, 1.0 + 3 * 2**-11], np.float32)
    scaled = (rng.standard_normal(200000) * rng.choice([1e-3, 1e-1, 1, 30, 300], 200000)).astype(np.float32)
    return np.concatenate([x, extra, -extra, scaled])


def test_bf16_matches_library():
    x = _samples()
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.convert(x, oracle.BF16), ref)


def test_fp16_matches_library():
    x = _samples()
    ref = torch.from_numpy(x).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.convert(x, oracle.FP16), ref)


def test_e4m3_matches_library_in_range_and_saturates():
    x = _samples()
    inr = x[np.abs(x) < 448.0]
    ref = torch.from_numpy(inr).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.convert(inr, oracle.E4M3), ref)
    big = x[np.abs(x) >= 448.0]
    got = oracle.convert(big, oracle.E4M3)
    assert np.all(got == np.where(big > 0, 0x7E, 0xFE))
    # every finite e4m3 value converts to itself
    allv = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    fin = np.isfinite(allv)
    np.testing.assert_array_equal(oracle.convert(allv[fin], oracle.E4M3), np.arange(256, dtype=np.uint8)[fin])


def test_int8_round_half_even_and_clamp():
    x = np.array([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, 127.49, 127.5, 300, -127.5, -128.0, -1e9, 0.49999997],
                 np.float32)
    got = oracle.convert(x, oracle.INT8)
    assert list(got) == [0, 2, 2, 0, -2, -2, 126, 127, 127, 127, -127, -127, -127, 0]
    y = _samples()
    ref = np.clip(np.rint(y.astype(np.float64)), -127, 127).astype(np.int8)
    np.testing.assert_array_equal(oracle.convert(y, oracle.INT8), ref)


def test_uint8_offset_round_half_even_and_clamp():
    # [paper] App. B, Table 6: unsigned integer containers carry an offset; the decoder
    # adds it back: nearest integer (ties to even), clamped to [-128, 127], plus 128
    x = np.array([0.5, 1.5, -0.5, -1.5, 126.5, 127.5, 300, -127.5, -128.0, -128.5, -129.0, -1e9, 0.0, -0.0],
                 np.float32)
    got = oracle.convert(x, oracle.UINT8)
    assert list(got) == [128, 130, 128, 126, 254, 255, 255, 0, 0, 0, 0, 0, 128, 128]
    y = _samples()
    ref = (np.clip(np.rint(y.astype(np.float64)), -128, 127) + 128).astype(np.uint8)
    np.testing.assert_array_equal(oracle.convert(y, oracle.UINT8), ref)
    # the offset removed, UINT8 and INT8 agree wherever INT8 does not clamp
    z = y[(y > -127.5) & (y < 127.5)]
    np.testing.assert_array_equal(oracle.convert(z, oracle.UINT8).astype(np.int16) - 128,
                                  oracle.convert(z, oracle.INT8).astype(np.int16))
