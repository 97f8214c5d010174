"""Pins of the oracle's number-format conversions against library routines:
numpy's IEEE binary16 conversion and torch's bfloat16 conversion (both round to nearest,
ties to even), exhaustively over all 16-bit patterns where that is possible."""
import numpy as np
import torch

import oracle


def _edge_floats():
    f = np.float32
    vals = [0.0, -0.0, 1.0, -1.0, 65504.0, 65519.996, 65520.0, -65520.0, 65536.0, 1e-8, 5.96e-8,
            2.98e-8, 2.9802322e-08, 8.9406967e-08, 6.1035156e-05, 6.0975552e-05, 3.4028235e38,
            1.1754944e-38, 1e-45, np.inf, -np.inf, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11,
            1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 0.007874016, 1 / 7.0, 2049.0, 2051.0]
    return np.array(vals, dtype=f)


def _random_floats(n, seed):
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 2 ** 32, size=n, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    scaled = (rng.standard_normal(n) * np.exp(rng.uniform(-30, 14, n))).astype(np.float32)
    return np.concatenate([x, scaled, _edge_floats()])


def test_fp16_decode_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.fp16_to_f64(bits)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_bf16_decode_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_fp16_rounding_matches_numpy():
    x = _random_floats(400_000, 1)
    got = oracle.f32_to_fp16_rn(x)
    ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


def test_fp16_rounding_every_halfway_point():
    """All midpoints between adjacent finite binary16 values (ties go to the even one)."""
    pos = np.arange(0, 0x7bff, dtype=np.uint32).astype(np.uint16)
    lo = pos.view(np.float16).astype(np.float64)
    hi = (pos + 1).view(np.float16).astype(np.float64)
    mid = ((lo + hi) / 2).astype(np.float32)
    exact = mid.astype(np.float64) == (lo + hi) / 2
    mid = mid[exact]
    got = oracle.f32_to_fp16_rn(mid)
    ref = mid.astype(np.float16).view(np.uint16)
    assert mid.size > 30000
    assert np.array_equal(got, ref)
    assert np.all(got % 2 == 0)


def test_bf16_rounding_matches_torch():
    x = _random_floats(400_000, 2)
    got = oracle.f32_to_bf16_rn(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
