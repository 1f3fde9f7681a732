"""Pins of the oracle's FP8 KV storage (quantize / dequantize) against things other than itself.

The pages (mo.ai.kr, "Step 5 Preview agentic work design", section "long-horizon RL and run cost")
say the KV cache is trained for FP8 storage and give no format details. The reading: each (token,
group) row of K or V holds E4M3 values and one power-of-two scale, the smallest s = 2^e with
max |x| <= 448 s; values round to nearest, ties to even. Pinned by:
* torch's float8_e4m3fn cast of x / s (a library routine) for rows spanning many binades,
  subnormal codes included;
* closed forms: exactly representable rows round-trip unchanged; hand-chosen ties; the row's
  largest magnitude lands in (224, 448]; an all-zero row has scale 1 and zero codes;
* the error bound of a 3-bit mantissa (half an ulp: 2^-4 relative for normal codes, 2^-10 s
  absolute below 2^-6 s), and that every dequantized value is exact in bf16.
"""
import numpy as np
import pytest
import torch

import oracle
from sgqa_inputs import bf16_bits_to_f64, f64_to_bf16_bits


def _rows(seed, n=400, d=128):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, d)) * np.exp2(rng.integers(-20, 20, size=(n, 1)))
    x[::7, ::3] *= 1e-3  # many codes in the subnormal range
    return f64_to_bf16_bits(x)


def test_fp8_codes_match_torch_e4m3_cast(oracle_lib):
    xb = _rows(1)
    q, s = oracle.quantize_fp8(xb)
    xf = bf16_bits_to_f64(xb)
    want = torch.from_numpy(xf / s[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(q, want)
    assert ((q & 0x78) == 0).sum() > 100  # subnormal codes exercised
    back = torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float64).numpy() * s[:, None]
    np.testing.assert_array_equal(oracle.dequantize_fp8(q, s), back)


def test_fp8_scale_is_the_smallest_power_of_two(oracle_lib):
    xb = _rows(2)
    q, s = oracle.quantize_fp8(xb)
    amax = np.abs(bf16_bits_to_f64(xb)).max(axis=1)
    np.testing.assert_array_equal(np.exp2(np.round(np.log2(s))), s)
    assert (amax / s <= 448).all() and (amax / s > 224).all()
    z, sz = oracle.quantize_fp8(np.zeros((3, 128), dtype=np.uint16))
    assert (z == 0).all() and (sz == 1.0).all()


def test_fp8_closed_forms(oracle_lib):
    # exactly representable rows (E4M3 values times 2^e, largest 448 * 2^e) round-trip unchanged
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 0x7F, size=(50, 128)).astype(np.uint8)
    codes[:, 0] = 0x7E  # 448
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    vals *= np.exp2(rng.integers(-10, 10, size=(50, 1)))
    vals *= np.where(rng.random((50, 128)) < 0.5, -1.0, 1.0)
    xb = f64_to_bf16_bits(vals)
    assert np.array_equal(bf16_bits_to_f64(xb), vals)
    q, s = oracle.quantize_fp8(xb)
    np.testing.assert_array_equal(oracle.dequantize_fp8(q, s), vals)
    # ties at scale 1 (a row whose largest value is 448): to the even mantissa
    row = np.zeros(128)
    row[0] = 448.0
    row[1:7] = [1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, -1.0625, 2.0 ** -6 + 2.0 ** -10]
    q, s = oracle.quantize_fp8(f64_to_bf16_bits(row[None]))
    got = oracle.dequantize_fp8(q, s)[0, :7]
    assert s[0] == 1.0
    np.testing.assert_array_equal(got, [448.0, 1.0, 1.25, 0.0, 2.0 ** -8, -1.0, 2.0 ** -6])


def test_fp8_error_bound_and_bf16_exactness(oracle_lib):
    xb = _rows(4)
    q, s = oracle.quantize_fp8(xb)
    x = bf16_bits_to_f64(xb)
    y = oracle.dequantize_fp8(q, s)
    small = np.abs(x) < 2.0 ** -6 * s[:, None]
    err = np.abs(y - x)
    assert (err[~small] <= 2.0 ** -4 * np.abs(x[~small])).all()
    assert (err[small] <= (2.0 ** -10 * s[:, None] * np.ones_like(x))[small]).all()
    np.testing.assert_array_equal(bf16_bits_to_f64(f64_to_bf16_bits(y)), y)
