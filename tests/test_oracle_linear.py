"""Pins of the oracle's W4A16 and W4A4 linears.

Independent checks: an exact rational brute force on 4 x 32 x 16 inputs, a
library matmul over dequantized operands, and closed forms for degenerate
weights.
"""
from fractions import Fraction

import ml_dtypes
import numpy as np

import oracle
from bit_linear_moe_b200 import synth


def _lib_dequant_exact(codes, scales, gs):
    """Dequantize with library decoders into exact Fractions."""
    rows, half = codes.shape
    cols = half * 2
    c = np.empty((rows, cols), dtype=np.uint8)
    c[:, 0::2] = codes & 0xF
    c[:, 1::2] = codes >> 4
    e2 = c.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    e4 = scales.view(ml_dtypes.float8_e4m3fn).astype(np.float64).repeat(16, axis=1)
    g = Fraction(float(gs))
    return [[Fraction(float(e2[r, k])) * Fraction(float(e4[r, k])) * g for k in range(cols)]
            for r in range(rows)]


def test_w4a16_bruteforce_4x32x16_exact():
    rng = np.random.default_rng(3)
    x = synth.activations(rng, 4, 32)          # M = 4, K = 32 (two blocks)
    w = synth.weight(rng, 16, 32)              # N = 16
    q = oracle.quantize(w)
    wd = _lib_dequant_exact(*q)
    y, absdot = oracle.linear_w4a16(x, *q)
    for m in range(4):
        for n in range(16):
            exact = sum(Fraction(float(x[m, k])) * wd[n][k] for k in range(32))
            exact_abs = sum(abs(Fraction(float(x[m, k])) * wd[n][k]) for k in range(32))
            # the oracle's only rounding is the final multiply by gs (one fp64 rounding)
            assert abs(Fraction(y[m, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 52)
            assert abs(Fraction(absdot[m, n]) - exact_abs) <= exact_abs * Fraction(1, 2 ** 52)


def test_w4a4_bruteforce_exact():
    rng = np.random.default_rng(4)
    x = synth.activations(rng, 4, 32)
    w = synth.weight(rng, 16, 32)
    xq, wq = oracle.quantize(x), oracle.quantize(w)
    xd, wd = _lib_dequant_exact(*xq), _lib_dequant_exact(*wq)
    y, _ = oracle.linear_w4a4(xq, wq)
    for m in range(4):
        for n in range(16):
            exact = sum(xd[m][k] * wd[n][k] for k in range(32))
            assert abs(Fraction(y[m, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 51)


def test_w4a16_matches_library_matmul_over_dequantized():
    rng = np.random.default_rng(5)
    x = synth.activations(rng, 3, 1024)
    q = oracle.quantize(synth.weight(rng, 200, 1024))
    y, absdot = oracle.linear_w4a16(x, *q)
    wd = oracle.dequantize(*q)
    ref = x.astype(np.float64) @ wd.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-14)
    assert np.allclose(absdot, np.abs(x.astype(np.float64)) @ np.abs(wd).T, rtol=1e-12)


def test_w4a4_matches_library_matmul_over_dequantized():
    rng = np.random.default_rng(6)
    xq = oracle.quantize(synth.activations(rng, 5, 512))
    wq = oracle.quantize(synth.weight(rng, 64, 512))
    y, _ = oracle.linear_w4a4(xq, wq)
    ref = oracle.dequantize(*xq) @ oracle.dequantize(*wq).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_zero_weights_give_zero():
    x = synth.activations(np.random.default_rng(1), 2, 64)
    q = oracle.quantize(np.zeros((8, 64), np.float32))
    y, a = oracle.linear_w4a16(x, *q)
    assert not y.any() and not a.any()


def test_single_nonzero_code_selects_one_input():
    K, N = 64, 4
    x = synth.activations(np.random.default_rng(2), 1, K)
    codes = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, K // 16), np.uint8)
    codes[2, 9] = 0x50            # element k = 19 (high nibble of byte 9): E2M1 code 5 = 3.0
    scales[2, 1] = 0x38           # 1.0
    gs = np.float32(0.25)
    y, _ = oracle.linear_w4a16(x, codes, scales, gs)
    assert y[0, 2] == float(x[0, 19]) * 3.0 * 0.25
    assert not np.delete(y[0], 2).any()


def test_uniform_scales_reduce_to_plain_matmul_of_code_values():
    rng = np.random.default_rng(9)
    K, N = 128, 16
    x = synth.activations(rng, 2, K)
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    scales = np.full((N, K // 16), 0x40, np.uint8)   # every scale 2.0
    gs = np.float32(0.5)
    y, _ = oracle.linear_w4a16(x, codes, scales, gs)
    c = np.empty((N, K), np.uint8)
    c[:, 0::2], c[:, 1::2] = codes & 0xF, codes >> 4
    vals = c.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.allclose(y, x.astype(np.float64) @ vals.T, rtol=1e-13, atol=1e-15)
