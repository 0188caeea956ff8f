"""Pins of the oracle quantizer.

Independent checks: per-block rounding through ml_dtypes' fp8/fp4 conversions
(a library restatement of the same definition), round-trip identities, closed
forms for degenerate blocks and tensors.
"""
import ml_dtypes
import numpy as np

import oracle
from bit_linear_moe_b200 import synth


def test_global_scale_is_one_binary32_division():
    x = synth.weight(np.random.default_rng(5), 64, 128)
    amax = np.float32(np.abs(x).max())
    assert oracle.global_scale(x) == np.float32(amax / np.float32(2688.0))
    assert oracle.global_scale(np.zeros((4, 16), np.float32)) == np.float32(1.0)


def _quantize_via_library(x, gs):
    """The quantizer definition restated with ml_dtypes' RNE conversions."""
    rows, cols = x.shape
    gs = np.float32(gs)
    denom = np.float32(gs * np.float32(6.0))
    xb = x.reshape(rows, cols // 16, 16)
    amax_b = np.abs(xb).max(axis=2).astype(np.float32)
    ratio = (amax_b / denom).astype(np.float32)
    ratio = np.minimum(ratio, np.float32(448.0))  # satfinite; ml_dtypes overflows to NaN
    s = ratio.astype(ml_dtypes.float8_e4m3fn)
    sd = s.astype(np.float32)
    r = (sd * gs).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (xb / r[:, :, None]).astype(np.float32)
    c = q.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    c[np.broadcast_to(r[:, :, None] == 0, c.shape)] = 0
    c = c.reshape(rows, cols)
    packed = (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    return packed, s.view(np.uint8)


def test_quantize_matches_library_restatement():
    rng = np.random.default_rng(7)
    x = synth.weight(rng, 96, 256)
    x[3, 16:32] = 0.0                         # an all-zero block
    x[5, 32:48] = 0.0
    x[5, 40] = 1e-9                           # a block whose scale underflows to zero
    x[7, :16] *= 1e-3                         # subnormal-scale block
    codes, scales, gs = oracle.quantize(x)
    c2, s2 = _quantize_via_library(x, gs)
    assert np.array_equal(scales, s2)
    assert np.array_equal(codes, c2)
    assert scales[3, 1] == 0 and not codes[3, 8:16].any()
    assert scales[5, 2] == 0 and not codes[5, 16:24].any()


def test_quantize_with_given_scale_matches_library_and_saturates():
    x = synth.activations(np.random.default_rng(8), 32, 512)
    gs = np.float32(1e-4)                     # far too small: scales saturate at 448
    codes, scales, gs2 = oracle.quantize(x, gs=gs)
    assert gs2 == gs
    c2, s2 = _quantize_via_library(x, gs)
    assert np.array_equal(scales, s2) and np.array_equal(codes, c2)
    assert (scales == 0x7E).all()


def test_all_zero_tensor():
    codes, scales, gs = oracle.quantize(np.zeros((8, 64), np.float32))
    assert gs == np.float32(1.0) and not codes.any() and not scales.any()


def test_single_nonzero_block_element():
    x = np.zeros((1, 32), np.float32)
    x[0, 5] = -0.75
    codes, scales, gs = oracle.quantize(x)
    assert gs == np.float32(np.float32(0.75) / np.float32(2688))
    # amax / (6 gs) = 448 up to rounding -> scale 448, element -> -6 (code 15).
    assert scales[0, 0] == 0x7E and scales[0, 1] == 0
    assert codes[0, 2] == 0xF0  # element 5 is the high nibble of byte 2
    assert not np.delete(codes[0], 2).any()


def test_quantize_dequantize_roundtrip_is_identity():
    # quantize(dequantize(q), gs) == q with gs held fixed; holds for blocks whose
    # E4M3 scale is normal (>= 2^-6) or zero, which covers N(0, .02) weights.
    for seed in range(3):
        x = synth.weight(np.random.default_rng(seed), 64, 512)
        q = oracle.quantize(x)
        assert (q[1] >= 0x08).all()
        deq = oracle.dequantize(*q).astype(np.float32)
        q2 = oracle.quantize(deq, gs=q[2])
        assert np.array_equal(q[0], q2[0]) and np.array_equal(q[1], q2[1])


def test_permutation_commutes_with_quantize():
    x = synth.activations(np.random.default_rng(11), 40, 128)
    perm = np.random.default_rng(12).integers(0, 40, size=100)
    qa = oracle.quantize(x)
    qb = oracle.quantize(x[perm], gs=qa[2])
    assert np.array_equal(qa[0][perm], qb[0]) and np.array_equal(qa[1][perm], qb[1])


def test_dequantized_error_within_half_step():
    # Every dequantized value is within half an E2M1 step (times the block
    # scale) of the input, except where the step saturates at 6.
    x = synth.weight(np.random.default_rng(21), 32, 256)
    q = oracle.quantize(x)
    deq = oracle.dequantize(*q)
    sd = np.array([[oracle.e4m3_value(s) for s in row] for row in q[1]])
    r = (sd * np.float64(q[2])).repeat(16, axis=1)
    # largest gap between neighbouring E2M1 magnitudes is 2 (between 4 and 6)
    assert (np.abs(deq - x) <= r * 1.0 + 1e-12).all()
