"""Pins for the decode-stack glue oracle (rms renormalisation, silu * up,
bf16 rounding): closed forms, exact special cases and hand-computed values."""
import math
import struct

import numpy as np

from oracle import stack as ost


def _bits(f):
    return struct.unpack("<I", struct.pack("<f", np.float32(f)))[0]


def _from_bits(u):
    return struct.unpack("<f", struct.pack("<I", u))[0]


def test_bf16_round_ties_to_even_and_specials():
    one = 1.0
    # 1 + 2^-8 lies halfway between bf16 1.0 and 1 + 2^-7: ties to the even (1.0)
    assert ost.bf16_round([one + 2.0 ** -8])[0] == 1.0
    # 1 + 3 * 2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6: ties to 1 + 2^-6
    assert ost.bf16_round([one + 3 * 2.0 ** -8])[0] == np.float32(1 + 2.0 ** -6)
    # just above the halfway point rounds up
    assert ost.bf16_round([_from_bits(_bits(1 + 2.0 ** -8) + 1)])[0] == np.float32(1 + 2.0 ** -7)
    # bf16 values are fixed points; signs and zeros are kept
    for v in (0.0, -0.0, 1.5, -3.0, 2.0 ** -130, 3.3895313892515355e38):
        r = ost.bf16_round([v])[0]
        assert _bits(r) == _bits(v) or abs(v) > 3e38
    assert math.copysign(1.0, ost.bf16_round([-0.0])[0]) == -1.0
    # past the largest bf16 (0x7F7F0000 = 3.3895e38) the halfway case rounds to infinity
    assert np.isinf(ost.bf16_round([_from_bits(0x7F7F8000)])[0])
    assert np.isnan(ost.bf16_round([np.nan])[0])


def test_rms_norm_closed_forms():
    # a constant row normalises to +-1 exactly
    for c in (0.5, -3.0, 1e-20, 7e30):
        y = ost.rms_norm(np.full((1, 100), c, np.float32))
        assert np.all(y == np.float32(math.copysign(1.0, c)))
    # an all-zero row stays zero
    assert np.all(ost.rms_norm(np.zeros((2, 64), np.float32)) == 0.0)
    # scaling a row by a power of two changes nothing
    rng = np.random.default_rng(0)
    v = rng.standard_normal((3, 257)).astype(np.float32)
    assert np.array_equal(ost.rms_norm(v), ost.rms_norm(v * np.float32(2.0 ** 40)))
    # the normalised row has mean square 1 before rounding
    e = ost.rms_norm_exact(v)
    assert np.allclose(np.mean(e * e, axis=1), 1.0, rtol=0, atol=1e-12)


def test_rms_norm_hand_value():
    # [3, 4]: mean square 12.5, so the outputs are 3/sqrt(12.5) and 4/sqrt(12.5)
    y = ost.rms_norm(np.array([[3.0, 4.0]], np.float32))[0]
    s = math.sqrt(12.5)
    assert y[0] == ost.bf16_round([3.0 / s])[0] and y[1] == ost.bf16_round([4.0 / s])[0]
    assert abs(float(y[0]) - 0.848528) < 4e-3 and abs(float(y[1]) - 1.131371) < 4e-3
    # rows are independent
    two = ost.rms_norm(np.array([[3.0, 4.0], [0.0, 0.0], [-1.0, 1.0]], np.float32))
    assert np.array_equal(two[0], y) and np.all(two[1] == 0) and np.array_equal(two[2], [-1.0, 1.0])


def test_silu_mul_closed_forms():
    # silu(0) = 0 whatever the up value; silu(g) * 1 = g * sigmoid(g)
    g = np.array([[0.0, 1.0, -2.0, 20.0, 5.0, 1.0, 1.0, 1.0]], np.float32)
    e = ost.silu_mul_exact(g)[0]
    assert e[0] == 0.0
    assert abs(e[1] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15
    assert abs(e[2] - (-2.0 / (1.0 + math.exp(2.0)))) < 1e-15
    assert abs(e[3] - 20.0 / (1.0 + math.exp(-20.0))) < 1e-12
    # silu(-x) = silu(x) - x
    x = np.linspace(-8, 8, 33)
    gg = np.concatenate([x, np.ones_like(x)])[None, :]
    hh = np.concatenate([-x, np.ones_like(x)])[None, :]
    assert np.allclose(ost.silu_mul_exact(hh)[0], ost.silu_mul_exact(gg)[0] - x, rtol=0, atol=1e-12)
    # the product scales linearly in the up half, and the rounding is bf16's
    r = ost.silu_mul(np.array([[1.0, 3.0]], np.float32))[0]
    assert r == ost.bf16_round([3.0 / (1.0 + math.exp(-1.0))])[0]
