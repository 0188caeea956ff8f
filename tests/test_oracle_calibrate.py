"""Pins of the oracle's calibrated quantizer (closed forms, invariances and a
brute-force recomputation, independent of the code under test)."""
import math

import numpy as np

import oracle
from oracle import calibrate as cal
from bit_linear_moe_b200 import synth


def test_pow_eighths_exact_on_powers_of_two():
    for j in range(9):
        assert cal.pow_eighths(np.float32(256.0), j) == np.float32(2.0 ** j)
        assert cal.pow_eighths(np.float32(2.0 ** -24), j) == np.float32(2.0 ** (-3 * j))


def test_pow_eighths_close_to_the_real_power():
    rng = np.random.default_rng(0)
    a = rng.uniform(1e-3, 1e3, 200).astype(np.float32)
    for j in range(9):
        got = cal.pow_eighths(a, j).astype(np.float64)
        want = np.array([math.pow(float(v), j / 8) for v in a])
        ulp = np.spacing(want.astype(np.float32)).astype(np.float64)
        assert np.all(np.abs(got - want) <= 3 * ulp), j


def test_channel_stats_closed_forms():
    x = np.full((5, 32), -3.0, np.float32)
    a, m2 = cal.channel_stats(x)
    assert np.all(a == 3.0) and np.all(m2 == 9.0)
    x = np.zeros((4, 16), np.float32)
    x[2, 5] = 8.0
    a, m2 = cal.channel_stats(x)
    assert a[5] == 2.0 and m2[5] == 16.0 and np.count_nonzero(a) == 1


def test_alpha_zero_is_plain_rtn():
    rng = np.random.default_rng(1)
    w = synth.weight(rng, 64, 128)
    x, _ = synth.prefill_x(2, 32, 128)
    r = cal.calibrate(w, x)
    assert np.all(r["scales_all"][0] == 1.0)
    q0, qr = r["qs"][0], oracle.quantize(w)
    assert np.array_equal(q0[0], qr[0]) and np.array_equal(q0[1], qr[1]) and q0[2] == qr[2]
    assert r["err"][r["j"]] <= r["err"][0]


def test_error_matches_a_loop():
    rng = np.random.default_rng(2)
    w = synth.weight(rng, 3, 32)
    x = synth.activations(rng, 6, 32)
    r = cal.calibrate(w, x)
    a, m2 = cal.channel_stats(x)
    for j in (0, 4, 8):
        s = r["scales_all"][j]
        deq = oracle.dequantize(*r["qs"][j])
        e = 0.0
        for n in range(3):
            for k in range(32):
                d = deq[n, k] / float(s[k]) - float(w[n, k])
                e += float(m2[k]) * d * d
        assert math.isclose(e, r["err"][j], rel_tol=1e-12)


def test_scaling_the_calibration_batch_changes_nothing():
    """x -> 2^16 x scales a by 2^16 (every a^(j/8) by an exact 2^(2j)) and m2
    by 2^32: the normalised scales, the codes and the chosen alpha stay."""
    rng = np.random.default_rng(3)
    w = synth.weight(rng, 32, 64)
    x, _ = synth.prefill_x(3, 16, 64)
    r1 = cal.calibrate(w, x)
    r2 = cal.calibrate(w, (x * np.float32(2.0 ** 16)).astype(np.float32))
    assert r1["j"] == r2["j"]
    assert np.array_equal(r1["scales_all"], r2["scales_all"])
    assert np.allclose(r2["err"], r1["err"] * 2.0 ** 32, rtol=1e-12)


def test_outlier_channels_are_protected():
    """A few input channels carry 20x larger activations: some alpha > 0 lowers
    the weighted error below round-to-nearest."""
    rng = np.random.default_rng(4)
    K = 256
    w = synth.weight(rng, 128, K)
    x, cols = synth.prefill_x(5, 64, K)
    r = cal.calibrate(w, x)
    assert r["j"] > 0 and r["err"][r["j"]] < r["err"][0]
    assert np.all(r["s"][cols] > np.median(r["s"]))
