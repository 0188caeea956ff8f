"""Pins of the oracle's format layer (E2M1 / E4M3 decode and encode).

The oracle's tables and encoders are checked against things it does not share:
golden values from the published format definitions, the fp8/fp4 conversions
of two independent libraries (torch, ml_dtypes), and an exact rational brute
force.  No expected value here comes from the CUDA path.
"""
import math
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                a, b = line.split()
                rows.append((int(a, 0), float(b)))
    return rows


def test_e2m1_table_matches_format_definition():
    rows = _read_golden("e2m1_values.txt")
    assert len(rows) == 16
    for code, val in rows:
        got = oracle.e2m1_value(code)
        assert got == val and math.copysign(1, got) == math.copysign(1, val), (code, got, val)


def test_e2m1_table_matches_library_fp4():
    # torch stores two fp4 codes per byte (low nibble first); ml_dtypes decodes one per byte.
    codes = np.arange(16, dtype=np.uint8)
    lib_vals = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    ours = np.array([oracle.e2m1_value(c) for c in range(16)])
    assert np.array_equal(np.signbit(lib_vals), np.signbit(ours))
    assert np.array_equal(lib_vals, ours)


def test_e4m3_golden_points():
    for code, val in _read_golden("e4m3_points.txt"):
        got = oracle.e4m3_value(code)
        if math.isnan(val):
            assert math.isnan(got), code
        else:
            assert got == val and math.copysign(1, got) == math.copysign(1, val), (hex(code), got, val)


def test_e4m3_all_256_codes_match_torch_fp8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = np.array([oracle.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert set(np.flatnonzero(nan)) == {0x7F, 0xFF}
    assert np.array_equal(ref[~nan], ours[~nan])
    assert np.array_equal(np.signbit(ref[~nan]), np.signbit(ours[~nan]))
    assert np.nanmax(ours) == 448.0
    assert min(v for v in ours if v > 0) == 2.0 ** -9


def test_e4m3_round_trip_all_finite_codes():
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        v = np.float32(oracle.e4m3_value(c))
        assert int(oracle.e4m3_encode(v)) == c, hex(c)


def _probe_points(table):
    """Each representable value, every midpoint between neighbours, and the fp32
    neighbours one ulp either side of both."""
    mags = sorted(set(abs(v) for v in table if not math.isnan(v)))
    pts = []
    for a, b in zip(mags[:-1], mags[1:]):
        mid = np.float32((a + b) / 2)
        assert float(mid) == (a + b) / 2  # midpoints are exact in fp32 here
        pts += [np.float32(a), mid, np.nextafter(mid, np.float32(0)),
                np.nextafter(mid, np.float32(np.inf))]
    pts += [np.float32(mags[-1]), np.nextafter(np.float32(mags[-1]), np.float32(np.inf))]
    pts = np.array(pts, dtype=np.float32)
    return np.concatenate([pts, -pts])


def test_e2m1_encoder_matches_ml_dtypes_rne_with_saturation():
    pts = _probe_points([oracle.e2m1_value(c) for c in range(8)])
    extra = np.array([0.0, -0.0, 6.5, 7.0, -7.0, 1e30, -1e30, 1e-30, -1e-30,
                      2.0 ** -149, -(2.0 ** -149)], dtype=np.float32)
    pts = np.concatenate([pts, extra])
    ours = oracle.e2m1_encode(pts)
    ref = pts.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(ours, ref), np.stack([pts, ours, ref], 1)[ours != ref]


def _exact_nearest(f, mags, tie_even=True):
    """Brute force in exact rationals: nearest magnitude index, ties to even index."""
    a = abs(Fraction(float(f)))
    best, bestd = None, None
    for i, m in enumerate(mags):
        d = abs(a - Fraction(m))
        if bestd is None or d < bestd or (d == bestd and tie_even and i % 2 == 0):
            best, bestd = i, d
    return best


def test_e4m3_encoder_exact_rational_brute_force():
    mags = [oracle.e4m3_value(c) for c in range(127)]
    pts = _probe_points(mags)
    pts = np.concatenate([pts, np.array([500.0, 1e9, 2.0 ** -12, 2.0 ** -10, 3 * 2.0 ** -11],
                                        dtype=np.float32)])
    ours = oracle.e4m3_encode(pts)
    for f, c in zip(pts, ours):
        want = _exact_nearest(f, mags) | (0x80 if math.copysign(1, f) < 0 else 0)
        assert int(c) == want, (float(f), hex(c), hex(want))


def test_e4m3_encoder_matches_ml_dtypes_in_range():
    rng = np.random.default_rng(123)
    vals = np.concatenate([
        rng.uniform(0, 448, 20000), np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448), 20000)),
    ]).astype(np.float32)
    ours = oracle.e4m3_encode(vals)
    ref = vals.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(ours, ref)


def test_e4m3_encoder_saturates():
    for f in (448.0, 449.0, 464.0, 465.0, 1e6, 3e38):
        assert int(oracle.e4m3_encode(np.float32(f))) == 0x7E
