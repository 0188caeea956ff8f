"""Oracle for the glue between the linears of a dense decode stack.

TEST INFRASTRUCTURE ONLY (see :mod:`oracle`).

Ignis README, "The decode round": a decode step streams every layer's weights
once, so a whole stack of layers is timed as one pass over all of them.  The
pages do not say how one layer's output feeds the next; the plainest reading
that keeps the activations bounded over 64 layers, with attention left out, is

  q  = QKV(x)                          [M, 10240]
  o  = O(rms(q[:, :5120]))             [M, 5120]   (the Q slice stands in for attention)
  g  = GU(rms(o))                      [M, 34816]
  h  = silu(g[:, :17408]) * g[:, 17408:]
  x' = rms(Down(h))                    [M, 5120]

with rms(v) = v / sqrt(mean(v^2)) per row (an all-zero row stays zero) and
every activation handed to a linear rounded to bf16 (round to nearest even).
The arithmetic here is fp64; only the final rounding to bf16 is a format step.
"""
from __future__ import annotations

import numpy as np


def bf16_round(a) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returned as float32.

    NaN stays NaN; values that round past the largest bf16 become infinity.
    """
    x = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    out = r.astype(np.uint32).view(np.float32).copy()
    nan = np.isnan(x)
    out[nan] = x[nan]
    return out


def rms_norm(x) -> np.ndarray:
    """bf16(v / sqrt(mean(v^2))) for each row v of x (fp64 inside)."""
    v = np.asarray(x, dtype=np.float64)
    ms = np.mean(v * v, axis=-1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = np.where(ms > 0.0, v / np.sqrt(ms), 0.0)
    return bf16_round(y.astype(np.float32))


def rms_norm_exact(x) -> np.ndarray:
    """The same, unrounded (fp64): the value bf16_round is applied to."""
    v = np.asarray(x, dtype=np.float64)
    ms = np.mean(v * v, axis=-1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        return np.where(ms > 0.0, v / np.sqrt(ms), 0.0)


def silu_mul(g) -> np.ndarray:
    """bf16(silu(g[:, :n]) * g[:, n:]) with n = g.shape[-1] // 2 (fp64 inside)."""
    v = np.asarray(g, dtype=np.float64)
    n = v.shape[-1] // 2
    a, b = v[..., :n], v[..., n:]
    y = a / (1.0 + np.exp(-a)) * b
    return bf16_round(y.astype(np.float32))


def silu_mul_exact(g) -> np.ndarray:
    """The same, unrounded (fp64)."""
    v = np.asarray(g, dtype=np.float64)
    n = v.shape[-1] // 2
    a, b = v[..., :n], v[..., n:]
    return a / (1.0 + np.exp(-a)) * b
