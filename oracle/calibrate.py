"""Oracle for the activation-calibrated NVFP4 quantizer.

TEST INFRASTRUCTURE ONLY (see :mod:`oracle`).

imp v0.20.0 release notes, "Highlights": a first-party NVFP4 quantizer with
AWQ-class activation calibration.  The pages name the class of method only;
the reading restated here, step by step:

  1. channel statistics of the calibration activations x [S, K]:
         a_k = (sum_s |x_sk|) / S,  m2_k = (sum_s x_sk^2) / S
     in binary32, rows added in order;
  2. for alpha = j / 8, j = 0..8, channel scales s_k = a_k^alpha (1 where
     a_k == 0), with a^(j/8) composed from square roots and products (below),
     normalised by sqrt(max_k s_k * min_k s_k), all in binary32;
  3. W' = W diag(s) in binary32, quantized with the round-to-nearest rules
     (gs from amax(W'));
  4. err(alpha) = sum_k m2_k sum_n (dequant(W')_nk / s_k - W_nk)^2 in fp64;
  5. the alpha of least err is kept (lowest j on ties).
"""
from __future__ import annotations

import numpy as np

from . import dequantize, quantize

N_ALPHAS = 9


def channel_stats(x) -> tuple[np.ndarray, np.ndarray]:
    """(a, m2): mean |x| and mean x^2 per column, binary32, rows in order."""
    x = np.asarray(x, dtype=np.float32)
    S, K = x.shape
    sa = np.zeros(K, dtype=np.float32)
    s2 = np.zeros(K, dtype=np.float32)
    for s in range(S):
        row = x[s]
        sa = (sa + np.abs(row)).astype(np.float32)
        s2 = (s2 + (row * row).astype(np.float32)).astype(np.float32)
    return (sa / np.float32(S)).astype(np.float32), (s2 / np.float32(S)).astype(np.float32)


def pow_eighths(a, j: int) -> np.ndarray:
    """a^(j/8) in binary32 from r1 = sqrt(a), r2 = sqrt(r1), r3 = sqrt(r2)."""
    a = np.asarray(a, dtype=np.float32)
    r1 = np.sqrt(a).astype(np.float32)
    r2 = np.sqrt(r1).astype(np.float32)
    r3 = np.sqrt(r2).astype(np.float32)
    table = {0: np.ones_like(a), 1: r3, 2: r2, 3: r2 * r3, 4: r1, 5: r1 * r3, 6: r1 * r2, 7: (r1 * r2) * r3, 8: a}
    return np.asarray(table[j], dtype=np.float32)


def channel_scales(a) -> np.ndarray:
    """s [9, K]: the normalised channel scales of every alpha = j / 8."""
    a = np.asarray(a, dtype=np.float32)
    out = np.empty((N_ALPHAS, a.size), dtype=np.float32)
    for j in range(N_ALPHAS):
        raw = np.where(a > 0, pow_eighths(np.where(a > 0, a, np.float32(1)), j), np.float32(1)).astype(np.float32)
        norm = np.sqrt(np.float32(raw.max()) * np.float32(raw.min())).astype(np.float32)
        out[j] = (raw / norm).astype(np.float32)
    return out


def weighted_error(w, q, s, m2) -> float:
    """sum_k m2_k sum_n (dequant(q)_nk / s_k - w_nk)^2 in fp64."""
    deq = dequantize(*q)
    d = deq / np.asarray(s, dtype=np.float64)[None, :] - np.asarray(w, dtype=np.float64)
    return float(np.sum(np.asarray(m2, dtype=np.float64) * np.sum(d * d, axis=0)))


def calibrate(w, x):
    """Returns dict(j, s [K], q = (codes, scales, gs) of W diag(s), err [9], scales_all [9, K])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    a, m2 = channel_stats(x)
    s_all = channel_scales(a)
    err = np.empty(N_ALPHAS)
    qs = []
    for j in range(N_ALPHAS):
        wp = (w * s_all[j][None, :]).astype(np.float32)
        q = quantize(wp)
        qs.append(q)
        err[j] = weighted_error(w, q, s_all[j], m2)
    j = int(np.argmin(err))  # first index of the minimum: lowest j on ties
    return {"j": j, "s": s_all[j], "q": qs[j], "err": err, "scales_all": s_all, "qs": qs}
