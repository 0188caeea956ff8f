"""Oracle for the routed mixture-of-experts form of the NVFP4 linear layer.

TEST INFRASTRUCTURE ONLY (see :mod:`oracle`).

The pages give the shape of the layer and nothing of its math: every token is
routed to 10 of 512 experts in each layer (CHImp Alpha v1.0 model card, "How
it fits on one GPU"; Ignis README, "48 x 512 experts"), and only the chosen
experts' weights are read per token (CHImp, same section).  The steps below are
the plainest reading of a softmax-routed top-k SwiGLU expert layer:

  logits  l[t, e] = sum_h h[t, h] * Wr[e, h]  (+ bias[e])         fp64
  top-k   the k experts with the largest logits; equal logits go to the lower
          expert index; slots ordered by descending logit, then index
  weights w[t, j] = softmax(l[t, :])[idx_j] / sum_j' softmax(l[t, :])[idx_j'],
          which equals exp(l_j - l_max) / sum_{j' in top-k} exp(l_j' - l_max)
  permute rows grouped by expert (ascending), tokens ascending inside a group
  gate/up gu = x[tok] @ dequant(Wgu[e])^T, then a = silu(gu[:, :I]) * gu[:, I:]
  down    d = a @ dequant(Wd[e])^T
  combine y[t] = sum_j w[t, j] * d[row_of[t, j]], j ascending
"""
from __future__ import annotations

import numpy as np

from . import linear_w4a16


def router_logits(h: np.ndarray, w_router: np.ndarray, bias=None) -> np.ndarray:
    """fp64 logits ``h @ Wr^T (+ bias)``; h [T, H], Wr [E, H] hold bf16 values."""
    l = np.asarray(h, dtype=np.float64) @ np.asarray(w_router, dtype=np.float64).T
    if bias is not None:
        l = l + np.asarray(bias, dtype=np.float64)[None, :]
    return l


def topk(logits: np.ndarray, k: int):
    """Top-k experts per token by logit and their renormalised softmax weights.

    Selection: descending logit, equal logits ordered by ascending expert index.
    Returns ``(idx int32 [T, k], w float64 [T, k])``.
    """
    l = np.asarray(logits, dtype=np.float64)
    T, E = l.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    for t in range(T):
        row = l[t]
        order = sorted(range(E), key=lambda e: (-row[e], e))[:k]
        idx[t] = order
        sel = row[order]
        ex = np.exp(sel - sel.max())
        w[t] = ex / ex.sum()
    return idx, w


def permute(idx: np.ndarray, E: int):
    """Counting sort of the (token, slot) pairs by expert, stable in token order.

    Returns ``(offsets int32 [E+1], perm_tok int32 [R], perm_slot int32 [R],
    row_of int32 [T, k])`` with R = T*k: rows [offsets[e], offsets[e+1]) belong
    to expert e; row r holds token perm_tok[r] in its slot perm_slot[r]; and
    row_of[t, j] is the row of token t's slot j.
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    counts = [0] * E
    for t in range(T):
        for j in range(k):
            counts[int(idx[t, j])] += 1
    offsets = [0] * (E + 1)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    cursor = list(offsets[:E])
    R = T * k
    perm_tok = np.empty(R, dtype=np.int32)
    perm_slot = np.empty(R, dtype=np.int32)
    row_of = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            r = cursor[e]
            cursor[e] += 1
            perm_tok[r] = t
            perm_slot[r] = j
            row_of[t, j] = r
    return np.asarray(offsets, dtype=np.int32), perm_tok, perm_slot, row_of


def swiglu(gu: np.ndarray) -> np.ndarray:
    """a = silu(g) * u with g the first half of the columns, u the second; fp64."""
    gu = np.asarray(gu, dtype=np.float64)
    I = gu.shape[1] // 2
    g, u = gu[:, :I], gu[:, I:]
    return g / (1.0 + np.exp(-g)) * u


def combine(d: np.ndarray, w: np.ndarray, row_of: np.ndarray):
    """y[t] = sum_j w[t, j] * d[row_of[t, j]] in fp64, j ascending.

    Returns ``(y, bound)`` where bound = sum_j |w_j * d_j| feeds the error bound.
    """
    d = np.asarray(d, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    T, k = row_of.shape
    y = np.zeros((T, d.shape[1]), dtype=np.float64)
    b = np.zeros_like(y)
    for j in range(k):
        term = w[:, j:j + 1] * d[row_of[:, j]]
        y += term
        b += np.abs(term)
    return y, b


def grouped_linear_w4a16(x: np.ndarray, offsets, perm_tok, w_codes, w_scales, w_gs, gather: bool):
    """Per-expert W4A16 linear over the permuted rows.

    Row r of the result uses expert e's weights for r in [offsets[e], offsets[e+1])
    and input row ``x[perm_tok[r]]`` (gather) or ``x[r]``.  Weights are stacked
    ``[E, N, K/2]``, ``[E, N, K/16]``, ``gs [E]``.  Only experts with rows are read.
    Returns ``(y, absdot)`` fp64 [R, N].
    """
    offsets = np.asarray(offsets)
    E = len(offsets) - 1
    R = int(offsets[-1])
    N = w_codes.shape[1]
    y = np.zeros((R, N), dtype=np.float64)
    a = np.zeros((R, N), dtype=np.float64)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        rows = np.asarray(perm_tok[lo:hi]) if gather else np.arange(lo, hi)
        ye, ae = linear_w4a16(np.asarray(x, dtype=np.float32)[rows], w_codes[e], w_scales[e], w_gs[e])
        y[lo:hi] = ye
        a[lo:hi] = ae
    return y, a
