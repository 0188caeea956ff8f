"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds none of the layer's arithmetic: it only draws numbers.  Both
the CUDA path and the CPU oracle are fed from here, so a parity test compares
the two on identical bytes.

Workloads (weights N(0, 0.02), activations N(0, 1), both rounded as stated):

* ``single``  one 2048 x 2048 linear, M = 1 (seed 0: W first, then x).
* ``dense27b``  the four linears of a 27B-shaped decoder layer, hidden 5120:
  fused QKV (K 5120, N 10240), o_proj (5120, 5120), fused gate+up
  (5120, 34816), down (17408, 5120); seeds 1..4 in that order; decode
  activations from ``rng([seed, M])``.
* ``prefill``  the same weights; activations from ``rng([seed, 100 + M])`` with
  1 % of the columns (``rng.choice(K, K // 100, replace=False)``, drawn first)
  multiplied by 20 before rounding to bf16 (outlier channels).
* ``moe``  512 experts, hidden 2048, expert intermediate 512, top-10; router
  weight N(0, 0.02) rounded to bf16 (seed 10); expert e's gate+up [1024, 2048]
  from ``rng([10, 1, e])`` and down [2048, 512] from ``rng([10, 2, e])``;
  hidden states from ``rng([10, 3, T])``.  The skewed run adds
  ``bias[e] = -1.1 * ln(rank[e])`` with ranks a seeded permutation of 1..512
  (``rng([10, 4])``): a log-prior that makes expert popularity follow
  Zipf(1.1).
"""
from __future__ import annotations

import numpy as np
import torch

DENSE27B = (
    ("qkv", 5120, 10240, 1),
    ("o_proj", 5120, 5120, 2),
    ("gate_up", 5120, 34816, 3),
    ("down", 17408, 5120, 4),
)
DECODE_M = (1, 2, 4, 8, 16, 32)
VERIFY_M = (8, 16, 64)          # speculative-verify widths: 1 + draft tokens
PREFILL_M = (512, 2048, 8192)

MOE_E, MOE_H, MOE_I, MOE_K = 512, 2048, 512, 10
MOE_T = (1, 32, 4096)


def to_bf16(a: np.ndarray) -> np.ndarray:
    """Round to bf16 (nearest-even) and return the values as float32."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def weight(rng: np.random.Generator, n: int, k: int) -> np.ndarray:
    """[n, k] float32 weights, 0.02 * N(0, 1)."""
    return (0.02 * rng.standard_normal((n, k))).astype(np.float32)


def activations(rng: np.random.Generator, m: int, k: int) -> np.ndarray:
    """[m, k] bf16-valued float32 activations, N(0, 1)."""
    return to_bf16(rng.standard_normal((m, k)))


def single(seed: int = 0):
    """The 2048 x 2048, M = 1 case: returns ``(W float32 [2048, 2048], x [1, 2048])``."""
    rng = np.random.default_rng(seed)
    w = weight(rng, 2048, 2048)
    x = activations(rng, 1, 2048)
    return w, x


def dense_weight(seed: int, k: int, n: int) -> np.ndarray:
    return weight(np.random.default_rng(seed), n, k)


def decode_x(seed: int, m: int, k: int) -> np.ndarray:
    return activations(np.random.default_rng([seed, m]), m, k)


def prefill_x(seed: int, m: int, k: int):
    """Prefill activations with 1 % outlier columns; returns ``(x, outlier_cols)``."""
    rng = np.random.default_rng([seed, 100 + m])
    cols = rng.choice(k, k // 100, replace=False)
    x = rng.standard_normal((m, k))
    x[:, cols] *= 20.0
    return to_bf16(x), np.sort(cols)


def moe_router(seed: int = 10) -> np.ndarray:
    """Router weight [512, 2048], bf16-valued float32."""
    return to_bf16(0.02 * np.random.default_rng(seed).standard_normal((MOE_E, MOE_H)))


def moe_expert(e: int, seed: int = 10):
    """Expert e's fp32 weights: ``(gate_up [1024, 2048], down [2048, 512])``.

    Rows 0..511 of gate_up are the gate projection, rows 512..1023 the up one.
    """
    wgu = weight(np.random.default_rng([seed, 1, e]), 2 * MOE_I, MOE_H)
    wd = weight(np.random.default_rng([seed, 2, e]), MOE_H, MOE_I)
    return wgu, wd


def moe_hidden(t: int, seed: int = 10) -> np.ndarray:
    return activations(np.random.default_rng([seed, 3, t]), t, MOE_H)


def moe_zipf_bias(seed: int = 10, s: float = 1.1) -> np.ndarray:
    """Per-expert logit offset -s * ln(rank), ranks a seeded permutation of 1..E."""
    ranks = np.random.default_rng([seed, 4]).permutation(MOE_E) + 1
    return (-s * np.log(ranks)).astype(np.float32)
