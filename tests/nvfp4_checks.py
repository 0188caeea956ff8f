"""Comparison helpers for the parity tests (test-side only; no method arithmetic
of either implementation lives here).

* ``tiled_to_rowmajor``: reads scales stored in the tensor-core layout back into
  row-major order, from the layout's index map as stated in include/nvfp4.h.
* ``assert_within_bound``: the output bound |y - ref| <= 1e-4 * sum_k |x_k w_k|
  + 1e-6, plus one bf16 rounding step of ref for bf16 outputs.
"""
import numpy as np
import torch


def tiled_index(rows: int, cols: int) -> np.ndarray:
    """Byte offsets of scale (r, c), c < cols/16, in the TILED layout."""
    nsf = cols // 16
    cp4 = (nsf + 3) // 4
    r = np.arange(rows)[:, None]
    c = np.arange(nsf)[None, :]
    return ((r // 128) * cp4 + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (c % 4)


def tiled_to_rowmajor(buf: np.ndarray, rows: int, cols: int) -> np.ndarray:
    return np.asarray(buf).reshape(-1)[tiled_index(rows, cols)]


def rowmajor_to_tiled(sc: np.ndarray, rows: int, cols: int) -> np.ndarray:
    nsf = cols // 16
    rp = (rows + 127) // 128 * 128
    cp = (nsf + 3) // 4 * 4
    out = np.zeros(rp * cp, dtype=np.uint8)
    out[tiled_index(rows, cols)] = sc
    return out


def bf16_ulp(ref: np.ndarray) -> np.ndarray:
    a = np.abs(ref)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 7), 0.0)


def bound(absdot: np.ndarray, ref: np.ndarray, bf16: bool) -> np.ndarray:
    b = 1e-4 * absdot + 1e-6
    if bf16:
        b = b + bf16_ulp(ref)
    return b


def assert_within_bound(y, ref: np.ndarray, absdot: np.ndarray, bf16: bool, what: str = ""):
    if isinstance(y, torch.Tensor):
        y = y.float().cpu().numpy()
    y = np.asarray(y, dtype=np.float64)
    err = np.abs(y - ref)
    b = bound(absdot, ref, bf16)
    bad = err > b
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(
            f"{what}: {bad.sum()} of {bad.size} outside the bound; first at {tuple(i)}: "
            f"y={y[tuple(i)]!r} ref={ref[tuple(i)]!r} bound={b[tuple(i)]!r}; max err/bound={np.max(err / b):.3g}")
    return float(np.max(err / b)) if err.size else 0.0
