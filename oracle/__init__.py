"""CPU oracle for the NVFP4 linear layer and its mixture-of-experts form.

TEST INFRASTRUCTURE ONLY.  The test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The product path (the
C-ABI library under ``bit_linear_moe_b200``) never imports, links or calls it,
and the two share no code, tables or constants.  The only thing they share is
the seeded input generator module, which holds none of the method's arithmetic.

The quantizer and the linears live in ``nvfp4_oracle.c`` (binary32 quantizer
arithmetic in a fixed operation order, fp64 accumulation); the routing,
permutation, SwiGLU and combine steps are plain numpy in :mod:`oracle.moe`,
the decode-stack glue (rms renormalisation, silu * up, bf16 rounding) in
:mod:`oracle.stack`, and the activation-calibrated quantizer in
:mod:`oracle.calibrate`.
The format readings (rounding, ties, saturation, signed zero, zero-scale
blocks, packing order) are stated in the C file's header.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-Wall"]


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        i64, f32, p = ctypes.c_int64, ctypes.c_float, ctypes.c_void_p
        L.nvo_e2m1_value.argtypes = [ctypes.c_int]
        L.nvo_e2m1_value.restype = ctypes.c_double
        L.nvo_e4m3_value.argtypes = [ctypes.c_int]
        L.nvo_e4m3_value.restype = ctypes.c_double
        L.nvo_e2m1_encode.argtypes = [f32]
        L.nvo_e2m1_encode.restype = ctypes.c_int
        L.nvo_e4m3_encode.argtypes = [f32]
        L.nvo_e4m3_encode.restype = ctypes.c_int
        L.nvo_global_scale.argtypes = [p, i64]
        L.nvo_global_scale.restype = f32
        L.nvo_quantize.argtypes = [p, i64, i64, f32, p, p]
        L.nvo_quantize.restype = None
        L.nvo_dequantize.argtypes = [p, p, f32, i64, i64, p]
        L.nvo_dequantize.restype = None
        L.nvo_linear_w4a16.argtypes = [p, i64, i64, p, p, f32, i64, p, p]
        L.nvo_linear_w4a16.restype = None
        L.nvo_linear_w4a4.argtypes = [p, p, f32, i64, i64, p, p, f32, i64, p, p]
        L.nvo_linear_w4a4.restype = None
        L.nvo_num_threads.argtypes = []
        L.nvo_num_threads.restype = ctypes.c_int
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def num_threads() -> int:
    """OpenMP threads the oracle's parallel loops use."""
    return int(lib().nvo_num_threads())


# ---------------------------------------------------------------- format ----

def e2m1_value(code: int) -> float:
    return float(lib().nvo_e2m1_value(int(code)))


def e4m3_value(code: int) -> float:
    return float(lib().nvo_e4m3_value(int(code)))


def e2m1_encode(f) -> np.ndarray:
    """Element-wise E2M1 encoder (nearest, ties to even code, saturating, signed zero)."""
    f = np.asarray(f, dtype=np.float32)
    L = lib()
    return np.array([L.nvo_e2m1_encode(float(v)) for v in f.ravel()], dtype=np.uint8).reshape(f.shape)


def e4m3_encode(f) -> np.ndarray:
    """Element-wise E4M3 encoder (nearest, ties to even code, saturating at 448)."""
    f = np.asarray(f, dtype=np.float32)
    L = lib()
    return np.array([L.nvo_e4m3_encode(float(v)) for v in f.ravel()], dtype=np.uint8).reshape(f.shape)


def global_scale(x: np.ndarray) -> np.float32:
    """gs = amax / 2688 in binary32 (1.0 for an all-zero tensor)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return np.float32(lib().nvo_global_scale(_ptr(x), x.size))


def quantize(x: np.ndarray, gs=None):
    """Quantize fp32 ``x[rows, cols]`` to NVFP4.

    Returns ``(codes uint8 [rows, cols/2], scales uint8 [rows, cols/16], gs float32)``
    with row-major scales.  ``gs`` defaults to :func:`global_scale` of ``x``.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, cols = x.shape
    assert cols % 16 == 0
    if gs is None:
        gs = global_scale(x)
    gs = np.float32(gs)
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    scales = np.zeros((rows, cols // 16), dtype=np.uint8)
    lib().nvo_quantize(_ptr(x), rows, cols, float(gs), _ptr(codes), _ptr(scales))
    return codes, scales, gs


def dequantize(codes: np.ndarray, scales: np.ndarray, gs) -> np.ndarray:
    """fp64 values E2M1(code) * E4M3(scale) * gs of a quantized [rows, cols] tensor."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, cols = codes.shape[0], codes.shape[1] * 2
    out = np.empty((rows, cols), dtype=np.float64)
    lib().nvo_dequantize(_ptr(codes), _ptr(scales), float(np.float32(gs)), rows, cols, _ptr(out))
    return out


def linear_w4a16(x: np.ndarray, codes: np.ndarray, scales: np.ndarray, gs):
    """y = x @ dequant(W)^T in fp64, and the bound term sum_k |x_k w_k|.

    ``x`` is [M, K] fp32 holding bf16 values; W is given as ``codes [N, K/2]``,
    ``scales [N, K/16]`` (row-major) and ``gs``.  Returns ``(y, absdot)``, both
    float64 [M, N].
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    M, K = x.shape
    N = codes.shape[0]
    assert codes.shape == (N, K // 2) and scales.shape == (N, K // 16)
    y = np.empty((M, N), dtype=np.float64)
    a = np.empty((M, N), dtype=np.float64)
    lib().nvo_linear_w4a16(_ptr(x), M, K, _ptr(codes), _ptr(scales), float(np.float32(gs)), N,
                           _ptr(y), _ptr(a))
    return y, a


def linear_w4a4(xq, wq):
    """W4A4: both operands NVFP4 ``(codes, scales, gs)``; returns ``(y, absdot)`` fp64."""
    xc, xs, gsx = (np.ascontiguousarray(xq[0], dtype=np.uint8),
                   np.ascontiguousarray(xq[1], dtype=np.uint8), np.float32(xq[2]))
    wc, ws, gsw = (np.ascontiguousarray(wq[0], dtype=np.uint8),
                   np.ascontiguousarray(wq[1], dtype=np.uint8), np.float32(wq[2]))
    M, K = xc.shape[0], xc.shape[1] * 2
    N = wc.shape[0]
    assert wc.shape == (N, K // 2) and ws.shape == (N, K // 16) and xs.shape == (M, K // 16)
    y = np.empty((M, N), dtype=np.float64)
    a = np.empty((M, N), dtype=np.float64)
    lib().nvo_linear_w4a4(_ptr(xc), _ptr(xs), float(gsx), M, K, _ptr(wc), _ptr(ws), float(gsw), N,
                          _ptr(y), _ptr(a))
    return y, a
