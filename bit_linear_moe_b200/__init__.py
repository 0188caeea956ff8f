"""Python binding of libnvfp4, the NVFP4 linear layer for B200 (sm_100a).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  The functions carry the names of the C entry points declared in
``include/nvfp4.h`` and take torch CUDA tensors for device memory; outputs and
workspaces not passed in are allocated with torch (the library itself never
allocates).  Every call is enqueued on the current torch stream.

There is no fallback: if ``libnvfp4.so`` has not been built, importing the
library raises ``ImportError``; a non-zero status raises :class:`NVFP4Error`.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4.so")

# status codes, enumerations (values of include/nvfp4.h)
OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_DTYPE, ERR_WORKSPACE, ERR_ARCH, ERR_LAUNCH, ERR_LAYOUT, ERR_MODE, \
    ERR_DEVICE_TIMEOUT = range(11)
DTYPE_F32, DTYPE_BF16 = 0, 1
SF_ROWMAJOR, SF_TILED = 0, 1
MODE_AUTO, MODE_W4A16, MODE_W4A4 = 0, 1, 2
EPI_NONE, EPI_SWIGLU, EPI_COMBINE = 0, 1, 2


CHAIN_SRC_X, CHAIN_SRC_OP = 0, 1
CHAIN_XFORM_NONE, CHAIN_XFORM_RMS, CHAIN_XFORM_SILU_MUL = 0, 1, 2


class ChainOp(ctypes.Structure):
    """``nvfp4_chain_op`` of include/nvfp4.h."""
    _fields_ = [("w_codes", ctypes.c_void_p), ("w_scales", ctypes.c_void_p), ("w_gs", ctypes.c_void_p),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("src", ctypes.c_int32), ("src_op", ctypes.c_int32),
                ("x", ctypes.c_void_p), ("x_ld", ctypes.c_int64), ("xform", ctypes.c_int32),
                ("y_xform", ctypes.c_int32), ("y", ctypes.c_void_p), ("y_dtype", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, call: str):
        super().__init__(f"{call} failed: {status_string(status)} (status {status})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libnvfp4 (raises ImportError when it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m bit_linear_moe_b200.build` "
                              "(there is no fallback implementation)")
        L = ctypes.CDLL(LIB_PATH)
        p, i64, i32, sz, i = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t, ctypes.c_int
        sig = {
            "nvfp4_status_string": (ctypes.c_char_p, [i]),
            "nvfp4_version": (i, []),
            "nvfp4_scales_bytes": (sz, [i64, i64, i]),
            "nvfp4_read_device_status": (i, [p, p]),
            "nvfp4_debug_wait_timeout": (i, [i64, p]),
            "nvfp4_quantize_workspace": (sz, [i64, i64]),
            "nvfp4_quantize": (i, [p, i, i64, i64, p, i, p, p, p, p, sz, p]),
            "nvfp4_linear_workspace": (sz, [i64, i64, i64, i]),
            "nvfp4_linear": (i, [p, i, i64, i64, p, p, i, p, i64, p, i, i, p, sz, p]),
            "nvfp4_linear_w4a4q": (i, [p, p, p, i64, i64, p, p, p, i64, p, i, p]),
            "nvfp4_rms_norm": (i, [p, i, i64, i64, i64, p, p]),
            "nvfp4_chain_workspace": (sz, [p, i32, i64]),
            "nvfp4_calibrate_workspace": (sz, [i64, i64, i64]),
            "nvfp4_calibrate": (i, [p, i64, i64, p, i, i64, i, p, p, p, p, p, p, p, sz, p]),
            "nvfp4_chain": (i, [p, i32, i64, p, sz, p]),
            "nvfp4_silu_mul": (i, [p, i, i64, i64, p, p]),
            "nvfp4_rms_norm_quant_workspace": (sz, [i64]),
            "nvfp4_rms_norm_quant": (i, [p, i, i64, i64, i64, i, p, p, p, p, sz, p]),
            "moe_route_topk_workspace": (sz, [i64, i32, i32]),
            "moe_route_topk": (i, [p, p, p, i64, i64, i32, i32, p, p, p, p, p, p, p, p, sz, p]),
            "moe_route_topk_noalloc": (i, [p, p, p, i64, i64, i32, i32, p, p, p, p, p, p, p, p]),
            "moe_grouped_linear_workspace": (sz, [i64, i64, i64, i32, i32, i, i]),
            "nvfp4_linear_w4a4_ws_layout": (i, [i64, i64, p]),
            "moe_layer_decode_workspace": (sz, [i64, i64, i64, i32, i32]),
            "moe_layer_decode": (i, [p, p, p, i64, i64, i32, i32, p, p, p, i64, p, p, p, p, p, p, p, p, i, p, sz,
                                     p]),
            "moe_grouped_linear_w4a4_ws_layout": (i, [i64, i64, i64, i32, i32, i, p]),
            "moe_grouped_linear": (i, [p, i, i64, i, p, p, i32, i64, p, p, i, p, i64, i, p, p, i32, p, i, i,
                                       p, sz, p]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().nvfp4_status_string(int(status)).decode()


def _check(status: int, call: str):
    if status != OK:
        raise NVFP4Error(status, call)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return DTYPE_F32
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _workspace(nbytes: int, device, ws=None):
    if nbytes == 0:
        return None, 0
    if ws is None:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return ws, ws.numel() * ws.element_size()


def nvfp4_scales_bytes(rows: int, cols: int, sf_layout: int) -> int:
    return int(lib().nvfp4_scales_bytes(rows, cols, sf_layout))


def nvfp4_quantize(x: torch.Tensor, gs_in: torch.Tensor | None = None, sf_layout: int = SF_ROWMAJOR,
                   codes=None, scales=None, gs_out=None, ws=None):
    """Quantize ``x [rows, cols]`` (fp32 or bf16) to ``(codes, scales, gs)`` on the device."""
    rows, cols = x.shape
    dev = x.device
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty(nvfp4_scales_bytes(rows, cols, sf_layout), dtype=torch.uint8, device=dev)
    if gs_out is None:
        gs_out = torch.empty(1, dtype=torch.float32, device=dev)
    ws, wsb = _workspace(int(lib().nvfp4_quantize_workspace(rows, cols)), dev, ws)
    _check(lib().nvfp4_quantize(_ptr(x), _dtype_code(x), rows, cols, _ptr(gs_in), sf_layout, _ptr(codes),
                                _ptr(scales), _ptr(gs_out), _ptr(ws), wsb, _stream()), "nvfp4_quantize")
    return codes, scales, gs_out


def nvfp4_calibrate(w: torch.Tensor, x_calib: torch.Tensor, sf_layout: int = SF_ROWMAJOR, ws=None):
    """Activation-calibrated quantization of ``w [N, K]`` (fp32) from ``x_calib
    [S, K]`` (bf16).  Returns ``(codes, scales, gs, col_scale, err[9], alpha_idx)``:
    the quantized ``w * col_scale``; use it on activations divided by ``col_scale``."""
    N, K = w.shape
    S = x_calib.shape[0]
    dev = w.device
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty(nvfp4_scales_bytes(N, K, sf_layout), dtype=torch.uint8, device=dev)
    gs = torch.empty(1, dtype=torch.float32, device=dev)
    col = torch.empty(K, dtype=torch.float32, device=dev)
    err = torch.empty(9, dtype=torch.float32, device=dev)
    aidx = torch.empty(1, dtype=torch.int32, device=dev)
    ws, wsb = _workspace(int(lib().nvfp4_calibrate_workspace(N, K, S)), dev, ws)
    _check(lib().nvfp4_calibrate(_ptr(w), N, K, _ptr(x_calib), _dtype_code(x_calib), S, sf_layout, _ptr(codes),
                                 _ptr(scales), _ptr(gs), _ptr(col), _ptr(err), _ptr(aidx), _ptr(ws), wsb,
                                 _stream()), "nvfp4_calibrate")
    return codes, scales, gs, col, err, aidx


def nvfp4_rms_norm(x: torch.Tensor, cols: int | None = None, y=None):
    """``bf16(v / sqrt(mean(v^2)))`` for the first ``cols`` columns of each row v of
    ``x [rows, ld]`` (fp32 or bf16, rows contiguous); returns ``y [rows, cols]`` bf16."""
    rows, ld = x.shape
    if x.stride(1) != 1 or x.stride(0) != ld:
        raise ValueError("x must be a contiguous [rows, ld] tensor")
    cols = ld if cols is None else int(cols)
    if y is None:
        y = torch.empty((rows, cols), dtype=torch.bfloat16, device=x.device)
    _check(lib().nvfp4_rms_norm(_ptr(x), _dtype_code(x), rows, cols, ld, _ptr(y), _stream()), "nvfp4_rms_norm")
    return y


def nvfp4_rms_norm_quant(x: torch.Tensor, cols: int | None = None, sf_layout: int = SF_TILED, ws=None):
    """NVFP4 ``(codes, scales, gs)`` of ``nvfp4_rms_norm(x, cols)``, without the bf16 rows."""
    rows, ld = x.shape
    if x.stride(1) != 1 or x.stride(0) != ld:
        raise ValueError("x must be a contiguous [rows, ld] tensor")
    cols = ld if cols is None else int(cols)
    dev = x.device
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty(nvfp4_scales_bytes(rows, cols, sf_layout), dtype=torch.uint8, device=dev)
    gs = torch.empty(1, dtype=torch.float32, device=dev)
    ws, wsb = _workspace(int(lib().nvfp4_rms_norm_quant_workspace(rows)), dev, ws)
    _check(lib().nvfp4_rms_norm_quant(_ptr(x), _dtype_code(x), rows, cols, ld, sf_layout, _ptr(codes), _ptr(scales),
                                      _ptr(gs), _ptr(ws), wsb, _stream()), "nvfp4_rms_norm_quant")
    return codes, scales, gs


def nvfp4_silu_mul(g: torch.Tensor, h=None):
    """``bf16(silu(g[:, :n]) * g[:, n:])`` for ``g [rows, 2n]`` (fp32 or bf16, contiguous)."""
    rows, w = g.shape
    if not g.is_contiguous() or w % 2:
        raise ValueError("g must be a contiguous [rows, 2n] tensor")
    half = w // 2
    if h is None:
        h = torch.empty((rows, half), dtype=torch.bfloat16, device=g.device)
    _check(lib().nvfp4_silu_mul(_ptr(g), _dtype_code(g), rows, half, _ptr(h), _stream()), "nvfp4_silu_mul")
    return h


def nvfp4_linear(x: torch.Tensor, w_codes: torch.Tensor, w_scales: torch.Tensor, w_gs: torch.Tensor,
                 w_sf_layout: int = SF_ROWMAJOR, y=None, y_dtype=torch.float32, mode: int = MODE_AUTO, ws=None):
    """``y = x @ W^T`` with W NVFP4 ``(w_codes [N, K/2], w_scales, w_gs)``; x bf16 [M, K]."""
    M, K = x.shape
    N = w_codes.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=y_dtype, device=x.device)
    ws, wsb = _workspace(int(lib().nvfp4_linear_workspace(M, K, N, mode)), x.device, ws)
    _check(lib().nvfp4_linear(_ptr(x), _dtype_code(x), M, K, _ptr(w_codes), _ptr(w_scales), w_sf_layout,
                              _ptr(w_gs), N, _ptr(y), _dtype_code(y), mode, _ptr(ws), wsb, _stream()),
           "nvfp4_linear")
    return y


def nvfp4_linear_w4a4q(x_codes: torch.Tensor, x_scales: torch.Tensor, x_gs: torch.Tensor, w_codes: torch.Tensor,
                       w_scales: torch.Tensor, w_gs: torch.Tensor, y=None, y_dtype=torch.bfloat16):
    """W4A4 with pre-quantized activations (codes [M, K/2], TILED scales, device gs)."""
    M, K = x_codes.shape[0], x_codes.shape[1] * 2
    N = w_codes.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=y_dtype, device=x_codes.device)
    _check(lib().nvfp4_linear_w4a4q(_ptr(x_codes), _ptr(x_scales), _ptr(x_gs), M, K, _ptr(w_codes), _ptr(w_scales),
                                    _ptr(w_gs), N, _ptr(y), _dtype_code(y), _stream()), "nvfp4_linear_w4a4q")
    return y


def chain_ops(specs) -> "ctypes.Array":
    """Build the ``nvfp4_chain_op`` array from dicts with keys ``w`` = (codes,
    TILED scales, gs), ``src`` (a bf16 tensor [M, K] or the index of an earlier
    op), ``K`` (when ``src`` is an op index: the columns the transform reads),
    ``xform``, ``y`` (tensor or None) and ``y_xform``."""
    arr = (ChainOp * len(specs))()
    for i, sp in enumerate(specs):
        c, sc, g = sp["w"]
        o = arr[i]
        o.w_codes, o.w_scales, o.w_gs = c.data_ptr(), sc.data_ptr(), g.data_ptr()
        o.N, o.K = c.shape[0], c.shape[1] * 2
        src = sp["src"]
        if hasattr(src, "data_ptr"):
            o.src, o.src_op, o.x, o.x_ld = CHAIN_SRC_X, -1, src.data_ptr(), src.stride(0)
        else:
            o.src, o.src_op, o.x, o.x_ld = CHAIN_SRC_OP, int(src), None, 0
        o.xform = int(sp.get("xform", CHAIN_XFORM_NONE))
        y = sp.get("y")
        o.y = None if y is None else y.data_ptr()
        o.y_dtype = DTYPE_F32 if y is None else _dtype_code(y)
        o.y_xform = int(sp.get("y_xform", CHAIN_XFORM_NONE))
    return arr


def nvfp4_chain(specs, M: int, ws=None, ops=None):
    """Run a list of W4A16 decode linears in one persistent launch per 12 ops
    (see ``nvfp4_chain`` in include/nvfp4.h).  Outputs go to the ``y`` tensors
    of the specs.  ``ops`` may pass a prebuilt :func:`chain_ops` array."""
    if ops is None:
        ops = chain_ops(specs)
    n = len(ops)
    dev = torch.device("cuda", torch.cuda.current_device())
    optr = ctypes.cast(ops, ctypes.c_void_p)
    ws, wsb = _workspace(int(lib().nvfp4_chain_workspace(optr, n, M)), dev, ws)
    _check(lib().nvfp4_chain(optr, n, M, _ptr(ws), wsb, _stream()), "nvfp4_chain")
    return ws


def moe_route_topk(h: torch.Tensor, w_router: torch.Tensor, k: int, logit_bias=None, want_logits: bool = False,
                   out=None, ws=None):
    """Router, top-k and permutation.  Returns a dict of device tensors:
    ``logits`` (if wanted), ``topk_idx``, ``topk_w``, ``expert_offsets``, ``perm_tok``, ``perm_slot``, ``row_of``."""
    T, H = h.shape
    E = w_router.shape[0]
    dev = h.device
    o = dict(out or {})
    if want_logits and "logits" not in o:
        o["logits"] = torch.empty((T, E), dtype=torch.float32, device=dev)
    o.setdefault("topk_idx", torch.empty((T, k), dtype=torch.int32, device=dev))
    o.setdefault("topk_w", torch.empty((T, k), dtype=torch.float32, device=dev))
    o.setdefault("expert_offsets", torch.empty(E + 1, dtype=torch.int32, device=dev))
    o.setdefault("perm_tok", torch.empty(T * k, dtype=torch.int32, device=dev))
    o.setdefault("perm_slot", torch.empty(T * k, dtype=torch.int32, device=dev))
    o.setdefault("row_of", torch.empty((T, k), dtype=torch.int32, device=dev))
    ws, wsb = _workspace(int(lib().moe_route_topk_workspace(T, E, k)), dev, ws)
    _check(lib().moe_route_topk(_ptr(h), _ptr(w_router), _ptr(logit_bias), T, H, E, k, _ptr(o.get("logits")),
                                _ptr(o["topk_idx"]), _ptr(o["topk_w"]), _ptr(o["expert_offsets"]),
                                _ptr(o["perm_tok"]), _ptr(o["perm_slot"]), _ptr(o["row_of"]), _ptr(ws), wsb,
                                _stream()), "moe_route_topk")
    return o


def moe_route_topk_noalloc(h: torch.Tensor, w_router: torch.Tensor, k: int, logit_bias=None,
                           want_logits: bool = False, out=None):
    """``moe_route_topk`` without a workspace: for callers that cannot allocate
    device memory while routing.  The library's built-in 1 MiB scratch is used
    instead (shared by every call; overlapping calls race)."""
    T, H = h.shape
    E = w_router.shape[0]
    dev = h.device
    o = dict(out or {})
    if want_logits and "logits" not in o:
        o["logits"] = torch.empty((T, E), dtype=torch.float32, device=dev)
    o.setdefault("topk_idx", torch.empty((T, k), dtype=torch.int32, device=dev))
    o.setdefault("topk_w", torch.empty((T, k), dtype=torch.float32, device=dev))
    o.setdefault("expert_offsets", torch.empty(E + 1, dtype=torch.int32, device=dev))
    o.setdefault("perm_tok", torch.empty(T * k, dtype=torch.int32, device=dev))
    o.setdefault("perm_slot", torch.empty(T * k, dtype=torch.int32, device=dev))
    o.setdefault("row_of", torch.empty((T, k), dtype=torch.int32, device=dev))
    _check(lib().moe_route_topk_noalloc(_ptr(h), _ptr(w_router), _ptr(logit_bias), T, H, E, k,
                                        _ptr(o.get("logits")), _ptr(o["topk_idx"]), _ptr(o["topk_w"]),
                                        _ptr(o["expert_offsets"]), _ptr(o["perm_tok"]), _ptr(o["perm_slot"]),
                                        _ptr(o["row_of"]), _stream()), "moe_route_topk_noalloc")
    return o


def moe_grouped_linear(x: torch.Tensor, expert_offsets: torch.Tensor, w_codes: torch.Tensor,
                       w_scales: torch.Tensor, w_gs: torch.Tensor, R: int, perm_tok=None, gather: bool = True,
                       w_sf_layout: int = SF_ROWMAJOR, epilogue: int = EPI_NONE, topk_w=None, row_of=None,
                       k: int = 0, y=None, y_dtype=torch.float32, mode: int = MODE_AUTO, ws=None):
    """Expert linears over permuted rows; see ``moe_grouped_linear`` in ``include/nvfp4.h``."""
    K = x.shape[1]
    E, N = w_codes.shape[0], w_codes.shape[1]
    if y is None:
        if epilogue == EPI_SWIGLU:
            shape = (R, N // 2)
        elif epilogue == EPI_COMBINE:
            shape = (R // k, N)
        else:
            shape = (R, N)
        y = torch.empty(shape, dtype=y_dtype, device=x.device)
    ws, wsb = _workspace(int(lib().moe_grouped_linear_workspace(R, K, N, E, k, epilogue, mode)), x.device, ws)
    _check(lib().moe_grouped_linear(_ptr(x), _dtype_code(x), K, int(gather), _ptr(expert_offsets),
                                    _ptr(perm_tok), E, R, _ptr(w_codes), _ptr(w_scales), w_sf_layout, _ptr(w_gs),
                                    N, epilogue, _ptr(topk_w), _ptr(row_of), k, _ptr(y), _dtype_code(y), mode,
                                    _ptr(ws), wsb, _stream()), "moe_grouped_linear")
    return y


def moe_layer_decode(h: torch.Tensor, w_router: torch.Tensor, k: int, gate_up, down, logit_bias=None,
                     y=None, y_dtype=torch.float32, want_logits: bool = False, want_routing: bool = False,
                     want_a: bool = False, ws=None):
    """One expert layer for a decode batch (T <= 32): ``gate_up`` and ``down`` are
    the stacked ``(codes, TILED scales, gs)`` of the experts.  Returns ``y``, or
    ``(y, extras)`` with the requested ``logits``, ``topk_idx``/``topk_w`` and ``a``."""
    T, H = h.shape
    E = w_router.shape[0]
    I = gate_up[0].shape[1] // 2
    dev = h.device
    if y is None:
        y = torch.empty((T, H), dtype=y_dtype, device=dev)
    ex = {}
    if want_logits:
        ex["logits"] = torch.empty((T, E), dtype=torch.float32, device=dev)
    if want_routing:
        ex["topk_idx"] = torch.empty((T, k), dtype=torch.int32, device=dev)
        ex["topk_w"] = torch.empty((T, k), dtype=torch.float32, device=dev)
    if want_a:
        ex["a"] = torch.empty((T * k, I), dtype=torch.bfloat16, device=dev)
    ws, wsb = _workspace(int(lib().moe_layer_decode_workspace(T, H, I, E, k)), dev, ws)
    _check(lib().moe_layer_decode(_ptr(h), _ptr(w_router), _ptr(logit_bias), T, H, E, k, _ptr(gate_up[0]),
                                  _ptr(gate_up[1]), _ptr(gate_up[2]), I, _ptr(down[0]), _ptr(down[1]),
                                  _ptr(down[2]), _ptr(ex.get("logits")), _ptr(ex.get("topk_idx")),
                                  _ptr(ex.get("topk_w")), _ptr(ex.get("a")), _ptr(y), _dtype_code(y), _ptr(ws),
                                  wsb, _stream()), "moe_layer_decode")
    return (y, ex) if ex else y


def nvfp4_linear_w4a4_ws_layout(M: int, K: int) -> dict:
    """Byte offsets, inside a W4A4 ``nvfp4_linear`` workspace, of the quantized
    activations the call leaves there: ``gs_x``, ``codes``, ``scales``."""
    out = (ctypes.c_int64 * 3)()
    _check(lib().nvfp4_linear_w4a4_ws_layout(M, K, out), "nvfp4_linear_w4a4_ws_layout")
    return dict(zip(("gs_x", "codes", "scales"), (int(v) for v in out)))


def moe_grouped_linear_w4a4_ws_layout(R: int, K: int, N: int, E: int, k: int, epilogue: int) -> dict:
    """Byte offsets, inside a W4A4 ``moe_grouped_linear`` workspace, of the padded
    permuted activations the call leaves there (see include/nvfp4.h)."""
    out = (ctypes.c_int64 * 6)()
    _check(lib().moe_grouped_linear_w4a4_ws_layout(R, K, N, E, k, epilogue, out),
           "moe_grouped_linear_w4a4_ws_layout")
    return dict(zip(("gs_x", "pad_off", "src_rows", "codes", "scales", "rows_pad"), (int(v) for v in out)))


def nvfp4_debug_wait_timeout(limit_cycles: int):
    """Launch the library's wait-timeout probe (a bounded wait that runs out)."""
    _check(lib().nvfp4_debug_wait_timeout(int(limit_cycles), _stream()), "nvfp4_debug_wait_timeout")


def nvfp4_read_device_status() -> int:
    st = ctypes.c_int(0)
    _check(lib().nvfp4_read_device_status(_stream(), ctypes.byref(st)), "nvfp4_read_device_status")
    return st.value
