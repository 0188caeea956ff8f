"""The C-ABI library: exported symbols and host-side validation (no GPU needed).

Every entry point validates its arguments on the host before touching the
device, so these tests call it with fake (but aligned) pointers and check the
status codes; nothing is launched.  A fully valid call on a machine without a
B200 must return NVFP4_ERR_ARCH instead of launching.
"""
import ctypes
import os
import re

import pytest
import torch

import bit_linear_moe_b200 as nv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = ctypes.c_void_p(0x10000)           # aligned, never dereferenced
FAKE2 = ctypes.c_void_p(0x20000)
MISALIGNED = ctypes.c_void_p(0x10008)


@pytest.fixture(scope="module")
def L():
    from bit_linear_moe_b200 import build
    build.build()
    return nv.lib()


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    names = _declared_functions()
    assert "nvfp4_linear" in names and "moe_grouped_linear" in names and len(names) >= 12
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for s in range(11):
        assert nv.status_string(s) not in ("", "unknown status")
    assert nv.status_string(99) == "unknown status"


def test_scales_bytes(L):
    assert nv.nvfp4_scales_bytes(5, 48, nv.SF_ROWMAJOR) == 15
    assert nv.nvfp4_scales_bytes(5, 48, nv.SF_TILED) == 128 * 4
    assert nv.nvfp4_scales_bytes(129, 1024, nv.SF_TILED) == 256 * 64
    assert nv.nvfp4_scales_bytes(5, 40, nv.SF_TILED) == 0


def _linear(L, **kw):
    a = dict(x=FAKE, xd=nv.DTYPE_BF16, M=1, K=64, c=FAKE, s=FAKE, lay=nv.SF_ROWMAJOR, gs=FAKE, N=16,
             y=FAKE2, yd=nv.DTYPE_F32, mode=nv.MODE_W4A16, ws=None, wsb=0)
    a.update(kw)
    return L.nvfp4_linear(a["x"], a["xd"], a["M"], a["K"], a["c"], a["s"], a["lay"], a["gs"], a["N"], a["y"],
                          a["yd"], a["mode"], a["ws"], a["wsb"], None)


def test_linear_validation(L):
    assert _linear(L, x=None) == nv.ERR_NULL
    assert _linear(L, K=40) == nv.ERR_SHAPE
    assert _linear(L, M=0) == nv.ERR_SHAPE
    assert _linear(L, N=0) == nv.ERR_SHAPE
    assert _linear(L, c=MISALIGNED) == nv.ERR_ALIGN
    assert _linear(L, xd=nv.DTYPE_F32) == nv.ERR_DTYPE
    assert _linear(L, yd=7) == nv.ERR_DTYPE
    assert _linear(L, lay=5) == nv.ERR_LAYOUT
    assert _linear(L, mode=9) == nv.ERR_MODE
    need = L.nvfp4_linear_workspace(1, 64, 16, nv.MODE_W4A16)
    assert need >= 64 * 2 + 4
    assert _linear(L) == nv.ERR_WORKSPACE
    assert _linear(L, ws=FAKE2, wsb=need - 1) == nv.ERR_WORKSPACE
    assert _linear(L, ws=MISALIGNED, wsb=need) == nv.ERR_ALIGN
    assert _linear(L, N=200000, ws=FAKE2, wsb=need) == nv.ERR_SHAPE
    if not torch.cuda.is_available():
        assert _linear(L, ws=FAKE2, wsb=need) == nv.ERR_ARCH


def test_linear_w4a4_validation(L):
    ws_need = L.nvfp4_linear_workspace(512, 1024, 256, nv.MODE_W4A4)
    assert ws_need > 512 * 512
    assert _linear(L, M=512, K=1024, N=256, mode=nv.MODE_W4A4, lay=nv.SF_ROWMAJOR,
                   ws=FAKE, wsb=ws_need) == nv.ERR_LAYOUT
    assert _linear(L, M=512, K=1000 + 8, N=256, mode=nv.MODE_W4A4, lay=nv.SF_TILED,
                   ws=FAKE, wsb=ws_need) == nv.ERR_SHAPE
    assert _linear(L, M=512, K=1024, N=256, mode=nv.MODE_W4A4, lay=nv.SF_TILED,
                   ws=FAKE, wsb=ws_need - 1) == nv.ERR_WORKSPACE


def test_quantize_validation(L):
    def q(**kw):
        a = dict(x=FAKE, xd=nv.DTYPE_F32, rows=4, cols=64, gs=None, lay=nv.SF_ROWMAJOR, c=FAKE, s=FAKE,
                 go=FAKE2, ws=FAKE2, wsb=256)
        a.update(kw)
        return L.nvfp4_quantize(a["x"], a["xd"], a["rows"], a["cols"], a["gs"], a["lay"], a["c"], a["s"],
                                a["go"], a["ws"], a["wsb"], None)
    assert q(x=None) == nv.ERR_NULL
    assert q(cols=24) == nv.ERR_SHAPE
    assert q(rows=0) == nv.ERR_SHAPE
    assert q(wsb=16) == nv.ERR_WORKSPACE
    assert q(ws=None) == nv.ERR_WORKSPACE
    assert q(s=MISALIGNED) == nv.ERR_ALIGN
    assert q(xd=3) == nv.ERR_DTYPE
    assert q(lay=2) == nv.ERR_LAYOUT
    if not torch.cuda.is_available():
        assert q() == nv.ERR_ARCH


def test_route_validation(L):
    def r(**kw):
        a = dict(h=FAKE, w=FAKE, b=None, T=4, H=64, E=16, k=4, lo=None, ws=FAKE2)
        a.update(kw)
        wsb = a.pop("wsb", L.moe_route_topk_workspace(a["T"], a["E"], a["k"]))
        return L.moe_route_topk(a["h"], a["w"], a["b"], a["T"], a["H"], a["E"], a["k"], a["lo"], FAKE, FAKE,
                                FAKE, FAKE, FAKE, FAKE, a["ws"], wsb, None)
    assert r(h=None) == nv.ERR_NULL
    assert r(k=0) == nv.ERR_SHAPE
    assert r(k=17, E=16) == nv.ERR_SHAPE
    assert r(E=2048) == nv.ERR_SHAPE
    assert r(H=60) == nv.ERR_SHAPE
    assert r(wsb=8) == nv.ERR_WORKSPACE
    if not torch.cuda.is_available():
        assert r() == nv.ERR_ARCH


def test_grouped_validation(L):
    def g(**kw):
        a = dict(x=FAKE, K=64, gather=1, off=FAKE, pt=FAKE, E=8, R=16, c=FAKE, s=FAKE, lay=nv.SF_ROWMAJOR,
                 gs=FAKE, N=32, epi=nv.EPI_NONE, tw=None, ro=None, k=0, y=FAKE2, mode=nv.MODE_W4A16)
        a.update(kw)
        wsb = L.moe_grouped_linear_workspace(a["R"], a["K"], a["N"], a["E"], a["k"], a["epi"], a["mode"])
        return L.moe_grouped_linear(a["x"], nv.DTYPE_BF16, a["K"], a["gather"], a["off"], a["pt"], a["E"],
                                    a["R"], a["c"], a["s"], a["lay"], a["gs"], a["N"], a["epi"], a["tw"],
                                    a["ro"], a["k"], a["y"], nv.DTYPE_F32, a["mode"], FAKE2 if wsb else None,
                                    wsb, None)
    assert g(pt=None) == nv.ERR_NULL
    assert g(epi=nv.EPI_COMBINE) == nv.ERR_NULL
    assert g(epi=nv.EPI_COMBINE, tw=FAKE, ro=FAKE, k=3) == nv.ERR_SHAPE
    assert g(epi=nv.EPI_SWIGLU, N=33) == nv.ERR_SHAPE
    assert g(epi=7) == nv.ERR_MODE
    assert g(K=48) == nv.ERR_SHAPE
    if not torch.cuda.is_available():
        assert g() == nv.ERR_ARCH


def test_stack_glue_validation(L):
    ODD = ctypes.c_void_p(0x10001)

    def rms(**kw):
        a = dict(x=FAKE, xd=nv.DTYPE_F32, rows=2, cols=64, ld=128, y=FAKE2)
        a.update(kw)
        return L.nvfp4_rms_norm(a["x"], a["xd"], a["rows"], a["cols"], a["ld"], a["y"], None)

    assert rms(x=None) == nv.ERR_NULL
    assert rms(y=None) == nv.ERR_NULL
    assert rms(xd=3) == nv.ERR_DTYPE
    assert rms(rows=0) == nv.ERR_SHAPE
    assert rms(cols=0) == nv.ERR_SHAPE
    assert rms(ld=63) == nv.ERR_SHAPE
    assert rms(x=ctypes.c_void_p(0x10002)) == nv.ERR_ALIGN       # fp32 rows need 4-byte alignment
    assert rms(x=ctypes.c_void_p(0x10002), xd=nv.DTYPE_BF16) != nv.ERR_ALIGN
    assert rms(y=ODD) == nv.ERR_ALIGN

    def silu(**kw):
        a = dict(g=FAKE, gd=nv.DTYPE_BF16, rows=2, half=64, h=FAKE2)
        a.update(kw)
        return L.nvfp4_silu_mul(a["g"], a["gd"], a["rows"], a["half"], a["h"], None)

    assert silu(g=None) == nv.ERR_NULL
    assert silu(gd=7) == nv.ERR_DTYPE
    assert silu(half=0) == nv.ERR_SHAPE
    assert silu(g=ODD) == nv.ERR_ALIGN
    if not torch.cuda.is_available():
        assert rms() == nv.ERR_ARCH and silu() == nv.ERR_ARCH


def test_noalloc_scratch_limit(L):
    """The allocation-free router needs ceil(T/32) * E * 8 bytes of its 1 MiB
    scratch (plus T * E * 4 without a logits buffer) and says so before
    touching the device."""
    def route(T, logits):
        return L.moe_route_topk_noalloc(FAKE, FAKE2, None, T, 2048, 512, 10, logits, FAKE, FAKE, FAKE, FAKE,
                                        FAKE, FAKE, None)

    assert route(8192 + 1, FAKE) == nv.ERR_WORKSPACE            # 257 blocks x 512 x 8 > 1 MiB
    assert route(513, None) == nv.ERR_WORKSPACE                 # 513 x 512 x 4 B of logits alone > 1 MiB
    if not torch.cuda.is_available():
        assert route(8192, FAKE) == nv.ERR_ARCH                 # fits: validation passes, then no B200
        assert route(32, None) == nv.ERR_ARCH


def test_grouped_auto_mode_threshold(L):
    """AUTO runs the grouped linear as W4A16 for R <= 512 rows and as W4A4 above:
    the workspace query follows the same rule (k = 10, so the switch is not at
    32 * k = 320 rows)."""
    K, N, E, k = 2048, 1024, 512, 10
    for epi in (nv.EPI_NONE, nv.EPI_SWIGLU, nv.EPI_COMBINE):
        for R in (320, 321, 512, 513):
            auto = L.moe_grouped_linear_workspace(R, K, N, E, k, epi, nv.MODE_AUTO)
            want = nv.MODE_W4A16 if R <= 512 else nv.MODE_W4A4
            assert auto == L.moe_grouped_linear_workspace(R, K, N, E, k, epi, want), (epi, R)
        assert (L.moe_grouped_linear_workspace(512, K, N, E, k, epi, nv.MODE_W4A16)
                != L.moe_grouped_linear_workspace(512, K, N, E, k, epi, nv.MODE_W4A4))


def test_w4a4_workspace_layouts(L):
    """The documented places of the quantized activations inside the W4A4
    workspaces: inside the workspace the size query returns, 16-byte aligned,
    in the stated order."""
    M, K = 2048, 5120
    lay = nv.nvfp4_linear_w4a4_ws_layout(M, K)
    need = L.nvfp4_linear_workspace(M, K, 4096, nv.MODE_W4A4)
    assert lay["gs_x"] % 4 == 0 and lay["codes"] % 16 == 0 and lay["scales"] % 16 == 0
    assert lay["codes"] + M * K // 2 <= lay["scales"]
    assert lay["scales"] + nv.nvfp4_scales_bytes(M, K, nv.SF_TILED) <= need
    with pytest.raises(nv.NVFP4Error):
        nv.nvfp4_linear_w4a4_ws_layout(M, 5000)
    R, E, k, N = 40960, 512, 10, 1024
    for epi in (nv.EPI_NONE, nv.EPI_SWIGLU, nv.EPI_COMBINE):
        g = nv.moe_grouped_linear_w4a4_ws_layout(R, 2048, N, E, k, epi)
        need = L.moe_grouped_linear_workspace(R, 2048, N, E, k, epi, nv.MODE_W4A4)
        rp = g["rows_pad"]
        assert rp % 128 == 0 and rp >= R + 127 * E
        assert g["pad_off"] + 4 * (E + 1) <= g["src_rows"]
        assert g["src_rows"] + 4 * rp <= g["codes"]
        assert g["codes"] + rp * 1024 <= g["scales"]
        assert g["scales"] + nv.nvfp4_scales_bytes(rp, 2048, nv.SF_TILED) <= need
        assert all(v % 16 == 0 for key, v in g.items() if key != "rows_pad")
    with pytest.raises(nv.NVFP4Error):
        nv.moe_grouped_linear_w4a4_ws_layout(R, 2000, N, E, k, nv.EPI_NONE)


def test_debug_wait_timeout_validation(L):
    assert L.nvfp4_debug_wait_timeout(0, None) == nv.ERR_SHAPE
    assert L.nvfp4_debug_wait_timeout(5_000_000_000, None) == nv.ERR_SHAPE
    if not torch.cuda.is_available():
        assert L.nvfp4_debug_wait_timeout(1000, None) == nv.ERR_ARCH


def test_moe_layer_decode_validation(L):
    """The decode-time expert layer: workspace query and host-side checks."""
    need = L.moe_layer_decode_workspace(32, 2048, 512, 512, 10)
    assert need > 32 * 10 * 2048 * 4                      # holds the per-slot fp32 rows of the down projection
    assert L.moe_layer_decode_workspace(33, 2048, 512, 512, 10) == 0    # T > 32
    assert L.moe_layer_decode_workspace(1, 2000, 512, 512, 10) == 0     # H % 256
    assert L.moe_layer_decode_workspace(1, 2048, 500, 512, 10) == 0     # I % 256
    assert L.moe_layer_decode_workspace(1, 8192, 512, 512, 10) == 0     # H above 4096
    assert L.moe_layer_decode_workspace(1, 2048, 512, 8, 10) == 0       # k > E

    def call(**kw):
        a = dict(h=FAKE, wr=FAKE, T=1, H=2048, E=512, k=10, I=512, y=FAKE2, yd=nv.DTYPE_F32, ws=FAKE2,
                 wsb=L.moe_layer_decode_workspace(1, 2048, 512, 512, 10), ao=None)
        a.update(kw)
        return L.moe_layer_decode(a["h"], a["wr"], None, a["T"], a["H"], a["E"], a["k"], FAKE, FAKE, FAKE, a["I"],
                                  FAKE, FAKE, FAKE, None, None, None, a["ao"], a["y"], a["yd"], a["ws"], a["wsb"],
                                  None)

    assert call(h=None) == nv.ERR_NULL
    assert call(yd=5) == nv.ERR_DTYPE
    assert call(T=0) == nv.ERR_SHAPE
    assert call(T=40) == nv.ERR_SHAPE
    assert call(ao=MISALIGNED) == nv.ERR_ALIGN
    assert call(wsb=16) == nv.ERR_WORKSPACE
    if not torch.cuda.is_available():
        assert call() == nv.ERR_ARCH


def test_chain_validation(L):
    import bit_linear_moe_b200 as nvm

    class T:  # a stand-in tensor with a fixed aligned address
        def __init__(self, ptr, shape, stride0=None, dtype=torch.float32):
            self._p, self.shape, self.dtype = ptr, shape, dtype
            self._s = stride0 if stride0 is not None else shape[-1]

        def data_ptr(self):
            return self._p

        def stride(self, d):
            return self._s

    w = (T(0x10000, (128, 128)), T(0x20000, (128,)), T(0x30000, (1,)))
    def run(specs, M=1):
        ops = nvm.chain_ops(specs)
        n = len(ops)
        p = ctypes.cast(ops, ctypes.c_void_p)
        need = L.nvfp4_chain_workspace(p, n, M)
        return L.nvfp4_chain(p, n, M, FAKE2 if need else None, need, None), need

    xin = T(0x40000, (1, 256), dtype=torch.bfloat16)
    ok = [{"w": w, "src": xin, "y": T(0x50000, (1, 128))}]
    st, need = run(ok)
    assert need > 0
    if not torch.cuda.is_available():
        assert st == nv.ERR_ARCH
    assert run(ok, M=3)[0] == nv.ERR_SHAPE                                         # M > 2
    assert run([{"w": w, "src": 0}])[0] == nv.ERR_SHAPE                           # reads itself
    assert run([{"w": w, "src": xin, "xform": nv.CHAIN_XFORM_RMS}])[0] == nv.ERR_MODE
    assert run([{"w": w, "src": T(0x40008, (1, 256), dtype=torch.bfloat16)}])[0] == nv.ERR_ALIGN
    w_bad = (T(0x10000, (100, 128)), w[1], w[2])                                    # N % 8
    assert run([{"w": w_bad, "src": xin}])[0] == nv.ERR_SHAPE
    two = ok + [{"w": w, "src": 0, "xform": nv.CHAIN_XFORM_SILU_MUL}]              # silu needs N = 2K
    assert run(two)[0] == nv.ERR_SHAPE


def test_calibrate_validation(L):
    def c(**kw):
        a = dict(w=FAKE, N=64, K=128, x=FAKE2, xd=nv.DTYPE_BF16, S=16, lay=nv.SF_TILED)
        a.update(kw)
        need = L.nvfp4_calibrate_workspace(a["N"], a["K"], a["S"])
        wsb = a.pop("wsb", need)
        return L.nvfp4_calibrate(a["w"], a["N"], a["K"], a["x"], a["xd"], a["S"], a["lay"], FAKE, FAKE, FAKE, FAKE,
                                 None, None, FAKE2 if wsb else None, wsb, None)
    assert L.nvfp4_calibrate_workspace(64, 128, 16) > 64 * 128 * 4
    assert L.nvfp4_calibrate_workspace(64, 100, 16) == 0
    assert c(w=None) == nv.ERR_NULL
    assert c(xd=nv.DTYPE_F32) == nv.ERR_DTYPE
    assert c(K=100) == nv.ERR_SHAPE
    assert c(S=0) == nv.ERR_SHAPE
    assert c(lay=7) == nv.ERR_LAYOUT
    assert c(wsb=64) == nv.ERR_WORKSPACE
    if not torch.cuda.is_available():
        assert c() == nv.ERR_ARCH


def test_rms_norm_quant_validation(L):
    def r(**kw):
        a = dict(x=FAKE, xd=nv.DTYPE_BF16, rows=4, cols=64, ld=64, lay=nv.SF_TILED)
        a.update(kw)
        wsb = a.pop("wsb", L.nvfp4_rms_norm_quant_workspace(a["rows"]))
        return L.nvfp4_rms_norm_quant(a["x"], a["xd"], a["rows"], a["cols"], a["ld"], a["lay"], FAKE, FAKE, FAKE2,
                                      FAKE2, wsb, None)
    assert r(x=None) == nv.ERR_NULL
    assert r(xd=5) == nv.ERR_DTYPE
    assert r(cols=40) == nv.ERR_SHAPE
    assert r(ld=60) == nv.ERR_SHAPE
    assert r(ld=68) == nv.ERR_ALIGN                      # bf16 rows need a stride of 8 elements
    assert r(wsb=4) == nv.ERR_WORKSPACE
    if not torch.cuda.is_available():
        assert r() == nv.ERR_ARCH
