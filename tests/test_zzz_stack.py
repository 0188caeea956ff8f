"""GPU decode-stack glue (rms renormalisation, silu * up) against the oracle,
and one stack layer on small shapes checked stage by stage (each stage on the
GPU's own input to it).  bf16 outputs may differ from the oracle's bf16 by one
bf16 step: the GPU sums in fp32, in another order, before the same rounding."""
import numpy as np
import pytest
import torch

import bit_linear_moe_b200 as nv
import oracle
from oracle import stack as ost
from bit_linear_moe_b200 import synth
from nvfp4_checks import assert_within_bound, bf16_ulp, rowmajor_to_tiled, tiled_to_rowmajor

pytestmark = pytest.mark.gpu


def _close_bf16(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    lim = bf16_ulp(ref) + 1e-30
    assert (err <= lim).all(), f"{what}: {(err > lim).sum()} elements off by more than one bf16 step"


@pytest.mark.parametrize("rows,cols,ld,dtype", [(1, 5120, 10240, torch.float32), (8, 5120, 5120, torch.bfloat16),
                                                (3, 100, 100, torch.float32), (32, 5120, 5120, torch.float32),
                                                (4, 777, 800, torch.bfloat16)])
def test_rms_norm(rows, cols, ld, dtype):
    rng = np.random.default_rng(rows * 7 + cols)
    x = (rng.standard_normal((rows, ld)) * rng.uniform(0.01, 100, (rows, 1))).astype(np.float32)
    if rows > 2:
        x[1] = 0.0                                  # an all-zero row stays zero
    xd = torch.from_numpy(x).to(dtype).cuda()
    y = nv.nvfp4_rms_norm(xd, cols=cols)
    torch.cuda.synchronize()
    xin = xd.float().cpu().numpy()[:, :cols]
    ref = ost.rms_norm(xin)
    _close_bf16(y.float().cpu().numpy(), ref, f"rms {rows}x{cols}")
    if rows > 2:
        assert not y[1].float().any()


@pytest.mark.parametrize("rows,half,dtype", [(1, 17408, torch.float32), (32, 17408, torch.bfloat16),
                                             (5, 33, torch.float32)])
def test_silu_mul(rows, half, dtype):
    rng = np.random.default_rng(rows + half)
    g = (4 * rng.standard_normal((rows, 2 * half))).astype(np.float32)
    gd = torch.from_numpy(g).to(dtype).cuda()
    h = nv.nvfp4_silu_mul(gd)
    torch.cuda.synchronize()
    ref = ost.silu_mul(gd.float().cpu().numpy())
    _close_bf16(h.float().cpu().numpy(), ref, f"silu_mul {rows}x{half}")


@pytest.mark.parametrize("M", [1, 8])
def test_stack_layer_small(M):
    """One layer of the stack on small shapes: hidden 512, QKV 1024, GU 2 x 768."""
    d, nq, ni = 512, 1024, 768
    rng = np.random.default_rng(900 + M)
    shapes = {"qkv": (nq, d), "o": (d, d), "gu": (2 * ni, d), "down": (d, ni)}
    q_w = {k: oracle.quantize(synth.weight(np.random.default_rng([900, i]), n, kk))
           for i, (k, (n, kk)) in enumerate(shapes.items())}
    dev_w = {}
    for k, (c, s, g) in q_w.items():
        n, kk = shapes[k]
        dev_w[k] = (torch.from_numpy(np.ascontiguousarray(c)).cuda(),
                    torch.from_numpy(np.ascontiguousarray(rowmajor_to_tiled(s, n, kk)).ravel()).cuda(),
                    torch.tensor([g], dtype=torch.float32, device="cuda"))

    def lin(x_bf16, k):
        c, s, g = dev_w[k]
        return nv.nvfp4_linear(x_bf16, c, s, g, w_sf_layout=nv.SF_TILED, y_dtype=torch.float32,
                               mode=nv.MODE_W4A16)

    x0 = ost.rms_norm(rng.standard_normal((M, d)).astype(np.float32))
    x = torch.from_numpy(x0).to(torch.bfloat16).cuda()
    q = lin(x, "qkv")
    o_in = nv.nvfp4_rms_norm(q, cols=d)
    o = lin(o_in, "o")
    gu_in = nv.nvfp4_rms_norm(o)
    g = lin(gu_in, "gu")
    h = nv.nvfp4_silu_mul(g)
    dn = lin(h, "down")
    x1 = nv.nvfp4_rms_norm(dn)
    torch.cuda.synchronize()

    def host(t):
        return t.float().cpu().numpy()

    ref, ad = oracle.linear_w4a16(x0, *q_w["qkv"])
    assert_within_bound(q, ref, ad, False, "qkv")
    _close_bf16(host(o_in), ost.rms_norm(host(q)[:, :d]), "rms(q slice)")
    ref, ad = oracle.linear_w4a16(host(o_in), *q_w["o"])
    assert_within_bound(o, ref, ad, False, "o")
    _close_bf16(host(gu_in), ost.rms_norm(host(o)), "rms(o)")
    ref, ad = oracle.linear_w4a16(host(gu_in), *q_w["gu"])
    assert_within_bound(g, ref, ad, False, "gate/up")
    _close_bf16(host(h), ost.silu_mul(host(g)), "silu * up")
    ref, ad = oracle.linear_w4a16(host(h), *q_w["down"])
    assert_within_bound(dn, ref, ad, False, "down")
    _close_bf16(host(x1), ost.rms_norm(host(dn)), "rms(down)")
    # the renormalised output has mean square 1 up to the bf16 rounding
    ms = np.mean(host(x1).astype(np.float64) ** 2, axis=1)
    assert np.allclose(ms, 1.0, atol=2e-2)


# ---- the 64-layer stack at the 27B shapes ------------------------------------------

_SH = synth.DENSE27B        # (name, K, N, seed): qkv, o_proj, gate_up, down


def _stack_layer(li):
    """Layer li of the stack as the bench builds it: 0.02 N(0, 1) weights drawn on
    the device (seed 1000 + 4 li + j), quantized by nvfp4_quantize (TILED)."""
    mats = {}
    for j, (name, K, N, _) in enumerate(_SH):
        gen = torch.Generator(device="cuda")
        gen.manual_seed(1000 + 4 * li + j)
        w = 0.02 * torch.randn((N, K), generator=gen, device="cuda")
        mats[name] = (w,) + tuple(nv.nvfp4_quantize(w, sf_layout=nv.SF_TILED))
    return mats


def _host_weights(li, mats):
    """The layer's NVFP4 weights on the host (row-major scales), after checking
    on 16 seeded rows per matrix that they are the oracle's quantization of
    the fp32 weights (gs from the whole tensor's amax)."""
    out = {}
    rng = np.random.default_rng([li, 77])
    for name, K, N, _ in _SH:
        w, c, s, g = mats[name]
        gs = oracle.global_scale(np.array([w.abs().max().item()], dtype=np.float32))
        assert np.float32(g.item()) == gs, f"layer {li} {name}: gs"
        codes = c.cpu().numpy()
        scales = tiled_to_rowmajor(s.cpu().numpy(), N, K)
        rows = np.sort(rng.choice(N, 16, replace=False))
        q = oracle.quantize(w[torch.from_numpy(rows).cuda()].cpu().numpy(), gs=gs)
        assert np.array_equal(codes[rows], q[0]) and np.array_equal(scales[rows], q[1]), \
            f"layer {li} {name}: weights differ from the oracle's quantization"
        out[name] = (codes, scales, gs)
    return out


@pytest.mark.parametrize("M", [1, 8, 32])
def test_stack_27b_stagewise(M):
    """The 64-layer decode stack at the 27B shapes, run as the bench runs it.
    Every stage (the four linears, the three renormalisations, silu * up) of
    layers 0, 1, 31 and 63 (all 64 layers at M = 1) is checked against the
    oracle on the GPU's own input to that stage."""
    kq = _SH[0][1]
    check = set(range(64)) if M == 1 else {0, 1, 31, 63}
    gx = torch.Generator(device="cuda")
    gx.manual_seed(999)
    x = nv.nvfp4_rms_norm(torch.randn((M, kq), generator=gx, device="cuda"))

    def host(t):
        return t.float().cpu().numpy()

    for li in range(64):
        mats = _stack_layer(li)

        def lin(xin, name):
            _, c, s, g = mats[name]
            return nv.nvfp4_linear(xin, c, s, g, w_sf_layout=nv.SF_TILED, y_dtype=torch.float32,
                                   mode=nv.MODE_W4A16)

        q = lin(x, "qkv")
        o_in = nv.nvfp4_rms_norm(q, cols=kq)
        o = lin(o_in, "o_proj")
        gu_in = nv.nvfp4_rms_norm(o)
        g = lin(gu_in, "gate_up")
        h = nv.nvfp4_silu_mul(g)
        dn = lin(h, "down")
        x_next = nv.nvfp4_rms_norm(dn)
        torch.cuda.synchronize()
        if li in check:
            wq = _host_weights(li, mats)
            ref, ad = oracle.linear_w4a16(host(x), *wq["qkv"])
            assert_within_bound(q, ref, ad, False, f"layer {li} qkv")
            _close_bf16(host(o_in), ost.rms_norm(host(q)[:, :kq]), f"layer {li} rms(q slice)")
            ref, ad = oracle.linear_w4a16(host(o_in), *wq["o_proj"])
            assert_within_bound(o, ref, ad, False, f"layer {li} o_proj")
            _close_bf16(host(gu_in), ost.rms_norm(host(o)), f"layer {li} rms(o)")
            ref, ad = oracle.linear_w4a16(host(gu_in), *wq["gate_up"])
            assert_within_bound(g, ref, ad, False, f"layer {li} gate_up")
            _close_bf16(host(h), ost.silu_mul(host(g)), f"layer {li} silu * up")
            ref, ad = oracle.linear_w4a16(host(h), *wq["down"])
            assert_within_bound(dn, ref, ad, False, f"layer {li} down")
            _close_bf16(host(x_next), ost.rms_norm(host(dn)), f"layer {li} rms(down)")
            del wq
        del mats
        x = x_next
    xf = host(x).astype(np.float64)
    assert np.isfinite(xf).all()
    assert np.allclose(np.mean(xf ** 2, axis=1), 1.0, atol=2e-2)
