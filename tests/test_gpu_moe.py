"""GPU mixture-of-experts path vs the CPU oracle.

Routing: the GPU's fp32 logits are within the linear bound of the fp64 logits;
top-k indices are bit-exact against the oracle's top-k taken on the GPU's own
fp32 logits; the permutation is bit-exact against the oracle's counting sort of
the GPU's indices.  Expert linears are checked stage by stage: each stage's
reference is computed by the oracle from the GPU's inputs to that stage.
"""
import functools

import numpy as np
import pytest
import torch

import bit_linear_moe_b200 as nv
import oracle
from oracle import moe as omoe
from bit_linear_moe_b200 import synth
from nvfp4_checks import assert_within_bound, bf16_ulp

pytestmark = pytest.mark.gpu
E, H, I, K_TOP = synth.MOE_E, synth.MOE_H, synth.MOE_I, synth.MOE_K


@functools.lru_cache(maxsize=1)
def _router():
    return synth.moe_router()


def _route(T, zipf):
    h = synth.moe_hidden(T)
    wr = _router()
    bias = synth.moe_zipf_bias() if zipf else None
    hd = torch.from_numpy(h).to(torch.bfloat16).cuda()
    wd = torch.from_numpy(wr).to(torch.bfloat16).cuda()
    bd = None if bias is None else torch.from_numpy(bias).cuda()
    out = nv.moe_route_topk(hd, wd, K_TOP, logit_bias=bd, want_logits=True)
    torch.cuda.synchronize()
    return h, wr, bias, hd, {k: v.cpu().numpy() for k, v in out.items()}, out


@pytest.mark.parametrize("T", synth.MOE_T)
@pytest.mark.parametrize("zipf", [False, True])
def test_route_topk_permutation(T, zipf):
    h, wr, bias, _, g, _ = _route(T, zipf)
    ref = omoe.router_logits(h, wr, bias)
    absdot = np.abs(h.astype(np.float64)) @ np.abs(wr.astype(np.float64)).T
    assert_within_bound(g["logits"], ref, absdot, False, "router logits")
    idx, w = omoe.topk(g["logits"].astype(np.float64), K_TOP)
    assert np.array_equal(g["topk_idx"], idx)
    assert np.allclose(g["topk_w"], w, rtol=2e-6, atol=1e-7)
    off, pt, ps, ro = omoe.permute(g["topk_idx"], E)
    assert np.array_equal(g["expert_offsets"], off)
    assert np.array_equal(g["perm_tok"], pt)
    assert np.array_equal(g["perm_slot"], ps)
    assert np.array_equal(g["row_of"], ro)
    # near-ties between the k-th and (k+1)-th fp64 logits are reported, not gated
    s = np.sort(ref, axis=1)[:, ::-1]
    near = int((s[:, K_TOP - 1] - s[:, K_TOP] < 2e-4 * absdot.max(axis=1)).sum())
    print(f"T={T} zipf={zipf}: {near} near-tie tokens; touched experts {int((np.diff(off) > 0).sum())}")


def test_route_ties_go_to_lower_index():
    T, Hs, Es = 4, 64, 40
    h = np.zeros((T, Hs), np.float32)
    h[:, 0] = 1.0
    wr = np.zeros((Es, Hs), np.float32)
    wr[[3, 7, 11, 20, 33], 0] = 0.5          # five equal top logits
    wr[[1, 2], 0] = 0.25
    out = nv.moe_route_topk(torch.from_numpy(h).to(torch.bfloat16).cuda(),
                            torch.from_numpy(wr).to(torch.bfloat16).cuda(), 6, want_logits=True)
    idx = out["topk_idx"].cpu().numpy()
    assert (idx == np.array([3, 7, 11, 20, 33, 1])).all()
    assert np.allclose(out["topk_w"].cpu().numpy()[:, :5], np.exp(0.5) / (5 * np.exp(0.5) + np.exp(0.25)))


@pytest.mark.parametrize("T,Hs,Es,with_bias", [(300, 128, 96, True), (129, 1088, 90, False), (65, 64, 512, True),
                                                (1000, 2048, 130, True), (200, 128, 700, False)])
def test_router_tensor_core_shapes(T, Hs, Es, with_bias):
    """Token counts above 64 run the tensor-core router: ragged token and
    expert tiles, a K ring that wraps, expert counts that are not a multiple
    of 4 (scalar stores)."""
    rng = np.random.default_rng(T + Hs + Es)
    h = synth.to_bf16(rng.standard_normal((T, Hs)).astype(np.float32))
    wr = synth.to_bf16((0.05 * rng.standard_normal((Es, Hs))).astype(np.float32))
    bias = (0.1 * rng.standard_normal(Es)).astype(np.float32) if with_bias else None
    k = 6
    out = nv.moe_route_topk(torch.from_numpy(h).to(torch.bfloat16).cuda(), torch.from_numpy(wr).to(torch.bfloat16).cuda(),
                            k, logit_bias=None if bias is None else torch.from_numpy(bias).cuda(), want_logits=True)
    torch.cuda.synchronize()
    g = {n: v.cpu().numpy() for n, v in out.items()}
    ref = omoe.router_logits(h, wr, bias)
    absdot = np.abs(h.astype(np.float64)) @ np.abs(wr.astype(np.float64)).T
    assert_within_bound(g["logits"], ref, absdot, False, f"router logits T={T} H={Hs} E={Es}")
    idx, _ = omoe.topk(g["logits"].astype(np.float64), k)
    assert np.array_equal(g["topk_idx"], idx)


def test_route_ties_go_to_lower_index_tensor_core():
    T, Hs, Es = 100, 64, 40
    h = np.zeros((T, Hs), np.float32)
    h[:, 0] = 1.0
    wr = np.zeros((Es, Hs), np.float32)
    wr[[3, 7, 11, 20, 33], 0] = 0.5
    wr[[1, 2], 0] = 0.25
    out = nv.moe_route_topk(torch.from_numpy(h).to(torch.bfloat16).cuda(),
                            torch.from_numpy(wr).to(torch.bfloat16).cuda(), 6, want_logits=True)
    idx = out["topk_idx"].cpu().numpy()
    assert (idx == np.array([3, 7, 11, 20, 33, 1])).all()


class _Experts:
    """Expert weights for the routed-expert tests.  The oracle quantizes every
    expert it checks; untouched experts hold zeros (they are never read)."""

    def __init__(self, experts):
        self.gu = {}
        self.dn = {}
        for e in experts:
            wgu, wd = synth.moe_expert(int(e))
            self.gu[int(e)] = oracle.quantize(wgu)
            self.dn[int(e)] = oracle.quantize(wd)

    @staticmethod
    def _stack(qs, N, K):
        codes = np.zeros((E, N, K // 2), np.uint8)
        scales = np.zeros((E, N, K // 16), np.uint8)
        gs = np.ones(E, np.float32)
        for e, q in qs.items():
            codes[e], scales[e], gs[e] = q
        return (torch.from_numpy(codes).cuda(), torch.from_numpy(scales.reshape(-1)).cuda(),
                torch.from_numpy(gs).cuda())

    def gate_up(self):
        return self._stack(self.gu, 2 * I, H)

    def down(self):
        return self._stack(self.dn, H, I)


@pytest.mark.parametrize("T", [1, 32])
@pytest.mark.parametrize("zipf", [False, True])
def test_expert_layer_w4a16(T, zipf):
    h, _, _, hd, g, dev = _route(T, zipf)
    touched = np.flatnonzero(np.diff(g["expert_offsets"]) > 0)
    ex = _Experts(touched)
    R = T * K_TOP
    gc, gsc, ggs = ex.gate_up()
    a = nv.moe_grouped_linear(hd, dev["expert_offsets"], gc, gsc, ggs, R, perm_tok=dev["perm_tok"], gather=True,
                              epilogue=nv.EPI_SWIGLU, y_dtype=torch.bfloat16, mode=nv.MODE_W4A16)
    torch.cuda.synchronize()
    # stage 1: gate/up + SwiGLU against the oracle on the GPU's routing
    off, pt = g["expert_offsets"], g["perm_tok"]
    wc = np.zeros((E, 2 * I, H // 2), np.uint8); ws = np.zeros((E, 2 * I, H // 16), np.uint8)
    wg = np.ones(E, np.float32)
    for e in touched:
        wc[e], ws[e], wg[e] = ex.gu[int(e)]
    gu, gu_ad = omoe.grouped_linear_w4a16(h, off, pt, wc, ws, wg, gather=True)
    ref_a = omoe.swiglu(gu)
    gg, uu = gu[:, :I], gu[:, I:]
    sig = 1.0 / (1.0 + np.exp(-gg))
    dg = 1e-4 * gu_ad[:, :I] + 1e-6
    du = 1e-4 * gu_ad[:, I:] + 1e-6
    # first-order propagation of the gate/up bound through silu(g) * u
    bound = np.abs(uu) * np.abs(sig * (1 + gg * (1 - sig))) * dg + np.abs(gg * sig) * du + dg * du
    bound = bound + 1e-5 * np.abs(ref_a) + 1e-6 + bf16_ulp(ref_a)
    a_np = a.float().cpu().numpy()
    err = np.abs(a_np - ref_a)
    assert (err <= bound).all(), f"swiglu stage: {(err > bound).sum()} outside, max ratio {np.max(err / bound)}"
    # stage 2: down + combine from the GPU's own a
    dc, dsc, dgs = ex.down()
    y = nv.moe_grouped_linear(a, dev["expert_offsets"], dc, dsc, dgs, R, gather=False,
                              epilogue=nv.EPI_COMBINE, topk_w=dev["topk_w"], row_of=dev["row_of"], k=K_TOP,
                              y_dtype=torch.float32, mode=nv.MODE_W4A16)
    torch.cuda.synchronize()
    dwc = np.zeros((E, H, I // 2), np.uint8); dws = np.zeros((E, H, I // 16), np.uint8)
    dwg = np.ones(E, np.float32)
    for e in touched:
        dwc[e], dws[e], dwg[e] = ex.dn[int(e)]
    d, d_ad = omoe.grouped_linear_w4a16(a_np, off, pt, dwc, dws, dwg, gather=False)
    ref_y, _ = omoe.combine(d, g["topk_w"].astype(np.float64), g["row_of"])
    ybound_ad, _ = omoe.combine(d_ad, np.abs(g["topk_w"].astype(np.float64)), g["row_of"])
    assert_within_bound(y, ref_y, ybound_ad, False, "down + combine")


def test_untouched_experts_are_not_read():
    """Experts without rows may hold unreadable garbage: give them NaN scales
    and check the outputs stay finite and equal to the clean run."""
    T = 1
    h, _, _, hd, g, dev = _route(T, False)
    touched = np.flatnonzero(np.diff(g["expert_offsets"]) > 0)
    ex = _Experts(touched)
    gc, gsc, ggs = ex.gate_up()
    a1 = nv.moe_grouped_linear(hd, dev["expert_offsets"], gc, gsc, ggs, T * K_TOP, perm_tok=dev["perm_tok"],
                               epilogue=nv.EPI_SWIGLU, mode=nv.MODE_W4A16)
    sc = gsc.view(E, -1).clone()
    mask = torch.ones(E, dtype=torch.bool)
    mask[torch.from_numpy(touched)] = False
    sc[mask.cuda()] = 0x7F                   # E4M3 NaN everywhere an untouched expert has a scale
    a2 = nv.moe_grouped_linear(hd, dev["expert_offsets"], gc, sc.reshape(-1), ggs, T * K_TOP,
                               perm_tok=dev["perm_tok"], epilogue=nv.EPI_SWIGLU, mode=nv.MODE_W4A16)
    torch.cuda.synchronize()
    assert torch.isfinite(a2).all() and torch.equal(a1, a2)


# ---- grouped W4A4 (tensor-core) expert layer ---------------------------------

def _w4a4_layer(E, T, zipf_like, seed=20):
    """E experts with the per-expert shapes of the 512-expert layer; weights
    quantized on the GPU (bit-exactness of that quantizer is tested in
    test_gpu_quantize) and by the oracle for the experts it checks."""
    rng = np.random.default_rng(seed)
    wr = synth.to_bf16(0.02 * rng.standard_normal((E, H)))
    h = synth.activations(np.random.default_rng([seed, T]), T, H)
    bias = (-1.1 * np.log(np.random.default_rng([seed, 1]).permutation(E) + 1)).astype(np.float32) if zipf_like \
        else None
    gu_f = [synth.weight(np.random.default_rng([seed, 2, e]), 2 * I, H) for e in range(E)]
    dn_f = [synth.weight(np.random.default_rng([seed, 3, e]), H, I) for e in range(E)]

    def stack(ws):
        N, K = ws[0].shape
        sb = nv.nvfp4_scales_bytes(N, K, nv.SF_TILED)
        codes = torch.empty((E, N, K // 2), dtype=torch.uint8, device="cuda")
        scales = torch.empty(E * sb, dtype=torch.uint8, device="cuda")
        gs = torch.empty(E, dtype=torch.float32, device="cuda")
        for e, w in enumerate(ws):
            nv.nvfp4_quantize(torch.from_numpy(w).cuda(), sf_layout=nv.SF_TILED, codes=codes[e],
                              scales=scales[e * sb:(e + 1) * sb], gs_out=gs[e:e + 1])
        return codes, scales, gs

    return h, wr, bias, gu_f, dn_f, stack(gu_f), stack(dn_f)


@pytest.mark.parametrize("zipf", [False, True])
def test_expert_layer_w4a4_4096_tokens(zipf):
    E_, T = 64, 4096
    h, wr, bias, gu_f, dn_f, (gc, gsc, ggs), (dc, dsc, dgs) = _w4a4_layer(E_, T, zipf)
    hd = torch.from_numpy(h).to(torch.bfloat16).cuda()
    out = nv.moe_route_topk(hd, torch.from_numpy(wr).to(torch.bfloat16).cuda(), K_TOP,
                            logit_bias=None if bias is None else torch.from_numpy(bias).cuda())
    R = T * K_TOP
    a = nv.moe_grouped_linear(hd, out["expert_offsets"], gc, gsc, ggs, R, perm_tok=out["perm_tok"], gather=True,
                              w_sf_layout=nv.SF_TILED, epilogue=nv.EPI_SWIGLU, y_dtype=torch.bfloat16,
                              mode=nv.MODE_W4A4)
    y = nv.moe_grouped_linear(a, out["expert_offsets"], dc, dsc, dgs, R, gather=False, w_sf_layout=nv.SF_TILED,
                              epilogue=nv.EPI_COMBINE, topk_w=out["topk_w"], row_of=out["row_of"], k=K_TOP,
                              y_dtype=torch.float32, mode=nv.MODE_W4A4)
    torch.cuda.synchronize()
    assert nv.nvfp4_read_device_status() == nv.OK
    g = {k2: v.cpu().numpy() for k2, v in out.items()}
    a_np = a.float().cpu().numpy()
    y_np = y.cpu().numpy()
    off, pt, row_of, tw = g["expert_offsets"], g["perm_tok"], g["row_of"], g["topk_w"].astype(np.float64)
    expert_of_row = np.searchsorted(off, np.arange(R), side="right") - 1
    toks = np.sort(np.random.default_rng(5).choice(T, 24, replace=False))
    gs_h = oracle.global_scale(h)
    gs_a = oracle.global_scale(a_np)
    q_gu, q_dn = {}, {}
    for t in toks:
        for j in range(K_TOP):
            r = int(row_of[t, j])
            e = int(expert_of_row[r])
            if e not in q_gu:
                q_gu[e] = oracle.quantize(gu_f[e])
                q_dn[e] = oracle.quantize(dn_f[e])
            # stage 1: gate/up (W4A4 on the gathered, quantized hidden state) + SwiGLU
            xq = oracle.quantize(h[pt[r]:pt[r] + 1], gs=gs_h)
            gu, gu_ad = oracle.linear_w4a4(xq, q_gu[e])
            ref_a = omoe.swiglu(gu)[0]
            gg, uu = gu[0, :I], gu[0, I:]
            sig = 1.0 / (1.0 + np.exp(-gg))
            dg, du = 1e-4 * gu_ad[0, :I] + 1e-6, 1e-4 * gu_ad[0, I:] + 1e-6
            bound = (np.abs(uu) * np.abs(sig * (1 + gg * (1 - sig))) * dg + np.abs(gg * sig) * du + dg * du
                     + 1e-5 * np.abs(ref_a) + 1e-6 + bf16_ulp(ref_a))
            err = np.abs(a_np[r] - ref_a)
            assert (err <= bound).all(), f"swiglu row {r}: max ratio {np.max(err / bound)}"
        # stage 2: down projection of the GPU's own a, then the weighted combine
        ref_y = np.zeros(H)
        ref_b = np.zeros(H)
        for j in range(K_TOP):
            r = int(row_of[t, j])
            e = int(expert_of_row[r])
            aq = oracle.quantize(a_np[r:r + 1], gs=gs_a)
            d, d_ad = oracle.linear_w4a4(aq, q_dn[e])
            ref_y += tw[t, j] * d[0]
            ref_b += abs(tw[t, j]) * d_ad[0]
        assert_within_bound(y_np[t], ref_y, ref_b, False, f"down+combine token {t}")
