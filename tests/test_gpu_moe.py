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
from moe_fixtures import moe512_q, quantize_experts, stack_tiled, swiglu_bound
from nvfp4_checks import assert_within_bound, bf16_ulp, tiled_to_rowmajor

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

def _grouped_ws_activations(ws, R, K, N, E_, epi):
    lay = nv.moe_grouped_linear_w4a4_ws_layout(R, K, N, E_, K_TOP, epi)
    b = ws.cpu().numpy()
    rp = lay["rows_pad"]
    gs = b[lay["gs_x"]:lay["gs_x"] + 4].view(np.float32)[0]
    pad_off = b[lay["pad_off"]:lay["pad_off"] + 4 * (E_ + 1)].view(np.int32).copy()
    src = b[lay["src_rows"]:lay["src_rows"] + 4 * rp].view(np.int32).copy()
    codes = b[lay["codes"]:lay["codes"] + rp * K // 2].reshape(rp, K // 2).copy()
    sc = tiled_to_rowmajor(b[lay["scales"]:lay["scales"] + nv.nvfp4_scales_bytes(rp, K, nv.SF_TILED)], rp, K)
    return gs, pad_off, src, codes, sc


def _check_permuted_activations(ws, x_np, xd, R, K, N, E_, epi, off, perm_tok):
    """The padded, permuted activations a grouped W4A4 call quantized: the row
    map is each expert's rows padded to whole 128-row tiles; codes, scales and
    gs equal the oracle's quantization of the gathered rows (bit-exact, every
    row); and quantize(permute(x)) == permute(quantize(x)) on the GPU."""
    gs, pad_off, src, codes, sc = _grouped_ws_activations(ws, R, K, N, E_, epi)
    cnt = np.diff(off)
    want_pad = np.concatenate([[0], np.cumsum((cnt + 127) // 128 * 128)]).astype(np.int32)
    assert np.array_equal(pad_off, want_pad)
    used = int(want_pad[-1])
    want_src = np.full(used, -1, np.int32)
    for e in np.flatnonzero(cnt):
        rows = np.arange(off[e], off[e + 1])
        want_src[want_pad[e]:want_pad[e] + cnt[e]] = perm_tok[rows] if perm_tok is not None else rows
    assert np.array_equal(src[:used], want_src)
    real = want_src >= 0
    gathered = x_np[want_src[real]]
    q = oracle.quantize(gathered, gs=oracle.global_scale(gathered))
    assert gs == q[2], f"gs_x {gs!r} != {q[2]!r}"
    assert np.array_equal(codes[:used][real], q[0]), f"{(codes[:used][real] != q[0]).sum()} code bytes differ"
    assert np.array_equal(sc[:used][real], q[1]), f"{(sc[:used][real] != q[1]).sum()} scales differ"
    assert not codes[:used][~real].any() and not sc[:used][~real].any(), "padding rows must be zero"
    # the same identity on the GPU: the dense quantizer with the same gs, then the row map
    gsd = torch.tensor([gs], dtype=torch.float32, device="cuda")
    c_full, s_full, _ = nv.nvfp4_quantize(xd, gs_in=gsd, sf_layout=nv.SF_ROWMAJOR)
    torch.cuda.synchronize()
    c_full, s_full = c_full.cpu().numpy(), s_full.cpu().numpy().reshape(-1, K // 16)
    assert np.array_equal(codes[:used][real], c_full[want_src[real]])
    assert np.array_equal(sc[:used][real], s_full[want_src[real]])


def _check_w4a4_layer(E_, T, h, wr, bias, gu_q, dn_q, ntok, seed):
    """One W4A4 expert layer, stage by stage: the routed gate/up + SwiGLU, the
    down projection (bf16 rows, the NONE epilogue) and the weighted combine,
    each against the oracle on the GPU's own input to that stage; the permuted
    activations of both projections bit-exact; the combine deterministic."""
    R = T * K_TOP
    gc, gsc, ggs = stack_tiled(gu_q)
    dc, dsc, dgs = stack_tiled(dn_q)
    hd = torch.from_numpy(h).to(torch.bfloat16).cuda()
    out = nv.moe_route_topk(hd, torch.from_numpy(wr).to(torch.bfloat16).cuda(), K_TOP,
                            logit_bias=None if bias is None else torch.from_numpy(bias).cuda())
    ws1 = torch.empty(int(nv.lib().moe_grouped_linear_workspace(R, H, 2 * I, E_, K_TOP, nv.EPI_SWIGLU,
                                                                nv.MODE_W4A4)), dtype=torch.uint8, device="cuda")
    a = nv.moe_grouped_linear(hd, out["expert_offsets"], gc, gsc, ggs, R, perm_tok=out["perm_tok"], gather=True,
                              w_sf_layout=nv.SF_TILED, epilogue=nv.EPI_SWIGLU, y_dtype=torch.bfloat16,
                              mode=nv.MODE_W4A4, ws=ws1)
    ws2 = torch.empty(int(nv.lib().moe_grouped_linear_workspace(R, I, H, E_, K_TOP, nv.EPI_NONE, nv.MODE_W4A4)),
                      dtype=torch.uint8, device="cuda")
    d = nv.moe_grouped_linear(a, out["expert_offsets"], dc, dsc, dgs, R, gather=False, w_sf_layout=nv.SF_TILED,
                              epilogue=nv.EPI_NONE, y_dtype=torch.bfloat16, mode=nv.MODE_W4A4, ws=ws2)
    ys = [nv.moe_grouped_linear(a, out["expert_offsets"], dc, dsc, dgs, R, gather=False, w_sf_layout=nv.SF_TILED,
                                epilogue=nv.EPI_COMBINE, topk_w=out["topk_w"], row_of=out["row_of"], k=K_TOP,
                                y_dtype=torch.float32, mode=nv.MODE_W4A4) for _ in range(2)]
    yb = nv.moe_grouped_linear(a, out["expert_offsets"], dc, dsc, dgs, R, gather=False, w_sf_layout=nv.SF_TILED,
                               epilogue=nv.EPI_COMBINE, topk_w=out["topk_w"], row_of=out["row_of"], k=K_TOP,
                               y_dtype=torch.bfloat16, mode=nv.MODE_W4A4)
    torch.cuda.synchronize()
    assert nv.nvfp4_read_device_status() == nv.OK
    assert torch.equal(ys[0], ys[1]), "the combine is not bitwise reproducible"
    assert torch.equal(yb, ys[0].to(torch.bfloat16)), "bf16 combine != bf16(fp32 combine)"
    g = {k2: v.cpu().numpy() for k2, v in out.items()}
    off, pt, row_of, tw = g["expert_offsets"], g["perm_tok"], g["row_of"], g["topk_w"].astype(np.float64)
    a_np = a.float().cpu().numpy()
    d_np = d.float().cpu().numpy()
    y_np = ys[0].cpu().numpy()
    _check_permuted_activations(ws1, h, hd, R, H, 2 * I, E_, nv.EPI_SWIGLU, off, pt)
    _check_permuted_activations(ws2, a_np, a, R, I, H, E_, nv.EPI_NONE, off, None)
    del ws1, ws2
    # combine, every token, on the GPU's own bf16 expert rows
    ref_y, ref_b = omoe.combine(d_np, tw, row_of)
    assert_within_bound(y_np, ref_y, ref_b, False, "combine")
    # gate/up + SwiGLU and down on the rows of `ntok` seeded tokens, grouped by expert
    expert_of_row = np.searchsorted(off, np.arange(R), side="right") - 1
    toks = np.sort(np.random.default_rng(seed).choice(T, ntok, replace=False))
    rows = np.sort(row_of[toks].ravel())
    gs_h = oracle.global_scale(h)
    gs_a = oracle.global_scale(a_np)
    for e in np.unique(expert_of_row[rows]):
        re = rows[expert_of_row[rows] == e]
        gu, gu_ad = oracle.linear_w4a4(oracle.quantize(h[pt[re]], gs=gs_h), gu_q[e])
        ref_a = omoe.swiglu(gu)
        err = np.abs(a_np[re] - ref_a)
        bound = swiglu_bound(gu, gu_ad, ref_a)
        assert (err <= bound).all(), f"swiglu expert {e}: max ratio {np.max(err / bound)}"
        ref_d, d_ad = oracle.linear_w4a4(oracle.quantize(a_np[re], gs=gs_a), dn_q[e])
        assert_within_bound(d_np[re], ref_d, d_ad, True, f"down expert {e}")
    return int((np.diff(off) > 0).sum())


@pytest.mark.parametrize("zipf", [False, True])
def test_expert_layer_w4a4_64_experts(zipf):
    """A 64-expert layer with the 512-expert layer's per-expert shapes: about
    640 rows per expert, so most tiles are full."""
    E_, T, seed = 64, 4096, 20
    rng = np.random.default_rng(seed)
    wr = synth.to_bf16(0.02 * rng.standard_normal((E_, H)))
    h = synth.activations(np.random.default_rng([seed, T]), T, H)
    bias = (-1.1 * np.log(np.random.default_rng([seed, 1]).permutation(E_) + 1)).astype(np.float32) if zipf \
        else None
    gu_q = quantize_experts([synth.weight(np.random.default_rng([seed, 2, e]), 2 * I, H) for e in range(E_)])
    dn_q = quantize_experts([synth.weight(np.random.default_rng([seed, 3, e]), H, I) for e in range(E_)])
    _check_w4a4_layer(E_, T, h, wr, bias, gu_q, dn_q, 64, 5)


@pytest.mark.parametrize("zipf", [False, True])
def test_expert_layer_w4a4_512_experts_4096_tokens(zipf):
    """The 512-expert layer at 4,096 tokens (the W4A4 configuration): about 80
    rows per expert under uniform routing, so every expert's tile is partial
    and padding dominates; the Zipf run concentrates rows on a few experts.
    256 seeded tokens (2,560 rows) are checked stage by stage."""
    T = 4096
    gu_q, dn_q = moe512_q()
    h = synth.moe_hidden(T)
    bias = synth.moe_zipf_bias() if zipf else None
    touched = _check_w4a4_layer(E, T, h, _router(), bias, gu_q, dn_q, 256, 11)
    print(f"E=512 T=4096 zipf={zipf}: {touched} experts touched")
