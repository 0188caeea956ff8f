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
