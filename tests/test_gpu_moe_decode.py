"""The fused decode-time expert layer (moe_layer_decode, T <= 32) against the
oracle, stage by stage: routing (logits within the linear bound, top-k bit-exact
on the GPU's own logits), the gate/up + SwiGLU rows a on the GPU's routing, and
the down projection + weighted combine y on the GPU's own a and weights."""
import numpy as np
import pytest
import torch

import bit_linear_moe_b200 as nv
import oracle
from oracle import moe as omoe
from bit_linear_moe_b200 import synth
from moe_fixtures import moe512_device, moe512_q, quantize_experts, stack_tiled, swiglu_bound
from nvfp4_checks import assert_within_bound

pytestmark = pytest.mark.gpu


def _check_layer(h, wr, bias, k, gu_q, dn_q, gu_d, dn_d, y_dtype=torch.float32):
    T, H = h.shape
    E = wr.shape[0]
    I = gu_q[0][0].shape[0] // 2
    hd = torch.from_numpy(h).to(torch.bfloat16).cuda()
    wd = torch.from_numpy(wr).to(torch.bfloat16).cuda()
    bd = None if bias is None else torch.from_numpy(bias).cuda()
    y, ex = nv.moe_layer_decode(hd, wd, k, gu_d, dn_d, logit_bias=bd, y_dtype=y_dtype, want_logits=True,
                                want_routing=True, want_a=True)
    y2 = nv.moe_layer_decode(hd, wd, k, gu_d, dn_d, logit_bias=bd, y_dtype=y_dtype)
    torch.cuda.synchronize()
    assert nv.nvfp4_read_device_status() == nv.OK
    assert torch.equal(y, y2), "the layer is not bitwise reproducible"
    g = {n: v.float().cpu().numpy() if v.dtype == torch.bfloat16 else v.cpu().numpy() for n, v in ex.items()}
    # routing
    ref_l = omoe.router_logits(h, wr, bias)
    absdot = np.abs(h.astype(np.float64)) @ np.abs(wr.astype(np.float64)).T
    assert_within_bound(g["logits"], ref_l, absdot, False, "router logits")
    idx, w = omoe.topk(g["logits"].astype(np.float64), k)
    assert np.array_equal(g["topk_idx"], idx), "top-k differs from the oracle's on the GPU's logits"
    assert np.allclose(g["topk_w"], w, rtol=2e-6, atol=1e-7)
    # gate/up + SwiGLU, row t * k + j, on the GPU's routing
    a = g["a"]
    for e in np.unique(idx):
        tj = np.argwhere(idx == e)
        rows = tj[:, 0] * k + tj[:, 1]
        gu, gu_ad = oracle.linear_w4a16(h[tj[:, 0]], *gu_q[e])
        ref_a = omoe.swiglu(gu)
        err = np.abs(a[rows] - ref_a)
        bound = swiglu_bound(gu, gu_ad, ref_a)
        assert (err <= bound).all(), f"swiglu expert {e}: max ratio {np.max(err / bound)}"
    # down + combine on the GPU's own a
    d = np.zeros((T * k, H))
    d_ad = np.zeros((T * k, H))
    for e in np.unique(idx):
        tj = np.argwhere(idx == e)
        rows = tj[:, 0] * k + tj[:, 1]
        d[rows], d_ad[rows] = oracle.linear_w4a16(a[rows], *dn_q[e])
    tw = g["topk_w"].astype(np.float64)
    ref_y = np.einsum("tj,tjn->tn", tw, d.reshape(T, k, H))
    bnd = np.einsum("tj,tjn->tn", np.abs(tw), d_ad.reshape(T, k, H))
    assert_within_bound(y, ref_y, bnd, y_dtype == torch.bfloat16, "down + combine")
    return int(len(np.unique(idx)))


@pytest.mark.parametrize("T", [1, 32])
@pytest.mark.parametrize("zipf", [False, True])
def test_moe_layer_decode_512_experts(T, zipf):
    """The 512-expert, top-10 layer at the decode batch sizes, uniform and
    Zipf-skewed routing."""
    gu_q, dn_q = moe512_q()
    gu_d, dn_d = moe512_device()
    h = synth.moe_hidden(T)
    bias = synth.moe_zipf_bias() if zipf else None
    n = _check_layer(h, synth.moe_router(), bias, synth.MOE_K, gu_q, dn_q, gu_d, dn_d)
    print(f"T={T} zipf={zipf}: {n} experts touched")


@pytest.mark.parametrize("T,E,k,H,I,y_bf16", [(5, 16, 4, 512, 256, False), (32, 16, 4, 512, 256, True),
                                               (17, 40, 6, 768, 512, False), (32, 8, 8, 256, 256, False),
                                               (3, 1024, 2, 256, 256, True)])
def test_moe_layer_decode_shapes(T, E, k, H, I, y_bf16):
    """Ragged token counts; few experts, so most experts hold 4+ tokens (groups
    of four, several groups per expert: the hot-expert path); every token on
    every expert (k = E = 8); E = 1024."""
    rng = np.random.default_rng(T * 1000 + E)
    wr = synth.to_bf16(0.05 * rng.standard_normal((E, H)))
    h = synth.activations(rng, T, H)
    bias = (0.1 * rng.standard_normal(E)).astype(np.float32)
    gu_q = quantize_experts([synth.weight(np.random.default_rng([T, E, 1, e]), 2 * I, H) for e in range(E)])
    dn_q = quantize_experts([synth.weight(np.random.default_rng([T, E, 2, e]), H, I) for e in range(E)])
    _check_layer(h, wr, bias, k, gu_q, dn_q, stack_tiled(gu_q), stack_tiled(dn_q),
                 torch.bfloat16 if y_bf16 else torch.float32)


def test_moe_layer_decode_matches_unfused_routing():
    """The fused layer routes exactly as moe_route_topk does (same logits kernel
    for T <= 64, same top-k order)."""
    T = 32
    h = torch.from_numpy(synth.moe_hidden(T)).to(torch.bfloat16).cuda()
    wr = torch.from_numpy(synth.moe_router()).to(torch.bfloat16).cuda()
    gu_d, dn_d = moe512_device()
    _, ex = nv.moe_layer_decode(h, wr, synth.MOE_K, gu_d, dn_d, want_logits=True, want_routing=True)
    r = nv.moe_route_topk(h, wr, synth.MOE_K, want_logits=True)
    torch.cuda.synchronize()
    assert torch.equal(ex["logits"], r["logits"])
    assert torch.equal(ex["topk_idx"], r["topk_idx"])
    assert torch.equal(ex["topk_w"], r["topk_w"])
