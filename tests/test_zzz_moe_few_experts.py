"""Grouped W4A16 expert layer with few experts (8 experts, 32 tokens, top-4:
16 rows per expert on average), so each grouped projection takes two
activation rows per pass.  Stage-wise parity against the oracle as in
test_gpu_moe.py (each stage on the GPU's own input to it)."""
import numpy as np
import pytest
import torch

import bit_linear_moe_b200 as nv
import oracle
from oracle import moe as omoe
from bit_linear_moe_b200 import synth
from nvfp4_checks import assert_within_bound, bf16_ulp

pytestmark = pytest.mark.gpu
H, I = synth.MOE_H, synth.MOE_I


def test_expert_layer_w4a16_few_experts():
    """8 experts, 32 tokens, top-4: 16 rows per expert on average, so each
    grouped projection takes two activation rows per pass (the many-rows
    configuration of both the SwiGLU and the short-K down kernels)."""
    Es, T, k = 8, 32, 4
    rng = np.random.default_rng(77)
    h = synth.moe_hidden(T)
    wr = synth.to_bf16((0.05 * rng.standard_normal((Es, H))).astype(np.float32))
    out = nv.moe_route_topk(torch.from_numpy(h).to(torch.bfloat16).cuda(),
                            torch.from_numpy(wr).to(torch.bfloat16).cuda(), k)
    torch.cuda.synchronize()
    off = out["expert_offsets"].cpu().numpy()
    pt = out["perm_tok"].cpu().numpy()
    R = T * k
    gu_q = [oracle.quantize(synth.moe_expert(e)[0]) for e in range(Es)]
    dn_q = [oracle.quantize(synth.moe_expert(e)[1]) for e in range(Es)]

    def stack(qs):
        return (torch.from_numpy(np.stack([q[0] for q in qs])).cuda(),
                torch.from_numpy(np.stack([q[1] for q in qs]).reshape(-1)).cuda(),
                torch.from_numpy(np.array([q[2] for q in qs], np.float32)).cuda())

    gc, gsc, ggs = stack(gu_q)
    hd = torch.from_numpy(h).to(torch.bfloat16).cuda()
    a = nv.moe_grouped_linear(hd, out["expert_offsets"], gc, gsc, ggs, R, perm_tok=out["perm_tok"], gather=True,
                              epilogue=nv.EPI_SWIGLU, y_dtype=torch.bfloat16, mode=nv.MODE_W4A16)
    torch.cuda.synchronize()
    wc = np.stack([q[0] for q in gu_q]); ws = np.stack([q[1] for q in gu_q])
    wg = np.array([q[2] for q in gu_q], np.float32)
    gu, gu_ad = omoe.grouped_linear_w4a16(h, off, pt, wc, ws, wg, gather=True)
    ref_a = omoe.swiglu(gu)
    gg, uu = gu[:, :I], gu[:, I:]
    sig = 1.0 / (1.0 + np.exp(-gg))
    dg, du = 1e-4 * gu_ad[:, :I] + 1e-6, 1e-4 * gu_ad[:, I:] + 1e-6
    bound = (np.abs(uu) * np.abs(sig * (1 + gg * (1 - sig))) * dg + np.abs(gg * sig) * du + dg * du
             + 1e-5 * np.abs(ref_a) + 1e-6 + bf16_ulp(ref_a))
    a_np = a.float().cpu().numpy()
    assert (np.abs(a_np - ref_a) <= bound).all(), "swiglu stage, few experts"
    dc, dsc, dgs = stack(dn_q)
    d = nv.moe_grouped_linear(a, out["expert_offsets"], dc, dsc, dgs, R, gather=False, y_dtype=torch.float32,
                              mode=nv.MODE_W4A16)
    torch.cuda.synchronize()
    dref, d_ad = omoe.grouped_linear_w4a16(a_np, off, pt, np.stack([q[0] for q in dn_q]),
                                          np.stack([q[1] for q in dn_q]), np.array([q[2] for q in dn_q], np.float32),
                                          gather=False)
    assert_within_bound(d, dref, d_ad, False, "down stage, few experts")
