"""Expert weights for the mixture-of-experts parity tests, quantized by the
oracle (test-side only; the arithmetic is the oracle's).  Both sides get the
same bytes: the oracle's codes and scales, uploaded with the scales rearranged
into the tensor-core layout by the index map of include/nvfp4.h."""
import functools
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
from bit_linear_moe_b200 import synth
from nvfp4_checks import rowmajor_to_tiled


def quantize_experts(ws_f, workers=8):
    """Oracle-quantize a list of weight matrices (threads: the C oracle releases the GIL)."""
    with ThreadPoolExecutor(workers) as ex:
        return list(ex.map(lambda w: oracle.quantize(w), ws_f))


def stack_tiled(qs):
    """Stacked [E, N, K/2] codes, per-expert TILED scale blocks and gs [E] on the device."""
    N, K = qs[0][0].shape[0], qs[0][0].shape[1] * 2
    codes = np.stack([q[0] for q in qs])
    scales = np.concatenate([rowmajor_to_tiled(q[1], N, K) for q in qs])
    gs = np.array([q[2] for q in qs], dtype=np.float32)
    return (torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), torch.from_numpy(gs).cuda())


@functools.lru_cache(maxsize=1)
def moe512_q():
    """The 512-expert layer's weights (synth.moe_expert, seed 10), quantized by
    the oracle: (gate/up list, down list) of (codes, row-major scales, gs)."""
    with ThreadPoolExecutor(8) as ex:
        w = list(ex.map(synth.moe_expert, range(synth.MOE_E)))
    gu = quantize_experts([a for a, _ in w])
    dn = quantize_experts([b for _, b in w])
    return gu, dn


@functools.lru_cache(maxsize=1)
def moe512_device():
    """moe512_q() stacked on the device: ((codes, scales, gs) gate/up, same for down)."""
    gu, dn = moe512_q()
    return stack_tiled(gu), stack_tiled(dn)


def swiglu_bound(gu, gu_ad, ref_a):
    """Bound of the SwiGLU stage: the gate/up output bound (1e-4 * sum|x w| +
    1e-6 per element) carried to first order through silu(g) * u, plus the
    stage's own 1e-5 relative slack and one bf16 rounding of the output."""
    from nvfp4_checks import bf16_ulp
    I = gu.shape[1] // 2
    gg, uu = gu[:, :I], gu[:, I:]
    sig = 1.0 / (1.0 + np.exp(-gg))
    dg, du = 1e-4 * gu_ad[:, :I] + 1e-6, 1e-4 * gu_ad[:, I:] + 1e-6
    return (np.abs(uu) * np.abs(sig * (1 + gg * (1 - sig))) * dg + np.abs(gg * sig) * du + dg * du
            + 1e-5 * np.abs(ref_a) + 1e-6 + bf16_ulp(ref_a))
