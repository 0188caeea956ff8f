"""The persistent chain of W4A16 decode linears (nvfp4_chain) against the
oracle.  Independent ops are checked like single linears.  Ops that read an
earlier op's output are checked stage by stage: the reference input is the
oracle's glue (rms / silu * up, rounded to bf16) applied to the GPU's own
output of the source op; because the GPU's glue sums in fp32 in another order,
its bf16 input may differ from the reference by one bf16 step per element, so
the bound adds sum_k ulp_bf16(x_k) |w_k| to 1e-4 sum_k |x_k w_k| + 1e-6."""
import functools

import numpy as np
import pytest
import torch

import bit_linear_moe_b200 as nv
import oracle
from oracle import stack as ost
from bit_linear_moe_b200 import synth
from nvfp4_checks import assert_within_bound, bf16_ulp, rowmajor_to_tiled

pytestmark = pytest.mark.gpu


@functools.lru_cache(maxsize=4)
def _dense_q(seed, K, N):
    return oracle.quantize(synth.dense_weight(seed, K, N))


def _upload(q):
    c, s, g = q
    N, K = c.shape[0], c.shape[1] * 2
    return (torch.from_numpy(np.ascontiguousarray(c)).cuda(),
            torch.from_numpy(rowmajor_to_tiled(s, N, K)).cuda(),
            torch.tensor([g], dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("M", [1, 2])
def test_chain_independent_27b(M):
    """The four 27B-shaped linears as independent ops of one call (the decode
    step of the benchmark), each against the oracle; two calls agree bitwise."""
    specs, refs = [], []
    for name, K, N, seed in synth.DENSE27B:
        q = _dense_q(seed, K, N)
        x = synth.decode_x(seed, M, K)
        specs.append({"w": _upload(q), "src": torch.from_numpy(x).to(torch.bfloat16).cuda(),
                      "y": torch.empty((M, N), dtype=torch.float32, device="cuda")})
        refs.append(oracle.linear_w4a16(x, *q))
    nv.nvfp4_chain(specs, M)
    first = [sp["y"].clone() for sp in specs]
    nv.nvfp4_chain(specs, M)
    torch.cuda.synchronize()
    assert nv.nvfp4_read_device_status() == nv.OK
    for sp, f, (ref, ad), (name, *_ ) in zip(specs, first, refs, synth.DENSE27B):
        assert torch.equal(sp["y"], f), f"{name}: two calls differ"
        assert_within_bound(sp["y"], ref, ad, False, f"chain {name} M={M}")


@pytest.mark.parametrize("M,K,N", [(1, 256, 8), (2, 768, 200), (1, 6144, 136), (2, 7168, 64)])
def test_chain_ragged_single(M, K, N):
    """One op: ragged row tiles, one stage, slices at the shared-memory limit."""
    rng = np.random.default_rng(M * 7 + K + N)
    q = oracle.quantize(synth.weight(rng, N, K))
    x = synth.activations(rng, M, K)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_chain([{"w": _upload(q), "src": torch.from_numpy(x).to(torch.bfloat16).cuda(), "y": y}], M)
    torch.cuda.synchronize()
    ref, ad = oracle.linear_w4a16(x, *q)
    assert_within_bound(y, ref, ad, True, f"chain single {M}x{K}x{N}")


def _glue_ref(v, xform, K):
    if xform == nv.CHAIN_XFORM_RMS:
        return ost.rms_norm(v[:, :K])
    if xform == nv.CHAIN_XFORM_SILU_MUL:
        return ost.silu_mul(v)
    return ost.bf16_round(v)


def _check_op(y_gpu, x_ref, q, what):
    ref, ad = oracle.linear_w4a16(x_ref, *q)
    _, ulp_ad = oracle.linear_w4a16(bf16_ulp(x_ref).astype(np.float32), *q)
    assert_within_bound(y_gpu, ref, ad + ulp_ad, False, what)


def _stack_specs(layers_q, x0_dev, M):
    """The stack's op list: per layer QKV (x), O (rms of the Q slice), GU (rms),
    Down (silu * up); every op returns its raw output as fp32."""
    specs = []
    kq = synth.DENSE27B[0][1]
    for li, wq in enumerate(layers_q):
        base = len(specs)
        first = x0_dev if li == 0 else base - 1
        for j, (name, K, N, _) in enumerate(synth.DENSE27B):
            if j == 0:
                src, xf = first, (nv.CHAIN_XFORM_NONE if li == 0 else nv.CHAIN_XFORM_RMS)
            elif j == 3:
                src, xf = base + 2, nv.CHAIN_XFORM_SILU_MUL
            else:
                src, xf = base + j - 1, nv.CHAIN_XFORM_RMS
            specs.append({"w": wq[name], "src": src, "xform": xf,
                          "y": torch.empty((M, N), dtype=torch.float32, device="cuda")})
    return specs


@pytest.mark.parametrize("M", [1, 2])
def test_chain_stack_27b(M):
    """Four stack layers at the 27B shapes in one call (16 ops, two launches):
    every op stage by stage; the last op's rms output in bf16."""
    L = 4
    gen = torch.Generator(device="cuda")
    layers_q, layers_dev = [], []
    for li in range(L):
        lq, ld = {}, {}
        for j, (name, K, N, _) in enumerate(synth.DENSE27B):
            w = synth.weight(np.random.default_rng([500 + li, j]), N, K)
            q = oracle.quantize(w)
            lq[name] = q
            ld[name] = _upload(q)
        layers_q.append(lq)
        layers_dev.append(ld)
    x0 = ost.rms_norm(np.random.default_rng([500, M]).standard_normal((M, synth.DENSE27B[0][1])).astype(np.float32))
    x0d = torch.from_numpy(x0).to(torch.bfloat16).cuda()
    specs = _stack_specs(layers_dev, x0d, M)
    nv.nvfp4_chain(specs, M)
    torch.cuda.synchronize()
    assert nv.nvfp4_read_device_status() == nv.OK
    outs = [sp["y"].cpu().numpy().astype(np.float64) for sp in specs]
    for i, sp in enumerate(specs):
        li, j = divmod(i, 4)
        name, K, N, _ = synth.DENSE27B[j]
        if isinstance(sp["src"], torch.Tensor):
            x_ref = x0
        else:
            x_ref = _glue_ref(outs[sp["src"]], sp["xform"], K)
        _check_op(outs[i], x_ref, layers_q[li][name], f"layer {li} {name}")
    # the stack output: rms of the last op, bf16, from a second call
    x_out = torch.empty((M, synth.DENSE27B[3][2]), dtype=torch.bfloat16, device="cuda")
    specs[-1]["y"], specs[-1]["y_xform"] = x_out, nv.CHAIN_XFORM_RMS
    nv.nvfp4_chain(specs, M)
    torch.cuda.synchronize()
    got = x_out.float().cpu().numpy()
    ref = ost.rms_norm(outs[-1])
    err = np.abs(got.astype(np.float64) - ref)
    assert (err <= bf16_ulp(ref) + 1e-30).all(), "stack output off by more than one bf16 step"
