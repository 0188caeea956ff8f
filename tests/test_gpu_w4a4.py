"""GPU W4A4 (tcgen05 block-scaled) linear vs the CPU oracle.

The oracle quantizes the activations itself (per-tensor gs from the whole
activation tensor, then per-16 E4M3 scales and E2M1 codes) and computes the
fp64 dot products of the two dequantized operands.  Bound: |y - ref| <=
1e-4 * sum_k |xq_k w_k| + 1e-6 (+ one bf16 rounding of ref for bf16 output).
Large shapes are checked on seeded row and column samples; the sampled rows
are quantized with the full tensor's gs, which is exact because quantization
is row-local once gs is fixed.
"""
import functools

import numpy as np
import pytest
import torch

import bit_linear_moe_b200 as nv
import oracle
from bit_linear_moe_b200 import synth
from nvfp4_checks import assert_within_bound, rowmajor_to_tiled, tiled_to_rowmajor

pytestmark = pytest.mark.gpu


def _upload_w(q, N, K):
    codes, scales, gs = q
    return (torch.from_numpy(np.ascontiguousarray(codes)).cuda(),
            torch.from_numpy(rowmajor_to_tiled(scales, N, K)).cuda(),
            torch.tensor([gs], dtype=torch.float32, device="cuda"))


def _gpu(x_np, wq, y_dtype):
    N, K = wq[0].shape[0], wq[0].shape[1] * 2
    c, s, g = _upload_w(wq, N, K)
    x = torch.from_numpy(x_np).to(torch.bfloat16).cuda()
    y = nv.nvfp4_linear(x, c, s, g, w_sf_layout=nv.SF_TILED, y_dtype=y_dtype, mode=nv.MODE_W4A4)
    torch.cuda.synchronize()
    return y.float().cpu().numpy()


def _ref(x_np, wq, rows=None, cols=None):
    gs_x = oracle.global_scale(x_np)
    xs = x_np if rows is None else x_np[rows]
    xq = oracle.quantize(xs, gs=gs_x)
    if cols is not None:
        wq = (wq[0][cols], wq[1][cols], wq[2])
    return oracle.linear_w4a4(xq, wq)


@pytest.mark.parametrize("M,K,N", [(1, 256, 128), (37, 512, 130), (128, 256, 256), (200, 1024, 64),
                                   (129, 768, 300), (256, 2048, 512)])
@pytest.mark.parametrize("y_dtype", [torch.float32, torch.bfloat16])
def test_small_and_ragged(M, K, N, y_dtype):
    rng = np.random.default_rng(M + K + N)
    wq = oracle.quantize(synth.weight(rng, N, K))
    x = synth.activations(rng, M, K)
    y = _gpu(x, wq, y_dtype)
    ref, ad = _ref(x, wq)
    assert_within_bound(y, ref, ad, y_dtype == torch.bfloat16, f"w4a4 {M}x{K}x{N}")


def test_outlier_columns_small():
    x, cols = synth.prefill_x(2, 256, 1024)
    wq = oracle.quantize(synth.weight(np.random.default_rng(3), 256, 1024))
    y = _gpu(x, wq, torch.float32)
    ref, ad = _ref(x, wq)
    assert_within_bound(y, ref, ad, False, "w4a4 outliers")


@functools.lru_cache(maxsize=1)
def _dense_q(seed, K, N):
    return oracle.quantize(synth.dense_weight(seed, K, N))


def _ws_activations(ws, M, K):
    """The quantized activations a W4A4 nvfp4_linear call leaves in its workspace."""
    lay = nv.nvfp4_linear_w4a4_ws_layout(M, K)
    b = ws.cpu().numpy()
    gs = b[lay["gs_x"]:lay["gs_x"] + 4].view(np.float32)[0]
    codes = b[lay["codes"]:lay["codes"] + M * K // 2].reshape(M, K // 2)
    sc = b[lay["scales"]:lay["scales"] + nv.nvfp4_scales_bytes(M, K, nv.SF_TILED)]
    return gs, codes, tiled_to_rowmajor(sc, M, K)


@pytest.mark.parametrize("M", synth.PREFILL_M)
@pytest.mark.parametrize("name,K,N,seed", synth.DENSE27B)
def test_prefill_shapes(name, K, N, seed, M):
    """The prefill configurations on every 27B-shaped linear.  The activation
    codes, scales and gs that nvfp4_linear quantizes into its workspace are
    compared with the oracle's in full (bit-exact); the output on 256 seeded
    rows x all N and on all M x 64 seeded columns."""
    wq = _dense_q(seed, K, N)
    x, _ = synth.prefill_x(seed, M, K)
    c, s, g = _upload_w(wq, N, K)
    xd = torch.from_numpy(x).to(torch.bfloat16).cuda()
    ws = torch.empty(int(nv.lib().nvfp4_linear_workspace(M, K, N, nv.MODE_W4A4)), dtype=torch.uint8,
                     device="cuda")
    y = nv.nvfp4_linear(xd, c, s, g, w_sf_layout=nv.SF_TILED, y_dtype=torch.bfloat16, mode=nv.MODE_W4A4, ws=ws)
    torch.cuda.synchronize()
    assert nv.nvfp4_read_device_status() == nv.OK
    del c, s, g, xd
    gs_w, codes_w, sc_w = _ws_activations(ws, M, K)
    del ws
    xq = oracle.quantize(x)
    assert gs_w == xq[2], f"{name} M={M}: gs_x {gs_w!r} != {xq[2]!r}"
    assert np.array_equal(codes_w, xq[0]), f"{name} M={M}: {(codes_w != xq[0]).sum()} activation code bytes differ"
    assert np.array_equal(sc_w, xq[1]), f"{name} M={M}: {(sc_w != xq[1]).sum()} activation scales differ"
    y = y.float().cpu().numpy()
    rng = np.random.default_rng([seed, M, 7])
    rows = np.sort(rng.choice(M, min(M, 256), replace=False))
    cols = np.sort(rng.choice(N, 64, replace=False))
    ref, ad = oracle.linear_w4a4((xq[0][rows], xq[1][rows], xq[2]), wq)
    assert_within_bound(y[rows], ref, ad, True, f"{name} M={M} sampled rows")
    ref, ad = oracle.linear_w4a4(xq, (wq[0][cols], wq[1][cols], wq[2]))
    assert_within_bound(y[:, cols], ref, ad, True, f"{name} M={M} sampled cols")
