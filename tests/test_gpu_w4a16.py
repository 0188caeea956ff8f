"""GPU W4A16 linear vs the CPU oracle, within |y-ref| <= 1e-4 sum|x w| + 1e-6
(+ one bf16 rounding of ref for bf16 outputs).  Weights are quantized by the
oracle and uploaded; activations are bf16."""
import functools

import numpy as np
import pytest
import torch

import bit_linear_moe_b200 as nv
import oracle
from bit_linear_moe_b200 import synth
from nvfp4_checks import assert_within_bound, rowmajor_to_tiled

pytestmark = pytest.mark.gpu


def _upload(q, layout, rows, cols):
    codes, scales, gs = q
    s = scales if layout == nv.SF_ROWMAJOR else rowmajor_to_tiled(scales, rows, cols)
    return (torch.from_numpy(np.ascontiguousarray(codes)).cuda(),
            torch.from_numpy(np.ascontiguousarray(s).ravel()).cuda(),
            torch.tensor([gs], dtype=torch.float32, device="cuda"))


def _run(x_np, q, layout, y_dtype):
    N, K = q[0].shape[0], q[0].shape[1] * 2
    c, s, g = _upload(q, layout, N, K)
    x = torch.from_numpy(x_np).to(torch.bfloat16).cuda()
    y = nv.nvfp4_linear(x, c, s, g, w_sf_layout=layout, y_dtype=y_dtype, mode=nv.MODE_W4A16)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("y_dtype", [torch.float32, torch.bfloat16])
def test_single_2048(y_dtype):
    w, x = synth.single(0)
    q = oracle.quantize(w)
    ref, ad = oracle.linear_w4a16(x, *q)
    for layout in (nv.SF_ROWMAJOR, nv.SF_TILED):
        y = _run(x, q, layout, y_dtype)
        assert_within_bound(y, ref, ad, y_dtype == torch.bfloat16, "single 2048")


@functools.lru_cache(maxsize=1)
def _dense_q(seed, K, N):
    return oracle.quantize(synth.dense_weight(seed, K, N))


@pytest.mark.parametrize("name,K,N,seed", synth.DENSE27B)
@pytest.mark.parametrize("M", synth.DECODE_M)
def test_dense27b_decode(name, K, N, seed, M):
    q = _dense_q(seed, K, N)
    x = synth.decode_x(seed, M, K)
    ref, ad = oracle.linear_w4a16(x, *q)
    layout = nv.SF_ROWMAJOR if M == 2 else nv.SF_TILED
    y = _run(x, q, layout, torch.float32)
    assert_within_bound(y, ref, ad, False, f"{name} M={M}")
    if M == 1:
        y = _run(x, q, layout, torch.bfloat16)
        assert_within_bound(y, ref, ad, True, f"{name} M={M} bf16")


@pytest.mark.parametrize("M,K,N", [(1, 16, 1), (3, 48, 3), (5, 80, 130), (2, 4096, 257), (7, 1040, 1000),
                                   (33, 256, 64), (1, 17408, 8), (4, 32, 2048), (1, 256, 19277), (2, 512, 37000),
                                   (1, 256, 40000), (2, 512, 60000)])
@pytest.mark.parametrize("layout", [nv.SF_ROWMAJOR, nv.SF_TILED])
def test_ragged(M, K, N, layout):
    rng = np.random.default_rng(M * 1000 + K + N)
    q = oracle.quantize(synth.weight(rng, N, K))
    x = synth.activations(rng, M, K)
    ref, ad = oracle.linear_w4a16(x, *q)
    y = _run(x, q, layout, torch.float32)
    assert_within_bound(y, ref, ad, False, f"ragged {M}x{K}x{N}")


def test_degenerate_weights():
    rng = np.random.default_rng(3)
    K, N = 256, 64
    x = synth.activations(rng, 2, K)
    q = oracle.quantize(np.zeros((N, K), np.float32))
    y = _run(x, q, nv.SF_ROWMAJOR, torch.float32)
    assert not y.any()
    codes = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, K // 16), np.uint8)
    codes[5, 9] = 0x70                       # element 19 of row 5 = E2M1 code 7 (6.0)
    scales[5, 1] = 0x38                      # 1.0
    y = _run(x, (codes, scales, np.float32(0.5)), nv.SF_ROWMAJOR, torch.float32).cpu().numpy()
    assert y[0, 5] == np.float32(x[0, 19] * 6.0 * 0.5) and y[1, 5] == np.float32(x[1, 19] * 3.0)
    assert np.count_nonzero(y) == 2


@pytest.mark.parametrize("M,K,N", [(5, 256, 128), (8, 512, 200), (13, 1024, 1000), (16, 256, 64), (17, 768, 130),
                                   (32, 5120, 256), (24, 2048, 384), (33, 256, 64), (48, 1024, 300),
                                   (64, 5120, 256), (64, 768, 130)])
def test_tensor_core_widths(M, K, N):
    """Widths 5..64 with tensor-core scales run the tensor-memory kernel."""
    rng = np.random.default_rng(M * 7 + K + N)
    q = oracle.quantize(synth.weight(rng, N, K))
    x = synth.activations(rng, M, K)
    ref, ad = oracle.linear_w4a16(x, *q)
    for y_dtype in (torch.float32, torch.bfloat16):
        y = _run(x, q, nv.SF_TILED, y_dtype)
        assert_within_bound(y, ref, ad, y_dtype == torch.bfloat16, f"tc {M}x{K}x{N}")


@pytest.mark.parametrize("name,K,N,seed", synth.DENSE27B)
def test_dense27b_verify_width_64(name, K, N, seed):
    """The widest speculative-verify width (64 tokens) on the 27B-shaped
    linears, W4A16, every output checked."""
    M = 64
    q = _dense_q(seed, K, N)
    x = synth.decode_x(seed, M, K)
    ref, ad = oracle.linear_w4a16(x, *q)
    y = _run(x, q, nv.SF_TILED, torch.bfloat16)
    assert_within_bound(y, ref, ad, True, f"{name} M={M}")
