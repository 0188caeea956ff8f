"""The calibrated quantizer on the GPU against the oracle.  The chosen alpha
is a decision taken on fp64 error sums that may differ in their last bits
between the two sides, so it is checked for validity (its oracle error is the
least one, to 1e-9 relative); everything downstream of it is checked bit for
bit: the channel scales, codes, scales and gs of the scaled weight."""
import numpy as np
import pytest
import torch

import bit_linear_moe_b200 as nv
import oracle
from oracle import calibrate as cal
from bit_linear_moe_b200 import synth
from nvfp4_checks import assert_within_bound, tiled_to_rowmajor

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,K,S,layout", [(96, 256, 32, nv.SF_ROWMAJOR), (512, 1024, 64, nv.SF_TILED),
                                          (5120, 5120, 128, nv.SF_TILED)])
def test_calibrate_matches_oracle(N, K, S, layout):
    rng = np.random.default_rng(N + K + S)
    w = synth.weight(rng, N, K)
    x, _ = synth.prefill_x(7, S, K)
    codes, scales, gs, col, err, aidx = nv.nvfp4_calibrate(torch.from_numpy(w).cuda(),
                                                           torch.from_numpy(x).to(torch.bfloat16).cuda(), layout)
    torch.cuda.synchronize()
    r = cal.calibrate(w, x)
    j = int(aidx.item())
    e_gpu = err.cpu().numpy().astype(np.float64)
    assert np.allclose(e_gpu, r["err"], rtol=1e-6), (e_gpu, r["err"])
    assert r["err"][j] <= r["err"].min() * (1 + 1e-9), f"alpha {j}/8 is not a least-error choice"
    assert np.array_equal(col.cpu().numpy(), r["scales_all"][j])
    q = r["qs"][j]
    sc = scales.cpu().numpy()
    sc = tiled_to_rowmajor(sc, N, K) if layout == nv.SF_TILED else sc.reshape(N, K // 16)
    assert np.array_equal(codes.cpu().numpy(), q[0])
    assert np.array_equal(sc, q[1])
    assert np.float32(gs.item()) == q[2]
    print(f"N={N} K={K}: alpha {j}/8, err {r['err'][j]:.4g} vs RTN {r['err'][0]:.4g}")


def test_calibrated_linear():
    """The calibrated weight on activations divided by the channel scales."""
    N, K, S, M = 256, 512, 64, 8
    rng = np.random.default_rng(11)
    w = synth.weight(rng, N, K)
    xc, _ = synth.prefill_x(8, S, K)
    codes, scales, gs, col, _, _ = nv.nvfp4_calibrate(torch.from_numpy(w).cuda(),
                                                      torch.from_numpy(xc).to(torch.bfloat16).cuda(), nv.SF_TILED)
    x, _ = synth.prefill_x(9, M, K)
    s = col.cpu().numpy()
    xs = synth.to_bf16((x / s[None, :]).astype(np.float32))
    y = nv.nvfp4_linear(torch.from_numpy(xs).to(torch.bfloat16).cuda(), codes, scales, gs,
                        w_sf_layout=nv.SF_TILED, mode=nv.MODE_W4A16)
    torch.cuda.synchronize()
    q = (codes.cpu().numpy(), tiled_to_rowmajor(scales.cpu().numpy(), N, K), np.float32(gs.item()))
    ref, ad = oracle.linear_w4a16(xs, *q)
    assert_within_bound(y, ref, ad, False, "calibrated linear")
