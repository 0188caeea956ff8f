"""The fused rms-renormalisation + quantization (nvfp4_rms_norm_quant) equals
the unfused chain nvfp4_rms_norm -> nvfp4_quantize bit for bit (codes,
scales, gs), and that chain's quantization equals the oracle's on the GPU's
own normalised rows; the normalised rows themselves are within one bf16 step
of the oracle's."""
import numpy as np
import pytest
import torch

import bit_linear_moe_b200 as nv
import oracle
from oracle import stack as ost
from nvfp4_checks import bf16_ulp, tiled_to_rowmajor

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,cols,ld,dtype,layout", [
    (1, 5120, 10240, torch.float32, nv.SF_TILED),        # the Q slice of a decode QKV output
    (5, 5120, 5120, torch.bfloat16, nv.SF_ROWMAJOR),
    (8, 1024, 1040, torch.float32, nv.SF_TILED),
    (9, 17408, 17408, torch.bfloat16, nv.SF_TILED),      # 256-thread rows
    (2048, 5120, 5120, torch.bfloat16, nv.SF_TILED),     # a prefill chunk
])
def test_rms_norm_quant(rows, cols, ld, dtype, layout):
    rng = np.random.default_rng(rows + cols + ld)
    x = (rng.standard_normal((rows, ld)) * rng.uniform(0.01, 50, (rows, 1))).astype(np.float32)
    if rows > 2:
        x[1] = 0.0                                        # an all-zero row stays zero
    xd = torch.from_numpy(x).to(dtype).cuda()
    c, s, g = nv.nvfp4_rms_norm_quant(xd, cols=cols, sf_layout=layout)
    y = nv.nvfp4_rms_norm(xd, cols=cols)
    c2, s2, g2 = nv.nvfp4_quantize(y, sf_layout=layout)
    torch.cuda.synchronize()
    assert torch.equal(c, c2) and torch.equal(s, s2) and torch.equal(g, g2), "fused != rms_norm -> quantize"
    yh = y.float().cpu().numpy()
    ref_y = ost.rms_norm(xd.float().cpu().numpy()[:, :cols])
    assert (np.abs(yh.astype(np.float64) - ref_y) <= bf16_ulp(ref_y) + 1e-30).all()
    q = oracle.quantize(yh)
    sc = s.cpu().numpy()
    sc = tiled_to_rowmajor(sc, rows, cols) if layout == nv.SF_TILED else sc.reshape(rows, cols // 16)
    assert np.array_equal(c.cpu().numpy(), q[0]) and np.array_equal(sc, q[1]) and np.float32(g.item()) == q[2]
