"""GPU quantizer vs the CPU oracle: codes, scales and gs bit-exact."""
import numpy as np
import pytest
import torch

import bit_linear_moe_b200 as nv
import oracle
from bit_linear_moe_b200 import synth
from nvfp4_checks import tiled_to_rowmajor

pytestmark = pytest.mark.gpu


def _gpu_quant(x_np, dtype, layout, gs_in=None):
    x = torch.from_numpy(x_np).to(dtype).cuda()
    g = None if gs_in is None else torch.tensor([gs_in], dtype=torch.float32, device="cuda")
    c, s, gs = nv.nvfp4_quantize(x, gs_in=g, sf_layout=layout)
    torch.cuda.synchronize()
    rows, cols = x_np.shape
    s = s.cpu().numpy()
    if layout == nv.SF_TILED:
        full = s
        s = tiled_to_rowmajor(s, rows, cols)
        mask = np.ones(full.size, bool)
        from nvfp4_checks import tiled_index
        mask[tiled_index(rows, cols).ravel()] = False
        assert not full[mask].any(), "tiled padding must be zero"
    else:
        s = s.reshape(rows, cols // 16)
    return c.cpu().numpy(), s, np.float32(gs.item())


def _check(x_np, dtype, layout, gs_in=None):
    xq = x_np if dtype == torch.float32 else synth.to_bf16(x_np)
    c, s, gs = _gpu_quant(xq, dtype, layout, gs_in)
    rc, rs, rgs = oracle.quantize(xq, gs=gs_in)
    assert gs == rgs, (gs, rgs)
    nbad_s = int((s != rs).sum())
    nbad_c = int((c != rc).sum())
    assert nbad_s == 0 and nbad_c == 0, f"scales differ at {nbad_s}, code bytes differ at {nbad_c}"


@pytest.mark.parametrize("layout", [nv.SF_ROWMAJOR, nv.SF_TILED])
def test_single_linear_weights_fp32(layout):
    w, _ = synth.single(0)
    _check(w, torch.float32, layout)


@pytest.mark.parametrize("layout", [nv.SF_ROWMAJOR, nv.SF_TILED])
@pytest.mark.parametrize("shape", [(1, 16), (3, 48), (130, 80), (257, 272), (5, 4096)])
def test_ragged_shapes(shape, layout):
    rng = np.random.default_rng(sum(shape))
    _check(synth.weight(rng, *shape), torch.float32, layout)
    _check(rng.standard_normal(shape).astype(np.float32), torch.bfloat16, layout)


def test_edge_values():
    rng = np.random.default_rng(1)
    x = synth.weight(rng, 64, 256)
    x[0] = 0.0                           # zero row
    x[1, :16] = 0.0                      # zero block
    x[2, 16:32] = -0.0                   # negative zeros
    x[3, 32:48] = 1e-12                  # block whose scale underflows
    x[4, :16] = -x[4, :16]
    x[5, 7] = 3.0                        # tensor max
    x[6, :] = np.float32(0.5) * 3.0 / 2688 * 6   # exact E2M1 * scale products
    x[7, 0:16] = np.linspace(-1, 1, 16, dtype=np.float32) * 1e-3
    for layout in (nv.SF_ROWMAJOR, nv.SF_TILED):
        _check(x, torch.float32, layout)
        _check(x, torch.bfloat16, layout)


def test_all_zero_tensor():
    _check(np.zeros((8, 64), np.float32), torch.float32, nv.SF_ROWMAJOR)


def test_given_global_scale_saturates():
    x = synth.activations(np.random.default_rng(2), 32, 512)
    _check(x, torch.bfloat16, nv.SF_ROWMAJOR, gs_in=np.float32(1e-4))
    _check(x, torch.bfloat16, nv.SF_TILED, gs_in=np.float32(0.37))


def test_prefill_activations_with_outliers():
    x, cols = synth.prefill_x(1, 512, 5120)
    assert len(cols) == 51
    _check(x, torch.bfloat16, nv.SF_TILED)


@pytest.mark.parametrize("name,K,N,seed", synth.DENSE27B)
def test_dense27b_weights_full(name, K, N, seed):
    w = synth.dense_weight(seed, K, N)
    _check(w, torch.float32, nv.SF_ROWMAJOR)


def _e4m3_value(b):
    """Value of an E4M3 byte (OCP FP8 format: bias 7, subnormals at exponent 0)."""
    e, m = (b >> 3) & 15, b & 7
    v = (1 + m / 8) * 2.0 ** (e - 7) if e else (m / 8) * 2.0 ** -6
    return -v if b & 0x80 else v


def test_quotients_at_e2m1_rounding_boundaries():
    """Elements placed on, and a few fp32 ulps either side of, every E2M1
    rounding boundary (the midpoints 0.25, 0.75, ..., 5 between E2M1 values)
    of their block's scale r: the code must follow the IEEE-rounded quotient
    x / r, ties to even, exactly as the oracle takes it."""
    gs = np.float32(0.3712345)
    mids = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)
    rng = np.random.default_rng(11)
    rows = []
    for _ in range(96):
        x = np.zeros(16 * 16, np.float32)
        for blk in range(16):
            A = np.float32(rng.uniform(0.05, 40.0))
            _, s, _ = oracle.quantize(np.concatenate([[A], np.zeros(15, np.float32)])[None, :].astype(np.float32),
                                      gs=gs)
            r = np.float32(np.float32(_e4m3_value(int(s[0, 0]))) * gs)
            vals = [A]
            for j in range(15):
                v = np.float32(mids[j % 7] * np.float64(r))
                for _ in range(abs(int(rng.integers(-3, 4)))):
                    v = np.nextafter(v, np.float32(np.inf) if rng.random() < 0.5 else np.float32(0))
                vals.append(-v if rng.random() < 0.5 else v)
            x[16 * blk:16 * blk + 16] = vals
        rows.append(x)
    x = np.stack(rows)
    _check(x, torch.float32, nv.SF_ROWMAJOR, gs_in=gs)
    _check(x, torch.float32, nv.SF_TILED, gs_in=gs)
    _check(x, torch.float32, nv.SF_TILED)  # the tensor's own gs: same boundaries, other scales
