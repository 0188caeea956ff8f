"""Bounded waits: a wait whose producer never delivers ends with
NVFP4_ERR_DEVICE_TIMEOUT in the library's status word instead of hanging, and
the device stays usable.  The producer here is the library's probe kernel (an
mbarrier nothing arrives on, nothing in flight), so no GPU fault or hang is
provoked."""
import numpy as np
import pytest
import torch

import bit_linear_moe_b200 as nv
import oracle
from bit_linear_moe_b200 import synth
from nvfp4_checks import assert_within_bound

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_device_stays_usable(cuda_device):
    assert nv.nvfp4_read_device_status() == nv.OK
    nv.nvfp4_debug_wait_timeout(20_000_000)            # ~10-20 ms of SM clock
    assert nv.nvfp4_read_device_status() == nv.ERR_DEVICE_TIMEOUT
    assert nv.nvfp4_read_device_status() == nv.OK       # the read resets the word
    # the context is intact: a normal call runs and is right
    w, x = synth.single(0)
    c, s, g = nv.nvfp4_quantize(torch.from_numpy(w).cuda(), sf_layout=nv.SF_TILED)
    y = nv.nvfp4_linear(torch.from_numpy(x).to(torch.bfloat16).cuda(), c, s, g, w_sf_layout=nv.SF_TILED,
                        mode=nv.MODE_W4A16)
    torch.cuda.synchronize()
    assert nv.nvfp4_read_device_status() == nv.OK
    ref, ad = oracle.linear_w4a16(x, *oracle.quantize(w))
    assert_within_bound(y, ref, ad, False, "linear after a timed-out wait")
