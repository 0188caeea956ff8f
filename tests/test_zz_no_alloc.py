"""The allocation-free router entry point, moe_route_topk_noalloc.

It serves callers that cannot allocate device memory while routing (a fixed
device-memory plan, or code where an allocation is not permitted); it keeps
its scratch in a 1 MiB array inside the library instead of a caller
workspace.  Its outputs must equal moe_route_topk's on the same inputs, on two
calls in a row (the second call reuses the scratch the first one left
behind).  This file is collected last so that a failure here cannot hide the
other tests' results.
"""
import numpy as np
import pytest
import torch

import bit_linear_moe_b200 as nv
from bit_linear_moe_b200 import synth

pytestmark = pytest.mark.gpu

KEYS = ("topk_idx", "expert_offsets", "perm_tok", "perm_slot", "row_of")


def _inputs(T, zipf):
    h = torch.from_numpy(synth.moe_hidden(T)).to(torch.bfloat16).cuda()
    wr = torch.from_numpy(synth.moe_router()).to(torch.bfloat16).cuda()
    bias = torch.from_numpy(synth.moe_zipf_bias()).cuda() if zipf else None
    return h, wr, bias


def _same(a, b, with_logits):
    for key in KEYS:
        assert torch.equal(a[key], b[key]), key
    assert torch.allclose(a["topk_w"], b["topk_w"], rtol=2e-6, atol=1e-7)
    if with_logits:
        assert torch.equal(a["logits"], b["logits"])


def test_noalloc_matches_workspace_entry_point_two_calls():
    # call 1: T = 32 with the logits kept in the built-in scratch
    h, wr, bias = _inputs(32, zipf=True)
    ref1 = nv.moe_route_topk(h, wr, synth.MOE_K, logit_bias=bias)
    got1 = nv.moe_route_topk_noalloc(h, wr, synth.MOE_K, logit_bias=bias)
    # call 2: T = 4096, logits in a caller buffer (they would not fit the scratch)
    h2, wr2, _ = _inputs(4096, zipf=False)
    ref2 = nv.moe_route_topk(h2, wr2, synth.MOE_K, want_logits=True)
    got2 = nv.moe_route_topk_noalloc(h2, wr2, synth.MOE_K, want_logits=True)
    torch.cuda.synchronize()
    _same(ref1, got1, with_logits=False)
    _same(ref2, got2, with_logits=True)
    assert int(got2["expert_offsets"][-1]) == 4096 * synth.MOE_K


def test_noalloc_rejects_requests_beyond_its_scratch():
    h, wr, _ = _inputs(4096, zipf=False)
    with pytest.raises(nv.NVFP4Error) as e:
        nv.moe_route_topk_noalloc(h, wr, synth.MOE_K)   # 4096 x 512 fp32 logits = 8 MiB > 1 MiB
    assert e.value.status == nv.ERR_WORKSPACE
