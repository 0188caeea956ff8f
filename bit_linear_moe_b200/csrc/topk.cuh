// Warp-level top-k of one token's router logits (CHImp Alpha v1.0 model card,
// "How it fits on one GPU": each token goes to 10 of 512 experts).
//
// Lane l holds logits l, l + 32, ... (PER of them).  Order: larger logit
// first, equal logits -> lower expert index.  Each lane keeps the best of its
// untaken values; a round is a warp arg-max over the lanes' bests, after which
// only the winning lane rescans its own values.  The weights are the softmax
// over the k winners (the full softmax renormalised over them).
#pragma once

#include "common.cuh"

namespace nvfp4 {

NVFP4_DEV bool topk_better(float v, int i, float bv, int bi) { return v > bv || (v == bv && i < bi); }

// After the call, lane j < k holds slot j: *idx_out = expert, *w_out = weight.
template <int PER>
NVFP4_DEV void warp_topk(const float* __restrict__ row, int E, int k, int lane, int* idx_out, float* w_out) {
    float v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = i * 32 + lane;
        v[i] = e < E ? row[e] : -INFINITY;
    }
    uint32_t taken = 0;  // bit i: v[i] already selected
    auto rescan = [&](float& lbv, int& lbi) {
        lbv = -INFINITY;
        lbi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = i * 32 + lane;
            if (e < E && !((taken >> i) & 1u) && topk_better(v[i], e, lbv, lbi)) {
                lbv = v[i];
                lbi = e;
            }
        }
    };
    float lbv;
    int lbi;
    rescan(lbv, lbi);
    float lmax = 0.0f, mywl = 0.0f;
    int myidx = 0;
    for (int j = 0; j < k; ++j) {
        float bv = lbv;
        int bi = lbi;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (topk_better(ov, oi, bv, bi)) {
                bv = ov;
                bi = oi;
            }
        }
        if ((bi & 31) == lane) {
            taken |= 1u << (bi >> 5);
            rescan(lbv, lbi);
        }
        if (j == 0) lmax = bv;
        if (lane == j) {
            myidx = bi;
            mywl = bv;
        }
    }
    const float ex = lane < k ? expf(mywl - lmax) : 0.0f;
    const float den = warp_sum(ex);
    *idx_out = myidx;
    *w_out = ex / den;
}

}  // namespace nvfp4
