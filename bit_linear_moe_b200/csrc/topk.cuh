// Warp-level top-k of one token's router logits (CHImp Alpha v1.0 model card,
// "How it fits on one GPU": each token goes to 10 of 512 experts).
//
// Lane l holds logits l, l + 32, ... (PER of them).  Order: larger logit
// first, equal logits -> lower expert index.  The weights are the softmax
// over the k winners (the full softmax renormalised over them).
#pragma once

#include "common.cuh"

namespace nvfp4 {

// Order-preserving 32-bit key of a float: for non-NaN a, b, a > b exactly when
// key(a) > key(b) as unsigned integers, and a == b exactly when the keys are
// equal (-0 is keyed as +0).  Every key of a finite or infinite value is > 0.
NVFP4_DEV uint32_t order_key(float v) {
    const uint32_t u = __float_as_uint(v == 0.0f ? 0.0f : v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

NVFP4_DEV float key_value(uint32_t kk) { return __uint_as_float((kk & 0x80000000u) ? (kk & 0x7FFFFFFFu) : ~kk); }

// Largest of n 64-bit values by a pairwise tree (depth log2 n).
template <int N>
NVFP4_DEV uint64_t tree_max(const uint64_t (&a)[N]) {
    uint64_t b[N];
#pragma unroll
    for (int i = 0; i < N; ++i) b[i] = a[i];
#pragma unroll
    for (int w = 1; w < N; w *= 2)
#pragma unroll
        for (int i = 0; i + w < N; i += 2 * w) b[i] = b[i] > b[i + w] ? b[i] : b[i + w];
    return b[0];
}

// After the call, lane j < k holds slot j: *idx_out = expert, *w_out = weight.
// Each lane keys its values once as (order key << 32 | PER - 1 - i), so the
// largest 64-bit value is its best logit with the lowest index; a round is
// two single-instruction warp reductions, the largest key among the lanes'
// bests (redux.sync.max) and the lowest expert index among the lanes holding
// it (redux.sync.min); the winning lane clears that value and takes the tree
// maximum again.  The winning logit is recovered from its key.
template <int PER>
NVFP4_DEV void warp_topk(const float* __restrict__ row, int E, int k, int lane, int* idx_out, float* w_out) {
    uint64_t kv[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = i * 32 + lane;
        kv[i] = e < E ? ((uint64_t)order_key(row[e]) << 32) | (uint32_t)(PER - 1 - i) : 0ull;
    }
    uint64_t best = tree_max(kv);
    float lmax = 0.0f, mywl = 0.0f;
    int myidx = 0;
    for (int j = 0; j < k; ++j) {
        const uint32_t mk = (uint32_t)(best >> 32);
        const uint32_t bk = __reduce_max_sync(0xffffffffu, mk);
        const uint32_t me = (uint32_t)(PER - 1 - (int)(best & 0xFFFFFFFFu)) * 32u + (uint32_t)lane;
        const int bi = (int)__reduce_min_sync(0xffffffffu, mk == bk ? me : 0xffffffffu);
        if ((bi & 31) == lane) {
#pragma unroll
            for (int i = 0; i < PER; ++i)
                if (i == (bi >> 5)) kv[i] = 0ull;
            best = tree_max(kv);
        }
        const float val = key_value(bk);
        if (j == 0) lmax = val;
        if (lane == j) {
            myidx = bi;
            mywl = val;
        }
    }
    const float ex = lane < k ? expf(mywl - lmax) : 0.0f;
    const float den = warp_sum(ex);
    *idx_out = myidx;
    *w_out = ex / den;
}

}  // namespace nvfp4
