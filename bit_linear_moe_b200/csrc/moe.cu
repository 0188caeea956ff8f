// K5/K6/K8: router, top-k, token permutation and combine of a routed
// mixture-of-experts layer (CHImp Alpha v1.0 model card, "How it fits on one
// GPU": each token is routed to 10 of 512 experts per layer).
//
// Router logits  l[t, e] = sum_h h[t, h] * Wr[e, h] (+ bias[e]), bf16 inputs,
//                fp32 accumulation (products of two bf16 are exact in fp32;
//                sums are kept in 32-term tile partials).
// Top-k          one warp per token; k rounds of a warp arg-max that orders by
//                (logit descending, expert index ascending); weights are the
//                softmax over the k winners.
// Permutation    counting sort by expert, stable in token order, without
//                atomics on the result: per block of 32 tokens a bitmask per
//                expert marks the tokens that chose it, so a token's rank inside
//                its block is a popcount; block bases come from a scan.
// Combine        y[t, n] = sum_j w[t, j] * d[row_of[t, j], n], j ascending.
#include "common.cuh"
#include "internal.h"
#include "tma.cuh"
#include "topk.cuh"

namespace nvfp4 {

// ---- router logits: 64 x 64 output tile per CTA, 256 threads, 4 x 4 each ----
constexpr int RT = 64, RK = 32;

__global__ void __launch_bounds__(256) router_logits_kernel(const __nv_bfloat16* __restrict__ h,
                                                            const __nv_bfloat16* __restrict__ wr,
                                                            const float* __restrict__ bias, int64_t T,
                                                            int64_t H, int32_t E, float* __restrict__ logits) {
    __shared__ float sh[RK][RT + 1];
    __shared__ float sw[RK][RT + 1];
    const int tid = threadIdx.x;
    const int64_t t0 = (int64_t)blockIdx.x * RT, e0 = (int64_t)blockIdx.y * RT;
    const int ty = tid / 16, tx = tid % 16;  // 16 x 16 threads, 4 x 4 outputs each
    float acc[4][4] = {};
    for (int64_t k0 = 0; k0 < H; k0 += RK) {
        // load 64 rows x 32 cols of h and of wr (bf16 -> fp32), 8 elements per thread
        {
            const int r = tid / 4, q = (tid % 4) * 8;
            float hv[8] = {}, wv[8] = {};
            if (t0 + r < T && k0 + q < H) {
                uint4 v = ldg_v4(h + (t0 + r) * H + k0 + q);
                uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) { hv[2 * j] = bf16lo_to_f32(u[j]); hv[2 * j + 1] = bf16hi_to_f32(u[j]); }
            }
            if (e0 + r < E && k0 + q < H) {
                uint4 v = ldg_v4(wr + (e0 + r) * H + k0 + q);
                uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) { wv[2 * j] = bf16lo_to_f32(u[j]); wv[2 * j + 1] = bf16hi_to_f32(u[j]); }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) { sh[q + j][r] = hv[j]; sw[q + j][r] = wv[j]; }
        }
        __syncthreads();
        float part[4][4] = {};
#pragma unroll 8
        for (int kk = 0; kk < RK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) { a[i] = sh[kk][ty * 4 + i]; b[i] = sw[kk][tx * 4 + i]; }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) part[i][j] = fmaf(a[i], b[j], part[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] += part[i][j];
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t t = t0 + ty * 4 + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t e = e0 + tx * 4 + j;
            if (e < E) logits[t * E + e] = acc[i][j] + (bias ? bias[e] : 0.0f);
        }
    }
}

// ---- router logits for a few tokens: one warp per (expert, group of up to 8
// tokens); the expert's row is streamed once per group, the tokens' rows come
// from L1/L2 ----
constexpr int kRouterTokGroup = 8;

__global__ void __launch_bounds__(256) router_logits_small_kernel(const __nv_bfloat16* __restrict__ h,
                                                                  const __nv_bfloat16* __restrict__ wr,
                                                                  const float* __restrict__ bias, int64_t T,
                                                                  int64_t H, int32_t E, float* __restrict__ logits) {
    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);  // global warp
    const int64_t ngroups = (T + kRouterTokGroup - 1) / kRouterTokGroup;
    // as a programmatic dependent: the next kernel may launch at once; the
    // hidden states (written by the kernel before) are read after the wait
    griddep_launch_dependents();
    griddep_wait();
    if (gw >= (int64_t)E * ngroups) return;
    const int64_t e = gw / ngroups, t0 = (gw % ngroups) * kRouterTokGroup;
    const int nt = (int)((T - t0) < kRouterTokGroup ? (T - t0) : kRouterTokGroup);
    float acc[kRouterTokGroup] = {};
    for (int64_t k0 = 8 * lane; k0 < H; k0 += 256) {
        const uint4 wv = ldg_v4(wr + e * H + k0);
        const uint32_t wu[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int t = 0; t < kRouterTokGroup; ++t) {
            if (t < nt) {
                const uint4 hv = ldg_v4(h + (t0 + t) * H + k0);
                const uint32_t hu[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[t] = fmaf(bf16lo_to_f32(hu[j]), bf16lo_to_f32(wu[j]), acc[t]);
                    acc[t] = fmaf(bf16hi_to_f32(hu[j]), bf16hi_to_f32(wu[j]), acc[t]);
                }
            }
        }
    }
#pragma unroll
    for (int t = 0; t < kRouterTokGroup; ++t) {
        const float v = warp_sum(acc[t]);
        if (lane == 0 && t < nt) logits[(t0 + t) * E + e] = v + (bias ? bias[e] : 0.0f);
    }
}

int launch_router_logits_small_pdl(const void* h, const void* wr, const float* bias, int64_t T, int64_t H,
                                   int32_t E, float* logits, cudaStream_t st) {
    const int64_t warps = (int64_t)E * ((T + kRouterTokGroup - 1) / kRouterTokGroup);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((warps + 7) / 8), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    set_pdl_attr(attr[0]);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, router_logits_small_kernel, (const __nv_bfloat16*)h, (const __nv_bfloat16*)wr,
                              bias, T, H, E, logits) == cudaSuccess
               ? NVFP4_OK
               : NVFP4_ERR_LAUNCH;
}

int launch_router_logits(const void* h, const void* wr, const float* bias, int64_t T, int64_t H, int32_t E,
                         float* logits, cudaStream_t st) {
    if (router_tcs_supported(h, wr, T, H, E))
        return launch_router_logits_tcs(h, wr, bias, T, H, E, logits, device_status_ptr(), st);
    if (T <= 64 && H % 8 == 0) {
        const int64_t warps = (int64_t)E * ((T + kRouterTokGroup - 1) / kRouterTokGroup);
        router_logits_small_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(
            (const __nv_bfloat16*)h, (const __nv_bfloat16*)wr, bias, T, H, E, logits);
        return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
    }
    if (router_tc_supported(h, wr, T, H, E))
        return launch_router_logits_tc(h, wr, bias, T, H, E, logits, device_status_ptr(), st);
    dim3 grid((unsigned)((T + RT - 1) / RT), (unsigned)((E + RT - 1) / RT));
    router_logits_kernel<<<grid, 256, 0, st>>>((const __nv_bfloat16*)h, (const __nv_bfloat16*)wr, bias, T, H, E,
                                               logits);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

// ---- top-k + per-block expert counts ------------------------------------
// CTA = 1024 threads = 32 warps, kPermBlockTokens tokens; a warp takes
// kPermBlockTokens / 32 of them (warp_topk, topk.cuh).
constexpr int kMaxE = 1024, kTopkThreads = 1024;

template <int PER>
__global__ void __launch_bounds__(kTopkThreads) topk_count_kernel(const float* __restrict__ logits, int64_t T,
                                                                  int32_t E, int32_t k, int32_t* __restrict__ topk_idx,
                                                                  float* __restrict__ topk_w,
                                                                  int32_t* __restrict__ blk_counts) {
    __shared__ uint32_t mask[kMaxE][kPermBlockTokens / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < E * (kPermBlockTokens / 32); i += blockDim.x) (&mask[0][0])[i] = 0;
    __syncthreads();
    const int64_t tb = (int64_t)blockIdx.x * kPermBlockTokens;
    for (int tt = warp; tt < kPermBlockTokens; tt += kTopkThreads / 32) {
        const int64_t t = tb + tt;
        if (t >= T) break;
        int myidx;
        float myw;
        warp_topk<PER>(logits + t * E, E, k, lane, &myidx, &myw);
        if (lane < k) {
            topk_idx[t * k + lane] = myidx;
            topk_w[t * k + lane] = myw;
            atomicOr(&mask[myidx][tt >> 5], 1u << (tt & 31));
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int c = 0;
#pragma unroll
        for (int w = 0; w < kPermBlockTokens / 32; ++w) c += __popc(mask[e][w]);
        blk_counts[(int64_t)blockIdx.x * E + e] = c;
    }
}

int launch_topk_count(const float* logits, int64_t T, int32_t E, int32_t k, int32_t* topk_idx, float* topk_w,
                      int32_t* blk_counts, cudaStream_t st) {
    const int64_t nblk = (T + kPermBlockTokens - 1) / kPermBlockTokens;
    const int per = (E + 31) / 32;
    if (per <= 8)
        topk_count_kernel<8><<<(unsigned)nblk, kTopkThreads, 0, st>>>(logits, T, E, k, topk_idx, topk_w, blk_counts);
    else if (per <= 16)
        topk_count_kernel<16><<<(unsigned)nblk, kTopkThreads, 0, st>>>(logits, T, E, k, topk_idx, topk_w, blk_counts);
    else
        topk_count_kernel<32><<<(unsigned)nblk, kTopkThreads, 0, st>>>(logits, T, E, k, topk_idx, topk_w, blk_counts);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

// ---- scan: expert offsets and per-block bases -----------------------------
__global__ void __launch_bounds__(1024) perm_scan_kernel(const int32_t* __restrict__ blk_counts, int64_t nblk,
                                                         int32_t E, int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ blk_base) {
    __shared__ int32_t tot[kMaxE];
    const int e = threadIdx.x;
    constexpr int kU = 8;  // counts loaded per round trip
    int32_t run = 0;
    if (e < E)
        for (int64_t b0 = 0; b0 < nblk; b0 += kU) {
            int32_t c[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) c[u] = b0 + u < nblk ? blk_counts[(b0 + u) * E + e] : 0;
#pragma unroll
            for (int u = 0; u < kU; ++u) run += c[u];
        }
    tot[e] = e < E ? run : 0;
    __syncthreads();
    // Hillis-Steele inclusive scan over 1024 entries.
    for (int o = 1; o < kMaxE; o <<= 1) {
        const int32_t add = e >= o ? tot[e - o] : 0;
        __syncthreads();
        tot[e] += add;
        __syncthreads();
    }
    if (e < E) {
        const int32_t excl = tot[e] - run;
        offsets[e] = excl;
        if (e == E - 1) offsets[E] = tot[e];
        int32_t base = excl;
        for (int64_t b0 = 0; b0 < nblk; b0 += kU) {
            int32_t c[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) c[u] = b0 + u < nblk ? blk_counts[(b0 + u) * E + e] : 0;
#pragma unroll
            for (int u = 0; u < kU; ++u)
                if (b0 + u < nblk) {
                    blk_base[(b0 + u) * E + e] = base;
                    base += c[u];
                }
        }
    }
}

int launch_perm_scan(const int32_t* blk_counts, int64_t nblk, int32_t E, int32_t* offsets, int32_t* blk_base,
                     cudaStream_t st) {
    perm_scan_kernel<<<1, kMaxE, 0, st>>>(blk_counts, nblk, E, offsets, blk_base);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

// ---- scatter: one thread per token -----------------------------------------
__global__ void __launch_bounds__(kPermBlockTokens) perm_scatter_kernel(
    const int32_t* __restrict__ topk_idx, int64_t T, int32_t E, int32_t k, const int32_t* __restrict__ blk_base,
    int32_t* __restrict__ perm_tok, int32_t* __restrict__ perm_slot, int32_t* __restrict__ row_of) {
    __shared__ uint32_t mask[kMaxE][kPermBlockTokens / 32];
    for (int i = threadIdx.x; i < E * (kPermBlockTokens / 32); i += blockDim.x) (&mask[0][0])[i] = 0;
    __syncthreads();
    const int tt = threadIdx.x;
    const int64_t t = (int64_t)blockIdx.x * kPermBlockTokens + tt;
    if (t < T)
        for (int j = 0; j < k; ++j) atomicOr(&mask[topk_idx[t * k + j]][tt >> 5], 1u << (tt & 31));
    __syncthreads();
    if (t >= T) return;
    for (int j = 0; j < k; ++j) {
        const int e = topk_idx[t * k + j];
        int rank = __popc(mask[e][tt >> 5] & ((1u << (tt & 31)) - 1u));
        for (int w = 0; w < (tt >> 5); ++w) rank += __popc(mask[e][w]);
        const int32_t row = blk_base[(int64_t)blockIdx.x * E + e] + rank;
        perm_tok[row] = (int32_t)t;
        perm_slot[row] = j;
        row_of[t * k + j] = row;
    }
}

int launch_perm_scatter(const int32_t* topk_idx, int64_t T, int32_t E, int32_t k, const int32_t* blk_base,
                        int32_t* perm_tok, int32_t* perm_slot, int32_t* row_of, cudaStream_t st) {
    const int64_t nblk = (T + kPermBlockTokens - 1) / kPermBlockTokens;
    perm_scatter_kernel<<<(unsigned)nblk, kPermBlockTokens, 0, st>>>(topk_idx, T, E, k, blk_base, perm_tok,
                                                                      perm_slot, row_of);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

// ---- combine ---------------------------------------------------------------
// One thread per 4 output columns of a token: the k slots are read in order
// j = 0..k-1 and summed in fp32, so the result does not depend on scheduling.
template <typename InT>
NVFP4_DEV float4 load4(const InT* p);
template <>
NVFP4_DEV float4 load4<float>(const float* p) {
    return *reinterpret_cast<const float4*>(p);
}
template <>
NVFP4_DEV float4 load4<__nv_bfloat16>(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    return make_float4(bf16lo_to_f32(u.x), bf16hi_to_f32(u.x), bf16lo_to_f32(u.y), bf16hi_to_f32(u.y));
}

template <typename InT, typename OutT>
__global__ void __launch_bounds__(256) combine_kernel(const InT* __restrict__ d, const float* __restrict__ w,
                                                      const int32_t* __restrict__ row_of, int64_t T, int32_t k,
                                                      int64_t N, OutT* __restrict__ y) {
    const int64_t n4 = N / 4;
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= T * n4) return;
    const int64_t t = i / n4, c = (i % n4) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
        const float wj = w[t * k + j];
        const int32_t r = row_of[t * k + j];
        if (r < 0 || (int64_t)r >= T * k) continue;  // row_of must index the T * k rows of d
        const float4 v = load4<InT>(d + (int64_t)r * N + c);
        acc.x = fmaf(wj, v.x, acc.x);
        acc.y = fmaf(wj, v.y, acc.y);
        acc.z = fmaf(wj, v.z, acc.z);
        acc.w = fmaf(wj, v.w, acc.w);
    }
    if constexpr (sizeof(OutT) == 4) {
        *reinterpret_cast<float4*>(y + t * N + c) = acc;
    } else {
        const __nv_bfloat162 b0 = __floats2bfloat162_rn(acc.x, acc.y);
        const __nv_bfloat162 b1 = __floats2bfloat162_rn(acc.z, acc.w);
        *reinterpret_cast<uint2*>(y + t * N + c) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&b0), *reinterpret_cast<const uint32_t*>(&b1));
    }
}

int launch_combine(const void* d, int d_dtype, const float* topk_w, const int32_t* row_of, int64_t T, int32_t k,
                   int64_t N, void* y, int y_dtype, cudaStream_t st) {
    const int64_t n = T * (N / 4);
    const unsigned grid = (unsigned)((n + 255) / 256);
#define NVFP4_C(IT, OT) \
    combine_kernel<IT, OT><<<grid, 256, 0, st>>>((const IT*)d, topk_w, row_of, T, k, N, (OT*)y)
    if (d_dtype == NVFP4_DTYPE_BF16) {
        if (y_dtype == NVFP4_DTYPE_BF16) NVFP4_C(__nv_bfloat16, __nv_bfloat16);
        else NVFP4_C(__nv_bfloat16, float);
    } else {
        if (y_dtype == NVFP4_DTYPE_BF16) NVFP4_C(float, __nv_bfloat16);
        else NVFP4_C(float, float);
    }
#undef NVFP4_C
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

}  // namespace nvfp4

namespace nvfp4 {

// ---- padded expert layout for the grouped tensor-core GEMM ------------------
// Each expert's rows are padded to whole 128-row tiles.  pad_off[e] is the
// first padded row of expert e; tile_info[t] = {expert, first output row,
// real rows} for the used tiles and {-1, 0, 0} for the rest.
__global__ void __launch_bounds__(1024) moe_pad_kernel(const int32_t* __restrict__ offsets, int32_t E,
                                                       int64_t n_mtiles, int32_t* __restrict__ pad_off,
                                                       int32_t* __restrict__ tile_info) {
    __shared__ int32_t tiles[kMaxE];
    const int e = threadIdx.x;
    const int32_t cnt = e < E ? offsets[e + 1] - offsets[e] : 0;
    const int32_t mine = (cnt + 127) / 128;
    tiles[e] = mine;
    __syncthreads();
    for (int o = 1; o < kMaxE; o <<= 1) {
        const int32_t add = e >= o ? tiles[e - o] : 0;
        __syncthreads();
        tiles[e] += add;
        __syncthreads();
    }
    const int32_t first = tiles[e] - mine;
    const int32_t total = tiles[kMaxE - 1];
    if (e < E) {
        pad_off[e] = first * 128;
        for (int32_t t = 0; t < mine; ++t) {
            int32_t* ti = tile_info + 3 * (int64_t)(first + t);
            ti[0] = e;
            ti[1] = offsets[e] + 128 * t;
            ti[2] = min(128, cnt - 128 * t);
        }
    }
    if (e == 0) pad_off[E] = total * 128;
    for (int64_t t = total + e; t < n_mtiles; t += blockDim.x) {
        int32_t* ti = tile_info + 3 * t;
        ti[0] = -1;
        ti[1] = 0;
        ti[2] = 0;
    }
}

// src_rows[pr] = activation row read by padded row pr (-1 for padding).
__global__ void __launch_bounds__(256) moe_src_rows_kernel(const int32_t* __restrict__ pad_off,
                                                           const int32_t* __restrict__ offsets, int32_t E,
                                                           const int32_t* __restrict__ gather, int64_t rows_pad,
                                                           int32_t* __restrict__ src_rows) {
    const int64_t pr = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (pr >= rows_pad) return;
    int32_t src = -1;
    if (pr < pad_off[E]) {
        int lo = 0, hi = E;  // last e with pad_off[e] <= pr
        while (hi - lo > 1) {
            const int mid = (lo + hi) / 2;
            if (pad_off[mid] <= pr) lo = mid; else hi = mid;
        }
        const int64_t local = pr - pad_off[lo];
        const int32_t cnt = offsets[lo + 1] - offsets[lo];
        if (local < cnt) {
            const int64_t r = offsets[lo] + local;
            src = gather ? gather[r] : (int32_t)r;
        }
    }
    src_rows[pr] = src;
}

int launch_moe_pad(const int32_t* offsets, int32_t E, int64_t rows_pad, const int32_t* gather, int32_t* pad_off,
                   int32_t* tile_info, int32_t* src_rows, cudaStream_t st) {
    moe_pad_kernel<<<1, kMaxE, 0, st>>>(offsets, E, rows_pad / 128, pad_off, tile_info);
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_LAUNCH;
    moe_src_rows_kernel<<<(unsigned)((rows_pad + 255) / 256), 256, 0, st>>>(pad_off, offsets, E, gather, rows_pad,
                                                                            src_rows);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

// ---- touched experts: list[j] = the j-th expert with rows, -1 past the last ----
__global__ void __launch_bounds__(1024) touched_experts_kernel(const int32_t* __restrict__ offsets, int32_t E,
                                                               int32_t nslots, int32_t* __restrict__ list) {
    __shared__ int32_t warp_tot[32];
    const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
    const bool has = e < E && offsets[e + 1] > offsets[e];
    const uint32_t bal = __ballot_sync(0xffffffffu, has);
    if (lane == 0) warp_tot[warp] = __popc(bal);
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += warp_tot[w];
    int total = 0;
    for (int w = 0; w < 32; ++w) total += warp_tot[w];
    const int pos = base + __popc(bal & ((1u << lane) - 1u));
    if (has && pos < nslots) list[pos] = e;
    for (int j = total + e; j < nslots; j += 1024) list[j] = -1;
}

int launch_touched_experts(const int32_t* offsets, int32_t E, int32_t nslots, int32_t* list, cudaStream_t st) {
    if (E < 1 || E > 1024) return NVFP4_ERR_SHAPE;
    touched_experts_kernel<<<1, 1024, 0, st>>>(offsets, E, nslots, list);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

}  // namespace nvfp4
