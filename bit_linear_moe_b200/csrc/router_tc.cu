// K5 (tensor-core form): router logits of a routed mixture-of-experts layer
// for prefill-sized token counts (CHImp Alpha v1.0 model card, "How it fits on
// one GPU": 512 experts, 10 per token).
//
//   l[t, e] = sum_h h[t, h] * Wr[e, h] (+ bias[e])
//
// A dense bf16 x bf16 contraction with fp32 accumulation: tcgen05.mma of
// kind::f16 (both operands bf16), M = 128 tokens, N = 128 experts, K = 16 per
// instruction, accumulator in tensor memory.  Products of two bf16 values are
// exact in fp32, as in the CUDA-core router; only the order of the fp32 sums
// differs.
//
// CTA (6 warps) computes one 128 x 128 logit tile:
//   warp 0   allocates 128 tensor-memory columns; lane 0 streams, per
//            64-element K stage, the 128 x 128-byte h and Wr tiles (2D TMA,
//            128-byte swizzle, no multicast; rows past T or E read as zero)
//            into a 3-stage ring;
//   warp 1   lane 0 issues the stage's 4 MMAs and commits to the stage's
//            empty barrier;
//   warps 2-5 wait for the last commit, read their 32-lane quadrant of the
//            accumulator with tcgen05.ld, add the bias and store fp32 logits.
#include <cuda.h>

#include <mutex>

#include "internal.h"
#include "tcgen05.cuh"

namespace nvfp4 {

namespace router_tc {
constexpr int BT = 128, BE = 128, BKB = 128;  // tile rows, K bytes per stage (64 bf16)
constexpr int kStages = 3;
constexpr int kTile = 128 * BKB;
constexpr int kStageBytes = 2 * kTile;
constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 256;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 128;
}  // namespace router_tc

// kind::f16 instruction descriptor: fp32 accumulator, A and B bf16, K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] x B[smem]^T, kind::f16.
NVFP4_DEV void mma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__global__ void __launch_bounds__(router_tc::kThreads, 1)
    router_logits_tc_kernel(const __grid_constant__ CUtensorMap map_h, const __grid_constant__ CUtensorMap map_w,
                            const float* __restrict__ bias, int64_t T, int64_t H, int32_t E,
                            float* __restrict__ logits, int* status) {
    using namespace router_tc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* accum = empty + kStages;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(accum + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * BT;
    const int64_t e0 = (int64_t)blockIdx.y * BE;
    const int nk = (int)(H * 2 / BKB);

    if (warp == 0) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 32) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accum, 1);
        fence_barrier_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&map_h);
            prefetch_tensormap(&map_w);
            for (int kt = 0; kt < nk; ++kt) {
                const int slot = kt % kStages;
                if (kt >= kStages && !mbar_wait(&empty[slot], ((kt / kStages) - 1) & 1, status)) break;
                uint8_t* st = smem + slot * kStageBytes;
                mbar_expect_tx(&full[slot], kStageBytes);
                tma_load_2d(st, &map_h, &full[slot], kt * BKB, (int)t0);
                tma_load_2d(st + kTile, &map_w, &full[slot], kt * BKB, (int)e0);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(BT, BE);
            bool ok = true;
            for (int kt = 0; kt < nk; ++kt) {
                const int slot = kt % kStages;
                if (!mbar_wait(&full[slot], (kt / kStages) & 1, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t st = smem_u32(smem + slot * kStageBytes);
#pragma unroll
                for (int j = 0; j < 4; ++j)  // K = 16 bf16 = 32 bytes per instruction
                    mma_f16_ss(tmem, sdesc_sw128_kmajor(st + 32 * j), sdesc_sw128_kmajor(st + kTile + 32 * j), idesc,
                               (kt > 0 || j > 0) ? 1u : 0u);
                tc_commit(&empty[slot]);
            }
            if (ok) tc_commit(accum);
        }
    } else {
        // epilogue: warps 2..5 -> tensor-memory lane quadrants 2, 3, 0, 1
        const int q = warp & 3;
        const bool ok = mbar_wait(accum, 0, status);
        tc_fence_after();
        const int64_t t = t0 + 32 * q + lane;
        for (int c0 = 0; c0 < BE; c0 += 32) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + c0, r);
            tmem_ld_wait();
            if (!ok || t >= T) continue;
            const int64_t e = e0 + c0;
            float* row = logits + t * E + e;
            if (e + 32 <= E && (E & 3) == 0) {
#pragma unroll
                for (int u = 0; u < 32; u += 4) {
                    float4 v = make_float4(__uint_as_float(r[u]), __uint_as_float(r[u + 1]),
                                           __uint_as_float(r[u + 2]), __uint_as_float(r[u + 3]));
                    if (bias) {
                        v.x += bias[e + u];
                        v.y += bias[e + u + 1];
                        v.z += bias[e + u + 2];
                        v.w += bias[e + u + 3];
                    }
                    *reinterpret_cast<float4*>(row + u) = v;
                }
            } else {
                for (int u = 0; u < 32; ++u)
                    if (e + u < E) row[u] = __uint_as_float(r[u]) + (bias ? bias[e + u] : 0.0f);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---- small token counts (T <= 64): experts as M, tokens as N, split K ----------
//
// For a decode batch the token count is far below an M = 128 tile, so the
// roles swap: A = 128 router rows (experts), B = the T token rows padded to
// NP = 16, 32, 48 or 64 (TMA reads rows past T as zero), D = [128 experts, NP
// tokens] in tensor memory.  K is split over a cluster of QS CTAs so that the
// 2 MB router weight streams over many SMs; each CTA's fp32 partial goes to
// rank 0 through distributed shared memory and rank 0 adds the QS partials in
// rank order (deterministic) plus the bias.
//   warp 0   tensor memory; lane 0 streams its K stages: the router rows first
//            (weights: requested before griddepcontrol.wait), the token rows
//            after it
//   warp 1   lane 0 issues 4 MMAs (K = 16) per 64-element stage
//   warps 2-5 read their 32-expert quadrant of the partial with tcgen05.ld
namespace router_tcs {
constexpr int kMaxStages = 8;
constexpr int kATile = 128 * 128;         // 128 experts x 64 bf16
constexpr int kBTile = 64 * 128;          // up to 64 tokens x 64 bf16
constexpr int kStageBytes = kATile + kBTile;
constexpr int kRedBytes = 128 * 1024;     // QS partials of [NP][128] fp32 (reuses the ring)
constexpr int kSmemBytes = 1024 + (kMaxStages * kStageBytes > kRedBytes ? kMaxStages * kStageBytes : kRedBytes) + 256;
}  // namespace router_tcs

template <int NP>
__global__ void __launch_bounds__(router_tc::kThreads, 1)
    router_logits_tcs_kernel(const __grid_constant__ CUtensorMap map_h, const __grid_constant__ CUtensorMap map_w,
                             const float* __restrict__ bias, int64_t T, int64_t H, int32_t E, int QS,
                             float* __restrict__ logits, int* status) {
    using namespace router_tcs;
    constexpr uint32_t kCols = NP <= 32 ? 32 : 64;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int nk = (int)(H / 64);
    const int q = (int)(blockIdx.x % QS);
    const int64_t e0 = (int64_t)(blockIdx.x / QS) * 128;
    const int k_begin = nk * q / QS, k_end = nk * (q + 1) / QS, ns = k_end - k_begin;
    const int ring = ns < kMaxStages ? ns : kMaxStages;
    uint8_t* bars_base = smem + (kMaxStages * kStageBytes > kRedBytes ? kMaxStages * kStageBytes : kRedBytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(bars_base);
    uint64_t* empty = full + kMaxStages;
    uint64_t* accum = empty + kMaxStages;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(accum + 1);
    float* s_red = reinterpret_cast<float*>(smem);  // [QS][NP][128], after every MMA of the cluster is done

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0) {
        tmem_alloc(s_tmem, kCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 32) {
        for (int s = 0; s < kMaxStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accum, 1);
        fence_barrier_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    griddep_launch_dependents();

    float part[NP];
    bool ok = true;
    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&map_h);
            prefetch_tensormap(&map_w);
            // the router rows of the first ring of stages go out before the wait
            for (int s = 0; s < ring; ++s) {
                mbar_expect_tx(&full[s], kATile + NP * 128);
                tma_load_2d(smem + s * kStageBytes, &map_w, &full[s], (k_begin + s) * 128, (int)e0);
            }
            griddep_wait();
            for (int s = 0; s < ns; ++s) {
                const int slot = s % ring;
                uint8_t* st = smem + slot * kStageBytes;
                if (s >= ring) {
                    if (!mbar_wait(&empty[slot], ((s / ring) - 1) & 1, status)) break;
                    mbar_expect_tx(&full[slot], kATile + NP * 128);
                    tma_load_2d(st, &map_w, &full[slot], (k_begin + s) * 128, (int)e0);
                }
                tma_load_2d(st + kATile, &map_h, &full[slot], (k_begin + s) * 128, 0);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(128, NP);
            for (int s = 0; s < ns; ++s) {
                const int slot = s % ring;
                if (!mbar_wait(&full[slot], (s / ring) & 1, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t st = smem_u32(smem + slot * kStageBytes);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_f16_ss(tmem, sdesc_sw128_kmajor(st + 32 * j), sdesc_sw128_kmajor(st + kATile + 32 * j), idesc,
                               (s > 0 || j > 0) ? 1u : 0u);
                tc_commit(&empty[slot]);
            }
            if (ok) tc_commit(accum);
        }
    } else {
        const int qd = warp & 3;
        ok = mbar_wait(accum, 0, status);
        tc_fence_after();
        uint32_t r[32];
#pragma unroll
        for (int c0 = 0; c0 < NP; c0 += 32) {
            tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * qd) << 16) + c0, r);
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 32; ++u)
                if (c0 + u < NP) part[c0 + u] = ok ? __uint_as_float(r[u]) : 0.0f;
        }
    }
    tc_fence_before();
    __syncwarp();
    cluster_sync();  // every MMA of the cluster has completed: rank 0's ring is free for the partials
    if (warp >= 2) {
        const int el = 32 * (warp & 3) + lane;  // expert within the tile
#pragma unroll
        for (int t = 0; t < NP; ++t) {
            float* slot = s_red + ((int64_t)q * NP + t) * 128 + el;
            if (q == 0) *slot = part[t];
            else st_dsmem_f32(slot, 0, part[t]);
        }
    }
    cluster_sync();  // the partials are in rank 0's shared memory
    if (q == 0) {
        for (int idx = threadIdx.x; idx < NP * 128; idx += router_tc::kThreads) {
            const int t = idx >> 7, el = idx & 127;
            const int64_t e = e0 + el;
            if (t >= T || e >= E) continue;
            float v = s_red[idx];
            for (int qq = 1; qq < QS; ++qq) v += s_red[(int64_t)qq * NP * 128 + idx];
            logits[(int64_t)t * E + e] = v + (bias ? bias[e] : 0.0f);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kCols);
    }
}

bool router_tcs_supported(const void* h, const void* wr, int64_t T, int64_t H, int32_t E) {
    return T >= 1 && T <= 64 && H % 64 == 0 && H >= 64 && H * 2 <= ((int64_t)1 << 32) && E <= 65535 * 16 &&
           ((uintptr_t)h & 15) == 0 && ((uintptr_t)wr & 15) == 0;
}

template <int NP>
static int launch_tcs(const CUtensorMap& mh, const CUtensorMap& mw, const float* bias, int64_t T, int64_t H,
                      int32_t E, float* logits, int* status, cudaStream_t st) {
    using namespace router_tcs;
    auto kern = router_logits_tcs_kernel<NP>;
    static std::once_flag once;
    std::call_once(once, [&] { cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes); });
    const int nk = (int)(H / 64);
    int QS = kRedBytes / (NP * 128 * 4);  // partials that fit the reduction buffer
    if (QS > 8) QS = 8;
    if (QS > nk) QS = nk;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(((E + 127) / 128) * QS), 1, 1);
    cfg.blockDim = dim3(router_tc::kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)QS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    set_pdl_attr(attr[1]);
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, mh, mw, bias, T, H, E, QS, logits, status) == cudaSuccess ? NVFP4_OK
                                                                                                    : NVFP4_ERR_LAUNCH;
}

int launch_router_logits_tcs(const void* h, const void* wr, const float* bias, int64_t T, int64_t H, int32_t E,
                             float* logits, int* status, cudaStream_t st) {
    const int NP = (int)((T + 15) / 16 * 16);
    CUtensorMap mh, mw;
    if (!make_tmap_2d_u8(&mh, h, (uint64_t)(H * 2), (uint64_t)T, 128, (uint32_t)NP, 1)) return NVFP4_ERR_LAUNCH;
    if (!make_tmap_2d_u8(&mw, wr, (uint64_t)(H * 2), (uint64_t)E, 128, 128, 1)) return NVFP4_ERR_LAUNCH;
    switch (NP) {
        case 16: return launch_tcs<16>(mh, mw, bias, T, H, E, logits, status, st);
        case 32: return launch_tcs<32>(mh, mw, bias, T, H, E, logits, status, st);
        case 48: return launch_tcs<48>(mh, mw, bias, T, H, E, logits, status, st);
        default: return launch_tcs<64>(mh, mw, bias, T, H, E, logits, status, st);
    }
}

bool router_tc_supported(const void* h, const void* wr, int64_t T, int64_t H, int32_t E) {
    return T > 64 && H % 64 == 0 && H * 2 <= ((int64_t)1 << 32) && T < ((int64_t)1 << 31) - router_tc::BT &&
           E <= 65535 * router_tc::BE && ((uintptr_t)h & 15) == 0 && ((uintptr_t)wr & 15) == 0;
}

int launch_router_logits_tc(const void* h, const void* wr, const float* bias, int64_t T, int64_t H, int32_t E,
                            float* logits, int* status, cudaStream_t st) {
    using namespace router_tc;
    CUtensorMap mh, mw;
    if (!make_tmap_2d_u8(&mh, h, (uint64_t)(H * 2), (uint64_t)T, BKB, BT, 1)) return NVFP4_ERR_LAUNCH;
    if (!make_tmap_2d_u8(&mw, wr, (uint64_t)(H * 2), (uint64_t)E, BKB, BE, 1)) return NVFP4_ERR_LAUNCH;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaFuncSetAttribute(router_logits_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    });
    dim3 grid((unsigned)((T + BT - 1) / BT), (unsigned)((E + BE - 1) / BE));
    router_logits_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(mh, mw, bias, T, H, E, logits, status);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

}  // namespace nvfp4
