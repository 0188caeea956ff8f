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
