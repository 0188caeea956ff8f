// K4: W4A4 linear on tcgen05 block-scaled tensor cores (kind::mxf4nvf4).
//
// Prefill runs in 2,048-token chunks on FP4 tensor cores (Ignis README,
// "How fast"; "Credits": split-K prefill, the NVFP4-full target).  With both
// operands NVFP4,
//
//   y[m, n] = gs_x * gs_w * sum_k E2M1(cx[m,k]) E4M3(sx[m,k/16]) E2M1(cw[n,k]) E4M3(sw[n,k/16])
//
// is one block-scaled MMA chain: the tensor core applies the per-16 E4M3
// scales of both operands and accumulates in fp32 in tensor memory; the two
// per-tensor scales are applied in the epilogue.
//
// CTA (6 warps) computes one 128 x 128 output tile:
//   warp 0   allocates tensor memory; lane 0 streams, per 256-element K tile,
//            A (128 x 128 B) and B (128 x 128 B) with 2D TMA (128-byte
//            swizzle, no multicast) and their scale factors (two 2 KB runs of
//            512-byte atoms, bulk copies) into a 3-stage ring;
//   warp 1   lane 0 copies the scale atoms to tensor memory (tcgen05.cp,
//            32x128b.warpx4) and issues 4 MMAs of K = 64 per stage, then
//            commits to the stage's empty barrier;
//   warps 2-5 wait for the last commit, read the 128 x 128 fp32 accumulator
//            with tcgen05.ld (each warp its 32-lane quadrant), scale by
//            gs_x * gs_w and store.
// Two CTAs fit on an SM (108 KB of shared memory, 256 tensor-memory columns
// each), so one CTA's epilogue overlaps the other's main loop.
#include <cuda.h>

#include <mutex>

#include "internal.h"
#include "tcgen05.cuh"

namespace nvfp4 {

namespace w4a4 {
constexpr int BM = 128, BN = 128, BK = 256;   // BK elements = 128 bytes per row
constexpr int kStages = 3;
constexpr int kABytes = BM * 128, kBBytes = BN * 128, kSfBytes = 2048;
constexpr int kStageBytes = kABytes + kBBytes + 2 * kSfBytes;
constexpr int kThreads = 192;
constexpr int kTmemCols = 256;                // 128 accumulator + 2 x 32 scale-factor columns
constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 256;
}  // namespace w4a4

struct GemmArgs {
    int64_t M, N, K;
    const uint8_t* sfa;   // activation scales, TILED layout for M rows
    const uint8_t* sfb;   // weight scales, TILED layout for N rows
    const float* gs_a;
    const float* gs_b;
    void* y;
    int64_t ldy;
    int* status;
};

template <typename OutT>
__global__ void __launch_bounds__(w4a4::kThreads, 2)
    gemm_w4a4_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                     const GemmArgs a) {
    using namespace w4a4;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* accum = empty + kStages;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(accum + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t m0 = (int64_t)blockIdx.x * BM, n0 = (int64_t)blockIdx.y * BN;
    const int nk = (int)(a.K / BK);
    const int64_t cp4 = a.K / 64;   // scale atoms per 128 rows

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
            prefetch_tensormap(&map_a);
            prefetch_tensormap(&map_b);
            const uint8_t* sfa = a.sfa + (m0 / 128) * cp4 * 512;
            const uint8_t* sfb = a.sfb + (n0 / 128) * cp4 * 512;
            for (int kt = 0; kt < nk; ++kt) {
                const int slot = kt % kStages;
                if (kt >= kStages && !mbar_wait(&empty[slot], ((kt / kStages) - 1) & 1, a.status)) break;
                uint8_t* st = smem + slot * kStageBytes;
                mbar_expect_tx(&full[slot], kStageBytes);
                tma_load_2d(st, &map_a, &full[slot], kt * 128, (int)m0);
                tma_load_2d(st + kABytes, &map_b, &full[slot], kt * 128, (int)n0);
                bulk_load(st + kABytes + kBBytes, sfa + (int64_t)kt * 4 * 512, kSfBytes, &full[slot]);
                bulk_load(st + kABytes + kBBytes + kSfBytes, sfb + (int64_t)kt * 4 * 512, kSfBytes, &full[slot]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_nvf4(BM, BN);
            bool ok = true;
            for (int kt = 0; kt < nk; ++kt) {
                const int slot = kt % kStages;
                if (!mbar_wait(&full[slot], (kt / kStages) & 1, a.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t st = smem_u32(smem + slot * kStageBytes);
                const uint32_t sf_col = 128 + (kt & 1) * 32;   // double-buffered scale-factor columns
                for (int j = 0; j < 4; ++j) {
                    tmem_cp_sf_atom(tmem + sf_col + 4 * j, sdesc_sf_atom(st + kABytes + kBBytes + 512 * j));
                    tmem_cp_sf_atom(tmem + sf_col + 16 + 4 * j,
                                    sdesc_sf_atom(st + kABytes + kBBytes + kSfBytes + 512 * j));
                }
                for (int j = 0; j < 4; ++j) {
                    mma_nvf4(tmem, sdesc_sw128_kmajor(st + 32 * j), sdesc_sw128_kmajor(st + kABytes + 32 * j), idesc,
                             tmem + sf_col + 4 * j, tmem + sf_col + 16 + 4 * j, (kt > 0 || j > 0) ? 1u : 0u);
                }
                tc_commit(&empty[slot]);
            }
            if (ok) tc_commit(accum);
        }
    } else {
        // epilogue: warps 2..5 -> tensor-memory lane quadrants 2, 3, 0, 1
        const int q = warp & 3;
        const bool ok = mbar_wait(accum, 0, a.status);
        tc_fence_after();
        const float g = ok ? a.gs_a[0] * a.gs_b[0] : 0.0f;
        const int64_t row = m0 + 32 * q + lane;
        OutT* yrow = reinterpret_cast<OutT*>(a.y) + row * a.ldy;
        for (int c0 = 0; c0 < BN; c0 += 32) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + c0, r);
            tmem_ld_wait();
            if (!ok || row >= a.M) continue;
            const int64_t col = n0 + c0;
            if (col + 32 <= a.N && (a.ldy & 7) == 0) {
                if constexpr (sizeof(OutT) == 4) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4*>(yrow + col + i) =
                            make_float4(__uint_as_float(r[i]) * g, __uint_as_float(r[i + 1]) * g,
                                        __uint_as_float(r[i + 2]) * g, __uint_as_float(r[i + 3]) * g);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint32_t w[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(r[i + 2 * u]) * g,
                                                                            __uint_as_float(r[i + 2 * u + 1]) * g);
                            w[u] = *reinterpret_cast<const uint32_t*>(&b2);
                        }
                        *reinterpret_cast<uint4*>(yrow + col + i) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            } else {
                for (int i = 0; i < 32; ++i)
                    if (col + i < a.N) store_out<OutT>(yrow + col + i, __uint_as_float(r[i]) * g);
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

template <typename OutT>
static int launch_typed(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& a, cudaStream_t st) {
    using namespace w4a4;
    auto kern = gemm_w4a4_kernel<OutT>;
    static std::once_flag once;
    std::call_once(once, [&] { cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes); });
    dim3 grid((unsigned)((a.M + BM - 1) / BM), (unsigned)((a.N + BN - 1) / BN));
    kern<<<grid, kThreads, kSmemBytes, st>>>(ma, mb, a);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

int launch_gemm_w4a4(const uint8_t* a_codes, const uint8_t* a_scales, const float* gs_a, int64_t M, int64_t K,
                     const uint8_t* b_codes, const uint8_t* b_scales, const float* gs_b, int64_t N, void* y,
                     int y_dtype, int* status, cudaStream_t st) {
    if ((M + w4a4::BM - 1) / w4a4::BM > 0x7fffffff || (N + w4a4::BN - 1) / w4a4::BN > 65535) return NVFP4_ERR_SHAPE;
    CUtensorMap ma, mb;
    if (!make_tmap_2d_u8(&ma, a_codes, (uint64_t)(K / 2), (uint64_t)M, 128, w4a4::BM, 1)) return NVFP4_ERR_LAUNCH;
    if (!make_tmap_2d_u8(&mb, b_codes, (uint64_t)(K / 2), (uint64_t)N, 128, w4a4::BN, 1)) return NVFP4_ERR_LAUNCH;
    GemmArgs a{};
    a.M = M;
    a.N = N;
    a.K = K;
    a.sfa = a_scales;
    a.sfb = b_scales;
    a.gs_a = gs_a;
    a.gs_b = gs_b;
    a.y = y;
    a.ldy = N;
    a.status = status;
    if (y_dtype == NVFP4_DTYPE_BF16) return launch_typed<__nv_bfloat16>(ma, mb, a, st);
    return launch_typed<float>(ma, mb, a, st);
}

}  // namespace nvfp4
