// K4 / K7: W4A4 linear on tcgen05 block-scaled tensor cores (kind::mxf4nvf4),
// dense and grouped by expert.
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
// CTA (6 warps) computes one 128-row tile against one (or, for SwiGLU, two)
// 128-row weight tiles:
//   warp 0   allocates tensor memory; lane 0 streams, per 256-element K tile,
//            A and B (128 x 128 B each, 2D TMA with 128-byte swizzle, no
//            multicast) and their scale factors (2 KB runs of 512-byte atoms,
//            bulk copies) into a 3-stage ring;
//   warp 1   lane 0 copies the scale atoms to tensor memory (tcgen05.cp
//            32x128b.warpx4) and issues 4 MMAs of K = 64 per B tile and stage,
//            then commits to the stage's empty barrier;
//   warps 2-5 wait for the last commit, read the fp32 accumulators with
//            tcgen05.ld (each warp its 32-lane quadrant) into registers and
//            apply the epilogue; warp 0 then frees the tensor memory while
//            they stage the tile in the idle ring's shared memory and write
//            it out one contiguous output-row run per warp instruction.
//
// Grouped form (mixture of experts; CHImp Alpha v1.0 model card, "How it fits
// on one GPU"): the permuted activations are laid out with each expert's rows
// padded to whole 128-row tiles, and a tile table gives each 128-row tile its
// expert, its first output row and its number of real rows; tiles past the
// last expert exit at once.  The weight tile comes from the expert's rows of
// the stacked [E * N, K/2] codes and the expert's scale block and gs.
// Epilogues: NONE (y = acc * g); SWIGLU (gate tile = rows j0.. of the expert,
// up tile = rows N/2 + j0..: two N = 128 MMAs into two accumulators, then
// y = silu(g) * u).  The weighted combine of the experts' rows runs after the
// GEMM, as a gather in slot order (moe.cu), so its sums are deterministic.
#include <cuda.h>

#include <mutex>

#include "internal.h"
#include "tcgen05.cuh"

namespace nvfp4 {

namespace w4a4 {
constexpr int BM = 128, BN = 128, BK = 256;  // BK elements = 128 bytes per row
constexpr int kStages = 3;
constexpr int kTile = 128 * 128, kSf = 2048;
constexpr int kThreads = 192;
constexpr int kOutStride = BN + 4;  // staged output row, floats (16-byte rows, conflict-free float4 stores)
template <int NB>
struct Cfg {
    static constexpr int kStageBytes = kTile * (1 + NB) + kSf * (1 + NB);
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 256;
    static constexpr int kSfCols = 16 * (1 + NB);                 // per scale-factor buffer
    static constexpr int kTmemCols = (128 * NB + 2 * kSfCols) <= 256 ? 256 : 512;
};
}  // namespace w4a4

struct GemmArgs {
    int64_t M, N, K;           // M: rows of A (padded rows when grouped); N: weight rows per expert
    const uint8_t* sfa;        // A scales, TILED
    const uint8_t* sfb;        // B scales, TILED (grouped: expert e at sfb + e * sf_stride)
    int64_t sf_stride;
    const float* gs_a;
    const float* gs_b;         // [1] or [E]
    const int32_t* tile_info;  // grouped: per 128-row tile {expert, first output row, real rows}
    void* y;
    int64_t ldy;
    int* status;
};

// silu(g) = g * sigmoid(g) with the hardware exponential and divide (a few
// ulp; the IEEE-rounded expf and division cost 10x more here, where one warp
// per scheduler runs the epilogue and nothing hides their latency).
NVFP4_DEV float silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

template <typename OutT, int EPI, bool GROUPED>
__global__ void __launch_bounds__(w4a4::kThreads, 1)
    gemm_w4a4_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                     const GemmArgs a) {
    using namespace w4a4;
    constexpr int NB = (EPI == NVFP4_EPI_SWIGLU) ? 2 : 1;
    using C = Cfg<NB>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * C::kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* accum = empty + kStages;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(accum + 1);

    // tile -> expert, output rows (uniform for the CTA; exits before any setup)
    int expert = 0, nvalid;
    int64_t out_row0;
    const int64_t m0 = (int64_t)blockIdx.x * BM;
    if constexpr (GROUPED) {
        const int32_t* ti = a.tile_info + 3 * (int64_t)blockIdx.x;
        expert = ti[0];
        if (expert < 0) return;
        out_row0 = ti[1];
        nvalid = ti[2];
    } else {
        out_row0 = m0;
        nvalid = (int)((a.M - m0) < BM ? (a.M - m0) : BM);
    }
    const int64_t col0 = (int64_t)blockIdx.y * BN;  // output column tile (SWIGLU: of N/2)
    int64_t brow[NB];                               // first weight row of each B tile, within the expert
    if constexpr (EPI == NVFP4_EPI_SWIGLU) {
        brow[0] = col0;
        brow[NB - 1] = a.N / 2 + col0;
    } else {
        brow[0] = col0;
    }

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = (int)(a.K / BK);
    const int64_t cp4 = a.K / 64;  // scale atoms per 128 rows

    if (warp == 0) {
        tmem_alloc(s_tmem, C::kTmemCols);
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
    // A programmatic dependent of the activation quantizer: the setup above
    // overlaps its tail; nothing it writes is read before this point.
    griddep_wait();

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&map_a);
            prefetch_tensormap(&map_b);
            const uint8_t* sfa = a.sfa + (m0 / 128) * cp4 * 512;
            const uint8_t* sfb_e = a.sfb + (int64_t)expert * a.sf_stride;
            for (int kt = 0; kt < nk; ++kt) {
                const int slot = kt % kStages;
                if (kt >= kStages && !mbar_wait(&empty[slot], ((kt / kStages) - 1) & 1, a.status)) break;
                uint8_t* st = smem + slot * C::kStageBytes;
                mbar_expect_tx(&full[slot], C::kStageBytes);
                tma_load_2d(st, &map_a, &full[slot], kt * 128, (int)m0);
#pragma unroll
                for (int b = 0; b < NB; ++b)
                    tma_load_2d(st + kTile * (1 + b), &map_b, &full[slot], kt * 128,
                                (int)((int64_t)expert * a.N + brow[b]));
                uint8_t* sf = st + kTile * (1 + NB);
                bulk_load(sf, sfa + (int64_t)kt * 4 * 512, kSf, &full[slot]);
#pragma unroll
                for (int b = 0; b < NB; ++b)
                    bulk_load(sf + kSf * (1 + b), sfb_e + ((brow[b] / 128) * cp4 + (int64_t)kt * 4) * 512, kSf,
                              &full[slot]);
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
                const uint32_t st = smem_u32(smem + slot * C::kStageBytes);
                const uint32_t sf = st + kTile * (1 + NB);
                const uint32_t sf_col = 128 * NB + (kt & 1) * C::kSfCols;  // double-buffered scale columns
                for (int j = 0; j < 4; ++j)
                    for (int b = 0; b <= NB; ++b)  // b = 0: A's atoms, b >= 1: B tile b-1's atoms
                        tmem_cp_sf_atom(tmem + sf_col + 16 * b + 4 * j, sdesc_sf_atom(sf + kSf * b + 512 * j));
                for (int b = 0; b < NB; ++b)
                    for (int j = 0; j < 4; ++j)
                        mma_nvf4(tmem + 128 * b, sdesc_sw128_kmajor(st + 32 * j),
                                 sdesc_sw128_kmajor(st + kTile * (1 + b) + 32 * j), idesc, tmem + sf_col + 4 * j,
                                 tmem + sf_col + 16 * (1 + b) + 4 * j, (kt > 0 || j > 0) ? 1u : 0u);
                tc_commit(&empty[slot]);
            }
            if (ok) tc_commit(accum);
        }
    } else {
        // epilogue: warps 2..5 -> tensor-memory lane quadrants 2, 3, 0, 1.  The
        // whole accumulator row goes to registers first; then warp 0 frees the
        // tensor memory while the stores run.
        const int q = warp & 3;
        const bool ok = mbar_wait(accum, 0, a.status);
        tc_fence_after();
        const int i = 32 * q + lane;  // row within the tile
        const float g = ok ? a.gs_a[0] * a.gs_b[GROUPED ? expert : 0] : 0.0f;
        uint32_t r[BN / 32][32];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
            tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + 32 * c, r[c]);
            if constexpr (EPI == NVFP4_EPI_SWIGLU) {
                uint32_t u[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + 128 + 32 * c, u);
                tmem_ld_wait();
#pragma unroll
                for (int t = 0; t < 32; ++t)
                    r[c][t] = __float_as_uint(silu(__uint_as_float(r[c][t]) * g) * (__uint_as_float(u[t]) * g));
            } else {
                tmem_ld_wait();
#pragma unroll
                for (int t = 0; t < 32; ++t) r[c][t] = __float_as_uint(__uint_as_float(r[c][t]) * g);
            }
        }
        tc_fence_before();
        asm volatile("bar.arrive 2, 160;" ::: "memory");  // warps 2-5 done with tensor memory
        // Stage the tile in shared memory (the ring is idle: every MMA that read
        // it has completed), then write it out row by row so that a warp's
        // stores (or reductions) cover contiguous runs of one output row.
        float* so = reinterpret_cast<float*>(smem);  // [BM][kOutStride]
#pragma unroll
        for (int c = 0; c < BN / 32; ++c)
#pragma unroll
            for (int t = 0; t < 32; t += 4)
                *reinterpret_cast<float4*>(so + i * kOutStride + 32 * c + t) =
                    make_float4(__uint_as_float(r[c][t]), __uint_as_float(r[c][t + 1]), __uint_as_float(r[c][t + 2]),
                                __uint_as_float(r[c][t + 3]));
        asm volatile("bar.sync 3, 128;" ::: "memory");
        const int64_t ncols = (EPI == NVFP4_EPI_SWIGLU) ? a.N / 2 : a.N;
        const int64_t col = col0 + 4 * lane;  // this lane's 4 columns
        const int nrows = ok ? nvalid : 0;
        for (int rr = warp - 2; rr < nrows; rr += 4) {
            const float4 v = *reinterpret_cast<const float4*>(so + rr * kOutStride + 4 * lane);
            const float vv[4] = {v.x, v.y, v.z, v.w};
            const int64_t orow = out_row0 + rr;
            {
                OutT* yp = reinterpret_cast<OutT*>(a.y) + orow * a.ldy + col;
                if (col + 4 <= ncols && (a.ldy & 3) == 0) {
                    if constexpr (sizeof(OutT) == 4) {
                        *reinterpret_cast<float4*>(yp) = v;
                    } else {
                        const __nv_bfloat162 b0 = __floats2bfloat162_rn(v.x, v.y);
                        const __nv_bfloat162 b1 = __floats2bfloat162_rn(v.z, v.w);
                        *reinterpret_cast<uint2*>(yp) =
                            make_uint2(*reinterpret_cast<const uint32_t*>(&b0), *reinterpret_cast<const uint32_t*>(&b1));
                    }
                } else {
                    for (int t = 0; t < 4; ++t)
                        if (col + t < ncols) store_out<OutT>(yp + t, vv[t]);
                }
            }
        }
    }
    if (warp == 0) {
        // every MMA completed before the epilogue read the accumulator
        asm volatile("bar.sync 2, 160;" ::: "memory");
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <typename OutT, int EPI, bool GROUPED>
static int launch_typed(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& a, int64_t m_tiles,
                        cudaStream_t st) {
    using namespace w4a4;
    constexpr int NB = (EPI == NVFP4_EPI_SWIGLU) ? 2 : 1;
    auto kern = gemm_w4a4_kernel<OutT, EPI, GROUPED>;
    static std::once_flag once;
    std::call_once(once,
                   [&] { cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<NB>::kSmemBytes); });
    const int64_t ncols = (EPI == NVFP4_EPI_SWIGLU) ? a.N / 2 : a.N;
    cudaLaunchAttribute attr[1];
    set_pdl_attr(attr[0]);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)m_tiles, (unsigned)((ncols + BN - 1) / BN));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = Cfg<NB>::kSmemBytes;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, ma, mb, a) == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
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
    const int64_t mt = (M + w4a4::BM - 1) / w4a4::BM;
    if (y_dtype == NVFP4_DTYPE_BF16) return launch_typed<__nv_bfloat16, NVFP4_EPI_NONE, false>(ma, mb, a, mt, st);
    return launch_typed<float, NVFP4_EPI_NONE, false>(ma, mb, a, mt, st);
}

int launch_gemm_w4a4_grouped(const uint8_t* a_codes, const uint8_t* a_scales, const float* gs_a, int64_t rows_pad,
                             int64_t K, const int32_t* tile_info, const uint8_t* w_codes, const uint8_t* w_scales,
                             int64_t sf_stride, const float* w_gs, int32_t E, int64_t N, int epilogue, void* y,
                             int y_dtype, int* status, cudaStream_t st) {
    CUtensorMap ma, mb;
    if (!make_tmap_2d_u8(&ma, a_codes, (uint64_t)(K / 2), (uint64_t)rows_pad, 128, w4a4::BM, 1)) return NVFP4_ERR_LAUNCH;
    if (!make_tmap_2d_u8(&mb, w_codes, (uint64_t)(K / 2), (uint64_t)E * (uint64_t)N, 128, w4a4::BN, 1))
        return NVFP4_ERR_LAUNCH;
    GemmArgs a{};
    a.M = rows_pad;
    a.N = N;
    a.K = K;
    a.sfa = a_scales;
    a.sfb = w_scales;
    a.sf_stride = sf_stride;
    a.gs_a = gs_a;
    a.gs_b = w_gs;
    a.tile_info = tile_info;
    a.y = y;
    a.status = status;
    const int64_t mt = rows_pad / w4a4::BM;
    if (epilogue == NVFP4_EPI_SWIGLU) {
        a.ldy = N / 2;
        if (y_dtype == NVFP4_DTYPE_BF16) return launch_typed<__nv_bfloat16, NVFP4_EPI_SWIGLU, true>(ma, mb, a, mt, st);
        return launch_typed<float, NVFP4_EPI_SWIGLU, true>(ma, mb, a, mt, st);
    }
    a.ldy = N;
    if (y_dtype == NVFP4_DTYPE_BF16) return launch_typed<__nv_bfloat16, NVFP4_EPI_NONE, true>(ma, mb, a, mt, st);
    return launch_typed<float, NVFP4_EPI_NONE, true>(ma, mb, a, mt, st);
}

}  // namespace nvfp4
