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
// Persistent CTAs (6 warps) walk 128 x 128 output tiles (for SwiGLU: 128
// rows x 128 outputs from two 128-row weight tiles) in a static round-robin
// order.  The CTAs running at one time cover consecutive tiles, so the
// operand they share stays in L2: dense, the row tile runs fastest when the
// activations are the smaller operand (each weight tile is then fetched from
// DRAM once) and the column tile otherwise; grouped, the column tile runs
// fastest (a row tile's activations are reused across the expert's columns):
//   warp 0   allocates tensor memory; lane 0 streams, per 256-element K
//            step, A and B (128 x 128 B each, 2D TMA with 128-byte swizzle,
//            no multicast) and their scale factors (2 KB runs of 512-byte
//            atoms, bulk copies) into a 3-stage ring that runs on across
//            tile boundaries, so the next tile's operands arrive while the
//            current tile's epilogue runs;
//   warp 1   lane 0 copies the scale atoms to tensor memory (tcgen05.cp
//            32x128b.warpx4) and issues 4 MMAs of K = 64 per B tile and
//            step, commits each step to the stage's empty barrier and each
//            finished tile to the accumulator barrier; before a tile's first
//            MMA it waits until the epilogue has read the previous tile's
//            accumulator out of tensor memory;
//   warps 2-5 read the fp32 accumulators with tcgen05.ld (each warp its
//            32-lane quadrant) into registers, release the accumulator, then
//            apply the epilogue and store each thread's output row.
// Two CTAs share an SM (one for SwiGLU, whose two accumulators fill tensor
// memory), so one CTA's MMAs run while the other's issuing thread waits.
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
    int64_t m_tiles;           // 128-row tiles of A
    int m_fast;                // tile order: 1 row tile fastest, 0 column tile fastest
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

// Output tile `tile` -> (128-row tile m, column tile n), m or n fastest; for
// the grouped form, the m tile's expert, first output row and real rows
// (expert < 0: a padding tile, skipped by every role alike).
struct TileRef {
    int64_t m0, out_row0, col0;
    int expert, nvalid;
};

template <bool GROUPED>
NVFP4_DEV TileRef tile_ref(const GemmArgs& a, int64_t tile, int64_t ntn) {
    TileRef t;
    int64_t mt, nt;
    if (a.m_fast) {
        nt = tile / a.m_tiles;
        mt = tile - nt * a.m_tiles;
    } else {
        mt = tile / ntn;
        nt = tile - mt * ntn;
    }
    t.col0 = nt * w4a4::BN;
    t.m0 = mt * w4a4::BM;
    if constexpr (GROUPED) {
        const int32_t* ti = a.tile_info + 3 * mt;
        t.expert = ti[0];
        t.out_row0 = ti[1];
        t.nvalid = ti[2];
    } else {
        t.expert = 0;
        t.out_row0 = t.m0;
        t.nvalid = (int)((a.M - t.m0) < w4a4::BM ? (a.M - t.m0) : w4a4::BM);
    }
    return t;
}

template <typename OutT, int EPI, bool GROUPED>
__global__ void __launch_bounds__(w4a4::kThreads, EPI == NVFP4_EPI_SWIGLU ? 1 : 2)
    gemm_w4a4_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                     const GemmArgs a) {
    using namespace w4a4;
    constexpr int NB = (EPI == NVFP4_EPI_SWIGLU) ? 2 : 1;
    using C = Cfg<NB>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * C::kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* acc_full = empty + kStages;
    uint64_t* acc_empty = acc_full + 1;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(acc_empty + 1);

    const int64_t ncols = (EPI == NVFP4_EPI_SWIGLU) ? a.N / 2 : a.N;  // output columns
    const int64_t ntn = (ncols + BN - 1) / BN;
    const int64_t ntiles = a.m_tiles * ntn;
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
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 4);  // one arrival per epilogue warp
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
            int64_t g = 0;  // K steps issued over all tiles: ring slot and phase
            bool ok = true;
            for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                const TileRef t = tile_ref<GROUPED>(a, tile, ntn);
                if (t.expert < 0) continue;
                int64_t brow[NB];
                brow[0] = t.col0;
                if constexpr (NB == 2) brow[1] = a.N / 2 + t.col0;
                const uint8_t* sfa = a.sfa + (t.m0 / 128) * cp4 * 512;
                const uint8_t* sfb_e = a.sfb + (int64_t)t.expert * a.sf_stride;
                for (int kt = 0; kt < nk; ++kt, ++g) {
                    const int slot = (int)(g % kStages);
                    if (g >= kStages && !mbar_wait(&empty[slot], (uint32_t)((g / kStages) - 1) & 1, a.status)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + slot * C::kStageBytes;
                    mbar_expect_tx(&full[slot], C::kStageBytes);
                    tma_load_2d(st, &map_a, &full[slot], kt * 128, (int)t.m0);
#pragma unroll
                    for (int b = 0; b < NB; ++b)
                        tma_load_2d(st + kTile * (1 + b), &map_b, &full[slot], kt * 128,
                                    (int)((int64_t)t.expert * a.N + brow[b]));
                    uint8_t* sf = st + kTile * (1 + NB);
                    bulk_load(sf, sfa + (int64_t)kt * 4 * 512, kSf, &full[slot]);
#pragma unroll
                    for (int b = 0; b < NB; ++b)
                        bulk_load(sf + kSf * (1 + b), sfb_e + ((brow[b] / 128) * cp4 + (int64_t)kt * 4) * 512, kSf,
                                  &full[slot]);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_nvf4(BM, BN);
            int64_t g = 0;
            uint32_t j = 0;  // tiles computed
            bool ok = true;
            for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                if (tile_ref<GROUPED>(a, tile, ntn).expert < 0) continue;
                // the epilogue has read the previous tile's accumulator
                if (j > 0 && !mbar_wait(acc_empty, (j - 1) & 1, a.status)) break;
                tc_fence_after();
                for (int kt = 0; kt < nk; ++kt, ++g) {
                    const int slot = (int)(g % kStages);
                    if (!mbar_wait(&full[slot], (uint32_t)(g / kStages) & 1, a.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + slot * C::kStageBytes);
                    const uint32_t sf = st + kTile * (1 + NB);
                    const uint32_t sf_col = 128 * NB + (uint32_t)(g & 1) * C::kSfCols;  // double-buffered scales
                    for (int q = 0; q < 4; ++q)
                        for (int b = 0; b <= NB; ++b)  // b = 0: A's atoms, b >= 1: B tile b-1's atoms
                            tmem_cp_sf_atom(tmem + sf_col + 16 * b + 4 * q, sdesc_sf_atom(sf + kSf * b + 512 * q));
                    for (int b = 0; b < NB; ++b)
                        for (int q = 0; q < 4; ++q)
                            mma_nvf4(tmem + 128 * b, sdesc_sw128_kmajor(st + 32 * q),
                                     sdesc_sw128_kmajor(st + kTile * (1 + b) + 32 * q), idesc, tmem + sf_col + 4 * q,
                                     tmem + sf_col + 16 * (1 + b) + 4 * q, (kt > 0 || q > 0) ? 1u : 0u);
                    tc_commit(&empty[slot]);
                }
                if (!ok) break;
                tc_commit(acc_full);
                ++j;
            }
        }
    } else {
        // epilogue: warps 2..5 -> tensor-memory lane quadrants 2, 3, 0, 1
        const int q = warp & 3;
        const int i = 32 * q + lane;  // row within the tile
        uint32_t j = 0;
        for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
            const TileRef t = tile_ref<GROUPED>(a, tile, ntn);
            if (t.expert < 0) continue;
            if (!mbar_wait(acc_full, j & 1, a.status)) break;
            ++j;
            tc_fence_after();
            const float g = a.gs_a[0] * a.gs_b[GROUPED ? t.expert : 0];
            // the tile row in registers: bf16 outputs packed two to a word
            constexpr bool kPack = sizeof(OutT) == 2;
            constexpr int kW = kPack ? 16 : 32;  // words per 32 columns
            uint32_t o[BN / 32][kW];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + 32 * c, r);
                float v[32];
                if constexpr (EPI == NVFP4_EPI_SWIGLU) {
                    uint32_t u[32];
                    tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + 128 + 32 * c, u);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = silu(__uint_as_float(r[e]) * g) * (__uint_as_float(u[e]) * g);
                } else {
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(r[e]) * g;
                }
#pragma unroll
                for (int e = 0; e < kW; ++e) {
                    if constexpr (kPack) {
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
                        o[c][e] = *reinterpret_cast<const uint32_t*>(&b2);
                    } else {
                        o[c][e] = __float_as_uint(v[e]);
                    }
                }
            }
            // the accumulator is in registers: the next tile's MMAs may start
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
            if (i < t.nvalid) {
                OutT* yp = reinterpret_cast<OutT*>(a.y) + (t.out_row0 + i) * a.ldy + t.col0;
                // 16-byte stores need a whole tile and 16-byte aligned rows (y itself is)
                if (t.col0 + BN <= ncols && (a.ldy * (int64_t)sizeof(OutT)) % 16 == 0) {
#pragma unroll
                    for (int c = 0; c < BN / 32; ++c)
#pragma unroll
                        for (int e = 0; e < kW; e += 4)
                            *reinterpret_cast<uint4*>(reinterpret_cast<uint32_t*>(yp + 32 * c) + e) =
                                make_uint4(o[c][e], o[c][e + 1], o[c][e + 2], o[c][e + 3]);
                } else {
#pragma unroll
                    for (int c = 0; c < BN / 32; ++c)
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            if (t.col0 + 32 * c + e >= ncols) continue;
                            float v;
                            if constexpr (kPack) {
                                const uint32_t w = o[c][e >> 1];
                                v = (e & 1) ? bf16hi_to_f32(w) : bf16lo_to_f32(w);
                            } else {
                                v = __uint_as_float(o[c][e]);
                            }
                            store_out<OutT>(yp + 32 * c + e, v);
                        }
                }
            }
        }
        tc_fence_before();
        asm volatile("bar.arrive 2, 160;" ::: "memory");  // warps 2-5 are done with tensor memory
    }
    if (warp == 0) {
        asm volatile("bar.sync 2, 160;" ::: "memory");
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int NB>
constexpr bool tmem_fits_two() { return w4a4::Cfg<NB>::kTmemCols <= 256; }

// Persistent grid: as many CTAs as fit on the GPU at once (occupancy of the
// kernel times the SM count), at most one per output tile.
template <typename OutT, int EPI, bool GROUPED>
static int launch_typed(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& a, cudaStream_t st) {
    using namespace w4a4;
    constexpr int NB = (EPI == NVFP4_EPI_SWIGLU) ? 2 : 1;
    auto kern = gemm_w4a4_kernel<OutT, EPI, GROUPED>;
    static std::once_flag once;
    static int per_sm = 1;
    std::call_once(once, [&] {
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<NB>::kSmemBytes);
        // two CTAs per SM when their registers, shared memory and tensor
        // memory (256 columns each) fit; CTAs never wait on one another, so a
        // grid larger than what is resident only queues
        cudaFuncAttributes fa;
        int dev = 0, smem_sm = 0;
        if (tmem_fits_two<NB>() && cudaFuncGetAttributes(&fa, kern) == cudaSuccess && cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) == cudaSuccess &&
            2 * fa.numRegs * kThreads <= 65536 && 2 * (Cfg<NB>::kSmemBytes + 1024) <= smem_sm)
            per_sm = 2;
    });
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        return NVFP4_ERR_LAUNCH;
    const int64_t ncols = (EPI == NVFP4_EPI_SWIGLU) ? a.N / 2 : a.N;
    const int64_t ntiles = a.m_tiles * ((ncols + BN - 1) / BN);
    const int64_t grid = ntiles < (int64_t)sms * per_sm ? ntiles : (int64_t)sms * per_sm;
    cudaLaunchAttribute attr[1];
    set_pdl_attr(attr[0]);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(grid > 0 ? grid : 1));
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
    a.m_tiles = (M + w4a4::BM - 1) / w4a4::BM;
    a.m_fast = M <= N;  // the smaller operand stays resident (A and B have the same row length)
    if (y_dtype == NVFP4_DTYPE_BF16) return launch_typed<__nv_bfloat16, NVFP4_EPI_NONE, false>(ma, mb, a, st);
    return launch_typed<float, NVFP4_EPI_NONE, false>(ma, mb, a, st);
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
    a.m_tiles = rows_pad / w4a4::BM;
    a.m_fast = 0;
    if (epilogue == NVFP4_EPI_SWIGLU) {
        a.ldy = N / 2;
        if (y_dtype == NVFP4_DTYPE_BF16) return launch_typed<__nv_bfloat16, NVFP4_EPI_SWIGLU, true>(ma, mb, a, st);
        return launch_typed<float, NVFP4_EPI_SWIGLU, true>(ma, mb, a, st);
    }
    a.ldy = N;
    if (y_dtype == NVFP4_DTYPE_BF16) return launch_typed<__nv_bfloat16, NVFP4_EPI_NONE, true>(ma, mb, a, st);
    return launch_typed<float, NVFP4_EPI_NONE, true>(ma, mb, a, st);
}

}  // namespace nvfp4
