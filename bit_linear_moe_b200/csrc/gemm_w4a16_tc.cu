// K3: W4A16 skinny GEMM (decode widths) with the dequantized weights in tensor
// memory (Ignis README, "The decode round": decode is weight streaming at the
// card's bandwidth; imp home page, "How does it work?": weights stay NVFP4).
//
//   y[m, n] = gs * 2^-p_m * sum_k xh[m, k] * (E2M1(c[n, k]) * E4M3(s[n, k/16]))
//
// with xh = x * 2^p_m in fp16 (x_prep_kernel).  E2M1 * E4M3 has at most 6
// significant bits and lies in [2^-10, 2688], so it is exact in fp16; the
// tensor core multiplies fp16 x fp16 exactly and accumulates in fp32.
//
// Why tensor cores for a bandwidth-bound op: on CUDA cores the unpack plus one
// FMA per weight per token costs >= 2.3 instructions per weight element at
// M = 1 and grows with M, above what the SMs can issue at HBM rate.  Here the
// CUDA cores only unpack (one cvt.rn.f16x2.e2m1x2 and one HMUL2 by the block
// scale per two weights) and the multiply-accumulate for all M tokens runs in
// tcgen05.mma with the weights as the A operand read from tensor memory.
//
// CTA = 10 warps, one 128-row weight tile, a range of 256-element K stages:
//   warp 0     tensor-memory allocation; lane 0 streams per stage the code
//              tile (128 x 128 B, 2D TMA, 128-byte swizzle), its 2 KB of scale
//              atoms (bulk copy) and the fp16 activation tile (NT x 256, four
//              2D TMA boxes, 128-byte swizzle; rows past M read as zero) into a
//              3-stage ring;
//   warps 2-9  dequantizers: a stage is 4 chunks of 64 K-elements; warp
//              group (w - 2) / 4 takes chunks of its parity, and each of its
//              4 warps covers the 32 weight rows of tensor-memory lane quadrant
//              w % 4 -- each thread its own row -- storing 32 columns of packed
//              fp16 per chunk with tcgen05.st into a ring of 6 A chunks (so the
//              unpacking runs 1.5 stages ahead of the MMAs);
//   warp 1     lane 0 issues, per chunk, 4 MMAs (M 128, N = NT, K 16) reading A
//              from tensor memory and the activation tile from shared memory,
//              then commits to the chunk's "A free" barrier and, after a
//              stage's last chunk, to the stage's empty barrier.
// K is split over a cluster of QS CTAs; partial sums meet through distributed
// shared memory (reusing the ring's memory) and rank 0 writes y.
#include <cuda.h>

#include <mutex>

#include "internal.h"
#include "tcgen05.cuh"

namespace nvfp4 {

namespace w4a16tc {
constexpr int kStages = 3;
constexpr int kCodes = 128 * 128, kSf = 2048;
constexpr int kThreads = 320;
constexpr int kTmemCols = 256;  // A ring: 6 x 32 columns, D: NT (<= 64) columns at 192
constexpr int kAChunks = 6;
template <int NT>
struct Cfg {
    static constexpr int kX = 4 * NT * 128;
    static constexpr int kStageBytes = kCodes + kX + kSf;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 256;
};
}  // namespace w4a16tc

struct TcArgs {
    int64_t M, K, N;
    const uint8_t* scales;  // TILED
    const float* gs;
    const float* inv_scale;
    void* y;
    int64_t ldy;
    int QS;
    int* status;
};

template <int NT>
NVFP4_DEV void tmem_ld_acc(uint32_t taddr, float (&v)[NT]) {
#pragma unroll
    for (int c0 = 0; c0 < NT; c0 += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + c0, r);  // 32 columns at a time; columns >= NT are unused
        tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < 32; ++t)
            if (c0 + t < NT) v[c0 + t] = __uint_as_float(r[t]);
    }
}

template <int NT, typename OutT>
__global__ void __launch_bounds__(w4a16tc::kThreads, 1)
    gemm_w4a16_tc_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                         const TcArgs a) {
    using namespace w4a16tc;
    using C = Cfg<NT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * C::kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* a_full = empty + kStages;   // [kAChunks]
    uint64_t* a_free = a_full + kAChunks;  // [kAChunks]
    uint64_t* accum = a_free + kAChunks;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(accum + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int QS = a.QS;
    const int q = (int)(blockIdx.x % QS);
    const int tile = (int)(blockIdx.x / QS);
    const int64_t row0 = (int64_t)tile * 128;
    const int nst = (int)(a.K / 256);
    const int st_begin = (int)((int64_t)nst * q / QS), st_end = (int)((int64_t)nst * (q + 1) / QS);
    const int ns = st_end - st_begin;
    const int64_t cp4 = a.K / 64;

    if (warp == 0) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 32) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 8 + 1);  // 8 dequant warps + the MMA commit
        }
        for (int c = 0; c < kAChunks; ++c) {
            mbar_init(&a_full[c], 4);
            mbar_init(&a_free[c], 1);
        }
        mbar_init(accum, 1);
        fence_barrier_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t d_col = 32 * kAChunks;
    bool ok = true;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&map_w);
            prefetch_tensormap(&map_x);
            const uint64_t pol = l2_evict_first_policy();  // weights are read once per call
            const uint8_t* sf_tile = a.scales + (int64_t)tile * cp4 * 512;
            for (int s = 0; s < ns; ++s) {
                const int slot = s % kStages;
                if (s >= kStages && !mbar_wait(&empty[slot], ((s / kStages) - 1) & 1, a.status)) break;
                uint8_t* st = smem + slot * C::kStageBytes;
                const int kst = st_begin + s;
                mbar_expect_tx(&full[slot], C::kStageBytes);
                tma_load_2d_hint(st, &map_w, &full[slot], kst * 128, (int)row0, pol);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    tma_load_2d(st + kCodes + c * NT * 128, &map_x, &full[slot], kst * 512 + c * 128, 0);
                bulk_load_hint(st + kCodes + C::kX, sf_tile + (int64_t)kst * 4 * 512, kSf, &full[slot], pol);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16(128, NT);
            for (int s = 0; s < ns && ok; ++s) {
                const int slot = s % kStages;
                if (!mbar_wait(&full[slot], (s / kStages) & 1, a.status)) { ok = false; break; }
                const uint32_t xs = smem_u32(smem + slot * C::kStageBytes + kCodes);
                for (int c = 0; c < 4; ++c) {
                    const int g = 4 * s + c, ac = g % kAChunks;
                    if (!mbar_wait(&a_full[ac], (g / kAChunks) & 1, a.status)) { ok = false; break; }
                    tc_fence_after();
                    for (int j = 0; j < 4; ++j) {
                        const int kk = 64 * c + 16 * j;  // element offset within the stage
                        const uint64_t bdesc = sdesc_sw128_kmajor(xs + (kk / 64) * NT * 128 + (kk % 64) * 2);
                        mma_f16_ts(tmem + d_col, tmem + 32 * ac + 8 * j, bdesc, idesc, (g > 0 || j > 0) ? 1u : 0u);
                    }
                    tc_commit(&a_free[ac]);
                }
                tc_commit(&empty[slot]);
            }
            if (ok) tc_commit(accum);
        }
    } else {
        // dequantizers: warps 2..9; group = (warp - 2) / 4 takes chunks c with c % 2 == group
        const int grp = (warp - 2) >> 2;
        const int quad = warp & 3;
        const int r = 32 * quad + lane;  // weight row within the tile == tensor-memory lane
        const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
        for (int s = 0; s < ns && ok; ++s) {
            const int slot = s % kStages;
            if (!mbar_wait(&full[slot], (s / kStages) & 1, a.status)) { ok = false; break; }
            const uint8_t* st = smem + slot * C::kStageBytes;
            const uint8_t* sf = st + kCodes + C::kX;
            uint32_t dep = 0;
            for (int c = grp; c < 4; c += 2) {
                const int g = 4 * s + c, ac = g % kAChunks;
                // this row's 32 code bytes of the chunk (2 swizzled 16-byte pieces) and its 4 block scales
                uint4 cw[2];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int piece = 2 * c + j;
                    cw[j] = *reinterpret_cast<const uint4*>(st + r * 128 + ((piece ^ (r & 7)) << 4));
                }
                const uint32_t sw = *reinterpret_cast<const uint32_t*>(sf + c * 512 + (r & 31) * 16 + (r >> 5) * 4);
                if (g >= kAChunks && !mbar_wait(&a_free[ac], ((g / kAChunks) - 1) & 1, a.status)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    // piece j holds blocks 2j, 2j+1 of the chunk (16 codes each)
                    uint32_t v[16];
                    const uint32_t w[4] = {cw[j].x, cw[j].y, cw[j].z, cw[j].w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int blk = 2 * j + (u >> 1);
                        const uint32_t sbyte = (sw >> (8 * blk)) & 0xFF;
                        const uint32_t s2 = e4m3x2_to_f16x2((uint16_t)(sbyte | (sbyte << 8)));
                        uint32_t hh[4];
                        e2m1x8_to_f16x2(w[u], hh);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            uint32_t prod;
                            asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(prod) : "r"(hh[e]), "r"(s2));
                            v[4 * u + e] = prod;
                        }
                    }
                    tmem_st_32x32b_x16(tmem + lane_off + 32 * ac + 16 * j, v);
                    dep ^= v[0] ^ v[15];
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&a_full[ac]);
            }
            // the code/scale slot is free once this warp's loads are done (they fed the stores)
            warp_release_after(&empty[slot], dep);
        }
    }

    // ---- epilogue: warps 2..5 read D (lane = weight row, column = token) ----
    float* s_red = reinterpret_cast<float*>(smem);  // ring memory is free after the main loop
    const bool epi = warp >= 2 && warp < 6;
    float acc[NT];
    if (epi) {
        const int quad = warp & 3;
        const int r = 32 * quad + lane;
        ok = mbar_wait(accum, 0, a.status) && ok;
        tc_fence_after();
        tmem_ld_acc<NT>(tmem + ((uint32_t)(32 * quad) << 16) + d_col, acc);
        if (QS == 1) {
            if (ok && row0 + r < a.N) {
                const float g = a.gs[0];
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    if (t < a.M) store_out<OutT>(reinterpret_cast<OutT*>(a.y) + t * a.ldy + row0 + r, acc[t] * g * a.inv_scale[t]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();  // ring and tensor memory no longer in use by the async units
    if (QS > 1) {
        if (epi) {
            const int r = 32 * (warp & 3) + lane;
#pragma unroll
            for (int t = 0; t < NT; ++t) s_red[t * 128 + r] = acc[t];
        }
        cluster_sync();
        if (q == 0) {
            const float g = a.gs[0];
            for (int idx = threadIdx.x; idx < 128 * NT; idx += kThreads) {
                const int t = idx / 128, r = idx % 128;
                if (t >= a.M || row0 + r >= a.N) continue;
                float v = s_red[idx];
                for (int qq = 1; qq < QS; ++qq) v += ld_dsmem_f32(&s_red[idx], (uint32_t)qq);
                store_out<OutT>(reinterpret_cast<OutT*>(a.y) + t * a.ldy + row0 + r, v * g * a.inv_scale[t]);
            }
        }
        cluster_sync();
    }
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---- host -------------------------------------------------------------------

template <int NT, typename OutT>
static int run(TcArgs a, const uint8_t* codes, const void* xh, cudaStream_t st) {
    using namespace w4a16tc;
    auto kern = gemm_w4a16_tc_kernel<NT, OutT>;
    static std::once_flag once;
    std::call_once(once, [&] {
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<NT>::kSmemBytes);
    });
    CUtensorMap mw, mx;
    if (!make_tmap_2d_u8(&mw, codes, (uint64_t)(a.K / 2), (uint64_t)a.N, 128, 128, 1)) return NVFP4_ERR_LAUNCH;
    if (!make_tmap_2d_u8(&mx, xh, (uint64_t)(a.K * 2), (uint64_t)a.M, 128, NT, 1)) return NVFP4_ERR_LAUNCH;
    // split K so that the grid is about one CTA per resident slot (two per SM
    // for 16 and 32 tokens, ~80-104 KB of shared memory and 256 tensor-memory
    // columns each; one per SM for 64 tokens, ~150 KB)
    const int64_t tiles = (a.N + 127) / 128;
    const int nst = (int)(a.K / 256);
    const int slots = (Cfg<NT>::kSmemBytes <= 110 * 1024 ? 2 : 1) * 148;
    int qs = (int)((slots + tiles / 2) / tiles);
    if (qs > 8) qs = 8;
    if (qs > nst) qs = nst;
    if (qs < 1) qs = 1;
    a.QS = qs;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles * qs), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = Cfg<NT>::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)qs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, mw, mx, a) == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

bool w4a16_tc_supported(int64_t M, int64_t K, int64_t N, int sf_layout) {
    return sf_layout == NVFP4_SF_TILED && M >= 3 && M <= 64 && K % 256 == 0 && N <= ((int64_t)1 << 30);
}

int launch_w4a16_tc(const void* xh, const float* inv_scale, int64_t M, int64_t K, const uint8_t* codes,
                    const uint8_t* scales, const float* gs, int64_t N, void* y, int y_dtype, int* status,
                    cudaStream_t st) {
    TcArgs a{};
    a.M = M;
    a.K = K;
    a.N = N;
    a.scales = scales;
    a.gs = gs;
    a.inv_scale = inv_scale;
    a.y = y;
    a.ldy = N;
    a.status = status;
    if (M <= 16) {
        if (y_dtype == NVFP4_DTYPE_BF16) return run<16, __nv_bfloat16>(a, codes, xh, st);
        return run<16, float>(a, codes, xh, st);
    }
    if (M <= 32) {
        if (y_dtype == NVFP4_DTYPE_BF16) return run<32, __nv_bfloat16>(a, codes, xh, st);
        return run<32, float>(a, codes, xh, st);
    }
    if (y_dtype == NVFP4_DTYPE_BF16) return run<64, __nv_bfloat16>(a, codes, xh, st);
    return run<64, float>(a, codes, xh, st);
}

}  // namespace nvfp4
