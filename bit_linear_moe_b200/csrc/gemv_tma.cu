// K2 (pipelined form): W4A16 decode for M <= 2 with K % 256 == 0 (wider
// batches go to the tensor-memory kernel in gemm_w4a16_tc.cu).
//
// Ignis README, "The decode round": decode linears are weight streaming at
// the card's bandwidth; this kernel is built so that the HBM stream never
// waits on the arithmetic.
//
//   y[m, n] = gs * sum_q 2^-p_{q,m} * sum_{b in split q} E4M3(s[n, b]) *
//                                       sum_{k in b} xh_q[m, k] * E2M1(c[n, k])
//
// Each CTA loads the bf16 activations of its K split into shared memory with
// plain loads (a bulk copy would queue behind the weight stages already
// requested), takes their largest magnitude, and rewrites them as fp16 scaled by a
// power of two p that puts that maximum in [2^14, 2^15): exact for every
// element within 2^28 of the split's maximum.  The split's partial sums are
// multiplied by 2^-p (exact) before the splits are added.
//
// CTA = 1 producer warp + 8 consumer warps, one 128-row tile of W and a
// contiguous range of 256-element K stages.  The producer streams, per stage,
// the 128 x 128-byte code tile (2D TMA, no multicast) and its 2 KB of scales
// (one bulk copy of four 512-byte tensor-core scale atoms, or a 2D TMA box of
// the row-major scales) into a 4-deep shared-memory ring guarded by
// mbarriers.  A consumer warp copies its slice of a slot into registers and
// releases the slot (data-dependent on all 32 lanes' reads) before doing the
// arithmetic, so the refill overlaps the math.  Each consumer lane owns one
// 32-element chunk column of a stage
// and 4 rows, so the activation chunk it loads from shared memory is reused 4
// times; codes are unpacked with cvt.rn.f16x2.e2m1x2 and multiplied with the
// mixed-precision fma.rn.f32.f16.  The K range of a tile is split over a
// cluster of QS CTAs (QS chosen so that the grid is one wave over the SMs);
// each CTA stores its partial sums into its own slot of rank 0's shared memory
// (remote stores, one cluster barrier) and rank 0 adds them and writes the
// output.  Launched as a programmatic dependent: the first ring of weight
// stages is requested before the previous kernel in the stream completes, the
// activations after it.
#include <cuda.h>

#include <map>
#include <mutex>
#include <tuple>

#include "internal.h"
#include "tma.cuh"

namespace nvfp4 {

constexpr int kStages = 4;
constexpr int kTileRows = 128;
constexpr int kStageK = 256;                    // elements per stage
constexpr int kCodeBytes = kTileRows * 128;     // 16 KB
constexpr int kScaleBytes = 2048;
constexpr int kThreads = 288;
constexpr int kMaxQS = 8;                        // K splits per tile (cluster size)

struct DecodeArgs {
    const __nv_bfloat16* x;
    int64_t M, K, N;
    const uint8_t* scales;  // TILED scales base (bulk copies)
    const float* gs;
    void* y;
    int64_t ldy;
    int QS;
    int64_t cp4;            // scale atoms along K (= K / 64)
    int* status;
};

NVFP4_DEV float fma_f16h(uint16_t a, uint16_t b, float c) {
    float d;
    asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
    return d;
}

// 32 code x activation products as two 16-element block partials.
NVFP4_DEV void dot32(const uint4& wq, const uint32_t (&xw)[16], float& p0, float& p1) {
    const uint32_t w[4] = {wq.x, wq.y, wq.z, wq.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t h[4];
        e2m1x8_to_f16x2(w[j], h);
        float p = (j < 2) ? p0 : p1;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint16_t hl, hh, xl, xhi;
            asm("mov.b32 {%0, %1}, %2;" : "=h"(hl), "=h"(hh) : "r"(h[q]));
            asm("mov.b32 {%0, %1}, %2;" : "=h"(xl), "=h"(xhi) : "r"(xw[4 * j + q]));
            p = fma_f16h(hl, xl, p);
            p = fma_f16h(hh, xhi, p);
        }
        if (j < 2) p0 = p; else p1 = p;
    }
}

static size_t decode_smem_bytes(int MT, int64_t kr_max) {
    return 1024 + (size_t)kStages * (kCodeBytes + kScaleBytes) + (size_t)MT * kr_max * 2 +
           (size_t)kMaxQS * kTileRows * MT * 4 +
           8 * (2 * kStages + 1);
}

template <int MT, int LAYOUT, typename OutT>
__global__ void __launch_bounds__(kThreads, 2)
    gemv_tma_kernel(const __grid_constant__ CUtensorMap codes_map, const __grid_constant__ CUtensorMap sc_map,
                    const DecodeArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int QS = a.QS;
    const int nst = (int)(a.K / kStageK);
    const int kr_max = (nst + QS - 1) / QS * kStageK;
    uint8_t* s_codes = smem;
    uint8_t* s_scales = s_codes + kStages * kCodeBytes;
    __half* s_x = reinterpret_cast<__half*>(s_scales + kStages * kScaleBytes);
    float* s_red = reinterpret_cast<float*>(s_x + MT * kr_max);  // [kMaxQS][kTileRows][MT] (rank 0 gathers)
    uint64_t* bars = reinterpret_cast<uint64_t*>(s_red + kMaxQS * kTileRows * MT);
    uint64_t* full = bars;
    uint64_t* empty = bars + kStages;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = (int)(blockIdx.x % QS);
    const int tile = (int)(blockIdx.x / QS);
    const int64_t row0 = (int64_t)tile * kTileRows;
    const int st_begin = (int)((int64_t)nst * q / QS), st_end = (int)((int64_t)nst * (q + 1) / QS);
    const int ns = st_end - st_begin;
    const int64_t k_begin = (int64_t)st_begin * kStageK;
    const int64_t m0 = (int64_t)blockIdx.y * MT;
    const int nt = (int)((a.M - m0) < MT ? (a.M - m0) : MT);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 8);  // one release per consumer warp
        }
        fence_barrier_init();
    }
    __syncthreads();

    float acc[4][MT];
    float inv_p[MT];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int t = 0; t < MT; ++t) acc[i][t] = 0.0f;
#pragma unroll
    for (int t = 0; t < MT; ++t) inv_p[t] = 1.0f;

    if (QS > 1) cluster_arrive_relaxed();  // waited on before the partial sums are pushed to rank 0
    griddep_launch_dependents();
    if (warp == 8) {
        // ---------------- producer ----------------
        if (lane == 0) {
            prefetch_tensormap(&codes_map);
            const uint64_t pol = l2_evict_first_policy();  // weights are read once per call
            if (LAYOUT == NVFP4_SF_ROWMAJOR) prefetch_tensormap(&sc_map);
            // weights only: the first ring's worth goes out before the previous
            // kernel has finished (the consumers fetch the activations)
            for (int s = 0; s < ns; ++s) {
                const int slot = s % kStages;
                if (s >= kStages) {
                    if (!mbar_wait(&empty[slot], ((s / kStages) - 1) & 1, a.status)) break;
                    fence_proxy_async();  // consumers' generic reads before the async-proxy refill
                }
                mbar_expect_tx(&full[slot], kCodeBytes + kScaleBytes);
                const int st = st_begin + s;
                tma_load_2d_hint(s_codes + slot * kCodeBytes, &codes_map, &full[slot], st * 128, (int)row0, pol);
                if (LAYOUT == NVFP4_SF_TILED)
                    bulk_load_hint(s_scales + slot * kScaleBytes,
                                   a.scales + ((int64_t)tile * a.cp4 + (int64_t)st * 4) * 512, kScaleBytes, &full[slot],
                                   pol);
                else
                    tma_load_2d_hint(s_scales + slot * kScaleBytes, &sc_map, &full[slot], st * 16, (int)row0, pol);
            }
        }
        if (QS > 1) cluster_wait();
    } else {
        griddep_wait();
        // ---------------- consumers ----------------
        const int ch = lane & 7, rsub = lane >> 3;
        bool ok = true;
        // this split's activations, straight from global memory with plain loads
        // (a bulk copy would queue behind the weight stages already in flight),
        // then bf16 -> fp16 * 2^p in place, p per token from the split's maximum
        {
            const int ctid = threadIdx.x;  // 0..255 (consumer threads)
            const int nv8 = ns * kStageK / 8;
            float* s_max = s_red;          // reused before the reduction needs it
            // every load of a thread is in flight before the first is used
            float mx[MT];
#pragma unroll
            for (int t = 0; t < MT; ++t) mx[t] = 0.0f;
            for (int base = ctid; base < nv8; base += 4 * 256) {
                uint4 q4[MT][4];
#pragma unroll
                for (int t = 0; t < MT; ++t)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int v = base + i * 256;
                        if (t < nt && v < nv8)
                            q4[t][i] = *reinterpret_cast<const uint4*>(a.x + (m0 + t) * a.K + k_begin + (int64_t)v * 8);
                    }
#pragma unroll
                for (int t = 0; t < MT; ++t)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int v = base + i * 256;
                        if (t < nt && v < nv8) {
                            reinterpret_cast<uint4*>(s_x + t * kr_max)[v] = q4[t][i];
                            const uint32_t u[4] = {q4[t][i].x, q4[t][i].y, q4[t][i].z, q4[t][i].w};
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                mx[t] = fmaxf(mx[t], fmaxf(fabsf(bf16lo_to_f32(u[j])), fabsf(bf16hi_to_f32(u[j]))));
                        }
                    }
            }
#pragma unroll
            for (int t = 0; t < MT; ++t) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) mx[t] = fmaxf(mx[t], __shfl_xor_sync(0xffffffffu, mx[t], o));
                if (lane == 0) s_max[t * 8 + warp] = mx[t];
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                float mx = 0.0f;
#pragma unroll
                for (int w = 0; w < 8; ++w) mx = fmaxf(mx, s_max[t * 8 + w]);
                int p = 0;
                if (mx > 0.0f) p = 141 - (int)((__float_as_uint(mx) >> 23) & 0xFF);
                p = p < -126 ? -126 : (p > 126 ? 126 : p);
                const float sc = __uint_as_float((uint32_t)(127 + p) << 23);
                inv_p[t] = __uint_as_float((uint32_t)(127 - p) << 23);
                if (t < nt)
                    for (int v = ctid; v < nv8; v += 256) {
                        uint4* qp = reinterpret_cast<uint4*>(s_x + t * kr_max) + v;
                        const uint4 q4 = *qp;
                        const uint32_t u[4] = {q4.x, q4.y, q4.z, q4.w};
                        uint32_t o[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const __half2 h = __floats2half2_rn(bf16lo_to_f32(u[j]) * sc, bf16hi_to_f32(u[j]) * sc);
                            o[j] = *reinterpret_cast<const uint32_t*>(&h);
                        }
                        *qp = make_uint4(o[0], o[1], o[2], o[3]);
                    }
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
        }
        for (int s = 0; s < ns && ok; ++s) {
            const int slot = s % kStages;
            if (!mbar_wait(&full[slot], (s / kStages) & 1, a.status)) {
                ok = false;
                break;
            }
            const uint8_t* cs = s_codes + slot * kCodeBytes;
            const uint8_t* ss = s_scales + slot * kScaleBytes;
            uint32_t xw[MT][16];
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                const uint4* xp = reinterpret_cast<const uint4*>(s_x + t * kr_max + s * kStageK + ch * 32);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint4 xv = xp[v];
                    xw[t][4 * v] = xv.x; xw[t][4 * v + 1] = xv.y; xw[t][4 * v + 2] = xv.z; xw[t][4 * v + 3] = xv.w;
                }
            }
            // copy this lane's slice of the slot to registers, release the slot,
            // then compute while the producer refills it
            uint4 wq[4];
            uint32_t sc2[4];
            uint32_t dep = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = 16 * warp + rsub + 4 * i;
                wq[i] = *reinterpret_cast<const uint4*>(cs + r * 128 + ch * 16);
                if (LAYOUT == NVFP4_SF_TILED)
                    sc2[i] = *reinterpret_cast<const uint16_t*>(ss + (ch >> 1) * 512 + (r & 31) * 16 + (r >> 5) * 4 +
                                                                2 * (ch & 1));
                else
                    sc2[i] = *reinterpret_cast<const uint16_t*>(ss + r * 16 + 2 * ch);
                dep ^= wq[i].x ^ wq[i].y ^ wq[i].z ^ wq[i].w ^ sc2[i];
            }
            warp_release_after(&empty[slot], dep);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 sd = f16x2_to_f32x2(e4m3x2_to_f16x2((uint16_t)sc2[i]));
#pragma unroll
                for (int t = 0; t < MT; ++t) {
                    float p0 = 0.0f, p1 = 0.0f;
                    dot32(wq[i], xw[t], p0, p1);
                    acc[i][t] = fmaf(p0, sd.x, acc[i][t]);
                    acc[i][t] = fmaf(p1, sd.y, acc[i][t]);
                }
            }
        }
        // reduce the 8 chunk columns of each row
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                float v = acc[i][t];
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                acc[i][t] = v;
            }
        if (QS > 1) cluster_wait();  // every CTA of the cluster is running: rank 0's memory can be written
        if (ch == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = 16 * warp + rsub + 4 * i;
                if (QS > 1) {
#pragma unroll
                    for (int t = 0; t < MT; ++t) {
                        float* slot = &s_red[((int64_t)q * kTileRows + r) * MT + t];
                        if (q == 0)
                            *slot = acc[i][t] * inv_p[t];
                        else
                            st_dsmem_f32(slot, 0, acc[i][t] * inv_p[t]);
                    }
                } else if (row0 + r < a.N) {
                    const float g = a.gs[0];
#pragma unroll
                    for (int t = 0; t < MT; ++t)
                        if (t < nt)
                            store_out<OutT>(reinterpret_cast<OutT*>(a.y) + (m0 + t) * a.ldy + row0 + r,
                                            acc[i][t] * inv_p[t] * g);
                }
            }
        }
    }

    if (QS > 1) {
        cluster_sync();  // every rank's partial sums are in rank 0's shared memory
        if (q == 0) {
            const float g = a.gs[0];
            for (int idx = threadIdx.x; idx < kTileRows * MT; idx += kThreads) {
                const int r = idx / MT, t = idx % MT;
                if (t >= nt || row0 + r >= a.N) continue;
                float v = s_red[idx];
                for (int qq = 1; qq < QS; ++qq) v += s_red[(int64_t)qq * kTileRows * MT + idx];
                store_out<OutT>(reinterpret_cast<OutT*>(a.y) + (m0 + t) * a.ldy + row0 + r, v * g);
            }
        }
    }
}

// ---- host ------------------------------------------------------------------

template <int MT, int LAYOUT, typename OutT>
static int launch_one(const DecodeArgs& a, const CUtensorMap& cm, const CUtensorMap& sm, cudaStream_t st) {
    auto kern = gemv_tma_kernel<MT, LAYOUT, OutT>;
    static std::once_flag once;
    std::call_once(once, [&] { cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024); });
    const int nst = (int)(a.K / kStageK);
    const int64_t tiles = (a.N + kTileRows - 1) / kTileRows;
    const int64_t kr_max = (int64_t)((nst + a.QS - 1) / a.QS) * kStageK;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles * a.QS), (unsigned)((a.M + MT - 1) / MT), 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = decode_smem_bytes(MT, kr_max);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)a.QS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    set_pdl_attr(attr[1]);
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, cm, sm, a) == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

// K-split of a tile: the largest QS <= 8 whose grid fits one wave of resident
// clusters (queried once per shape and cached).
template <int MT, int LAYOUT, typename OutT>
static int choose_qs(int64_t N, int64_t K, int64_t M) {
    static std::mutex mu;
    static std::map<std::tuple<int64_t, int64_t, int64_t>, int> cache;
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_tuple(N, K, M);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    auto kern = gemv_tma_kernel<MT, LAYOUT, OutT>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    const int nst = (int)(K / kStageK);
    const int64_t tiles = (N + kTileRows - 1) / kTileRows * ((M + MT - 1) / MT);
    int best = 1;
    for (int qs = (nst < 8 ? nst : 8); qs >= 2; --qs) {
        const int64_t kr_max = (int64_t)((nst + qs - 1) / qs) * kStageK;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(tiles * qs), 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = decode_smem_bytes(MT, kr_max);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)qs;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess) {
            cudaGetLastError();
            continue;
        }
        if ((int64_t)clusters >= tiles) {
            best = qs;
            break;
        }
    }
    cache[key] = best;
    return best;
}

template <int MT, int LAYOUT, typename OutT>
static int run(DecodeArgs a, const uint8_t* codes, const uint8_t* scales, cudaStream_t st) {
    CUtensorMap cm, sm;
    if (!make_tmap_2d_u8(&cm, codes, (uint64_t)(a.K / 2), (uint64_t)a.N, 128, kTileRows)) return NVFP4_ERR_LAUNCH;
    if (LAYOUT == NVFP4_SF_ROWMAJOR) {
        if (!make_tmap_2d_u8(&sm, scales, (uint64_t)(a.K / 16), (uint64_t)a.N, 16, kTileRows)) return NVFP4_ERR_LAUNCH;
    } else {
        sm = cm;
    }
    a.QS = choose_qs<MT, LAYOUT, OutT>(a.N, a.K, a.M);
    return launch_one<MT, LAYOUT, OutT>(a, cm, sm, st);
}

template <int LAYOUT, typename OutT>
static int run_mt(const DecodeArgs& a, const uint8_t* codes, const uint8_t* scales, cudaStream_t st) {
    if (a.M <= 1) return run<1, LAYOUT, OutT>(a, codes, scales, st);
    return run<2, LAYOUT, OutT>(a, codes, scales, st);
}

bool decode_tma_supported(int64_t M, int64_t K, int64_t N) {
    return M <= 2 && K % kStageK == 0 && K / 2 <= ((int64_t)1 << 31) && N <= ((int64_t)1 << 31);
}

int launch_decode_tma(const void* x, int64_t M, int64_t K, const uint8_t* codes, const uint8_t* scales,
                      int sf_layout, const float* gs, int64_t N, void* y, int y_dtype, int* status, cudaStream_t st) {
    DecodeArgs a{};
    a.x = (const __nv_bfloat16*)x;
    a.M = M;
    a.K = K;
    a.N = N;
    a.scales = scales;
    a.gs = gs;
    a.y = y;
    a.ldy = N;
    a.cp4 = K / 64;
    a.status = status;
    if (sf_layout == NVFP4_SF_TILED) {
        if (y_dtype == NVFP4_DTYPE_BF16) return run_mt<NVFP4_SF_TILED, __nv_bfloat16>(a, codes, scales, st);
        return run_mt<NVFP4_SF_TILED, float>(a, codes, scales, st);
    }
    if (y_dtype == NVFP4_DTYPE_BF16) return run_mt<NVFP4_SF_ROWMAJOR, __nv_bfloat16>(a, codes, scales, st);
    return run_mt<NVFP4_SF_ROWMAJOR, float>(a, codes, scales, st);
}

}  // namespace nvfp4
