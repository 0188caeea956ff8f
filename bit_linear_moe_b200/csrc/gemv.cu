// K2: W4A16 linear on CUDA cores, for decode widths (Ignis README, "The decode
// round": decode is weight streaming at the card's bandwidth).
//
//   y[m, n] = gs * 2^-p_m * sum_b E4M3(s[n, b]) * sum_{k in b} xh[m, k] * E2M1(c[n, k])
//
// where xh = x * 2^p_m in fp16 (prepared once per call by x_prep_kernel; p_m
// puts the row's largest magnitude in [2^14, 2^15), so xh equals x exactly
// for every element within 2^28 of the row maximum).  Each weight pair is
// unpacked by one cvt.rn.f16x2.e2m1x2 (exact) and multiplied with the
// mixed-precision fma.rn.f32.f16 (exact product, fp32 accumulate): one
// quarter-rate conversion per two elements and one FMA per element.  Per
// 16-element block the partial sum is scaled once by the E4M3 block scale.
//
// Work split: a CTA has 8 warps = RG row groups x QS K-splits.  A warp owns R
// weight rows (2: the activation chunk it loads is reused for both) and one
// K-split; its lanes stride over the split in 16-byte chunks (32 codes), and
// all of the warp's chunk loads for a batch are issued before any of them is
// consumed, so up to R*J 16-byte loads per lane are in flight.  Partial sums
// of the QS splits meet in shared memory.  QS is picked per shape so that
// small-N matrices still spread over all SMs.  The weight stream uses
// non-allocating 128-bit loads; activations and scales go through L1.
//
// Grouped form (mixture of experts; CHImp Alpha v1.0 model card, "How it fits
// on one GPU": only the chosen experts are read): grid.x walks the experts,
// expert e's rows are [offsets[e], offsets[e+1]); an expert without rows
// exits before touching its weights.  SWIGLU gives a warp gate rows j and the
// matching up rows N/2 + j and writes silu(g) * u.  For K <= 512 (at most 16 chunks
// per row) each half-warp takes its own rows, so no lane idles.
#include "common.cuh"
#include "internal.h"

namespace nvfp4 {

// ---- activation prep: bf16 -> fp16 * 2^p per row ----------------------------
__global__ void __launch_bounds__(256) x_prep_kernel(const __nv_bfloat16* __restrict__ x,
                                                     const int32_t* __restrict__ gather, int64_t K,
                                                     __half* __restrict__ xh, float* __restrict__ inv_scale) {
    const int64_t m = blockIdx.x;
    const __nv_bfloat16* xr = x + (gather ? (int64_t)gather[m] : m) * K;
    float mx = 0.0f;
    for (int64_t k = threadIdx.x * 8; k < K; k += blockDim.x * 8) {
        const uint4 v = ldg_v4(xr + k);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) mx = fmaxf(mx, fmaxf(fabsf(bf16lo_to_f32(u[j])), fabsf(bf16hi_to_f32(u[j]))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    __shared__ float red[8];
    __shared__ float s_scale;
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < 8; ++w) mx = fmaxf(mx, red[w]);
        // p = 14 - floor(log2(mx)) so that mx * 2^p lies in [2^14, 2^15)
        int p = 0;
        if (mx > 0.0f) p = 14 - (int)((__float_as_uint(mx) >> 23) & 0xFF) + 127;
        p = p < -126 ? -126 : (p > 126 ? 126 : p);
        s_scale = __uint_as_float((uint32_t)(127 + p) << 23);
        inv_scale[m] = __uint_as_float((uint32_t)(127 - p) << 23);
    }
    __syncthreads();
    const float sc = s_scale;
    for (int64_t k = threadIdx.x * 8; k < K; k += blockDim.x * 8) {
        const uint4 v = ldg_v4(xr + k);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __half2 h = __floats2half2_rn(bf16lo_to_f32(u[j]) * sc, bf16hi_to_f32(u[j]) * sc);
            o[j] = *reinterpret_cast<const uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(xh + m * K + k) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// ---- main kernel ---------------------------------------------------------------

NVFP4_DEV float fma_f16(uint16_t a, uint16_t b, float c) {
    float d;
    asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
    return d;
}

// 32 products of one 16-byte code chunk with 32 fp16 activations, as two
// block partials (elements 0..15 and 16..31).
NVFP4_DEV void chunk_dot(const uint4& wq, const uint32_t (&xw)[16], float& p0, float& p1) {
    const uint32_t w[4] = {wq.x, wq.y, wq.z, wq.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t h[4];
        e2m1x8_to_f16x2(w[j], h);
        float p = (j < 2) ? p0 : p1;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t xv = xw[4 * j + q];
            p = fma_f16((uint16_t)(h[q] & 0xFFFF), (uint16_t)(xv & 0xFFFF), p);
            p = fma_f16((uint16_t)(h[q] >> 16), (uint16_t)(xv >> 16), p);
        }
        if (j < 2) p0 = p; else p1 = p;
    }
}

// HALF: each half-warp takes its own R rows (for K of at most 512, where a
// row has no more 32-element chunks than 16 lanes can cover).
template <int MT, int R, int QS, int J, int LAYOUT, typename OutT, int EPI, int HALF = 0>
__global__ void __launch_bounds__(256) gemv_w4a16_kernel(const GemvArgs a) {
    constexpr int RG = 8 / QS;                                    // row groups per CTA
    constexpr int RW = (EPI == NVFP4_EPI_SWIGLU) ? R / 2 : R;     // output columns per warp (half-warp)
    constexpr int LW = HALF ? 16 : 32;                            // lanes per row group
    static_assert(EPI != NVFP4_EPI_SWIGLU || R % 2 == 0, "SwiGLU pairs gate rows with up rows");
    static_assert(!HALF || (QS == 1 && EPI == NVFP4_EPI_NONE), "half-warp rows: no K split, plain epilogue");
    __shared__ float red[8][R][MT];

    const int warp = threadIdx.x >> 5, lane32 = threadIdx.x & 31;
    const int lane = HALF ? (lane32 & 15) : lane32;               // lane within the row group
    const int half = HALF ? (lane32 >> 4) : 0;
    const int g = warp / QS, q = warp % QS;
    const int64_t K = a.K;
    const int64_t nch = K >> 5;                                   // 32-element chunks per row
    const int64_t nsf = K >> 4;
    const int64_t ncols_out = (EPI == NVFP4_EPI_SWIGLU) ? a.N / 2 : a.N;
    const int64_t c_begin = nch * q / QS, c_end = nch * (q + 1) / QS;

    const int64_t col0 = (((int64_t)blockIdx.y * RG + g) * (HALF ? 2 : 1) + half) * RW;
    const bool warp_active = col0 < ncols_out;

    int64_t row_begin, row_end;
    const uint8_t* codes = a.codes;
    const uint8_t* scales = a.scales;
    float gs;
    if (a.offsets) {
        const int e = a.experts ? a.experts[blockIdx.x] : (int)blockIdx.x;
        if (e < 0) return;  // slot past the last touched expert (CTA-uniform)
        row_begin = a.offsets[e];
        row_end = a.offsets[e + 1];
        if (row_end <= row_begin) return;  // untouched expert: its weights are never read (CTA-uniform)
        codes += (int64_t)e * a.N * (K >> 1);
        scales += (int64_t)e * a.sf_stride;
        gs = a.gs[e];
    } else {
        row_begin = (int64_t)blockIdx.x * MT;
        row_end = (a.M < row_begin + MT) ? a.M : row_begin + MT;
        gs = a.gs[0];
    }

    int64_t wrow[R];
    bool cvalid[RW];
#pragma unroll
    for (int i = 0; i < RW; ++i) {
        const int64_t c = col0 + i;
        cvalid[i] = c < ncols_out;
        const int64_t cc = cvalid[i] ? c : (warp_active ? col0 : 0);
        wrow[i] = cc;
        if constexpr (EPI == NVFP4_EPI_SWIGLU) wrow[RW + i] = a.N / 2 + cc;
    }

    const __half* xh = reinterpret_cast<const __half*>(a.xh);
    for (int64_t m0 = row_begin; m0 < row_end; m0 += MT) {
        const int nt = (int)((row_end - m0) < MT ? (row_end - m0) : MT);
        const __half* xr[MT];
#pragma unroll
        for (int t = 0; t < MT; ++t) xr[t] = xh + (m0 + (t < nt ? t : 0)) * K;
        float acc[R][MT];
#pragma unroll
        for (int i = 0; i < R; ++i)
#pragma unroll
            for (int t = 0; t < MT; ++t) acc[i][t] = 0.0f;

        if (warp_active) {
            for (int64_t cb = c_begin; cb < c_end; cb += LW * J) {
                // issue every load of the batch first
                uint4 wq[R][J];
                uint16_t s2[R][J];
#pragma unroll
                for (int j = 0; j < J; ++j) {
                    const int64_t c = cb + lane + LW * j;
                    const bool ok = c < c_end;
#pragma unroll
                    for (int i = 0; i < R; ++i) {
                        if (ok) {
                            wq[i][j] = ldg_stream(codes + wrow[i] * (K >> 1) + c * 16);
                            s2[i][j] = __ldg(reinterpret_cast<const uint16_t*>(
                                scales + sf_offset<LAYOUT>(wrow[i], 2 * c, nsf)));
                        } else {
                            wq[i][j] = make_uint4(0, 0, 0, 0);
                            s2[i][j] = 0;
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < J; ++j) {
                    const int64_t c = cb + lane + LW * j;
                    if (c >= c_end) break;
#pragma unroll
                    for (int t = 0; t < MT; ++t) {
                        uint32_t xw[16];
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            const uint4 xv = ldg_v4(xr[t] + c * 32 + v * 8);
                            xw[4 * v] = xv.x; xw[4 * v + 1] = xv.y; xw[4 * v + 2] = xv.z; xw[4 * v + 3] = xv.w;
                        }
#pragma unroll
                        for (int i = 0; i < R; ++i) {
                            float p0 = 0.0f, p1 = 0.0f;
                            chunk_dot(wq[i][j], xw, p0, p1);
                            const float2 sd = f16x2_to_f32x2(e4m3x2_to_f16x2(s2[i][j]));
                            acc[i][t] = fmaf(p0, sd.x, acc[i][t]);
                            acc[i][t] = fmaf(p1, sd.y, acc[i][t]);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int i = 0; i < R; ++i)
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                if constexpr (HALF) {
#pragma unroll
                    for (int o = 8; o > 0; o >>= 1) acc[i][t] += __shfl_xor_sync(0xffffffffu, acc[i][t], o);
                } else {
                    acc[i][t] = warp_sum(acc[i][t]);
                }
            }

        if constexpr (QS > 1) {
            if (lane == 0) {
#pragma unroll
                for (int i = 0; i < R; ++i)
#pragma unroll
                    for (int t = 0; t < MT; ++t) red[warp][i][t] = acc[i][t];
            }
            __syncthreads();
            if (q == 0) {
#pragma unroll
                for (int i = 0; i < R; ++i)
#pragma unroll
                    for (int t = 0; t < MT; ++t) {
                        float s = 0.0f;
#pragma unroll
                        for (int qq = 0; qq < QS; ++qq) s += red[g * QS + qq][i][t];
                        acc[i][t] = s;
                    }
            }
            __syncthreads();
        }

        if (q == 0 && warp_active) {
            OutT* y = reinterpret_cast<OutT*>(a.y);
#pragma unroll
            for (int i = 0; i < RW; ++i) {
#pragma unroll
                for (int t = 0; t < MT; ++t) {
                    if (lane == ((i * MT + t) & (LW - 1)) && t < nt && cvalid[i]) {
                        const float sc = gs * a.inv_scale[m0 + t];
                        float v;
                        if constexpr (EPI == NVFP4_EPI_SWIGLU) {
                            const float gg = acc[i][t] * sc, u = acc[RW + i][t] * sc;
                            v = gg / (1.0f + expf(-gg)) * u;
                        } else {
                            v = acc[i][t] * sc;
                        }
                        store_out<OutT>(y + (m0 + t) * a.ldy + col0 + i, v);
                    }
                }
            }
        }
    }
}

// ---- K % 32 == 16 tail path (8-byte rows): one warp per row, plain loads -----
template <int LAYOUT, typename OutT>
__global__ void __launch_bounds__(256) gemv_w4a16_odd_kernel(const GemvArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n = (int64_t)blockIdx.y * 8 + warp;
    if (n >= a.N) return;
    const int64_t K = a.K, nsf = K >> 4;
    const int64_t m = blockIdx.x;
    const __half* xr = reinterpret_cast<const __half*>(a.xh) + m * K;
    float acc = 0.0f;
    for (int64_t b = lane; b < nsf; b += 32) {   // one 16-element block per step
        uint2 wv;
        asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                     : "=r"(wv.x), "=r"(wv.y) : "l"(a.codes + n * (K >> 1) + b * 8));
        const uint4 xv0 = ldg_v4(xr + b * 16), xv1 = ldg_v4(xr + b * 16 + 8);
        const uint32_t xw[8] = {xv0.x, xv0.y, xv0.z, xv0.w, xv1.x, xv1.y, xv1.z, xv1.w};
        const uint32_t w[2] = {wv.x, wv.y};
        float p = 0.0f;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            uint32_t h[4];
            e2m1x8_to_f16x2(w[j], h);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                p = fma_f16((uint16_t)(h[qq] & 0xFFFF), (uint16_t)(xw[4 * j + qq] & 0xFFFF), p);
                p = fma_f16((uint16_t)(h[qq] >> 16), (uint16_t)(xw[4 * j + qq] >> 16), p);
            }
        }
        acc = fmaf(p, e4m3_to_f32(__ldg(a.scales + sf_offset<LAYOUT>(n, b, nsf))), acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) store_out<OutT>(reinterpret_cast<OutT*>(a.y) + m * a.ldy + n, acc * a.gs[0] * a.inv_scale[m]);
}

template <int MT, int R, int QS, int J, int LAYOUT, typename OutT, int EPI, int HALF = 0>
static int launch_cfg(const GemvArgs& a, cudaStream_t st) {
    constexpr int RG = 8 / QS;
    constexpr int RW = (EPI == NVFP4_EPI_SWIGLU) ? R / 2 : R;
    constexpr int CPB = RG * RW * (HALF ? 2 : 1);  // output columns per CTA
    const int64_t ncols = (EPI == NVFP4_EPI_SWIGLU) ? a.N / 2 : a.N;
    const int64_t tiles = (ncols + CPB - 1) / CPB;
    const int64_t gx = a.offsets ? (a.experts ? a.n_slots : a.E) : (a.M + MT - 1) / MT;
    if (tiles > 65535 || gx > 0x7fffffff) return NVFP4_ERR_SHAPE;
    dim3 grid((unsigned)gx, (unsigned)tiles);
    gemv_w4a16_kernel<MT, R, QS, J, LAYOUT, OutT, EPI, HALF><<<grid, 256, 0, st>>>(a);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

// K-split per CTA: enough CTAs for 148 SMs when N is small, 1 when N is large.
template <int MT, int LAYOUT, typename OutT, int EPI>
static int launch_qs(const GemvArgs& a, cudaStream_t st) {
    const int64_t ncols = (EPI == NVFP4_EPI_SWIGLU) ? a.N / 2 : a.N;
    const int64_t rows_per_warp = (EPI == NVFP4_EPI_SWIGLU) ? 1 : 2;
    const int64_t warps_at_qs1 = (ncols + rows_per_warp - 1) / rows_per_warp * (a.offsets ? 1 : (a.M + MT - 1) / MT);
    const int64_t nch = a.K >> 5;
    // target: >= ~8 resident-warp-slots of work per SM (148 SMs x 32 warps)
    int qs = 1;
    while (qs < 8 && warps_at_qs1 * qs < 148 * 48 && nch / (qs * 2) >= 16) qs *= 2;
    if (a.offsets) {
        // grouped (decode-time experts, a few rows each): two chunks in flight per
        // lane keep the register count, and so the resident warps per SM, up
        qs = nch >= 128 ? 2 : 1;
        // short rows (K <= 512): each half-warp takes four rows of its own
        if constexpr (EPI == NVFP4_EPI_NONE)
            if (nch <= 16) return launch_cfg<MT, 4, 1, 1, LAYOUT, OutT, EPI, 1>(a, st);
        // SwiGLU: two gate and two up rows per warp share each activation chunk
        if constexpr (EPI == NVFP4_EPI_SWIGLU) {
            if (qs == 1) return launch_cfg<MT, 4, 1, 2, LAYOUT, OutT, EPI>(a, st);
            return launch_cfg<MT, 4, 2, 2, LAYOUT, OutT, EPI>(a, st);
        }
        if (qs == 1) return launch_cfg<MT, 2, 1, 2, LAYOUT, OutT, EPI>(a, st);
        return launch_cfg<MT, 2, 2, 2, LAYOUT, OutT, EPI>(a, st);
    }
    switch (qs) {
        case 1: return launch_cfg<MT, 2, 1, 6, LAYOUT, OutT, EPI>(a, st);
        case 2: return launch_cfg<MT, 2, 2, 6, LAYOUT, OutT, EPI>(a, st);
        case 4: return launch_cfg<MT, 2, 4, 5, LAYOUT, OutT, EPI>(a, st);
        default: return launch_cfg<MT, 2, 8, 3, LAYOUT, OutT, EPI>(a, st);
    }
}

template <int LAYOUT, typename OutT, int EPI>
static int launch_mt(const GemvArgs& a, cudaStream_t st) {
    // grouped: most touched experts hold one or two rows at decode sizes; one
    // activation row per pass halves the activation reads for a single-row
    // expert (experts with more rows take more passes over their weights)
    const int64_t rows_hint = a.offsets ? (a.M <= 2 * (int64_t)a.n_slots ? 1 : 2) : a.M;
    if (rows_hint <= 1) return launch_qs<1, LAYOUT, OutT, EPI>(a, st);
    if (rows_hint <= 2) return launch_qs<2, LAYOUT, OutT, EPI>(a, st);
    return launch_qs<4, LAYOUT, OutT, EPI>(a, st);
}

template <int LAYOUT>
static int launch_layout(const GemvArgs& a, cudaStream_t st) {
    if (a.K % 32) {
        if (a.offsets || a.epilogue != NVFP4_EPI_NONE) return NVFP4_ERR_SHAPE;
        dim3 grid((unsigned)a.M, (unsigned)((a.N + 7) / 8));
        if (a.y_dtype == NVFP4_DTYPE_BF16)
            gemv_w4a16_odd_kernel<LAYOUT, __nv_bfloat16><<<grid, 256, 0, st>>>(a);
        else
            gemv_w4a16_odd_kernel<LAYOUT, float><<<grid, 256, 0, st>>>(a);
        return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
    }
    if (a.epilogue == NVFP4_EPI_SWIGLU) {
        if (a.y_dtype == NVFP4_DTYPE_BF16) return launch_mt<LAYOUT, __nv_bfloat16, NVFP4_EPI_SWIGLU>(a, st);
        return launch_mt<LAYOUT, float, NVFP4_EPI_SWIGLU>(a, st);
    }
    if (a.y_dtype == NVFP4_DTYPE_BF16) return launch_mt<LAYOUT, __nv_bfloat16, NVFP4_EPI_NONE>(a, st);
    return launch_mt<LAYOUT, float, NVFP4_EPI_NONE>(a, st);
}

int launch_x_prep(const void* x, const int32_t* gather, int64_t rows, int64_t K, void* xh, float* inv_scale,
                  cudaStream_t st) {
    if (rows > 0x7fffffff) return NVFP4_ERR_SHAPE;
    x_prep_kernel<<<(unsigned)rows, 256, 0, st>>>((const __nv_bfloat16*)x, gather, K, (__half*)xh, inv_scale);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

int launch_gemv_w4a16(const GemvArgs& a, cudaStream_t st) {
    if (a.sf_layout == NVFP4_SF_TILED) return launch_layout<NVFP4_SF_TILED>(a, st);
    return launch_layout<NVFP4_SF_ROWMAJOR>(a, st);
}

}  // namespace nvfp4
