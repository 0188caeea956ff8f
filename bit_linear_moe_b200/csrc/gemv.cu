// K2: W4A16 linear on CUDA cores, for decode widths (Ignis README, "The decode
// round": decode is weight streaming at the card's bandwidth).
//
// y[m, n] = gs * sum_b E4M3(s[n, b]) * sum_{k in block b} x[m, k] * E2M1(c[n, k])
//
// Work split: a warp owns R weight rows; its lanes stride over K in chunks of
// 2*VB elements (VB = 16: one 128-bit load of 32 codes + one 16-bit load of
// the two block scales per row).  The activation chunk is converted to fp32
// once and reused for all R rows.  Per block: 16 FMAs into a block partial,
// then one FMA by the block scale; gs is applied once at the end.  Lanes are
// reduced with warp shuffles.  The weight stream uses non-allocating 128-bit
// loads, so each weight byte crosses HBM once; activations come through the
// read-only cache.
//
// Grid: x = token groups (dense) or experts (grouped), y = row tiles.  With
// token groups fastest, the CTAs that read the same weight rows for different
// token groups run together and share the rows through L2.
//
// Grouped form (mixture of experts; CHImp Alpha v1.0 model card, "How it fits
// on one GPU": only the chosen experts are read): expert e's rows are
// [offsets[e], offsets[e+1]); an expert without rows exits before touching its
// weights.  SWIGLU pairs weight row j (gate) with row N/2 + j (up) in the same
// warp and writes silu(g) * u.
#include "common.cuh"
#include "internal.h"

namespace nvfp4 {

template <int VB>
NVFP4_DEV void load_codes(const uint8_t* p, uint32_t (&w)[VB / 4]) {
    if constexpr (VB == 16) {
        uint4 v = ldg_stream(p);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
        uint2 v;
        asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
        w[0] = v.x; w[1] = v.y;
    }
}

template <int MT, int R, int VB, int LAYOUT, typename OutT, int EPI>
__global__ void __launch_bounds__(256) gemv_w4a16_kernel(const GemvArgs a) {
    constexpr int CE = 2 * VB;          // elements per chunk
    constexpr int NB = CE / 16;         // blocks per chunk
    constexpr int RW = (EPI == NVFP4_EPI_SWIGLU) ? R / 2 : R;  // output columns per warp
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t K = a.K;
    const int64_t nchunk = K / CE;
    const int64_t nsf = K >> 4;
    const int64_t ncols_out = (EPI == NVFP4_EPI_SWIGLU) ? a.N / 2 : a.N;

    const int64_t col0 = ((int64_t)blockIdx.y * 8 + warp) * RW;
    if (col0 >= ncols_out) return;

    int64_t row_begin, row_end;
    const uint8_t* codes = a.codes;
    const uint8_t* scales = a.scales;
    float gs;
    if (a.offsets) {
        const int e = blockIdx.x;
        row_begin = a.offsets[e];
        row_end = a.offsets[e + 1];
        if (row_end <= row_begin) return;  // untouched expert: its weights are never read
        codes += (int64_t)e * a.N * (K >> 1);
        scales += (int64_t)e * a.sf_stride;
        gs = a.gs[e];
    } else {
        row_begin = (int64_t)blockIdx.x * MT;
        row_end = (a.M < row_begin + MT) ? a.M : row_begin + MT;
        gs = a.gs[0];
    }

    // Weight rows of this warp (clamped; invalid ones are computed and dropped).
    int64_t wrow[R];
    bool cvalid[RW];
#pragma unroll
    for (int i = 0; i < RW; ++i) {
        const int64_t c = col0 + i;
        cvalid[i] = c < ncols_out;
        const int64_t cc = cvalid[i] ? c : col0;
        wrow[i] = cc;
        if constexpr (EPI == NVFP4_EPI_SWIGLU) wrow[RW + i] = a.N / 2 + cc;
    }

    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(a.x);
    for (int64_t m0 = row_begin; m0 < row_end; m0 += MT) {
        const int nt = (int)((row_end - m0) < MT ? (row_end - m0) : MT);
        const __nv_bfloat16* xr[MT];
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            const int64_t r = m0 + (t < nt ? t : 0);
            const int64_t src = a.gather ? a.gather[r] : r;
            xr[t] = xb + src * K;
        }
        float acc[R][MT];
#pragma unroll
        for (int i = 0; i < R; ++i)
#pragma unroll
            for (int t = 0; t < MT; ++t) acc[i][t] = 0.0f;

        for (int64_t c = lane; c < nchunk; c += 32) {
            // activation chunk -> fp32
            float xf[MT][CE];
#pragma unroll
            for (int t = 0; t < MT; ++t) {
#pragma unroll
                for (int q = 0; q < CE / 8; ++q) {
                    uint4 v = ldg_v4(xr[t] + c * CE + q * 8);
                    uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        xf[t][q * 8 + 2 * j] = bf16lo_to_f32(u[j]);
                        xf[t][q * 8 + 2 * j + 1] = bf16hi_to_f32(u[j]);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < R; ++i) {
                uint32_t w[VB / 4];
                load_codes<VB>(codes + wrow[i] * (K >> 1) + c * VB, w);
                float sd[NB];
                if constexpr (NB == 2) {
                    const uint16_t s2 = __ldg(reinterpret_cast<const uint16_t*>(
                        scales + sf_offset<LAYOUT>(wrow[i], 2 * c, nsf)));
                    const float2 f = f16x2_to_f32x2(e4m3x2_to_f16x2(s2));
                    sd[0] = f.x;
                    sd[NB - 1] = f.y;
                } else {
                    sd[0] = e4m3_to_f32(__ldg(scales + sf_offset<LAYOUT>(wrow[i], c, nsf)));
                }
                float wf[CE];
#pragma unroll
                for (int j = 0; j < VB / 4; ++j) {
                    uint32_t h[4];
                    e2m1x8_to_f16x2(w[j], h);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float2 f = f16x2_to_f32x2(h[q]);
                        wf[8 * j + 2 * q] = f.x;
                        wf[8 * j + 2 * q + 1] = f.y;
                    }
                }
#pragma unroll
                for (int t = 0; t < MT; ++t) {
#pragma unroll
                    for (int bb = 0; bb < NB; ++bb) {
                        float p = 0.0f;
#pragma unroll
                        for (int j = 0; j < 16; ++j) p = fmaf(xf[t][16 * bb + j], wf[16 * bb + j], p);
                        acc[i][t] = fmaf(p, sd[bb], acc[i][t]);
                    }
                }
            }
        }

#pragma unroll
        for (int i = 0; i < R; ++i)
#pragma unroll
            for (int t = 0; t < MT; ++t) acc[i][t] = warp_sum(acc[i][t]);

        OutT* y = reinterpret_cast<OutT*>(a.y);
#pragma unroll
        for (int i = 0; i < RW; ++i) {
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                if (lane == ((i * MT + t) & 31) && t < nt && cvalid[i]) {
                    float v;
                    if constexpr (EPI == NVFP4_EPI_SWIGLU) {
                        const float g = acc[i][t] * gs, u = acc[RW + i][t] * gs;
                        v = g / (1.0f + expf(-g)) * u;
                    } else {
                        v = acc[i][t] * gs;
                    }
                    store_out<OutT>(y + (m0 + t) * a.ldy + col0 + i, v);
                }
            }
        }
    }
}

template <int MT, int R, int VB, int LAYOUT, typename OutT, int EPI>
static int launch_cfg(const GemvArgs& a, cudaStream_t st) {
    constexpr int RW = (EPI == NVFP4_EPI_SWIGLU) ? R / 2 : R;
    const int64_t ncols = (EPI == NVFP4_EPI_SWIGLU) ? a.N / 2 : a.N;
    const int64_t tiles = (ncols + 8 * RW - 1) / (8 * RW);
    const int64_t gx = a.offsets ? a.E : (a.M + MT - 1) / MT;
    if (tiles > 65535 || gx > 0x7fffffff) return NVFP4_ERR_SHAPE;
    dim3 grid((unsigned)gx, (unsigned)tiles);
    gemv_w4a16_kernel<MT, R, VB, LAYOUT, OutT, EPI><<<grid, 256, 0, st>>>(a);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

template <int VB, int LAYOUT, typename OutT, int EPI>
static int launch_mt(const GemvArgs& a, int64_t rows_hint, cudaStream_t st) {
    if (rows_hint <= 1) return launch_cfg<1, 4, VB, LAYOUT, OutT, EPI>(a, st);
    if (rows_hint <= 2) return launch_cfg<2, 2, VB, LAYOUT, OutT, EPI>(a, st);
    return launch_cfg<4, 2, VB, LAYOUT, OutT, EPI>(a, st);
}

template <int VB, int LAYOUT>
static int launch_out(const GemvArgs& a, int64_t rows_hint, cudaStream_t st) {
    if (a.epilogue == NVFP4_EPI_SWIGLU) {
        if (a.y_dtype == NVFP4_DTYPE_BF16) return launch_mt<VB, LAYOUT, __nv_bfloat16, NVFP4_EPI_SWIGLU>(a, rows_hint, st);
        return launch_mt<VB, LAYOUT, float, NVFP4_EPI_SWIGLU>(a, rows_hint, st);
    }
    if (a.y_dtype == NVFP4_DTYPE_BF16) return launch_mt<VB, LAYOUT, __nv_bfloat16, NVFP4_EPI_NONE>(a, rows_hint, st);
    return launch_mt<VB, LAYOUT, float, NVFP4_EPI_NONE>(a, rows_hint, st);
}

int launch_gemv_w4a16(const GemvArgs& a, cudaStream_t st) {
    // Dense: token-group width from M.  Grouped: rows per expert vary; the
    // widest group (4) amortises the weight read for hot experts.
    const int64_t rows_hint = a.offsets ? 4 : a.M;
    const bool v16 = (a.K % 32) == 0;
    if (a.sf_layout == NVFP4_SF_TILED)
        return v16 ? launch_out<16, NVFP4_SF_TILED>(a, rows_hint, st) : launch_out<8, NVFP4_SF_TILED>(a, rows_hint, st);
    return v16 ? launch_out<16, NVFP4_SF_ROWMAJOR>(a, rows_hint, st)
               : launch_out<8, NVFP4_SF_ROWMAJOR>(a, rows_hint, st);
}

}  // namespace nvfp4
