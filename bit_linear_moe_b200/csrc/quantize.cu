// K1: NVFP4 quantizer (imp v0.20.0 release notes, "Highlights": first-party
// NVFP4 quantizer; round-to-nearest part).
//
// Pass 1 (amax_kernel) reduces max|x| over the tensor into one word of the
// caller's workspace (non-negative floats order like their bit patterns, so an
// unsigned atomicMax is exact and order-independent).  Pass 2
// (quantize_kernel) gives one thread to each 16-element block:
//     gs     = gs_in, or amax / 2688 (1 if amax == 0)     binary32, one rounding
//     denom  = gs * 6
//     s      = E4M3(amax_block / denom)                    nearest-even, satfinite
//     r      = E4M3value(s) * gs
//     code_i = E2M1(x_i / r), or +0 for the whole block when r == 0
// The quotients are those of IEEE round-to-nearest division; a reciprocal
// product stands in for the division wherever it provably yields the same
// code (e2m1x8_of_quotients).  Nothing is contracted.
// HBM-bound: pass 1 reads x once, pass 2 reads x again (from L2 when x fits)
// and writes 9/32 of its bf16 size (codes + scales).  Pass 2 is a
// programmatic dependent of pass 1: its loads of x overlap pass 1's tail.
#include "common.cuh"
#include "internal.h"
#include "tma.cuh"

namespace nvfp4 {

// Eight consecutive elements (16 bytes of bf16, 32 of fp32) -> fp32.
template <typename T>
struct Vec8;

template <>
struct Vec8<__nv_bfloat16> {
    static NVFP4_DEV void load(const __nv_bfloat16* p, float (&v)[8]) {
        const uint4 a = ldg_v4(p);
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = bf16lo_to_f32(w[i]);
            v[2 * i + 1] = bf16hi_to_f32(w[i]);
        }
    }
};

template <>
struct Vec8<float> {
    static NVFP4_DEV void load(const float* p, float (&v)[8]) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint4 a = ldg_v4(p + 4 * i);
            v[4 * i] = __uint_as_float(a.x);
            v[4 * i + 1] = __uint_as_float(a.y);
            v[4 * i + 2] = __uint_as_float(a.z);
            v[4 * i + 3] = __uint_as_float(a.w);
        }
    }
};

NVFP4_DEV float amax8(const float (&v)[8]) {
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
    return m;
}

NVFP4_DEV void block_amax_to(float m, unsigned* amax_bits) {
    m = warp_max(m);
    __shared__ float red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
        atomicMax(amax_bits, __float_as_uint(m));
    }
}

// max|x| over n8 runs of eight elements, consecutive lanes on consecutive runs.
template <typename T>
__global__ void __launch_bounds__(256) amax_kernel(const T* __restrict__ x, int64_t n8,
                                                   unsigned* __restrict__ amax_bits) {
    griddep_launch_dependents();  // the quantizer may start loading x now
    float m = 0.0f;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    for (; i + 3 * stride < n8; i += 4 * stride) {  // four loads in flight per lane
        float v[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u) Vec8<T>::load(x + (i + u * stride) * 8, v[u]);
#pragma unroll
        for (int u = 0; u < 4; ++u) m = fmaxf(m, amax8(v[u]));
    }
    for (; i < n8; i += stride) {
        float v[8];
        Vec8<T>::load(x + i * 8, v);
        m = fmaxf(m, amax8(v));
    }
    block_amax_to(m, amax_bits);
}

// max|x| over the rows src_rows[r] (r < nrows, or < *row_bound when given;
// entries < 0 skipped).  A CTA's 256 threads are 256 / tpr rows of tpr
// 16-byte pieces (tpr = 2^lg_tpr, the largest power of two <= 256 dividing a
// row's pieces), four such row groups in flight at once; CTAs take row groups
// round-robin.
template <typename T>
__global__ void __launch_bounds__(256) amax_rows_kernel(const T* __restrict__ x, const int32_t* __restrict__ src_rows,
                                                        int64_t nrows, const int32_t* __restrict__ row_bound,
                                                        int64_t cols, int lg_tpr, unsigned* __restrict__ amax_bits) {
    griddep_launch_dependents();
    float m = 0.0f;
    const int64_t nb = cols / 8;
    const int rpp = 256 >> lg_tpr;  // rows per pass
    const int lr = threadIdx.x >> lg_tpr, c0 = threadIdx.x & ((1 << lg_tpr) - 1);
    const int64_t rend = row_bound && (int64_t)*row_bound < nrows ? (int64_t)*row_bound : nrows;
    for (int64_t r0 = (int64_t)blockIdx.x * 4 * rpp; r0 < rend; r0 += (int64_t)gridDim.x * 4 * rpp) {
        int32_t src[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t r = r0 + u * rpp + lr;
            src[u] = r < rend ? src_rows[r] : -1;
        }
        for (int64_t c = c0; c < nb; c += (1 << lg_tpr)) {
            float v[4][8];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (src[u] >= 0) Vec8<T>::load(x + (int64_t)src[u] * cols + c * 8, v[u]);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (src[u] >= 0) m = fmaxf(m, amax8(v[u]));
        }
    }
    block_amax_to(m, amax_bits);
}

NVFP4_DEV float global_scale_from(const float* gs_in, const unsigned* amax_bits) {
    if (gs_in) return *gs_in;
    const float amax = __uint_as_float(*amax_bits);
    return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);
}

// Approximate reciprocal (relative error below 2^-22 for normal inputs).
NVFP4_DEV float rcp_approx(float a) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(a));
    return r;
}

constexpr float kBracketLo = 0.99999618530273437500f;  // 1 - 2^-18
constexpr float kBracketHi = 1.00000381469726562500f;  // 1 + 2^-18

// E4M3 byte of RN(a / d), a >= 0 (the block scale).  inv ~ 1/d within 2^-22
// (0 when d is 0, subnormal or not finite).  t = RN(a * inv) lies within
// 2^-21 of RN(a / d); E4M3 rounding is monotone, so when t (1 - 2^-18) and
// t (1 + 2^-18) give the same byte (one cvt converts both) it is the byte of
// RN(a / d); otherwise the division decides.
NVFP4_DEV uint32_t e4m3_of_quotient(float a, float d, float inv) {
    if (inv != 0.0f) {
        const float t = __fmul_rn(a, inv);
        uint16_t pr;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
            : "=h"(pr)
            : "f"(__fmul_rn(t, kBracketHi)), "f"(__fmul_rn(t, kBracketLo)));
        if ((pr & 0xFF) == (pr >> 8)) return pr & 0xFF;
    }
    return f32_to_e4m3(__fdiv_rn(a, d));
}

// E2M1 code (low nibble) of RN(v / r).
NVFP4_DEV uint32_t e2m1_of_division(float v, float r) {
    uint16_t pr;
    asm("{\n\t.reg .b8 c;\n\tcvt.rn.satfinite.e2m1x2.f32 c, %1, %2;\n\tcvt.u16.u8 %0, c;\n\t}"
        : "=h"(pr)
        : "f"(0.0f), "f"(__fdiv_rn(v, r)));
    return pr & 0xF;
}

// E2M1 codes of v[j] / r (j < 16, two words), each quotient the IEEE-rounded
// division.  inv ~ 1/r within 2^-22 (0: always divide) and p = RN(v * inv)
// put p within 2^-21 |v / r| of RN(v / r).  E2M1 rounding is monotone over
// finite inputs (a NaN gives the same code either way), so where p (1 - 2^-18)
// and p (1 + 2^-18) round to the same code, that is the code of RN(v / r); an
// element whose bracket straddles a rounding boundary is divided.  (With bf16
// inputs that is not rare: an element with the mantissa of the tensor's amax
// makes v / r a boundary value in exact arithmetic, 0.75, 1.75 or 3.5, up to
// the roundings of gs and r.)  A block whose amax / r is not below 15 (an
// infinity, or near overflow) divides every element.
NVFP4_DEV uint2 e2m1x16_of_quotients(const float (&v)[16], float amax, float r, float inv) {
    uint32_t code[2], diff[2];
    if (inv != 0.0f && __fmul_rn(amax, inv) < 15.0f) {
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            float lo[8], hi[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float p = __fmul_rn(v[8 * w + j], inv);
                lo[j] = __fmul_rn(p, kBracketLo);
                hi[j] = __fmul_rn(p, kBracketHi);
            }
            code[w] = f32x8_to_e2m1(hi);
            diff[w] = f32x8_to_e2m1(lo) ^ code[w];
        }
    } else {
        code[0] = code[1] = 0u;
        diff[0] = diff[1] = 0xFFFFFFFFu;
    }
    if (diff[0] | diff[1]) {
#pragma unroll
        for (int w = 0; w < 2; ++w)
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (diff[w] & (0xFu << (4 * j)))
                    code[w] = (code[w] & ~(0xFu << (4 * j))) | (e2m1_of_division(v[8 * w + j], r) << (4 * j));
    }
    return make_uint2(code[0], code[1]);
}

// r is a normal float with a normal, finite reciprocal.
NVFP4_DEV bool rcp_safe(float r) { return r >= 1.17549435e-38f && r <= 1.0e37f; }

constexpr int kQThreads = 128;  // one CTA: 128 threads, one 16-element block each
constexpr int kQRows = 2;       // row passes per iteration: their loads are issued together

// Sixteen consecutive elements -> fp32 (two Vec8 loads).
template <typename T>
NVFP4_DEV void load16(const T* p, float (&v)[16]) {
    float a[8], b[8];
    Vec8<T>::load(p, a);
    Vec8<T>::load(p + 8, b);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        v[j] = a[j];
        v[8 + j] = b[j];
    }
}

// One thread per (row, 16-element block) of the padded scale grid (rows
// grid_rows, columns grid_cols).  A CTA's 128 threads are rpc = 128 / cw rows
// of cw consecutive blocks (cw = 2^lg_cw, the largest power of two <= 128
// dividing the padded column count, so short rows fill whole CTAs):
// thread t takes block blockIdx.x * cw + (t mod cw) of row
// r0 + i * rpc + t / cw, for i < 2 (both rows' loads in flight before either
// is used) and r0 = 2 rpc (blockIdx.y + j gridDim.y); the grid is capped so
// that each CTA walks several row groups.
// src_rows (nullable): dst row r reads source row src_rows[r]; -1 marks a
// padding row (zero codes and scales).  Rows >= dst_rows (tiled padding) and
// scale columns >= cols/16 get zero scales and no codes.
// row_bound (nullable): rows >= *row_bound are not touched at all.
// row_inv (nullable): source row r is first normalised, x -> bf16(x * row_inv[r])
// (the rows of nvfp4_rms_norm, recomputed instead of read back); x_ld is the
// source row stride in elements.
// Launched as a programmatic dependent of the pass that reduced amax_bits and
// row_inv: x (complete before that pass began) is loaded first, the pass's
// outputs only after griddep_wait().
template <typename T, int LAYOUT>
__global__ void __launch_bounds__(kQThreads) quantize_kernel(
    const T* __restrict__ x, const int32_t* __restrict__ src_rows, int64_t dst_rows, int64_t cols,
    int64_t grid_rows, int64_t grid_cols, const float* __restrict__ gs_in,
    const unsigned* __restrict__ amax_bits, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
    float* __restrict__ gs_out, const int32_t* __restrict__ row_bound, int64_t x_ld,
    const float* __restrict__ row_inv, int lg_cw) {
    griddep_launch_dependents();
    __shared__ float s_par[3];  // gs, denom, ~1/denom (0: divide)
    const int t = threadIdx.x;
    const int rpc = kQThreads >> lg_cw;
    const int64_t b = ((int64_t)blockIdx.x << lg_cw) + (t & ((1 << lg_cw) - 1));
    const int r_local = t >> lg_cw;
    const int64_t nsf = cols >> 4;
    const bool col_live = b < grid_cols, col_real = b < nsf;
    const int64_t rbound = row_bound ? (int64_t)*row_bound : grid_rows;
    const int64_t rend = rbound < grid_rows ? rbound : grid_rows;
    const T* xb = x + b * 16;
    uint8_t* cb = codes + b * 8;
    bool waited = false;
    for (int64_t r0 = (int64_t)blockIdx.y * rpc * kQRows; r0 < rend; r0 += (int64_t)gridDim.y * rpc * kQRows) {
        float v[kQRows][16];
        int64_t src[kQRows];
        bool real[kQRows];
#pragma unroll
        for (int i = 0; i < kQRows; ++i) {
            const int64_t r = r0 + i * rpc + r_local;
            src[i] = r;
            if (r < rend && r < dst_rows && src_rows) src[i] = src_rows[r];
            real[i] = col_real && r < rend && r < dst_rows && src[i] >= 0;
            if (real[i]) load16(xb + src[i] * x_ld, v[i]);
        }
        if (!waited) {
            griddep_wait();
            if (t == 0) {
                const float gs = global_scale_from(gs_in, amax_bits);
                const float denom = __fmul_rn(gs, 6.0f);
                s_par[0] = gs;
                s_par[1] = denom;
                s_par[2] = rcp_safe(denom) ? rcp_approx(denom) : 0.0f;
                if (gs_out && blockIdx.x == 0 && blockIdx.y == 0) *gs_out = gs;
            }
            __syncthreads();
            waited = true;
        }
        const float gs = s_par[0], denom = s_par[1], inv_denom = s_par[2];
#pragma unroll
        for (int i = 0; i < kQRows; ++i) {
            const int64_t r = r0 + i * rpc + r_local;
            if (!col_live || r >= rend) continue;
            const int64_t soff = sf_offset<LAYOUT>(r, b, nsf);
            uint2* cw = reinterpret_cast<uint2*>(cb + r * (cols >> 1));
            if (!real[i]) {
                scales[soff] = 0;
                if (r < dst_rows && col_real) *cw = make_uint2(0u, 0u);
                continue;
            }
            if (row_inv) {
                const float inv = row_inv[src[i]];
#pragma unroll
                for (int j = 0; j < 16; ++j) v[i][j] = __bfloat162float(__float2bfloat16_rn(v[i][j] * inv));
            }
            float amax_b = 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) amax_b = fmaxf(amax_b, fabsf(v[i][j]));
            const uint32_t sb = e4m3_of_quotient(amax_b, denom, inv_denom);
            const float rsc = __fmul_rn(e4m3_to_f32(sb), gs);
            uint2 packed = make_uint2(0u, 0u);
            if (rsc != 0.0f)
                packed = e2m1x16_of_quotients(v[i], amax_b, rsc, rcp_safe(rsc) ? rcp_approx(rsc) : 0.0f);
            *cw = packed;
            scales[soff] = (uint8_t)sb;
        }
    }
}

static int grid_for(int64_t n, int threads) {
    int64_t g = (n + threads - 1) / threads;
    return (int)(g < 1 ? 1 : g);
}

int launch_amax(const void* x, int x_dtype, int64_t n, unsigned* amax_bits, cudaStream_t st) {
    if (cudaMemsetAsync(amax_bits, 0, sizeof(unsigned), st) != cudaSuccess) return NVFP4_ERR_LAUNCH;
    const int64_t n8 = n / 8;
    int grid = grid_for(n8, 256);
    const int cap = 148 * 8;
    if (grid > cap) grid = cap;
    if (x_dtype == NVFP4_DTYPE_BF16)
        amax_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)x, n8, amax_bits);
    else
        amax_kernel<float><<<grid, 256, 0, st>>>((const float*)x, n8, amax_bits);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

int launch_amax_rows(const void* x, const int32_t* src_rows, int64_t nrows, int64_t cols, unsigned* amax_bits,
                     cudaStream_t st, const int32_t* row_bound) {
    if (cudaMemsetAsync(amax_bits, 0, sizeof(unsigned), st) != cudaSuccess) return NVFP4_ERR_LAUNCH;
    const int64_t nb = cols / 8;
    int lg_tpr = 0;  // the largest power of two <= 256 dividing a row's 16-byte pieces
    while (lg_tpr < 8 && nb % (2 << lg_tpr) == 0) ++lg_tpr;
    const int64_t rows_per_cta = (int64_t)(256 >> lg_tpr) * 4;
    int grid = grid_for((nrows + rows_per_cta - 1) / rows_per_cta, 1);
    if (grid > 148 * 8) grid = 148 * 8;
    amax_rows_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)x, src_rows, nrows, row_bound, cols,
                                                          lg_tpr, amax_bits);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

int launch_quantize(const void* x, int x_dtype, const int32_t* src_rows, int64_t dst_rows, int64_t cols,
                    int sf_layout, const float* gs_in, const unsigned* amax_bits, uint8_t* codes,
                    uint8_t* scales, float* gs_out, cudaStream_t st, const int32_t* row_bound, int64_t x_ld,
                    const float* row_inv) {
    if (x_ld <= 0) x_ld = cols;
    const int64_t nsf = cols / 16;
    const int64_t grid_rows = sf_layout == NVFP4_SF_TILED ? (dst_rows + 127) / 128 * 128 : dst_rows;
    const int64_t grid_cols = sf_layout == NVFP4_SF_TILED ? (nsf + 3) / 4 * 4 : nsf;
    int lg_cw = 0;  // the largest power of two <= 128 dividing grid_cols
    while (lg_cw < 7 && grid_cols % (2 << lg_cw) == 0) ++lg_cw;
    const int64_t gx = grid_cols >> lg_cw;
    if (gx > 0x7fffffff) return NVFP4_ERR_SHAPE;
    const int64_t rows_per_cta = (int64_t)(kQThreads >> lg_cw) * kQRows;
    int64_t gy = (grid_rows + rows_per_cta - 1) / rows_per_cta;
    // about four resident waves (8 CTAs of 128 threads per SM at 64
    // registers): enough CTAs to hide the tail, few enough that each walks
    // several row groups (measured: one wave left M = 8192 x 5120 at 64 us,
    // four give 55 us; uncapped 64-thread CTAs, 59 us)
    const int64_t gy_cap = (148 * 32 + gx - 1) / gx;
    if (gy > gy_cap) gy = gy_cap;
    if (gy > 65535) gy = 65535;
    if (gy < 1) gy = 1;
    // With amax_bits from the pass just launched (no gs_in), a programmatic
    // dependent of that pass; otherwise an ordinary launch.
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)gx, (unsigned)gy);
    cfg.blockDim = dim3(kQThreads);
    cfg.stream = st;
    if (!gs_in) {
        set_pdl_attr(attr[0]);
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    cudaError_t e;
#define NVFP4_Q(T, L)                                                                                         \
    e = cudaLaunchKernelEx(&cfg, quantize_kernel<T, L>, (const T*)x, src_rows, dst_rows, cols, grid_rows,      \
                           grid_cols, gs_in, amax_bits, codes, scales, gs_out, row_bound, x_ld, row_inv, lg_cw)
    if (x_dtype == NVFP4_DTYPE_BF16) {
        if (sf_layout == NVFP4_SF_TILED) NVFP4_Q(__nv_bfloat16, NVFP4_SF_TILED);
        else NVFP4_Q(__nv_bfloat16, NVFP4_SF_ROWMAJOR);
    } else {
        if (sf_layout == NVFP4_SF_TILED) NVFP4_Q(float, NVFP4_SF_TILED);
        else NVFP4_Q(float, NVFP4_SF_ROWMAJOR);
    }
#undef NVFP4_Q
    return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

}  // namespace nvfp4
