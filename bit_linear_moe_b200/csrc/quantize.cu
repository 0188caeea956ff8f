// K1: NVFP4 quantizer (imp v0.20.0 release notes, "Highlights": first-party
// NVFP4 quantizer; round-to-nearest part).
//
// Pass 1 (amax_kernel) reduces max|x| over the tensor into one word of the
// caller's workspace (non-negative floats order like their bit patterns, so an
// unsigned atomicMax is exact and order-independent).  Pass 2
// (quantize_kernel) gives one thread per 16-element block:
//     gs     = gs_in, or amax / 2688 (1 if amax == 0)     binary32, one rounding
//     denom  = gs * 6
//     s      = E4M3(amax_block / denom)                    nearest-even, satfinite
//     r      = E4M3value(s) * gs
//     code_i = E2M1(x_i / r), or +0 for the whole block when r == 0
// The divisions are IEEE round-to-nearest (__fdiv_rn); nothing is contracted.
// HBM-bound: pass 1 reads x once, pass 2 reads x again and writes 9/32 of its
// bf16 size (codes + scales).
#include "common.cuh"
#include "internal.h"

namespace nvfp4 {

template <typename T>
struct Vec16;  // 16 consecutive elements -> fp32

template <>
struct Vec16<__nv_bfloat16> {
    static NVFP4_DEV void load(const __nv_bfloat16* p, float (&v)[16]) {
        uint4 a = ldg_v4(p), b = ldg_v4(p + 8);
        uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v[2 * i] = bf16lo_to_f32(w[i]);
            v[2 * i + 1] = bf16hi_to_f32(w[i]);
        }
    }
};

template <>
struct Vec16<float> {
    static NVFP4_DEV void load(const float* p, float (&v)[16]) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint4 a = ldg_v4(p + 4 * i);
            v[4 * i] = __uint_as_float(a.x);
            v[4 * i + 1] = __uint_as_float(a.y);
            v[4 * i + 2] = __uint_as_float(a.z);
            v[4 * i + 3] = __uint_as_float(a.w);
        }
    }
};

template <typename T>
__global__ void __launch_bounds__(256) amax_kernel(const T* __restrict__ x, int64_t nvec16,
                                                   unsigned* __restrict__ amax_bits) {
    float m = 0.0f;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nvec16;
         i += (int64_t)gridDim.x * blockDim.x) {
        float v[16];
        Vec16<T>::load(x + i * 16, v);
#pragma unroll
        for (int j = 0; j < 16; ++j) m = fmaxf(m, fabsf(v[j]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
        atomicMax(amax_bits, __float_as_uint(m));
    }
}

// max|x| over the rows src_rows[r] (r < nrows, entries < 0 skipped), 16 columns per item.
template <typename T>
__global__ void __launch_bounds__(256) amax_rows_kernel(const T* __restrict__ x, const int32_t* __restrict__ src_rows,
                                                        int64_t nrows, int64_t cols, unsigned* __restrict__ amax_bits) {
    float m = 0.0f;
    const int64_t nb = cols / 16, n = nrows * nb;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / nb, b = i % nb;
        const int32_t src = src_rows[r];
        if (src < 0) continue;
        float v[16];
        Vec16<T>::load(x + (int64_t)src * cols + b * 16, v);
#pragma unroll
        for (int j = 0; j < 16; ++j) m = fmaxf(m, fabsf(v[j]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
        atomicMax(amax_bits, __float_as_uint(m));
    }
}

NVFP4_DEV float global_scale_from(const float* gs_in, const unsigned* amax_bits) {
    if (gs_in) return *gs_in;
    const float amax = __uint_as_float(*amax_bits);
    return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);
}

// One thread per (dst row, 16-element block) over the padded scale grid.
// src_rows (nullable): dst row r reads source row src_rows[r]; -1 marks a
// padding row (zero codes and scales).  Rows >= dst_rows (tiled padding) and
// scale columns >= cols/16 get zero scales and no codes.
// row_inv (nullable): source row r is first normalised, x -> bf16(x * row_inv[r])
// (the rows of nvfp4_rms_norm, recomputed instead of read back); x_ld is the
// source row stride in elements.
template <typename T, int LAYOUT>
__global__ void __launch_bounds__(256) quantize_kernel(
    const T* __restrict__ x, const int32_t* __restrict__ src_rows, int64_t dst_rows, int64_t cols,
    int64_t grid_rows, int64_t grid_cols, const float* __restrict__ gs_in,
    const unsigned* __restrict__ amax_bits, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
    float* __restrict__ gs_out, const int32_t* __restrict__ row_bound, int64_t x_ld,
    const float* __restrict__ row_inv) {
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const float gs = global_scale_from(gs_in, amax_bits);
    if (i == 0 && gs_out) *gs_out = gs;
    if (i >= grid_rows * grid_cols) return;
    const int64_t r = i / grid_cols, b = i % grid_cols;
    if (row_bound && r >= (int64_t)*row_bound) return;  // rows nobody reads (padded expert layout)
    const int64_t nsf = cols >> 4;
    const int64_t soff = sf_offset<LAYOUT>(r, b, nsf);
    int64_t src = r;
    if (r < dst_rows && src_rows) src = src_rows[r];
    if (r >= dst_rows || b >= nsf || src < 0) {
        scales[soff] = 0;
        if (r < dst_rows && b < nsf) *reinterpret_cast<uint2*>(codes + r * (cols >> 1) + b * 8) = make_uint2(0, 0);
        return;
    }
    float v[16];
    Vec16<T>::load(x + src * x_ld + b * 16, v);
    if (row_inv) {
        const float inv = row_inv[src];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = __bfloat162float(__float2bfloat16_rn(v[j] * inv));
    }
    float amax_b = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) amax_b = fmaxf(amax_b, fabsf(v[j]));
    const float denom = __fmul_rn(gs, 6.0f);
    const uint32_t s = f32_to_e4m3(__fdiv_rn(amax_b, denom));
    const float rsc = __fmul_rn(e4m3_to_f32(s), gs);
    uint2 packed = make_uint2(0, 0);
    if (rsc != 0.0f) {
        float q0[8], q1[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            q0[j] = __fdiv_rn(v[j], rsc);
            q1[j] = __fdiv_rn(v[8 + j], rsc);
        }
        packed.x = f32x8_to_e2m1(q0);
        packed.y = f32x8_to_e2m1(q1);
    }
    *reinterpret_cast<uint2*>(codes + r * (cols >> 1) + b * 8) = packed;
    scales[soff] = (uint8_t)s;
}

static int grid_for(int64_t n, int threads) {
    int64_t g = (n + threads - 1) / threads;
    return (int)(g < 1 ? 1 : g);
}

int launch_amax(const void* x, int x_dtype, int64_t n, unsigned* amax_bits, cudaStream_t st) {
    if (cudaMemsetAsync(amax_bits, 0, sizeof(unsigned), st) != cudaSuccess) return NVFP4_ERR_LAUNCH;
    const int64_t nvec = n / 16;
    int grid = grid_for(nvec, 256);
    const int cap = 148 * 8;
    if (grid > cap) grid = cap;
    if (x_dtype == NVFP4_DTYPE_BF16)
        amax_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)x, nvec, amax_bits);
    else
        amax_kernel<float><<<grid, 256, 0, st>>>((const float*)x, nvec, amax_bits);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

int launch_amax_rows(const void* x, const int32_t* src_rows, int64_t nrows, int64_t cols, unsigned* amax_bits,
                     cudaStream_t st) {
    if (cudaMemsetAsync(amax_bits, 0, sizeof(unsigned), st) != cudaSuccess) return NVFP4_ERR_LAUNCH;
    int grid = grid_for(nrows * (cols / 16), 256);
    if (grid > 148 * 8) grid = 148 * 8;
    amax_rows_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)x, src_rows, nrows, cols, amax_bits);
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
    const int grid = grid_for(grid_rows * grid_cols, 256);
#define NVFP4_Q(T, L)                                                                                 \
    quantize_kernel<T, L><<<grid, 256, 0, st>>>((const T*)x, src_rows, dst_rows, cols, grid_rows,     \
                                                grid_cols, gs_in, amax_bits, codes, scales, gs_out, row_bound, \
                                                x_ld, row_inv)
    if (x_dtype == NVFP4_DTYPE_BF16) {
        if (sf_layout == NVFP4_SF_TILED) NVFP4_Q(__nv_bfloat16, NVFP4_SF_TILED);
        else NVFP4_Q(__nv_bfloat16, NVFP4_SF_ROWMAJOR);
    } else {
        if (sf_layout == NVFP4_SF_TILED) NVFP4_Q(float, NVFP4_SF_TILED);
        else NVFP4_Q(float, NVFP4_SF_ROWMAJOR);
    }
#undef NVFP4_Q
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

}  // namespace nvfp4
