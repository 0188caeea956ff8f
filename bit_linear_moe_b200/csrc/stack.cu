// K9: glue between the linears of a dense decode stack (Ignis README, "The
// decode round": a decode step streams every layer's weights once).
//
//   rms_norm   y[r, c] = bf16(x[r, c] / sqrt(mean_c x[r, c]^2)), an all-zero
//              row gives zeros; rows of `cols` elements at stride `ld`, so a
//              slice of a wider output (the Q part of QKV) is read in place
//   silu_mul   h[r, j] = bf16(silu(g[r, j]) * g[r, half + j])
//
// Each is a few hundred KB at most per decode step: one CTA per row, fp32
// sums, IEEE-rounded square root, division and exponential.  Both run as
// programmatic dependents: they let the next kernel (the next linear, which
// fetches its weights before it waits) launch at once, and read their input
// only after griddepcontrol.wait.
#include "internal.h"
#include "tma.cuh"

namespace nvfp4 {

template <typename T>
NVFP4_DEV float load_f32(const T* p);
template <>
NVFP4_DEV float load_f32<float>(const float* p) {
    return __ldg(p);
}
template <>
NVFP4_DEV float load_f32<__nv_bfloat16>(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
}

// STATS: instead of writing y, store the row's factor in inv[r] and fold the
// largest |bf16(x * inv)| of the row into *amax_bits.
template <typename T, bool STATS = false>
__global__ void __launch_bounds__(1024) rms_norm_kernel(const T* __restrict__ x, int64_t cols, int64_t ld,
                                                       __nv_bfloat16* __restrict__ y, float* __restrict__ inv_out,
                                                       unsigned* __restrict__ amax_bits) {
    griddep_launch_dependents();
    griddep_wait();
    const int64_t r = blockIdx.x;
    const T* xr = x + r * ld;
    float ss = 0.0f;
    for (int64_t c = threadIdx.x; c < cols; c += blockDim.x) {
        const float v = load_f32<T>(xr + c);
        ss = fmaf(v, v, ss);
    }
    ss = warp_sum(ss);
    __shared__ float red[32];
    __shared__ float s_inv;
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.0f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
        s_inv = t > 0.0f ? 1.0f / sqrtf(t / (float)cols) : 0.0f;
    }
    __syncthreads();
    const float inv = s_inv;
    if constexpr (STATS) {
        float m = 0.0f;
        for (int64_t c = threadIdx.x; c < cols; c += blockDim.x)
            m = fmaxf(m, fabsf(__bfloat162float(__float2bfloat16_rn(load_f32<T>(xr + c) * inv))));
        m = warp_max(m);
        if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
        if (threadIdx.x == 0) inv_out[r] = inv;
    } else {
        __nv_bfloat16* yr = y + r * cols;
        for (int64_t c = threadIdx.x; c < cols; c += blockDim.x)
            yr[c] = __float2bfloat16_rn(load_f32<T>(xr + c) * inv);
    }
}

template <typename T>
__global__ void __launch_bounds__(256) silu_mul_kernel(const T* __restrict__ g, int64_t rows, int64_t half,
                                                       __nv_bfloat16* __restrict__ h) {
    griddep_launch_dependents();
    griddep_wait();
    const int64_t n = rows * half;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / half, j = i % half;
        const float a = load_f32<T>(g + r * 2 * half + j);
        const float b = load_f32<T>(g + r * 2 * half + half + j);
        h[i] = __float2bfloat16_rn(a / (1.0f + expf(-a)) * b);
    }
}

static cudaLaunchConfig_t glue_config(cudaLaunchAttribute* attr, unsigned grid, unsigned block, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.stream = st;
    set_pdl_attr(attr[0]);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

int launch_rms_norm(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld, void* y, cudaStream_t st) {
    if (rows > 0x7fffffff) return NVFP4_ERR_SHAPE;
    // a few rows (decode): 1024 threads per row, so a row's loads go out together
    const unsigned block = rows <= 8 ? 1024 : 256;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = glue_config(attr, (unsigned)rows, block, st);
    cudaError_t r;
    if (x_dtype == NVFP4_DTYPE_BF16)
        r = cudaLaunchKernelEx(&cfg, rms_norm_kernel<__nv_bfloat16, false>, (const __nv_bfloat16*)x, cols, ld,
                               (__nv_bfloat16*)y, (float*)nullptr, (unsigned*)nullptr);
    else
        r = cudaLaunchKernelEx(&cfg, rms_norm_kernel<float, false>, (const float*)x, cols, ld, (__nv_bfloat16*)y,
                               (float*)nullptr, (unsigned*)nullptr);
    return r == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

int launch_rms_stats(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld, float* inv,
                     unsigned* amax_bits, cudaStream_t st) {
    if (rows > 0x7fffffff) return NVFP4_ERR_SHAPE;
    if (cudaMemsetAsync(amax_bits, 0, sizeof(unsigned), st) != cudaSuccess) return NVFP4_ERR_LAUNCH;
    const unsigned block = rows <= 8 ? 1024 : 256;  // as launch_rms_norm: the same sums
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = glue_config(attr, (unsigned)rows, block, st);
    cudaError_t r;
    if (x_dtype == NVFP4_DTYPE_BF16)
        r = cudaLaunchKernelEx(&cfg, rms_norm_kernel<__nv_bfloat16, true>, (const __nv_bfloat16*)x, cols, ld,
                               (__nv_bfloat16*)nullptr, inv, amax_bits);
    else
        r = cudaLaunchKernelEx(&cfg, rms_norm_kernel<float, true>, (const float*)x, cols, ld,
                               (__nv_bfloat16*)nullptr, inv, amax_bits);
    return r == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

int launch_silu_mul(const void* g, int g_dtype, int64_t rows, int64_t half, void* h, cudaStream_t st) {
    const int64_t n = rows * half;
    int64_t grid = (n + 255) / 256;
    if (grid > 148 * 16) grid = 148 * 16;
    if (grid < 1) grid = 1;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = glue_config(attr, (unsigned)grid, 256, st);
    cudaError_t r;
    if (g_dtype == NVFP4_DTYPE_BF16)
        r = cudaLaunchKernelEx(&cfg, silu_mul_kernel<__nv_bfloat16>, (const __nv_bfloat16*)g, rows, half,
                               (__nv_bfloat16*)h);
    else
        r = cudaLaunchKernelEx(&cfg, silu_mul_kernel<float>, (const float*)g, rows, half, (__nv_bfloat16*)h);
    return r == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

}  // namespace nvfp4
