// K12: activation-calibrated NVFP4 quantization of a weight (imp v0.20.0
// release notes, "Highlights": a first-party NVFP4 quantizer with AWQ-class
// activation calibration).
//
// The pages name the method class only.  The reading implemented here: from
// a calibration batch X [S, K] of activations, per input channel k
//     a_k  = (sum_s |x_sk|) / S,   m2_k = (sum_s x_sk^2) / S
// (binary32, rows summed in order).  For alpha = j / 8, j = 0..8, channel
// scales s_k = a_k^alpha (1 for a channel with a_k == 0), normalised by
// sqrt(max_k s_k * min_k s_k); the weight W [N, K] is scaled per column,
// W' = W diag(s), and quantized by the round-to-nearest NVFP4 rules of
// nvfp4_quantize.  The effective weight is dequant(W') diag(1/s) (the
// activations are divided by s at inference).  alpha is chosen to minimise
//     err(alpha) = sum_k m2_k sum_n (dequant(W')_nk / s_k - w_nk)^2
// (the diagonal of the calibration Gram matrix weights the per-channel
// weight error), lowest j on ties; alpha = 0 is plain RTN, so the result is
// never worse than RTN by this measure.
//
// a^(j/8) is built from square roots and products in a fixed order
// (r1 = sqrt(a), r2 = sqrt(r1), r3 = sqrt(r2); a^(3/8) = r2 * r3, a^(5/8) =
// r1 * r3, a^(3/4) = r1 * r2, a^(7/8) = (r1 * r2) * r3): IEEE square root and
// multiplication are correctly rounded, so the scales, and with them the
// codes, are reproducible bit for bit by any IEEE implementation.
#include "common.cuh"
#include "internal.h"

namespace nvfp4 {

constexpr int kCalAlphas = 9;

// a_k, m2_k: one thread per channel, rows in order (binary32).
__global__ void __launch_bounds__(256) cal_stats_kernel(const __nv_bfloat16* __restrict__ x, int64_t S, int64_t K,
                                                        float* __restrict__ a, float* __restrict__ m2) {
    const int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (k >= K) return;
    float sa = 0.0f, s2 = 0.0f;
    for (int64_t s = 0; s < S; ++s) {
        const float v = __bfloat162float(x[s * K + k]);
        sa = __fadd_rn(sa, fabsf(v));
        s2 = __fadd_rn(s2, __fmul_rn(v, v));
    }
    a[k] = __fdiv_rn(sa, (float)S);
    m2[k] = __fdiv_rn(s2, (float)S);
}

NVFP4_DEV float pow_eighths(float a, int j) {
    const float r1 = __fsqrt_rn(a), r2 = __fsqrt_rn(r1), r3 = __fsqrt_rn(r2);
    switch (j) {
        case 0: return 1.0f;
        case 1: return r3;
        case 2: return r2;
        case 3: return __fmul_rn(r2, r3);
        case 4: return r1;
        case 5: return __fmul_rn(r1, r3);
        case 6: return __fmul_rn(r1, r2);
        case 7: return __fmul_rn(__fmul_rn(r1, r2), r3);
        default: return a;
    }
}

// s[j][k] for every alpha: one CTA of 1024 threads per j.
__global__ void __launch_bounds__(1024) cal_scales_kernel(const float* __restrict__ a, int64_t K, float* __restrict__ s) {
    const int j = blockIdx.x;
    __shared__ float s_max[32], s_min[32];
    float mx = 0.0f, mn = INFINITY;
    for (int64_t k = threadIdx.x; k < K; k += 1024) {
        const float v = a[k] > 0.0f ? pow_eighths(a[k], j) : 1.0f;
        mx = fmaxf(mx, v);
        mn = fminf(mn, v);
    }
    for (int o = 16; o > 0; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    if ((threadIdx.x & 31) == 0) {
        s_max[threadIdx.x >> 5] = mx;
        s_min[threadIdx.x >> 5] = mn;
    }
    __syncthreads();
    mx = 0.0f;
    mn = INFINITY;
    for (int w = 0; w < 32; ++w) {
        mx = fmaxf(mx, s_max[w]);
        mn = fminf(mn, s_min[w]);
    }
    const float norm = __fsqrt_rn(__fmul_rn(mx, mn));
    for (int64_t k = threadIdx.x; k < K; k += 1024) {
        const float v = a[k] > 0.0f ? pow_eighths(a[k], j) : 1.0f;
        s[(int64_t)j * K + k] = __fdiv_rn(v, norm);
    }
}

// w' = w * s[sel][k] (binary32), sel = *j_sel if j_sel, else j.
__global__ void __launch_bounds__(256) cal_scale_weight_kernel(const float* __restrict__ w, int64_t N, int64_t K,
                                                               const float* __restrict__ s, int j,
                                                               const int32_t* __restrict__ j_sel,
                                                               float* __restrict__ w_out, float* __restrict__ s_out) {
    const int jj = j_sel ? *j_sel : j;
    const float* sj = s + (int64_t)jj * K;
    const int64_t n4 = N * K / 4;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t k = (i * 4) % K;
        float4 v = reinterpret_cast<const float4*>(w)[i];
        v.x = __fmul_rn(v.x, sj[k]);
        v.y = __fmul_rn(v.y, sj[k + 1]);
        v.z = __fmul_rn(v.z, sj[k + 2]);
        v.w = __fmul_rn(v.w, sj[k + 3]);
        reinterpret_cast<float4*>(w_out)[i] = v;
        if (s_out && i < K / 4) reinterpret_cast<float4*>(s_out)[i] = reinterpret_cast<const float4*>(sj)[i];
    }
}

// Per-CTA partial of err(alpha_j) over 16-element blocks (fp64 sums); the
// weight's codes and row-major scales are those of w * s_j.
__global__ void __launch_bounds__(256) cal_error_kernel(const float* __restrict__ w, int64_t N, int64_t K,
                                                        const uint8_t* __restrict__ codes,
                                                        const uint8_t* __restrict__ scales, const float* __restrict__ gs,
                                                        const float* __restrict__ s, const float* __restrict__ m2,
                                                        double* __restrict__ partial) {
    const int64_t nb = N * (K / 16);
    double acc = 0.0;
    const double g = (double)*gs;
    for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < nb; b += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = b / (K / 16), k0 = (b % (K / 16)) * 16;
        const double sc = (double)e4m3_to_f32(scales[b]) * g;
        const uint2 cw = *reinterpret_cast<const uint2*>(codes + n * (K / 2) + k0 / 2);
        const uint32_t w2[2] = {cw.x, cw.y};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t hh[4];
            e2m1x8_to_f16x2(w2[h], hh);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 v = f16x2_to_f32x2(hh[e]);
                const int64_t k = k0 + 8 * h + 2 * e;
                const double d0 = (double)v.x * sc / (double)s[k] - (double)w[n * K + k];
                const double d1 = (double)v.y * sc / (double)s[k + 1] - (double)w[n * K + k + 1];
                acc += (double)m2[k] * d0 * d0 + (double)m2[k + 1] * d1 * d1;
            }
        }
    }
    __shared__ double red[256];
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) partial[blockIdx.x] = red[0];
}

// err[j] = the partials summed in order; after the last alpha, the argmin.
__global__ void cal_finish_kernel(const double* __restrict__ partial, int nparts, int j, double* __restrict__ err,
                                  int32_t* __restrict__ j_best, float* __restrict__ err_out) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    double e = 0.0;
    for (int i = 0; i < nparts; ++i) e += partial[i];
    err[j] = e;
    if (err_out) err_out[j] = (float)e;
    if (j == kCalAlphas - 1) {
        int best = 0;
        for (int i = 1; i < kCalAlphas; ++i)
            if (err[i] < err[best]) best = i;
        *j_best = best;
    }
}

int launch_calibrate(const float* w, int64_t N, int64_t K, const void* x, int64_t S, int sf_layout, uint8_t* codes,
                     uint8_t* scales, float* gs_out, float* col_scale_out, float* err_out, int32_t* alpha_idx_out,
                     const CalibrateWs& ws, cudaStream_t st) {
    const unsigned grid_k = (unsigned)((K + 255) / 256);
    cal_stats_kernel<<<grid_k, 256, 0, st>>>((const __nv_bfloat16*)x, S, K, ws.a, ws.m2);
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_LAUNCH;
    cal_scales_kernel<<<kCalAlphas, 1024, 0, st>>>(ws.a, K, ws.s);
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_LAUNCH;
    int64_t gw = (N * K / 4 + 255) / 256;
    if (gw > 148 * 16) gw = 148 * 16;
    for (int j = 0; j < kCalAlphas; ++j) {
        cal_scale_weight_kernel<<<(unsigned)gw, 256, 0, st>>>(w, N, K, ws.s, j, nullptr, ws.w_scaled, nullptr);
        if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_LAUNCH;
        NVFP4_TRY_INTERNAL(launch_amax(ws.w_scaled, NVFP4_DTYPE_F32, N * K, ws.amax, st));
        NVFP4_TRY_INTERNAL(launch_quantize(ws.w_scaled, NVFP4_DTYPE_F32, nullptr, N, K, NVFP4_SF_ROWMAJOR, nullptr,
                                           ws.amax, ws.codes, ws.scales, ws.gs, st));
        cal_error_kernel<<<kCalErrBlocks, 256, 0, st>>>(w, N, K, ws.codes, ws.scales, ws.gs, ws.s + (int64_t)j * K,
                                                        ws.m2, ws.partial);
        if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_LAUNCH;
        cal_finish_kernel<<<1, 32, 0, st>>>(ws.partial, kCalErrBlocks, j, ws.err, ws.j_best, err_out);
        if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_LAUNCH;
    }
    // the chosen alpha: its scales to the caller, its scaled weight quantized in the caller's layout
    cal_scale_weight_kernel<<<(unsigned)gw, 256, 0, st>>>(w, N, K, ws.s, 0, ws.j_best, ws.w_scaled, col_scale_out);
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_LAUNCH;
    if (alpha_idx_out &&
        cudaMemcpyAsync(alpha_idx_out, ws.j_best, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return NVFP4_ERR_LAUNCH;
    NVFP4_TRY_INTERNAL(launch_amax(ws.w_scaled, NVFP4_DTYPE_F32, N * K, ws.amax, st));
    return launch_quantize(ws.w_scaled, NVFP4_DTYPE_F32, nullptr, N, K, sf_layout, nullptr, ws.amax, codes, scales,
                           gs_out, st);
}

}  // namespace nvfp4
