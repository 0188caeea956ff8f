// Device helpers shared by the libnvfp4 kernels (sm_100a only).
//
// Format conversions use the hardware cvt instructions of sm_100:
//   cvt.rn.f16x2.e2m1x2          E2M1 pair  -> f16x2 (exact)
//   cvt.rn.f16x2.e4m3x2          E4M3 pair  -> f16x2 (exact; E4M3 fits f16)
//   cvt.rn.satfinite.e4m3x2.f32  f32 pair   -> E4M3 pair, nearest-even, saturating
//   cvt.rn.satfinite.e2m1x2.f32  f32 pair   -> E2M1 pair, nearest-even, saturating
// Element 2j of a packed pair always sits in the low nibble / low byte.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nvfp4.h"

#define NVFP4_DEV __device__ __forceinline__

namespace nvfp4 {

// ---- loads ------------------------------------------------------------------

// 16-byte streaming load through the non-coherent path, no L1 allocation:
// weights are read exactly once per launch.
NVFP4_DEV uint4 ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

NVFP4_DEV uint4 ldg_v4(const void* p) {
    return __ldg(reinterpret_cast<const uint4*>(p));
}

// ---- decode -----------------------------------------------------------------

// Eight E2M1 codes (one 32-bit word, element 0 in bits 3:0) -> four f16x2.
NVFP4_DEV void e2m1x8_to_f16x2(uint32_t w, uint32_t (&h)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
}

// Two E4M3 bytes (byte 0 in bits 7:0) -> f16x2 (exact).
NVFP4_DEV uint32_t e4m3x2_to_f16x2(uint16_t s) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(s));
    return h;
}

NVFP4_DEV float e4m3_to_f32(uint32_t byte) {
    uint32_t h = e4m3x2_to_f16x2((uint16_t)(byte & 0xFF));
    return __half2float(__ushort_as_half((unsigned short)(h & 0xFFFF)));
}

NVFP4_DEV float2 f16x2_to_f32x2(uint32_t h) {
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// Two bf16 values in one word (element 0 low) -> fp32 (exact).
NVFP4_DEV float bf16lo_to_f32(uint32_t u) { return __uint_as_float(u << 16); }
NVFP4_DEV float bf16hi_to_f32(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// ---- encode -----------------------------------------------------------------

// E4M3 code of a (a >= 0 here), nearest-even, saturating at 448.
NVFP4_DEV uint32_t f32_to_e4m3(float a) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(a));
    return r & 0xFF;
}

// Eight floats -> eight E2M1 codes packed in a word (element 0 in bits 3:0).
NVFP4_DEV uint32_t f32x8_to_e2m1(const float (&v)[8]) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return out;
}

// ---- products ---------------------------------------------------------------

// d = a * b + c with f16 a, b (exact product) and an fp32 accumulator.
NVFP4_DEV float fma_f32_f16(uint16_t a, uint16_t b, float c) {
    float d;
    asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
    return d;
}

// 32 products of one 16-byte chunk of E2M1 codes with 32 fp16 activations
// (xw: 16 words of f16 pairs), as two 16-element block partials.  The f16
// halves are taken as register halves (mov.b32 {lo, hi}), not by masking.
NVFP4_DEV void dot32_e2m1_f16(const uint4& wq, const uint32_t* xw, float& p0, float& p1) {
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
            p = fma_f32_f16(hl, xl, p);
            p = fma_f32_f16(hh, xhi, p);
        }
        if (j < 2) p0 = p; else p1 = p;
    }
}

// ---- scale layouts ----------------------------------------------------------

// Byte offset of scale (r, c) of a matrix with `ncols_sf` scale columns.
template <int LAYOUT>
NVFP4_DEV int64_t sf_offset(int64_t r, int64_t c, int64_t ncols_sf) {
    if constexpr (LAYOUT == NVFP4_SF_ROWMAJOR) {
        return r * ncols_sf + c;
    } else {
        const int64_t cp4 = (ncols_sf + 3) >> 2;  // atoms along the scale columns
        return (((r >> 7) * cp4 + (c >> 2)) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (c & 3);
    }
}

NVFP4_DEV float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

NVFP4_DEV float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <typename T>
NVFP4_DEV void store_out(T* p, float v);
template <>
NVFP4_DEV void store_out<float>(float* p, float v) { *p = v; }
template <>
NVFP4_DEV void store_out<__nv_bfloat16>(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

}  // namespace nvfp4
