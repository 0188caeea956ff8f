// Internal launchers behind the C ABI (not exported).  Every launcher takes
// validated arguments and returns an NVFP4_* status.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nvfp4.h"

namespace nvfp4 {

// Launch attribute for programmatic dependent launch (kernels that call
// griddep_wait() before touching activations or outputs).
inline void set_pdl_attr(cudaLaunchAttribute& a) {
    a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a.val.programmaticStreamSerializationAllowed = 1;
}

// stack.cu: decode-stack glue (bf16 outputs)
int launch_rms_norm(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld, void* y, cudaStream_t st);
int launch_silu_mul(const void* g, int g_dtype, int64_t rows, int64_t half, void* h, cudaStream_t st);
// The rms factor of every row (written to inv) and the largest |bf16(x * inv)|
// over all rows (atomicMax into *amax_bits, zeroed first): the same reduction
// as launch_rms_norm, so bf16(x * inv) equals its output.
int launch_rms_stats(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld, float* inv,
                     unsigned* amax_bits, cudaStream_t st);

// quantize.cu
int launch_amax(const void* x, int x_dtype, int64_t n, unsigned* amax_bits, cudaStream_t st);
// src_rows (nullable): dst row r quantizes source row src_rows[r]; -1 = zero row.
// row_bound (nullable, device): rows >= *row_bound are skipped entirely.
// x_ld (0: cols) is the source row stride; row_inv (nullable, device): source
// row r is normalised first, x -> bf16(x * row_inv[r]).
int launch_quantize(const void* x, int x_dtype, const int32_t* src_rows, int64_t dst_rows, int64_t cols,
                    int sf_layout, const float* gs_in, const unsigned* amax_bits, uint8_t* codes,
                    uint8_t* scales, float* gs_out, cudaStream_t st, const int32_t* row_bound = nullptr,
                    int64_t x_ld = 0, const float* row_inv = nullptr);
// amax over bf16 rows x[src_rows[r]], r < nrows (negative entries skipped);
// row_bound (nullable, device): rows >= *row_bound are not read.
int launch_amax_rows(const void* x, const int32_t* src_rows, int64_t nrows, int64_t cols, unsigned* amax_bits,
                     cudaStream_t st, const int32_t* row_bound = nullptr);

// gemv.cu: W4A16 on CUDA cores.
struct GemvArgs {
    const void* xh;           // fp16 activations x * 2^p (from launch_x_prep), [rows, K]
    const float* inv_scale;   // per activation row: 2^-p
    int64_t M;                // dense: number of rows of x / y
    int64_t K;
    const uint8_t* codes;     // [N, K/2]  (grouped: [E, N, K/2])
    const uint8_t* scales;    // per-matrix scale block (grouped: E of them, sf_stride apart)
    int64_t sf_stride;        // bytes between experts' scale blocks
    int sf_layout;
    const float* gs;          // [1] or [E]
    int64_t N;                // weight rows
    const int32_t* offsets;   // grouped: [E+1] row offsets (nullable for dense)
    int32_t E;
    const int32_t* experts;   // grouped: touched experts, one per grid slot, -1 = none (nullable: slot = expert)
    int32_t n_slots;          // grouped: grid slots when `experts` is set
    int epilogue;             // NVFP4_EPI_NONE or NVFP4_EPI_SWIGLU
    void* y;                  // output rows
    int y_dtype;              // NVFP4_DTYPE_F32 / BF16
    int64_t ldy;              // elements per output row
};
// Activation prep for W4A16: xh[r] = fp16(x[src(r)] * 2^p_r), inv_scale[r] = 2^-p_r,
// src(r) = gather[r] if gather else r.
int launch_x_prep(const void* x, const int32_t* gather, int64_t rows, int64_t K, void* xh, float* inv_scale,
                  cudaStream_t st);
int launch_gemv_w4a16(const GemvArgs& a, cudaStream_t st);

// gemm_w4a16_tc.cu: W4A16 with dequantized weights in tensor memory (3 <= M <= 64, TILED, K % 256 == 0).
bool w4a16_tc_supported(int64_t M, int64_t K, int64_t N, int sf_layout);
int launch_w4a16_tc(const void* xh, const float* inv_scale, int64_t M, int64_t K, const uint8_t* codes,
                    const uint8_t* scales, const float* gs, int64_t N, void* y, int y_dtype, int* status,
                    cudaStream_t st);

// gemv_tma.cu: pipelined W4A16 decode (TMA ring, cluster split-K) for M <= 4, K % 256 == 0.
bool decode_tma_supported(int64_t M, int64_t K, int64_t N);
int launch_decode_tma(const void* x, int64_t M, int64_t K, const uint8_t* codes, const uint8_t* scales,
                      int sf_layout, const float* gs, int64_t N, void* y, int y_dtype, int* status, cudaStream_t st);

// gemm_w4a4.cu: tcgen05 block-scaled W4A4 GEMM.  A = activations [M, K/2]
// codes + TILED scales, B = weights [N, K/2] + TILED scales; K % 256 == 0.
int launch_gemm_w4a4(const uint8_t* a_codes, const uint8_t* a_scales, const float* gs_a, int64_t M, int64_t K,
                     const uint8_t* b_codes, const uint8_t* b_scales, const float* gs_b, int64_t N, void* y,
                     int y_dtype, int* status, cudaStream_t st);

// moe.cu
// router_tc.cu: tensor-core router logits for T <= 64 (experts as M, split K
// over a cluster; H % 64 == 0, 16-byte aligned rows), programmatic dependent
bool router_tcs_supported(const void* h, const void* wr, int64_t T, int64_t H, int32_t E);
int launch_router_logits_tcs(const void* h, const void* wr, const float* bias, int64_t T, int64_t H, int32_t E,
                             float* logits, int* status, cudaStream_t st);
// router_tc.cu: tensor-core router logits (T > 64, H % 64 == 0, 16-byte aligned rows)
bool router_tc_supported(const void* h, const void* wr, int64_t T, int64_t H, int32_t E);
int launch_router_logits_tc(const void* h, const void* wr, const float* bias, int64_t T, int64_t H, int32_t E,
                            float* logits, int* status, cudaStream_t st);
// Device address of the library's status word (timeouts of bounded waits).
int* device_status_ptr();
int launch_router_logits(const void* h, const void* wr, const float* bias, int64_t T, int64_t H, int32_t E,
                         float* logits, cudaStream_t st);
int launch_topk_count(const float* logits, int64_t T, int32_t E, int32_t k, int32_t* topk_idx, float* topk_w,
                      int32_t* blk_counts, cudaStream_t st);
int launch_perm_scan(const int32_t* blk_counts, int64_t nblk, int32_t E, int32_t* offsets, int32_t* blk_base,
                     cudaStream_t st);
int launch_perm_scatter(const int32_t* topk_idx, int64_t T, int32_t E, int32_t k, const int32_t* blk_base,
                        int32_t* perm_tok, int32_t* perm_slot, int32_t* row_of, cudaStream_t st);
// y[t] = sum_{j<k} topk_w[t, j] * d[row_of[t, j]], j ascending, fp32; d [T*k, N] in d_dtype; N % 4 == 0.
int launch_combine(const void* d, int d_dtype, const float* topk_w, const int32_t* row_of, int64_t T, int32_t k,
                   int64_t N, void* y, int y_dtype, cudaStream_t st);

// Padded expert layout (rows_pad = multiple of 128 >= R + 127 E): pad_off[E+1],
// tile_info[3 * rows_pad/128], src_rows[rows_pad].
int launch_moe_pad(const int32_t* offsets, int32_t E, int64_t rows_pad, const int32_t* gather, int32_t* pad_off,
                   int32_t* tile_info, int32_t* src_rows, cudaStream_t st);
// experts with rows, compacted: list[j] for j < nslots (-1 past the last), E <= 1024.
int launch_touched_experts(const int32_t* offsets, int32_t E, int32_t nslots, int32_t* list, cudaStream_t st);

// gemm_w4a4.cu, grouped: A = padded permuted activations, B = stacked experts.
int launch_gemm_w4a4_grouped(const uint8_t* a_codes, const uint8_t* a_scales, const float* gs_a, int64_t rows_pad,
                             int64_t K, const int32_t* tile_info, const uint8_t* w_codes, const uint8_t* w_scales,
                             int64_t sf_stride, const float* w_gs, int32_t E, int64_t N, int epilogue, void* y,
                             int y_dtype, int* status, cudaStream_t st);

// moe_decode.cu: one routed expert layer for T <= 32 tokens (router, top-k,
// gate/up + SwiGLU, down, combine), five kernels chained by PDL.
struct MoeDecodeLaunch {
    const void* h;              // [T, H] bf16
    const void* w_router;       // [E, H] bf16
    const float* logit_bias;    // [E] or null
    int T, H, I, E, k;
    const uint8_t* gu_codes;    // [E, 2I, H/2]
    const uint8_t* gu_scales;   // E TILED blocks
    const float* gu_gs;         // [E]
    const uint8_t* dn_codes;    // [E, H, I/2]
    const uint8_t* dn_scales;
    const float* dn_gs;
    float* logits;              // [T, E]
    int32_t* topk_idx;          // [T, k]
    float* topk_w;              // [T, k]
    int32_t* n_groups;          // routing tables: [1]
    int32_t* groups;            // [T * k][8] token-group records
    void* h16;                  // [T, H] fp16, h prescaled per token
    void* a;                    // [T * k, I] bf16
    void* a16;                  // [T * k, I] fp16, a prescaled per (row, 64 columns)
    float* inv_a;               // [T * k, I / 64]
    float* d;                   // [T * k, H]
    void* y;                    // [T, H]
    int y_dtype;
    int* status;
};
size_t moe_decode_smem_bytes(int64_t H, int64_t I);
int launch_moe_decode(const MoeDecodeLaunch& L, cudaStream_t st);
// the small-batch router kernel as a programmatic dependent launch
int launch_router_logits_small_pdl(const void* h, const void* wr, const float* bias, int64_t T, int64_t H,
                                   int32_t E, float* logits, cudaStream_t st);

// chain.cu: W4A16 decode linears in a persistent launch per 12 ops.
int chain_validate(const nvfp4_chain_op* ops, int n_ops, int64_t M);
size_t chain_workspace(const nvfp4_chain_op* ops, int n_ops, int64_t M);
int launch_chain(const nvfp4_chain_op* ops, int n_ops, int64_t M, void* ws, size_t ws_bytes, int* status,
                 cudaStream_t st);

// calibrate.cu: activation-calibrated quantization of a weight (9 alphas).
constexpr int kCalErrBlocks = 296;
struct CalibrateWs {
    float* a;            // [K] mean |x|
    float* m2;           // [K] mean x^2
    float* s;            // [9][K] channel scales per alpha
    float* w_scaled;     // [N, K]
    unsigned* amax;
    uint8_t* codes;      // [N, K/2]
    uint8_t* scales;     // [N, K/16] row-major
    float* gs;
    double* partial;     // [kCalErrBlocks]
    double* err;         // [9]
    int32_t* j_best;
};
int launch_calibrate(const float* w, int64_t N, int64_t K, const void* x, int64_t S, int sf_layout, uint8_t* codes,
                     uint8_t* scales, float* gs_out, float* col_scale_out, float* err_out, int32_t* alpha_idx_out,
                     const CalibrateWs& ws, cudaStream_t st);

#define NVFP4_TRY_INTERNAL(expr)        \
    do {                                \
        const int _s = (expr);          \
        if (_s != NVFP4_OK) return _s;  \
    } while (0)

// Tokens per block of the routing permutation (top-k, counts, scatter): 32
// gives one CTA per 32 tokens, so a 4,096-token batch spreads over 128 SMs.
constexpr int kPermBlockTokens = 32;

}  // namespace nvfp4
