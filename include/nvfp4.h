/*
 * nvfp4.h -- C ABI of libnvfp4, the NVFP4 linear layer for B200 (sm_100a).
 *
 * The layer: a linear y = x W^T whose weight W [N, K] is stored as NVFP4, i.e.
 * E2M1 4-bit codes, one E4M3 scale per 16 consecutive values along K and one
 * fp32 scale per tensor:
 *
 *     W[n, k] = E2M1(code[n, k]) * E4M3(scale[n, k / 16]) * gs
 *
 * The pages this library follows name the format and the ways the layer runs,
 * but do not define either:
 *   - imp home page, "How does it work?": weights stay NVFP4 and the GPU
 *     multiplies in that format instead of unpacking to 16 bits;
 *   - Ignis README, "The decode round": decode linears are weight streaming at
 *     the card's bandwidth (the W4A16 decode path here);
 *   - Ignis README, "How fast" and "Credits": prefill in 2,048-token chunks,
 *     split-K prefill, attention on FP4 tensor cores (the W4A4 prefill path);
 *   - imp v0.20.0 release notes, "Highlights": a first-party NVFP4 quantizer
 *     (nvfp4_quantize);
 *   - CHImp Alpha v1.0 model card, "How it fits on one GPU": every token is
 *     routed to 10 of 512 experts per layer and only those experts' weights
 *     are read (moe_route_topk, moe_grouped_linear);
 *   - Ignis README, "What sets it apart" / "Building it": a flat,
 *     device-resident, step-level C ABI under a per-request error boundary
 *     (the style of this header).
 *
 * Conventions for every call below.
 *   - Every pointer argument is a DEVICE pointer (unless stated) owned by the
 *     caller; the library keeps no reference after the call returns.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL means the legacy default stream).  No call allocates or frees
 *     memory or synchronizes, except nvfp4_read_device_status.
 *   - Every call validates its arguments on the host before launching any
 *     kernel.  A call that returns an error has launched nothing and written
 *     nothing.  Values behind device pointers (e.g. a per-tensor scale) are not
 *     validated: they must be finite, and scales positive.
 *   - Data pointers must be 16-byte aligned.
 *   - Matrices are row-major.  Codes are packed two per byte, element 2j in
 *     the low nibble of byte j.  Scale bytes are raw E4M3 with sign bit 0.
 *   - Returns NVFP4_OK (0) or one of the NVFP4_ERR_* codes.
 *
 * Numerics.  W4A16 accumulates in fp32: per 16-element block, sum x * E2M1,
 * then multiply by the block's E4M3 scale, then by gs at the end.  The
 * tensor-core skinny path rounds activations to fp16 after a per-row
 * power-of-two prescale (exact for every element within 2^32 of its row's
 * largest magnitude).  W4A4 quantizes activations with the same rules as
 * nvfp4_quantize and accumulates E2M1 x E2M1 products in fp32 on the tensor
 * cores.  bf16 outputs are rounded to nearest even from fp32.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
enum {
    NVFP4_OK = 0,
    NVFP4_ERR_NULL = 1,           /* a required pointer is NULL                   */
    NVFP4_ERR_SHAPE = 2,          /* a size is out of range / not a multiple      */
    NVFP4_ERR_ALIGN = 3,          /* a pointer is not 16-byte aligned             */
    NVFP4_ERR_DTYPE = 4,          /* unsupported dtype code                       */
    NVFP4_ERR_WORKSPACE = 5,      /* ws is NULL or ws_bytes below the query value */
    NVFP4_ERR_ARCH = 6,           /* the current device is not sm_100             */
    NVFP4_ERR_LAUNCH = 7,         /* a kernel launch or driver call failed        */
    NVFP4_ERR_LAYOUT = 8,         /* scale layout not accepted by the chosen mode */
    NVFP4_ERR_MODE = 9,           /* unknown mode or epilogue code                */
    NVFP4_ERR_DEVICE_TIMEOUT = 10 /* a kernel's bounded wait ran out (read with
                                     nvfp4_read_device_status)                    */
};

/* ---- enumerations ------------------------------------------------------ */
enum { NVFP4_DTYPE_F32 = 0, NVFP4_DTYPE_BF16 = 1 };

/* Scale layouts.
 *   ROWMAJOR: scale (r, c) at byte r * (cols/16) + c.  rows * cols/16 bytes.
 *   TILED:    the tensor-core scale-factor layout.  Rows are padded to
 *             Rp = ceil(rows/128)*128 and scale columns to Cp = ceil((cols/16)/4)*4;
 *             the matrix is cut into 128 x 4 atoms of 512 bytes, atoms ordered
 *             with the column index fastest:
 *               byte(r, c) = ((r/128) * (Cp/4) + c/4) * 512
 *                            + (r%32) * 16 + ((r%128)/32) * 4 + (c%4).
 *             Rp * Cp bytes; padding bytes are written as 0 by nvfp4_quantize.
 *             This is the operand layout of tcgen05 block-scaled MMA, so a
 *             128-row x 64-column tile's scales are one contiguous 512 B atom. */
enum { NVFP4_SF_ROWMAJOR = 0, NVFP4_SF_TILED = 1 };

/* Modes of the linear.  AUTO picks W4A16 for M <= 32 and W4A4 above. */
enum { NVFP4_MODE_AUTO = 0, NVFP4_MODE_W4A16 = 1, NVFP4_MODE_W4A4 = 2 };

/* Epilogues of moe_grouped_linear. */
enum { NVFP4_EPI_NONE = 0, NVFP4_EPI_SWIGLU = 1, NVFP4_EPI_COMBINE = 2 };

/* ---- helpers ------------------------------------------------------------ */

/* Text of a status code (static storage). */
const char* nvfp4_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int nvfp4_version(void);

/* Bytes of a [rows, cols] tensor's scales in `sf_layout` (0 on bad arguments). */
size_t nvfp4_scales_bytes(int64_t rows, int64_t cols, int sf_layout);

/* Debug helper.  Copies the library's device status word (set by a kernel
 * whose bounded wait ran out) into *status_out, resets it to NVFP4_OK, and
 * synchronizes `stream`.  The only call that synchronizes. */
int nvfp4_read_device_status(void* stream, int* status_out);

/* Debug helper for the bounded waits (Ignis README, "Credits": a per-request
 * error boundary).  Launches one CTA that waits on an mbarrier nothing arrives
 * on, with the bounded wait every TMA / tensor-core kernel here uses, limited
 * to limit_cycles SM clock cycles (1 .. 4e9).  Nothing is in flight while it
 * waits; when the limit runs out the kernel records NVFP4_ERR_DEVICE_TIMEOUT
 * in the status word and returns, and the device stays usable.  Returns
 * NVFP4_ERR_SHAPE for a limit out of range. */
int nvfp4_debug_wait_timeout(int64_t limit_cycles, void* stream);

/* ---- nvfp4_quantize ------------------------------------------------------
 * NVFP4 quantization (imp v0.20.0 release notes, "Highlights": first-party
 * NVFP4 quantizer, round-to-nearest part).  For x [rows, cols]:
 *     gs      = *gs_in if gs_in != NULL, else amax(|x|) / 2688 (1.0 if amax == 0)
 *     s[r, b] = E4M3(amax_b / (gs * 6))               (binary32: denom = gs * 6)
 *     c[r, k] = E2M1(x[r, k] / (E4M3value(s) * gs))  (binary32 division)
 * Rounding is to nearest with ties to the even code, saturating at 448 / 6,
 * and keeps the sign (a negative value that rounds to 0 gives code 8).
 * A block whose E4M3value(s) * gs is 0 stores +0 codes.
 *   x       [rows, cols] in x_dtype (F32 or BF16)
 *   gs_in   device float or NULL
 *   codes   out, rows * cols/2 bytes
 *   scales  out, nvfp4_scales_bytes(rows, cols, sf_layout) bytes
 *   gs_out  out, one device float (the gs used)
 *   ws      scratch of nvfp4_quantize_workspace(rows, cols) bytes (holds the
 *           amax reduction); contents on entry are ignored.
 * Requires cols % 16 == 0, rows >= 1. */
size_t nvfp4_quantize_workspace(int64_t rows, int64_t cols);
int nvfp4_quantize(const void* x, int x_dtype, int64_t rows, int64_t cols,
                   const float* gs_in, int sf_layout,
                   uint8_t* codes, uint8_t* scales, float* gs_out,
                   void* ws, size_t ws_bytes, void* stream);

/* ---- nvfp4_calibrate -------------------------------------------------------
 * Activation-calibrated NVFP4 quantization of a weight (imp v0.20.0 release
 * notes, "Highlights": a first-party NVFP4 quantizer with AWQ-class
 * activation calibration).  From a calibration batch x [S, K] (bf16):
 *     a_k  = (sum_s |x[s, k]|) / S,  m2_k = (sum_s x[s, k]^2) / S
 *            (binary32, rows added in order)
 *     for alpha = j / 8, j = 0..8:
 *       s_k = a_k^alpha (1 where a_k == 0), then s_k /= sqrt(max s * min s);
 *             a^(j/8) is computed from r1 = sqrt(a), r2 = sqrt(r1),
 *             r3 = sqrt(r2) as 1, r3, r2, r2*r3, r1, r1*r3, r1*r2,
 *             (r1*r2)*r3, a (IEEE square roots and products)
 *       W'  = W diag(s) (binary32), quantized as nvfp4_quantize(W') (gs from
 *             amax(W'))
 *       err = sum_k m2_k sum_n (dequant(W')[n, k] / s_k - W[n, k])^2  (fp64)
 *     the alpha of least err (lowest j on ties) is kept.
 * The linear with the calibrated weight is y = (x / s) dequant(W')^T: the
 * caller divides the activations by col_scale_out (or folds 1/s into the
 * operation that produces them).  alpha = 0 is plain round-to-nearest.
 *   w              [N, K] fp32 (device)
 *   x              [S, K] bf16 calibration activations
 *   codes, scales  out: W' in sf_layout;  gs_out one float
 *   col_scale_out  out: s [K] of the chosen alpha
 *   err_out        NULL or out [9]: err of every alpha (as float)
 *   alpha_idx_out  NULL or out [1]: the chosen j (alpha = j / 8)
 *   ws             scratch of nvfp4_calibrate_workspace(N, K, S) bytes.
 * Requires K % 16 == 0. */
size_t nvfp4_calibrate_workspace(int64_t N, int64_t K, int64_t S);
int nvfp4_calibrate(const float* w, int64_t N, int64_t K, const void* x, int x_dtype, int64_t S, int sf_layout,
                    uint8_t* codes, uint8_t* scales, float* gs_out, float* col_scale_out, float* err_out,
                    int32_t* alpha_idx_out, void* ws, size_t ws_bytes, void* stream);

/* ---- nvfp4_linear --------------------------------------------------------
 * y[m, n] = sum_k x[m, k] * W[n, k], W NVFP4 as above (Ignis README, "The
 * decode round"; imp home page, "How does it work?").
 *   x        [M, K] bf16 (x_dtype must be NVFP4_DTYPE_BF16)
 *   w_codes  [N, K/2] bytes;  w_scales in w_sf_layout;  w_gs one device float
 *   y        [M, N] in y_dtype (F32 or BF16)
 *   mode     W4A16: weight-only, activations stay bf16.  Accepts either
 *                   scale layout.  Any M >= 1.
 *            W4A4:  activations quantized per call to NVFP4 (per-tensor gs,
 *                   same rules as nvfp4_quantize), tcgen05 block-scaled MMA.
 *                   Requires w_sf_layout == TILED and K % 256 == 0.
 *            AUTO:  W4A16 if M <= 32, else W4A4.
 *   ws       scratch of nvfp4_linear_workspace(M, K, N, mode) bytes (the
 *            quantized activations for W4A4, the fp16 activations for the
 *            tensor-core W4A16 path); contents on entry are ignored.
 * Requires K % 16 == 0, M, N >= 1. */
size_t nvfp4_linear_workspace(int64_t M, int64_t K, int64_t N, int mode);
int nvfp4_linear(const void* x, int x_dtype, int64_t M, int64_t K,
                 const uint8_t* w_codes, const uint8_t* w_scales, int w_sf_layout,
                 const float* w_gs, int64_t N,
                 void* y, int y_dtype, int mode,
                 void* ws, size_t ws_bytes, void* stream);

/* ---- nvfp4_linear_w4a4_ws_layout -------------------------------------------
 * Where a W4A4 nvfp4_linear call leaves the activations it quantized, inside
 * its workspace: once the call has run (stream order), the bytes at these
 * offsets from ws hold
 *   offsets[0]  gs_x, one float (amax(|x|) / 2688, as nvfp4_quantize)
 *   offsets[1]  codes [M, K/2]
 *   offsets[2]  scales, TILED for M rows
 * exactly what nvfp4_quantize(x, gs_in = NULL, TILED) writes, so a caller can
 * hand them to nvfp4_linear_w4a4q for another weight with the same input.
 * Requires K % 256 == 0, M >= 1. */
int nvfp4_linear_w4a4_ws_layout(int64_t M, int64_t K, int64_t offsets[3]);

/* ---- nvfp4_linear_w4a4q ---------------------------------------------------
 * The W4A4 linear with activations already in NVFP4 (e.g. written by a
 * previous layer's quantizing epilogue, or by nvfp4_quantize with
 * sf_layout = TILED): the tensor-core GEMM alone, without the quantize pass
 * (Ignis README, "Credits": the NVFP4-full target).
 *     y[m, n] = (*x_gs) * (*w_gs) * sum_k E2M1(xc) E4M3(xs) E2M1(wc) E4M3(ws)
 *   x_codes  [M, K/2];  x_scales TILED for M rows;  x_gs one device float
 *   w_codes  [N, K/2];  w_scales TILED for N rows;  w_gs one device float
 *   y        [M, N] in y_dtype (F32 or BF16)
 * Requires K % 256 == 0; no workspace. */
int nvfp4_linear_w4a4q(const uint8_t* x_codes, const uint8_t* x_scales, const float* x_gs, int64_t M, int64_t K,
                       const uint8_t* w_codes, const uint8_t* w_scales, const float* w_gs, int64_t N,
                       void* y, int y_dtype, void* stream);

/* ---- nvfp4_chain ----------------------------------------------------------
 * A list of W4A16 decode linears run in order by one persistent launch (a
 * launch per 12 ops): the decode chain of a layer stack, streamed without the
 * drain, prologue and tail of a launch per linear (Ignis README, "The decode
 * round": a decode step streams every layer's weights; "Credits": the decode
 * chain replayed as one unit).
 * Op i computes out_i = x_i W_i^T (W_i [N, K] NVFP4, TILED scales), M rows,
 * with x_i taken from
 *   SRC_X   a caller bf16 tensor x [M, K] (row stride x_ld elements), or
 *   SRC_OP  the output v of an earlier op src_op of the same call, through
 *           XFORM_NONE      x = bf16(v)                       (v has >= K columns)
 *           XFORM_RMS       x = bf16(v[:, :K] / sqrt(mean(v[:, :K]^2)))
 *                           (a row of zeros stays zero)
 *           XFORM_SILU_MUL  x[:, j] = bf16(silu(v[:, j]) * v[:, K + j]),
 *                           silu(a) = a / (1 + e^-a)        (v has 2K columns)
 * and, if y is not NULL, writes y = out_i (XFORM_NONE) or y = rms(out_i)
 * (XFORM_RMS, over all N columns) in y_dtype.  Ops without y keep their
 * output in the workspace only.  Outputs accumulate in fp32 (the split-K
 * partial sums of an output element are added in a fixed order: results are
 * deterministic).
 *   ws  scratch of nvfp4_chain_workspace(ops, n_ops, M) bytes; contents on
 *       entry are ignored.
 * Requires 1 <= M <= 2, K % 256 == 0, N % 8 == 0, 16-byte aligned pointers;
 * needs two resident CTAs per SM (returns NVFP4_ERR_LAUNCH otherwise); a grid
 * barrier that runs out reports NVFP4_ERR_DEVICE_TIMEOUT through
 * nvfp4_read_device_status. */
enum { NVFP4_CHAIN_SRC_X = 0, NVFP4_CHAIN_SRC_OP = 1 };
enum { NVFP4_CHAIN_XFORM_NONE = 0, NVFP4_CHAIN_XFORM_RMS = 1, NVFP4_CHAIN_XFORM_SILU_MUL = 2 };
typedef struct {
    const uint8_t* w_codes;   /* [N, K/2] */
    const uint8_t* w_scales;  /* TILED */
    const float* w_gs;        /* [1] */
    int64_t N, K;
    int32_t src;              /* NVFP4_CHAIN_SRC_X or NVFP4_CHAIN_SRC_OP */
    int32_t src_op;           /* SRC_OP: index of an earlier op */
    const void* x;            /* SRC_X: bf16 [M, x_ld] */
    int64_t x_ld;
    int32_t xform;            /* SRC_OP: NVFP4_CHAIN_XFORM_*; SRC_X: NONE */
    int32_t y_xform;          /* NONE or RMS */
    void* y;                  /* NULL or [M, N] */
    int32_t y_dtype;          /* F32 or BF16 */
    int32_t reserved;
} nvfp4_chain_op;
size_t nvfp4_chain_workspace(const nvfp4_chain_op* ops, int32_t n_ops, int64_t M);
int nvfp4_chain(const nvfp4_chain_op* ops, int32_t n_ops, int64_t M, void* ws, size_t ws_bytes, void* stream);

/* ---- nvfp4_rms_norm / nvfp4_silu_mul -------------------------------------
 * The glue between the linears of a dense decode stack (Ignis README, "The
 * decode round": a decode step streams the whole stack's weights once).  The
 * pages leave the chaining open; with attention left out each layer is
 *     q = QKV(x); o = O(rms(q[:, :K_o])); g = GU(rms(o));
 *     h = silu(g[:, :N/2]) * g[:, N/2:]; x' = rms(Down(h))
 * nvfp4_rms_norm:  y[r, c] = bf16(x[r, c] / sqrt(mean_c x[r, c]^2)), rounded
 *   to nearest even; an all-zero row gives zeros.
 *   x      rows of `cols` elements, row r starting at element r * ld
 *          (ld >= cols, so a column slice of a wider matrix is read in place);
 *          x_dtype F32 or BF16
 *   y      [rows, cols] bf16, densely packed
 * nvfp4_silu_mul:  h[r, j] = bf16(silu(g[r, j]) * g[r, half + j]),
 *   silu(v) = v / (1 + e^-v)
 *   g      [rows, 2 * half], g_dtype F32 or BF16;  h  [rows, half] bf16
 * Element-size alignment only; no workspace. */
int nvfp4_rms_norm(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld, void* y, void* stream);

/* nvfp4_rms_norm_quant:  the NVFP4 quantization of nvfp4_rms_norm(x) without
 * writing or reading back its bf16 rows (Ignis README, "Credits": activations
 * reach the prefill GEMM as NVFP4; the rms renormalisation is the producer).
 * codes, scales and gs_out equal, bit for bit, nvfp4_quantize of the rows
 * nvfp4_rms_norm(x, ...) returns, with gs_in = NULL: one pass takes each row's
 * rms factor and the largest normalised magnitude over all rows (the global
 * scale), a second writes codes and scales from x directly.  Feed the result
 * to nvfp4_linear_w4a4q (sf_layout TILED).
 *   x       rows of `cols` elements at stride ld (F32 or BF16), 16-byte
 *           aligned, ld a multiple of 8 (BF16) or 4 (F32)
 *   codes   out [rows, cols/2];  scales  out in sf_layout;  gs_out  out [1]
 *   ws      scratch of nvfp4_rms_norm_quant_workspace(rows) bytes.
 * Requires cols % 16 == 0. */
size_t nvfp4_rms_norm_quant_workspace(int64_t rows);
int nvfp4_rms_norm_quant(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld, int sf_layout,
                         uint8_t* codes, uint8_t* scales, float* gs_out, void* ws, size_t ws_bytes, void* stream);
int nvfp4_silu_mul(const void* g, int g_dtype, int64_t rows, int64_t half, void* h, void* stream);

/* ---- moe_route_topk ------------------------------------------------------
 * Router of a routed mixture-of-experts layer (CHImp Alpha v1.0 model card,
 * "How it fits on one GPU": 10 of 512 experts per token).
 *     l[t, e]   = sum_h h[t, h] * Wr[e, h] (+ logit_bias[e]), fp32 accumulate
 *     topk_idx  the k largest logits per token, equal logits -> lower index,
 *               slots in descending logit order
 *     topk_w    softmax over the k selected logits (= full softmax
 *               renormalised over the top k)
 *     expert_offsets[E+1]  exclusive prefix sum of per-expert counts
 *     perm_tok[r], perm_slot[r]  the (token, slot) of row r, rows grouped by
 *               expert ascending, tokens ascending within an expert
 *     row_of[t*k + j]  the row of token t's slot j (inverse of the above)
 *   h [T, H] bf16;  w_router [E, H] bf16;  logit_bias [E] fp32 or NULL;
 *   logits_out [T, E] fp32 or NULL;  topk_idx, row_of [T, k] int32;
 *   topk_w [T, k] fp32;  perm_tok, perm_slot [T*k] int32;
 *   ws  scratch of moe_route_topk_workspace(T, E, k) bytes (per-expert
 *       counters); contents on entry are ignored.
 * Requires 1 <= k <= 32, k <= E <= 1024, H % 8 == 0, T >= 1. */
size_t moe_route_topk_workspace(int64_t T, int32_t E, int32_t k);
int moe_route_topk(const void* h, const void* w_router, const float* logit_bias,
                   int64_t T, int64_t H, int32_t E, int32_t k,
                   float* logits_out, int32_t* topk_idx, float* topk_w,
                   int32_t* expert_offsets, int32_t* perm_tok, int32_t* perm_slot,
                   int32_t* row_of, void* ws, size_t ws_bytes, void* stream);

/* ---- moe_route_topk_noalloc ------------------------------------------------
 * The pages have no counterpart to this call.  It computes exactly what
 * moe_route_topk computes, for callers that cannot allocate device memory
 * when they route (an engine whose device memory plan is fixed at load and
 * must not grow inside a step, or code where an allocation would stall the
 * device or is not permitted), so it takes no workspace.  Its scratch is a
 * 1 MiB array inside the library that every GPU loading the library holds
 * until exit.  It needs ceil(T/32) * E * 8 bytes (rounded up to 256-byte
 * pieces), plus T * E * 4 bytes when logits_out is NULL; a request that does
 * not fit returns NVFP4_ERR_WORKSPACE before launching anything (pass
 * logits_out to route large T).  The first call on a device looks up the
 * array's device address, so make it before any stream capture; the address
 * stays cached for the process, so do not call this again after a device
 * reset (cudaDeviceReset) in the same process.  Every call
 * shares the array: calls that overlap on the GPU race and must be
 * serialized by the caller.  Arguments, layouts and errors are otherwise
 * those of moe_route_topk. */
int moe_route_topk_noalloc(const void* h, const void* w_router, const float* logit_bias,
                           int64_t T, int64_t H, int32_t E, int32_t k,
                           float* logits_out, int32_t* topk_idx, float* topk_w,
                           int32_t* expert_offsets, int32_t* perm_tok, int32_t* perm_slot,
                           int32_t* row_of, void* stream);

/* ---- moe_layer_decode ----------------------------------------------------
 * One routed mixture-of-experts layer for a decode batch of T <= 32 tokens,
 * from the router to the weighted combine, reading only the chosen experts'
 * weights (CHImp Alpha v1.0 model card, "How it fits on one GPU": each token
 * goes to 10 of 512 experts per layer and only those experts are read).
 *     l[t, e]  = sum_h h[t, h] * Wr[e, h] (+ logit_bias[e]), fp32
 *     topk_idx, topk_w as moe_route_topk (ties -> lower index; softmax over
 *                the k selected)
 *     a[t*k+j, c] = bf16(silu(g) * u), g = h[t] . Wgu[e][c],
 *                u = h[t] . Wgu[e][I + c], e = topk_idx[t, j]   (W4A16)
 *     y[t, n]  = sum_{j<k} topk_w[t, j] * (a[t*k+j] . Wd[e][n]), j ascending,
 *                fp32 (the per-slot dot products are fp32; y rounded to
 *                y_dtype at the end)
 *   h          [T, H] bf16;  w_router [E, H] bf16;  logit_bias [E] or NULL
 *   gu_codes   [E, 2I, H/2], gu_scales E consecutive TILED blocks of
 *              nvfp4_scales_bytes(2I, H, TILED), gu_gs [E]  (rows 0..I-1 of an
 *              expert are the gate projection, I..2I-1 the up projection)
 *   dn_codes   [E, H, I/2], dn_scales E TILED blocks of
 *              nvfp4_scales_bytes(H, I, TILED), dn_gs [E]
 *   logits_out [T, E] fp32, topk_idx [T, k] int32, topk_w [T, k] fp32,
 *   a_out      [T*k, I] bf16: optional outputs (NULL: kept in the workspace)
 *   y          [T, H] in y_dtype (F32 or BF16)
 *   ws         scratch of moe_layer_decode_workspace(T, H, I, E, k) bytes;
 *              contents on entry are ignored.
 * The layer runs as five kernels chained by programmatic dependent launch.
 * Requires 1 <= T <= 32, 1 <= k <= 32, k <= E <= 1024, H and I multiples of
 * 256 and at most 4096, TILED scales; the workspace query returns 0 for
 * shapes out of range. */
size_t moe_layer_decode_workspace(int64_t T, int64_t H, int64_t I, int32_t E, int32_t k);
int moe_layer_decode(const void* h, const void* w_router, const float* logit_bias,
                     int64_t T, int64_t H, int32_t E, int32_t k,
                     const uint8_t* gu_codes, const uint8_t* gu_scales, const float* gu_gs, int64_t I,
                     const uint8_t* dn_codes, const uint8_t* dn_scales, const float* dn_gs,
                     float* logits_out, int32_t* topk_idx, float* topk_w, void* a_out,
                     void* y, int y_dtype, void* ws, size_t ws_bytes, void* stream);

/* ---- moe_grouped_linear --------------------------------------------------
 * Expert linears over the permuted rows (CHImp, same section: only the chosen
 * experts' weights are read).  For each expert e and row r in
 * [expert_offsets[e], expert_offsets[e+1]):
 *     out[r, :] = xin(r) @ W_e^T,  xin(r) = x[perm_tok[r]] if gather else x[r]
 * then the epilogue:
 *     NONE     y[r, n]  = out[r, n]                               y [R, N]
 *     SWIGLU   y[r, j]  = silu(out[r, j]) * out[r, N/2 + j]        y [R, N/2]
 *              (gate = first half of W_e's rows, up = second half)
 *     COMBINE  y[t, n]  = sum_{j<k} topk_w[t, j] * out[row_of[t, j], n],
 *              j ascending, fp32                                    y [R/k, N]
 *              (W4A4 rounds out[r, :] to bf16 before the sum, the layer's
 *              bf16 expert output; W4A16 keeps it fp32.  Either way the
 *              sum is deterministic: the same inputs give the same bits.)
 *   x        [rows of x, K] bf16 (x_dtype BF16)
 *   w_codes  [E, N, K/2];  w_scales: E consecutive per-expert scale blocks of
 *            nvfp4_scales_bytes(N, K, w_sf_layout) bytes;  w_gs [E] fp32
 *   R        total rows (= T * k for routed input)
 *   topk_w, row_of, k: used by COMBINE only (may be NULL / 0 otherwise)
 *   y_dtype  F32 or BF16
 *   mode     W4A16, W4A4, or AUTO: W4A16 if R <= 512, else W4A4.  W4A4
 *            requires TILED scales, K % 256 == 0 and N % 128 == 0 (N % 256
 *            for SWIGLU).
 *   ws       scratch of moe_grouped_linear_workspace(...) bytes.
 * Experts with no rows are skipped: their weights are not read. */
size_t moe_grouped_linear_workspace(int64_t R, int64_t K, int64_t N, int32_t E, int32_t k,
                                    int epilogue, int mode);
int moe_grouped_linear(const void* x, int x_dtype, int64_t K, int gather,
                       const int32_t* expert_offsets, const int32_t* perm_tok,
                       int32_t E, int64_t R,
                       const uint8_t* w_codes, const uint8_t* w_scales, int w_sf_layout,
                       const float* w_gs, int64_t N,
                       int epilogue, const float* topk_w, const int32_t* row_of, int32_t k,
                       void* y, int y_dtype, int mode,
                       void* ws, size_t ws_bytes, void* stream);

/* ---- moe_grouped_linear_w4a4_ws_layout -------------------------------------
 * Where a W4A4 moe_grouped_linear call leaves the permuted activations it
 * quantized, inside its workspace.  Each expert's rows are padded to a whole
 * number of 128-row tiles; once the call has run (stream order), the bytes at
 * these offsets from ws hold
 *   out[0]  gs_x, one float: amax over the rows read (x[perm_tok[r]] when
 *           gathering, x[r] otherwise) / 2688
 *   out[1]  pad_off int32 [E+1]: first padded row of each expert; pad_off[E]
 *           is the number of padded rows in use
 *   out[2]  src_rows int32 [out[5]]: the row of x each padded row quantizes,
 *           -1 for padding
 *   out[3]  codes [out[5], K/2] of the padded rows (padding rows are 0)
 *   out[4]  scales, TILED for out[5] rows (padding rows are 0)
 *   out[5]  the padded row count the workspace is laid out for
 * Rows at or past pad_off[E] are not written.  Codes and scales of row pr
 * equal those nvfp4_quantize gives row src_rows[pr] of x with gs_in = gs_x.
 * Requires K % 256 == 0 and the other limits of moe_grouped_linear. */
int moe_grouped_linear_w4a4_ws_layout(int64_t R, int64_t K, int64_t N, int32_t E, int32_t k, int epilogue,
                                      int64_t out[6]);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_H */
