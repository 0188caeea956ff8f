// libnvfp4 C ABI: argument validation, workspace layout and dispatch.
// The declarations, argument meanings, layouts and error behaviour are in
// include/nvfp4.h.  Every entry point validates on the host and returns an
// error before launching anything.
#include <cuda_runtime.h>
#include <stdlib.h>

#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace nvfp4 {
__device__ int g_device_status = 0;

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Device address of the status word, looked up once per device (the slots are
// atomic: several host threads may make their first call at once; each stores
// the same address).  A device reset invalidates the cached address.
int* device_status_ptr() {
    static std::atomic<int*> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    int* p = cache[dev].load(std::memory_order_acquire);
    if (!p) {
        void* q = nullptr;
        if (cudaGetSymbolAddress(&q, g_device_status) != cudaSuccess) return nullptr;
        p = (int*)q;
        cache[dev].store(p, std::memory_order_release);
    }
    return p;
}
static size_t align256(size_t n) { return (n + 255) & ~(size_t)255; }

// The current device must be sm_100 (B200 / GB200 class).  Cached per device.
static int check_arch() {
    static std::atomic<int> cache[64];  // 0 unknown, 1 ok, 2 bad
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_ARCH;
    if (dev < 0 || dev >= 64) return NVFP4_ERR_ARCH;
    int c = cache[dev].load(std::memory_order_relaxed);
    if (c == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return NVFP4_ERR_ARCH;
        c = (major == 10 && minor == 0) ? 1 : 2;
        cache[dev].store(c, std::memory_order_relaxed);
    }
    return c == 1 ? NVFP4_OK : NVFP4_ERR_ARCH;
}

static bool dtype_ok(int d) { return d == NVFP4_DTYPE_F32 || d == NVFP4_DTYPE_BF16; }
static bool layout_ok(int l) { return l == NVFP4_SF_ROWMAJOR || l == NVFP4_SF_TILED; }

static size_t scales_bytes(int64_t rows, int64_t cols, int layout) {
    if (rows < 1 || cols < 16 || cols % 16) return 0;
    const int64_t nsf = cols / 16;
    if (layout == NVFP4_SF_ROWMAJOR) return (size_t)(rows * nsf);
    if (layout == NVFP4_SF_TILED) return (size_t)((rows + 127) / 128 * 128) * (size_t)((nsf + 3) / 4 * 4);
    return 0;
}

// Grid limits of the W4A16 kernels (row tiles of >= 2 rows on grid.y, token
// groups of <= 4 rows on grid.x).
constexpr int64_t kMaxW4A16N = 65535 * 2;
constexpr int64_t kMaxW4A16M = (int64_t)1 << 30;

// W4A16 workspace: fp16 activations and one inverse scale per row.
static size_t w4a16_ws(int64_t rows, int64_t K) { return align256((size_t)(rows * K) * 2) + align256((size_t)rows * 4); }

// Padded rows of the grouped W4A4 operand: every expert's rows padded to whole
// 128-row tiles (at most 127 padding rows per expert), rounded up to a tile.
static int64_t moe_w4a4_rows(int64_t R, int32_t E) { return (R + (int64_t)E * 127 + 127) / 128 * 128; }

struct GroupedW4A4Ws {
    unsigned* amax;
    float* gs_x;
    int32_t* pad_off;
    int32_t* tile_info;
    int32_t* src_rows;
    uint8_t* codes;
    uint8_t* scales;
    __nv_bfloat16* d;  // COMBINE: the experts' rows [R, N] before the weighted sum
    size_t bytes;
};
static GroupedW4A4Ws grouped_w4a4_ws(void* base, int64_t R, int64_t K, int64_t N, int32_t E, int32_t k,
                                     int epilogue) {
    GroupedW4A4Ws w{};
    const int64_t rp = moe_w4a4_rows(R, E);
    char* p = (char*)base;
    size_t off = 0;
    auto take = [&](size_t n) { char* q = p ? p + off : nullptr; off += align256(n); return q; };
    w.amax = (unsigned*)take(16);
    w.gs_x = (float*)take(16);
    w.pad_off = (int32_t*)take((size_t)(E + 1) * 4);
    w.tile_info = (int32_t*)take((size_t)(rp / 128) * 12);
    w.src_rows = (int32_t*)take((size_t)rp * 4);
    w.codes = (uint8_t*)take((size_t)(rp * K / 2));
    w.scales = (uint8_t*)take(scales_bytes(rp, K, NVFP4_SF_TILED));
    if (epilogue == NVFP4_EPI_COMBINE) w.d = (__nv_bfloat16*)take((size_t)R * (size_t)N * 2);
    w.bytes = off;
    return w;
}
}  // namespace nvfp4

using namespace nvfp4;

#define NVFP4_TRY(expr)                 \
    do {                                \
        const int _s = (expr);          \
        if (_s != NVFP4_OK) return _s;  \
    } while (0)

extern "C" {

const char* nvfp4_status_string(int status) {
    switch (status) {
        case NVFP4_OK: return "ok";
        case NVFP4_ERR_NULL: return "a required pointer is NULL";
        case NVFP4_ERR_SHAPE: return "a size is out of range or not a required multiple";
        case NVFP4_ERR_ALIGN: return "a pointer is not 16-byte aligned";
        case NVFP4_ERR_DTYPE: return "unsupported dtype";
        case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
        case NVFP4_ERR_ARCH: return "the current device is not sm_100";
        case NVFP4_ERR_LAUNCH: return "a kernel launch or driver call failed";
        case NVFP4_ERR_LAYOUT: return "scale layout not accepted by this mode";
        case NVFP4_ERR_MODE: return "unknown mode or epilogue";
        case NVFP4_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait ran out";
        default: return "unknown status";
    }
}

int nvfp4_version(void) { return 100; }

size_t nvfp4_scales_bytes(int64_t rows, int64_t cols, int sf_layout) { return scales_bytes(rows, cols, sf_layout); }

int nvfp4_read_device_status(void* stream, int* status_out) {
    if (!status_out) return NVFP4_ERR_NULL;
    cudaStream_t st = (cudaStream_t)stream;
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_device_status, sizeof(int), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return NVFP4_ERR_LAUNCH;
    if (cudaStreamSynchronize(st) != cudaSuccess) return NVFP4_ERR_LAUNCH;
    if (cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return NVFP4_ERR_LAUNCH;
    if (cudaStreamSynchronize(st) != cudaSuccess) return NVFP4_ERR_LAUNCH;
    *status_out = v;
    return NVFP4_OK;
}

// ---- quantize ----------------------------------------------------------------

size_t nvfp4_quantize_workspace(int64_t rows, int64_t cols) {
    (void)rows;
    (void)cols;
    return 256;
}

int nvfp4_quantize(const void* x, int x_dtype, int64_t rows, int64_t cols, const float* gs_in, int sf_layout,
                   uint8_t* codes, uint8_t* scales, float* gs_out, void* ws, size_t ws_bytes, void* stream) {
    if (!x || !codes || !scales || !gs_out) return NVFP4_ERR_NULL;
    if (!dtype_ok(x_dtype)) return NVFP4_ERR_DTYPE;
    if (!layout_ok(sf_layout)) return NVFP4_ERR_LAYOUT;
    if (rows < 1 || cols < 16 || cols % 16 || rows > (int64_t)1 << 31 || cols > (int64_t)1 << 31)
        return NVFP4_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return NVFP4_ERR_ALIGN;
    if (!ws || ws_bytes < nvfp4_quantize_workspace(rows, cols)) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(ws)) return NVFP4_ERR_ALIGN;
    NVFP4_TRY(check_arch());
    cudaStream_t st = (cudaStream_t)stream;
    unsigned* amax = (unsigned*)ws;
    if (!gs_in) NVFP4_TRY(launch_amax(x, x_dtype, rows * cols, amax, st));
    return launch_quantize(x, x_dtype, nullptr, rows, cols, sf_layout, gs_in, amax, codes, scales, gs_out, st);
}

// ---- calibrated quantizer ----------------------------------------------------------

static CalibrateWs calibrate_ws(void* base, int64_t N, int64_t K) {
    CalibrateWs w{};
    char* p = (char*)base;
    size_t off = 0;
    auto take = [&](size_t n) { char* q = p ? p + off : nullptr; off += align256(n); return q; };
    w.a = (float*)take((size_t)K * 4);
    w.m2 = (float*)take((size_t)K * 4);
    w.s = (float*)take((size_t)K * 4 * 9);
    w.w_scaled = (float*)take((size_t)(N * K) * 4);
    w.amax = (unsigned*)take(16);
    w.codes = (uint8_t*)take((size_t)(N * K / 2));
    w.scales = (uint8_t*)take((size_t)(N * K / 16));
    w.gs = (float*)take(16);
    w.partial = (double*)take((size_t)kCalErrBlocks * 8);
    w.err = (double*)take(9 * 8);
    w.j_best = (int32_t*)take(16);
    return w;
}
static size_t calibrate_ws_bytes(int64_t N, int64_t K) {
    CalibrateWs w = calibrate_ws((void*)(uintptr_t)256, N, K);  // offsets from a stand-in base
    return (size_t)((char*)w.j_best - (char*)(uintptr_t)256) + 256;
}

size_t nvfp4_calibrate_workspace(int64_t N, int64_t K, int64_t S) {
    if (N < 1 || K < 16 || K % 16 || S < 1) return 0;
    return calibrate_ws_bytes(N, K);
}

int nvfp4_calibrate(const float* w, int64_t N, int64_t K, const void* x, int x_dtype, int64_t S, int sf_layout,
                    uint8_t* codes, uint8_t* scales, float* gs_out, float* col_scale_out, float* err_out,
                    int32_t* alpha_idx_out, void* ws, size_t ws_bytes, void* stream) {
    if (!w || !x || !codes || !scales || !gs_out || !col_scale_out) return NVFP4_ERR_NULL;
    if (x_dtype != NVFP4_DTYPE_BF16) return NVFP4_ERR_DTYPE;
    if (!layout_ok(sf_layout)) return NVFP4_ERR_LAYOUT;
    if (N < 1 || K < 16 || K % 16 || S < 1 || N > ((int64_t)1 << 24) || K > ((int64_t)1 << 24) ||
        N * K > ((int64_t)1 << 34) || S > ((int64_t)1 << 24))
        return NVFP4_ERR_SHAPE;
    if (!aligned16(w) || !aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(col_scale_out))
        return NVFP4_ERR_ALIGN;
    if (!ws || ws_bytes < calibrate_ws_bytes(N, K)) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(ws)) return NVFP4_ERR_ALIGN;
    NVFP4_TRY(check_arch());
    return launch_calibrate(w, N, K, x, S, sf_layout, codes, scales, gs_out, col_scale_out, err_out, alpha_idx_out,
                            calibrate_ws(ws, N, K), (cudaStream_t)stream);
}

// ---- linear --------------------------------------------------------------------

static int resolve_mode(int mode, int64_t M) {
    if (mode == NVFP4_MODE_AUTO) return M <= 32 ? NVFP4_MODE_W4A16 : NVFP4_MODE_W4A4;
    return mode;
}

size_t nvfp4_linear_workspace(int64_t M, int64_t K, int64_t N, int mode) {
    (void)N;
    mode = resolve_mode(mode, M);
    if (mode == NVFP4_MODE_W4A4) {
        // amax word, gs, activation codes, tiled activation scales
        return align256(256) + align256((size_t)(M * K / 2)) + align256(scales_bytes(M, K, NVFP4_SF_TILED));
    }
    return decode_tma_supported(M, K, N) ? 0 : w4a16_ws(M, K);
}

int nvfp4_linear(const void* x, int x_dtype, int64_t M, int64_t K, const uint8_t* w_codes, const uint8_t* w_scales,
                 int w_sf_layout, const float* w_gs, int64_t N, void* y, int y_dtype, int mode, void* ws,
                 size_t ws_bytes, void* stream) {
    if (!x || !w_codes || !w_scales || !w_gs || !y) return NVFP4_ERR_NULL;
    if (x_dtype != NVFP4_DTYPE_BF16 || !dtype_ok(y_dtype)) return NVFP4_ERR_DTYPE;
    if (!layout_ok(w_sf_layout)) return NVFP4_ERR_LAYOUT;
    if (mode != NVFP4_MODE_AUTO && mode != NVFP4_MODE_W4A16 && mode != NVFP4_MODE_W4A4) return NVFP4_ERR_MODE;
    if (M < 1 || N < 1 || K < 16 || K % 16 || M > ((int64_t)1 << 31) || N > ((int64_t)1 << 31) ||
        K > ((int64_t)1 << 24))
        return NVFP4_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(y)) return NVFP4_ERR_ALIGN;
    mode = resolve_mode(mode, M);
    if (mode == NVFP4_MODE_W4A4) {
        if (w_sf_layout != NVFP4_SF_TILED) return NVFP4_ERR_LAYOUT;
        if (K % 256) return NVFP4_ERR_SHAPE;
        if ((N + 127) / 128 > 65535) return NVFP4_ERR_SHAPE;
    } else if (N > kMaxW4A16N || M > kMaxW4A16M) {
        return NVFP4_ERR_SHAPE;
    }
    const size_t need = nvfp4_linear_workspace(M, K, N, mode);
    if (need && (!ws || ws_bytes < need)) return NVFP4_ERR_WORKSPACE;
    if (need && !aligned16(ws)) return NVFP4_ERR_ALIGN;
    NVFP4_TRY(check_arch());
    cudaStream_t st = (cudaStream_t)stream;
    if (mode == NVFP4_MODE_W4A4) {
        // activations -> NVFP4 (per-tensor gs, tiled scales) in the workspace, then the tensor-core GEMM
        char* wp = (char*)ws;
        unsigned* amax = (unsigned*)wp;
        float* gs_x = (float*)(wp + 16);
        uint8_t* xc = (uint8_t*)(wp + 256);
        uint8_t* xs = xc + align256((size_t)(M * K / 2));
        NVFP4_TRY(launch_amax(x, NVFP4_DTYPE_BF16, M * K, amax, st));
        NVFP4_TRY(launch_quantize(x, NVFP4_DTYPE_BF16, nullptr, M, K, NVFP4_SF_TILED, nullptr, amax, xc, xs, gs_x, st));
        return launch_gemm_w4a4(xc, xs, gs_x, M, K, w_codes, w_scales, w_gs, N, y, y_dtype, device_status_ptr(), st);
    }
    if (decode_tma_supported(M, K, N))
        return launch_decode_tma(x, M, K, w_codes, w_scales, w_sf_layout, w_gs, N, y, y_dtype, device_status_ptr(),
                                 st);
    void* xh = ws;
    float* inv = (float*)((char*)ws + align256((size_t)(M * K) * 2));
    NVFP4_TRY(launch_x_prep(x, nullptr, M, K, xh, inv, st));
    if (w4a16_tc_supported(M, K, N, w_sf_layout))
        return launch_w4a16_tc(xh, inv, M, K, w_codes, w_scales, w_gs, N, y, y_dtype, device_status_ptr(), st);
    GemvArgs a{};
    a.xh = xh;
    a.inv_scale = inv;
    a.M = M;
    a.K = K;
    a.codes = w_codes;
    a.scales = w_scales;
    a.sf_layout = w_sf_layout;
    a.gs = w_gs;
    a.N = N;
    a.E = 1;
    a.epilogue = NVFP4_EPI_NONE;
    a.y = y;
    a.y_dtype = y_dtype;
    a.ldy = N;
    return launch_gemv_w4a16(a, st);
}

int nvfp4_linear_w4a4_ws_layout(int64_t M, int64_t K, int64_t* offsets) {
    if (!offsets) return NVFP4_ERR_NULL;
    if (M < 1 || K < 256 || K % 256 || M > ((int64_t)1 << 31) || K > ((int64_t)1 << 24)) return NVFP4_ERR_SHAPE;
    offsets[0] = 16;                                          // gs_x
    offsets[1] = 256;                                         // codes [M, K/2]
    offsets[2] = 256 + (int64_t)align256((size_t)(M * K / 2));  // TILED scales
    return NVFP4_OK;
}

int nvfp4_linear_w4a4q(const uint8_t* x_codes, const uint8_t* x_scales, const float* x_gs, int64_t M, int64_t K,
                       const uint8_t* w_codes, const uint8_t* w_scales, const float* w_gs, int64_t N, void* y,
                       int y_dtype, void* stream) {
    if (!x_codes || !x_scales || !x_gs || !w_codes || !w_scales || !w_gs || !y) return NVFP4_ERR_NULL;
    if (!dtype_ok(y_dtype)) return NVFP4_ERR_DTYPE;
    if (M < 1 || N < 1 || K < 256 || K % 256 || M > ((int64_t)1 << 31) || (N + 127) / 128 > 65535 ||
        K > ((int64_t)1 << 24))
        return NVFP4_ERR_SHAPE;
    if (!aligned16(x_codes) || !aligned16(x_scales) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(y))
        return NVFP4_ERR_ALIGN;
    NVFP4_TRY(check_arch());
    return launch_gemm_w4a4(x_codes, x_scales, x_gs, M, K, w_codes, w_scales, w_gs, N, y, y_dtype,
                            device_status_ptr(), (cudaStream_t)stream);
}

// ---- chains of decode linears ------------------------------------------------------

size_t nvfp4_chain_workspace(const nvfp4_chain_op* ops, int32_t n_ops, int64_t M) {
    return chain_workspace(ops, n_ops, M);
}

int nvfp4_chain(const nvfp4_chain_op* ops, int32_t n_ops, int64_t M, void* ws, size_t ws_bytes, void* stream) {
    NVFP4_TRY(chain_validate(ops, n_ops, M));
    const size_t need = chain_workspace(ops, n_ops, M);
    if (!ws || ws_bytes < need) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(ws)) return NVFP4_ERR_ALIGN;
    NVFP4_TRY(check_arch());
    return launch_chain(ops, n_ops, M, ws, ws_bytes, device_status_ptr(), (cudaStream_t)stream);
}

// ---- decode-stack glue ---------------------------------------------------------------

static bool float_dtype_ok(int d) { return d == NVFP4_DTYPE_F32 || d == NVFP4_DTYPE_BF16; }
static bool elem_aligned(const void* p, int d) {
    return ((uintptr_t)p & (uintptr_t)(d == NVFP4_DTYPE_F32 ? 3 : 1)) == 0;
}

int nvfp4_rms_norm(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld, void* y, void* stream) {
    if (!x || !y) return NVFP4_ERR_NULL;
    if (!float_dtype_ok(x_dtype)) return NVFP4_ERR_DTYPE;
    if (rows < 1 || cols < 1 || ld < cols || rows > ((int64_t)1 << 31) - 1 || cols > ((int64_t)1 << 31) ||
        ld > ((int64_t)1 << 40) / rows)
        return NVFP4_ERR_SHAPE;
    if (!elem_aligned(x, x_dtype) || !elem_aligned(y, NVFP4_DTYPE_BF16)) return NVFP4_ERR_ALIGN;
    NVFP4_TRY(check_arch());
    return launch_rms_norm(x, x_dtype, rows, cols, ld, y, (cudaStream_t)stream);
}

size_t nvfp4_rms_norm_quant_workspace(int64_t rows) {
    if (rows < 1) return 0;
    return align256(16) + align256((size_t)rows * 4);
}

int nvfp4_rms_norm_quant(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld, int sf_layout,
                         uint8_t* codes, uint8_t* scales, float* gs_out, void* ws, size_t ws_bytes, void* stream) {
    if (!x || !codes || !scales || !gs_out) return NVFP4_ERR_NULL;
    if (!float_dtype_ok(x_dtype)) return NVFP4_ERR_DTYPE;
    if (!layout_ok(sf_layout)) return NVFP4_ERR_LAYOUT;
    if (rows < 1 || cols < 16 || cols % 16 || ld < cols || rows > ((int64_t)1 << 31) - 1 ||
        cols > ((int64_t)1 << 31) || ld > ((int64_t)1 << 40) / rows)
        return NVFP4_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || ld % (x_dtype == NVFP4_DTYPE_F32 ? 4 : 8))
        return NVFP4_ERR_ALIGN;
    if (!ws || ws_bytes < nvfp4_rms_norm_quant_workspace(rows)) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(ws)) return NVFP4_ERR_ALIGN;
    NVFP4_TRY(check_arch());
    cudaStream_t st = (cudaStream_t)stream;
    unsigned* amax = (unsigned*)ws;
    float* inv = (float*)((char*)ws + align256(16));
    NVFP4_TRY(launch_rms_stats(x, x_dtype, rows, cols, ld, inv, amax, st));
    return launch_quantize(x, x_dtype, nullptr, rows, cols, sf_layout, nullptr, amax, codes, scales, gs_out, st,
                           nullptr, ld, inv);
}

int nvfp4_silu_mul(const void* g, int g_dtype, int64_t rows, int64_t half, void* h, void* stream) {
    if (!g || !h) return NVFP4_ERR_NULL;
    if (!float_dtype_ok(g_dtype)) return NVFP4_ERR_DTYPE;
    if (rows < 1 || half < 1 || rows > ((int64_t)1 << 31) || half > ((int64_t)1 << 40) / rows)
        return NVFP4_ERR_SHAPE;
    if (!elem_aligned(g, g_dtype) || !elem_aligned(h, NVFP4_DTYPE_BF16)) return NVFP4_ERR_ALIGN;
    NVFP4_TRY(check_arch());
    return launch_silu_mul(g, g_dtype, rows, half, h, (cudaStream_t)stream);
}

// ---- MoE routing -------------------------------------------------------------------

static int64_t perm_blocks(int64_t T) { return (T + kPermBlockTokens - 1) / kPermBlockTokens; }

size_t moe_route_topk_workspace(int64_t T, int32_t E, int32_t k) {
    (void)k;
    if (T < 1 || E < 1) return 0;
    return align256((size_t)(T * E) * 4) + 2 * align256((size_t)(perm_blocks(T) * E) * 4);
}

int moe_route_topk(const void* h, const void* w_router, const float* logit_bias, int64_t T, int64_t H, int32_t E,
                   int32_t k, float* logits_out, int32_t* topk_idx, float* topk_w, int32_t* expert_offsets,
                   int32_t* perm_tok, int32_t* perm_slot, int32_t* row_of, void* ws, size_t ws_bytes,
                   void* stream) {
    if (!h || !w_router || !topk_idx || !topk_w || !expert_offsets || !perm_tok || !perm_slot || !row_of)
        return NVFP4_ERR_NULL;
    if (T < 1 || T > ((int64_t)1 << 24) || H < 8 || H % 8 || E < 1 || E > 1024 || k < 1 || k > 32 || k > E)
        return NVFP4_ERR_SHAPE;
    if (!aligned16(h) || !aligned16(w_router)) return NVFP4_ERR_ALIGN;
    if (!ws || ws_bytes < moe_route_topk_workspace(T, E, k)) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(ws)) return NVFP4_ERR_ALIGN;
    NVFP4_TRY(check_arch());
    cudaStream_t st = (cudaStream_t)stream;
    char* p = (char*)ws;
    float* logits = (float*)p;
    p += align256((size_t)(T * E) * 4);
    int32_t* blk_counts = (int32_t*)p;
    p += align256((size_t)(perm_blocks(T) * E) * 4);
    int32_t* blk_base = (int32_t*)p;
    if (logits_out) logits = logits_out;
    NVFP4_TRY(launch_router_logits(h, w_router, logit_bias, T, H, E, logits, st));
    NVFP4_TRY(launch_topk_count(logits, T, E, k, topk_idx, topk_w, blk_counts, st));
    NVFP4_TRY(launch_perm_scan(blk_counts, perm_blocks(T), E, expert_offsets, blk_base, st));
    return launch_perm_scatter(topk_idx, T, E, k, blk_base, perm_tok, perm_slot, row_of, st);
}

// ---- MoE layer for a decode batch --------------------------------------------------

struct MoeDecodeWs {
    float* logits;
    int32_t* topk_idx;
    float* topk_w;
    int32_t* n_groups;
    int32_t* groups;
    void* h16;
    void* a;
    void* a16;
    float* inv_a;
    float* d;
    size_t bytes;
};
static MoeDecodeWs moe_decode_ws(void* base, int64_t T, int64_t H, int64_t I, int32_t E, int32_t k) {
    MoeDecodeWs w{};
    char* p = (char*)base;
    size_t off = 0;
    auto take = [&](size_t n) { char* q = p ? p + off : nullptr; off += align256(n); return q; };
    const size_t R = (size_t)(T * k);
    w.logits = (float*)take((size_t)(T * E) * 4);
    w.topk_idx = (int32_t*)take(R * 4);
    w.topk_w = (float*)take(R * 4);
    w.n_groups = (int32_t*)take(16);
    w.groups = (int32_t*)take(R * 32);
    w.h16 = take((size_t)(T * H) * 2);
    w.a = take(R * (size_t)I * 2);
    w.a16 = take(R * (size_t)I * 2);
    w.inv_a = (float*)take(R * (size_t)(I / 64) * 4);
    w.d = (float*)take(R * (size_t)H * 4);
    w.bytes = off;
    return w;
}

static bool moe_decode_shape_ok(int64_t T, int64_t H, int64_t I, int32_t E, int32_t k) {
    return T >= 1 && T <= 32 && E >= 1 && E <= 1024 && k >= 1 && k <= 32 && k <= E && H >= 256 && H % 256 == 0 &&
           I >= 256 && I % 256 == 0 && H <= 4096 && I <= 4096 && (int64_t)E * 2 * I < ((int64_t)1 << 31) &&
           (int64_t)E * H < ((int64_t)1 << 31) && moe_decode_smem_bytes(H, I) <= 227 * 1024;
}

size_t moe_layer_decode_workspace(int64_t T, int64_t H, int64_t I, int32_t E, int32_t k) {
    if (!moe_decode_shape_ok(T, H, I, E, k)) return 0;
    return moe_decode_ws(nullptr, T, H, I, E, k).bytes;
}

int moe_layer_decode(const void* h, const void* w_router, const float* logit_bias, int64_t T, int64_t H, int32_t E,
                     int32_t k, const uint8_t* gu_codes, const uint8_t* gu_scales, const float* gu_gs, int64_t I,
                     const uint8_t* dn_codes, const uint8_t* dn_scales, const float* dn_gs, float* logits_out,
                     int32_t* topk_idx, float* topk_w, void* a_out, void* y, int y_dtype, void* ws, size_t ws_bytes,
                     void* stream) {
    if (!h || !w_router || !gu_codes || !gu_scales || !gu_gs || !dn_codes || !dn_scales || !dn_gs || !y)
        return NVFP4_ERR_NULL;
    if (!dtype_ok(y_dtype)) return NVFP4_ERR_DTYPE;
    if (!moe_decode_shape_ok(T, H, I, E, k)) return NVFP4_ERR_SHAPE;
    if (!aligned16(h) || !aligned16(w_router) || !aligned16(gu_codes) || !aligned16(gu_scales) ||
        !aligned16(dn_codes) || !aligned16(dn_scales) || !aligned16(y) || !aligned16(a_out) ||
        !aligned16(logits_out))
        return NVFP4_ERR_ALIGN;
    const MoeDecodeWs need = moe_decode_ws(nullptr, T, H, I, E, k);
    if (!ws || ws_bytes < need.bytes) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(ws)) return NVFP4_ERR_ALIGN;
    NVFP4_TRY(check_arch());
    const MoeDecodeWs w = moe_decode_ws(ws, T, H, I, E, k);
    MoeDecodeLaunch L{};
    L.h = h;
    L.w_router = w_router;
    L.logit_bias = logit_bias;
    L.T = (int)T;
    L.H = (int)H;
    L.I = (int)I;
    L.E = E;
    L.k = k;
    L.gu_codes = gu_codes;
    L.gu_scales = gu_scales;
    L.gu_gs = gu_gs;
    L.dn_codes = dn_codes;
    L.dn_scales = dn_scales;
    L.dn_gs = dn_gs;
    L.logits = logits_out ? logits_out : w.logits;
    L.topk_idx = topk_idx ? topk_idx : w.topk_idx;
    L.topk_w = topk_w ? topk_w : w.topk_w;
    L.n_groups = w.n_groups;
    L.groups = w.groups;
    L.h16 = w.h16;
    L.a = a_out ? a_out : w.a;
    L.a16 = w.a16;
    L.inv_a = w.inv_a;
    L.d = w.d;
    L.y = y;
    L.y_dtype = y_dtype;
    L.status = device_status_ptr();
    return launch_moe_decode(L, (cudaStream_t)stream);
}

// ---- MoE grouped linear ------------------------------------------------------------

static int resolve_grouped_mode(int mode, int64_t R) {
    if (mode == NVFP4_MODE_AUTO) return R <= 512 ? NVFP4_MODE_W4A16 : NVFP4_MODE_W4A4;
    return mode;
}

size_t moe_grouped_linear_workspace(int64_t R, int64_t K, int64_t N, int32_t E, int32_t k, int epilogue, int mode) {
    (void)k;
    mode = resolve_grouped_mode(mode, R);
    size_t need = 0;
    if (mode == NVFP4_MODE_W4A16) {
        if (epilogue == NVFP4_EPI_COMBINE) need += align256((size_t)(R * N) * 4);
        need += w4a16_ws(R, K) + align256((size_t)E * 4);  // + the touched-expert list
    }
    if (mode == NVFP4_MODE_W4A4) need += grouped_w4a4_ws(nullptr, R, K, N, E, k, epilogue).bytes;
    return need;
}

int moe_grouped_linear_w4a4_ws_layout(int64_t R, int64_t K, int64_t N, int32_t E, int32_t k, int epilogue,
                                      int64_t* out) {
    if (!out) return NVFP4_ERR_NULL;
    if (epilogue != NVFP4_EPI_NONE && epilogue != NVFP4_EPI_SWIGLU && epilogue != NVFP4_EPI_COMBINE)
        return NVFP4_ERR_MODE;
    if (E < 1 || E > 1024 || R < 1 || R > ((int64_t)1 << 26) || N < 1 || N > ((int64_t)1 << 20) || K < 256 ||
        K % 256 || K > ((int64_t)1 << 20))
        return NVFP4_ERR_SHAPE;
    char* base = (char*)(uintptr_t)4096;  // offsets only: the layout from a stand-in base
    const GroupedW4A4Ws o = grouped_w4a4_ws(base, R, K, N, E, k, epilogue);
    out[0] = (char*)o.gs_x - base;
    out[1] = (char*)o.pad_off - base;
    out[2] = (char*)o.src_rows - base;
    out[3] = (char*)o.codes - base;
    out[4] = (char*)o.scales - base;
    out[5] = moe_w4a4_rows(R, E);
    return NVFP4_OK;
}

int moe_grouped_linear(const void* x, int x_dtype, int64_t K, int gather, const int32_t* expert_offsets,
                       const int32_t* perm_tok, int32_t E, int64_t R, const uint8_t* w_codes,
                       const uint8_t* w_scales, int w_sf_layout, const float* w_gs, int64_t N, int epilogue,
                       const float* topk_w, const int32_t* row_of, int32_t k, void* y, int y_dtype, int mode,
                       void* ws, size_t ws_bytes, void* stream) {
    if (!x || !expert_offsets || !w_codes || !w_scales || !w_gs || !y) return NVFP4_ERR_NULL;
    if (gather && !perm_tok) return NVFP4_ERR_NULL;
    if (x_dtype != NVFP4_DTYPE_BF16 || !dtype_ok(y_dtype)) return NVFP4_ERR_DTYPE;
    if (!layout_ok(w_sf_layout)) return NVFP4_ERR_LAYOUT;
    if (epilogue != NVFP4_EPI_NONE && epilogue != NVFP4_EPI_SWIGLU && epilogue != NVFP4_EPI_COMBINE)
        return NVFP4_ERR_MODE;
    if (mode != NVFP4_MODE_AUTO && mode != NVFP4_MODE_W4A16 && mode != NVFP4_MODE_W4A4) return NVFP4_ERR_MODE;
    if (E < 1 || E > 1024 || R < 1 || R > ((int64_t)1 << 26) || N < 1 || N > ((int64_t)1 << 20) || K < 16 ||
        K % 16 || K > ((int64_t)1 << 20))
        return NVFP4_ERR_SHAPE;
    if (epilogue == NVFP4_EPI_SWIGLU && N % 2) return NVFP4_ERR_SHAPE;
    if (epilogue == NVFP4_EPI_COMBINE) {
        if (!topk_w || !row_of) return NVFP4_ERR_NULL;
        if (k < 1 || R % k || N % 4) return NVFP4_ERR_SHAPE;
    }
    if (!aligned16(x) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(y)) return NVFP4_ERR_ALIGN;
    mode = resolve_grouped_mode(mode, R);
    if (mode == NVFP4_MODE_W4A4) {
        if (w_sf_layout != NVFP4_SF_TILED) return NVFP4_ERR_LAYOUT;
        if (K % 256 || N % 128 || (epilogue == NVFP4_EPI_SWIGLU && N % 256) || (int64_t)E * N > 0x7fffffff ||
            moe_w4a4_rows(R, E) / 128 > 0x7fffffff)
            return NVFP4_ERR_SHAPE;
    } else if (K % 32 || N > kMaxW4A16N) {
        return NVFP4_ERR_SHAPE;
    }
    const size_t need = moe_grouped_linear_workspace(R, K, N, E, k, epilogue, mode);
    if (need && (!ws || ws_bytes < need)) return NVFP4_ERR_WORKSPACE;
    if (need && !aligned16(ws)) return NVFP4_ERR_ALIGN;
    NVFP4_TRY(check_arch());
    cudaStream_t st = (cudaStream_t)stream;
    if (mode == NVFP4_MODE_W4A4) {
        const int64_t rp = moe_w4a4_rows(R, E);
        GroupedW4A4Ws w = grouped_w4a4_ws(ws, R, K, N, E, k, epilogue);
        NVFP4_TRY(launch_moe_pad(expert_offsets, E, rp, gather ? perm_tok : nullptr, w.pad_off, w.tile_info,
                                 w.src_rows, st));
        NVFP4_TRY(launch_amax_rows(x, w.src_rows, rp, K, w.amax, st, w.pad_off + E));
        NVFP4_TRY(launch_quantize(x, NVFP4_DTYPE_BF16, w.src_rows, rp, K, NVFP4_SF_TILED, nullptr, w.amax, w.codes,
                                  w.scales, w.gs_x, st, w.pad_off + E));
        const int64_t sf_stride = (int64_t)scales_bytes(N, K, NVFP4_SF_TILED);
        if (epilogue == NVFP4_EPI_COMBINE) {
            // the experts' rows in bf16, then the weighted sum in slot order
            NVFP4_TRY(launch_gemm_w4a4_grouped(w.codes, w.scales, w.gs_x, rp, K, w.tile_info, w_codes, w_scales,
                                               sf_stride, w_gs, E, N, NVFP4_EPI_NONE, w.d, NVFP4_DTYPE_BF16,
                                               device_status_ptr(), st));
            return launch_combine(w.d, NVFP4_DTYPE_BF16, topk_w, row_of, R / k, k, N, y, y_dtype, st);
        }
        return launch_gemm_w4a4_grouped(w.codes, w.scales, w.gs_x, rp, K, w.tile_info, w_codes, w_scales, sf_stride,
                                        w_gs, E, N, epilogue, y, y_dtype, device_status_ptr(), st);
    }
    char* wp = (char*)ws;
    float* d = nullptr;
    if (epilogue == NVFP4_EPI_COMBINE) {
        d = (float*)wp;
        wp += align256((size_t)(R * N) * 4);
    }
    void* xh = wp;
    float* inv = (float*)(wp + align256((size_t)(R * K) * 2));
    int32_t* touched = (int32_t*)(wp + w4a16_ws(R, K));
    // at most min(E, R) experts have rows: the grid covers those slots only
    const int32_t nslots = (int32_t)((int64_t)E < R ? (int64_t)E : R);
    NVFP4_TRY(launch_touched_experts(expert_offsets, E, nslots, touched, st));
    NVFP4_TRY(launch_x_prep(x, gather ? perm_tok : nullptr, R, K, xh, inv, st));
    GemvArgs a{};
    a.xh = xh;
    a.inv_scale = inv;
    a.M = R;
    a.K = K;
    a.codes = w_codes;
    a.scales = w_scales;
    a.sf_stride = (int64_t)scales_bytes(N, K, w_sf_layout);
    a.sf_layout = w_sf_layout;
    a.gs = w_gs;
    a.N = N;
    a.offsets = expert_offsets;
    a.E = E;
    a.experts = touched;
    a.n_slots = nslots;
    if (epilogue == NVFP4_EPI_COMBINE) {
        a.epilogue = NVFP4_EPI_NONE;
        a.y = d;
        a.y_dtype = NVFP4_DTYPE_F32;
        a.ldy = N;
        NVFP4_TRY(launch_gemv_w4a16(a, st));
        return launch_combine(d, NVFP4_DTYPE_F32, topk_w, row_of, R / k, k, N, y, y_dtype, st);
    }
    a.epilogue = epilogue;
    a.y = y;
    a.y_dtype = y_dtype;
    a.ldy = epilogue == NVFP4_EPI_SWIGLU ? N / 2 : N;
    return launch_gemv_w4a16(a, st);
}

}  // extern "C"
