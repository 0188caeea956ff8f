// moe_route_topk_noalloc: the router / top-k / permutation of moe_route_topk
// for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) when they route:
// an engine whose device memory plan is fixed when the model loads and must
// not grow inside a step, or code running where an allocation would stall
// the device or is not permitted.  This entry point takes the same inputs and
// outputs as moe_route_topk but no workspace: its scratch is the file-scope
// array below, which every GPU that loads the library holds until exit.
//
// The scratch holds the per-32-token-block expert counts and bases and, when
// the caller passes no logits buffer, the logits.  Every byte the kernels read
// from it they first write in the same call, so nothing needs clearing.  All
// calls share the one array: calls that overlap on the GPU (other streams,
// other threads) race on it and must be serialized by the caller.
#include <cuda_runtime.h>

#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace nvfp4 {
namespace {

constexpr size_t kNoallocScratchBytes = (size_t)1 << 20;  // 1 MiB
__device__ __align__(256) unsigned char g_route_scratch[kNoallocScratchBytes];

size_t round256(size_t n) { return (n + 255) & ~(size_t)255; }

// Device address of g_route_scratch for the current device.  In host code the
// array's name is only a host-side stand-in; the real address comes from
// cudaGetSymbolAddress, made once per device with that device current (the
// first call on a device does it, so that call should come before any stream
// capture).  The slots are atomic, so host threads making their first calls
// at the same time are safe (each stores the same address).  The cached
// address belongs to the device's primary context: after a device reset
// (cudaDeviceReset) it is stale, and this entry point must not be called again
// in that process.
unsigned char* scratch_ptr() {
    static std::atomic<unsigned char*> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    unsigned char* p = cache[dev].load(std::memory_order_acquire);
    if (!p) {
        void* q = nullptr;
        if (cudaGetSymbolAddress(&q, g_route_scratch) != cudaSuccess) return nullptr;
        p = (unsigned char*)q;
        cache[dev].store(p, std::memory_order_release);
    }
    return p;
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" int moe_route_topk_noalloc(const void* h, const void* w_router, const float* logit_bias, int64_t T,
                                      int64_t H, int32_t E, int32_t k, float* logits_out, int32_t* topk_idx,
                                      float* topk_w, int32_t* expert_offsets, int32_t* perm_tok,
                                      int32_t* perm_slot, int32_t* row_of, void* stream) {
    if (!h || !w_router || !topk_idx || !topk_w || !expert_offsets || !perm_tok || !perm_slot || !row_of)
        return NVFP4_ERR_NULL;
    if (T < 1 || T > ((int64_t)1 << 24) || H < 8 || H % 8 || E < 1 || E > 1024 || k < 1 || k > 32 || k > E)
        return NVFP4_ERR_SHAPE;
    if (((uintptr_t)h & 15u) || ((uintptr_t)w_router & 15u)) return NVFP4_ERR_ALIGN;
    const int64_t nblk = (T + kPermBlockTokens - 1) / kPermBlockTokens;
    const size_t logit_bytes = logits_out ? 0 : round256((size_t)(T * E) * 4);
    const size_t blk_bytes = round256((size_t)(nblk * E) * 4);
    if (logit_bytes + 2 * blk_bytes > kNoallocScratchBytes) return NVFP4_ERR_WORKSPACE;  // beyond the static scratch
    int major = 0, minor = 0, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess || major != 10 ||
        minor != 0)
        return NVFP4_ERR_ARCH;
    unsigned char* base = scratch_ptr();
    if (!base) return NVFP4_ERR_LAUNCH;
    cudaStream_t st = (cudaStream_t)stream;
    float* logits = logits_out ? logits_out : (float*)base;
    int32_t* blk_counts = (int32_t*)(base + logit_bytes);
    int32_t* blk_base = (int32_t*)(base + logit_bytes + blk_bytes);
    int s = launch_router_logits(h, w_router, logit_bias, T, H, E, logits, st);
    if (s == NVFP4_OK) s = launch_topk_count(logits, T, E, k, topk_idx, topk_w, blk_counts, st);
    if (s == NVFP4_OK) s = launch_perm_scan(blk_counts, nblk, E, expert_offsets, blk_base, st);
    if (s == NVFP4_OK) s = launch_perm_scatter(topk_idx, T, E, k, blk_base, perm_tok, perm_slot, row_of, st);
    return s;
}
