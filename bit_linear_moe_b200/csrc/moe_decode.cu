// K10: one routed mixture-of-experts layer for a decode batch of T <= 32
// tokens, fused from the router to the weighted combine (CHImp Alpha v1.0
// model card, "How it fits on one GPU": each token goes to 10 of 512 experts
// and only the chosen experts' weights are read).
//
//   l        = h Wr^T (+ bias)                         router_logits_small_kernel
//   top-k    k largest logits per token, softmax over them, and the routing
//            tables below                              moe_decode_route_kernel
//   a[t, j]  = silu(g) * u, [g; u] = h[t] Wgu[e]^T, e = topk_idx[t, j]   bf16
//   d[t, j]  = a[t, j] Wd[e]^T                                           fp32
//   y[t]     = sum_{j<k} topk_w[t, j] * d[t, j], j ascending, fp32
//            (gate/up + SwiGLU and down + combine: moe_decode_kernel)
//
// The four kernels run as a programmatic-dependent chain: each one launches
// while its predecessor drains and reads that predecessor's outputs only
// after griddepcontrol.wait.  No permutation of the activations is
// materialised: the route kernel writes, per expert, the list of (token, slot)
// pairs that chose it, cut into groups of at most four tokens.  Groups are
// ordered by size, largest first, so the experts many tokens chose (the hot
// experts of a skewed routing) are spread over the SMs before the rest.
//
// Expert kernel (one per projection, persistent over the SMs).  A work unit
// is (token group, 128-row weight tile): for gate/up the tile is 64 gate rows
// and the matching 64 up rows (two 2D TMA boxes of the stacked [E * 2I, H/2]
// codes), so SwiGLU pairs rows inside the CTA; for down it is 128 rows of the
// stacked [E * H, I/2] codes.  A producer warp streams, per 256-element K
// stage, the code boxes and their 2 KB scale-atom runs (bulk copies of the
// tensor-core scale layout) through an 8-deep shared-memory ring that runs
// across unit boundaries, so a whole gate/up unit (8 stages) is in flight at
// once.  Eight consumer warps do the arithmetic of the dense decode kernel:
// the group's activations, scaled per token by a power of two into fp16
// (exact for every element within 2^28 of the token's largest), E2M1 pairs
// unpacked with cvt.rn.f16x2.e2m1x2, products accumulated in fp32 with
// fma.rn.f32.f16, the E4M3 block scale applied per 16 elements.
//
// The combine: every down unit writes its fp32 rows d[t, j, tile] and counts
// one arrival per (token, tile) on a counter the route kernel zeroed; the unit
// that brings the count to k sums the k rows in slot order, so y does not
// depend on which unit finished last.
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "internal.h"
#include "tma.cuh"
#include "topk.cuh"

#define NVFP4_LAUNCH_TRY(expr)          \
    do {                                \
        const int _s = (expr);          \
        if (_s != NVFP4_OK) return _s;  \
    } while (0)

namespace nvfp4 {

// Uniform decision of the 256 consumer threads: true only if every one passes true.
NVFP4_DEV bool consumers_all(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 256, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

namespace moedec {
constexpr int kMT = 4;                            // tokens per group
constexpr int kStages = 8;
constexpr int kStageK = 256;                      // elements per stage
constexpr int kCodeBytes = 128 * 128;             // 128 rows x 128 B
constexpr int kScaleBytes = 4096;                 // two 2 KB scale runs (gate/up) or one (down)
constexpr int kThreads = 288;                     // 8 consumer warps + 1 producer warp
constexpr int kMaxE = 1024;

size_t smem_bytes(int K) {
    return 1024 + (size_t)kStages * (kCodeBytes + kScaleBytes) + (size_t)kMT * K * 2 + 128 * kMT * 4 +
           kMT * 8 * 4 + 16 + 8 * 2 * kStages;
}
}  // namespace moedec

struct MoeDecArgs {
    int T, H, I, E, k;
    const __nv_bfloat16* x;   // gate/up: h [T, H]; down: a [T * k, I]
    const uint8_t* scales;    // per-expert TILED scale blocks, sf_stride bytes apart
    int64_t sf_stride;
    int64_t cp4;              // scale atoms along K (K / 64)
    const float* gs;          // [E]
    const int32_t* n_groups;  // routing tables (route kernel)
    const int32_t* groups;    // [n_groups][3] = {expert, first pair, tokens}
    const int32_t* perm_t;    // pairs sorted by (expert, token): token
    const int32_t* perm_j;    //   and slot
    __nv_bfloat16* a;         // gate/up output [T * k, I], row t * k + j
    float* d;                 // down rows [T * k, H]
    int32_t* cnt;             // [T][H / 128] arrivals
    const float* topk_w;      // [T, k]
    void* y;                  // [T, H]
    int* status;
};

// ---- routing tables ----------------------------------------------------------

// Exclusive prefix sum over the 1024 threads of the CTA; *total = the sum.
NVFP4_DEV int block_excl_scan(int v, int* s_warp, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    __syncthreads();  // s_warp of an earlier scan fully read
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    int before = 0, tot = 0;
    for (int w = 0; w < 32; ++w) {
        const int t = s_warp[w];
        if (w < warp) before += t;
        tot += t;
    }
    *total = tot;
    return before + x - v;
}

// One CTA of 1024 threads: warp t takes token t's top-k; thread e takes
// expert e's token list.
template <int PER>
__global__ void __launch_bounds__(1024) moe_decode_route_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                                int ncnt, int32_t* __restrict__ topk_idx,
                                                                float* __restrict__ topk_w, int32_t* __restrict__ n_groups,
                                                                int32_t* __restrict__ groups,
                                                                int32_t* __restrict__ perm_t,
                                                                int32_t* __restrict__ perm_j, int32_t* __restrict__ cnt) {
    __shared__ uint32_t mask[moedec::kMaxE];  // bit t: token t chose expert e
    __shared__ int32_t s_off[moedec::kMaxE];
    __shared__ int s_warp[32];
    griddep_launch_dependents();
    griddep_wait();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < ncnt; i += 1024) cnt[i] = 0;
    mask[tid] = 0;
    __syncthreads();
    int myidx = 0;
    float myw = 0.0f;
    if (warp < T) {
        warp_topk<PER>(logits + (int64_t)warp * E, E, k, lane, &myidx, &myw);
        if (lane < k) {
            topk_idx[warp * k + lane] = myidx;
            topk_w[warp * k + lane] = myw;
            atomicOr(&mask[myidx], 1u << warp);
        }
    }
    __syncthreads();
    const int e = tid;
    const int c = e < E ? __popc(mask[e]) : 0;
    const int full = c >> 2, rem = c & 3;
    int tot_c, n_full, n3, n2, n1;
    const int off = block_excl_scan(c, s_warp, &tot_c);
    const int pf = block_excl_scan(full, s_warp, &n_full);
    const int p3 = block_excl_scan(rem == 3, s_warp, &n3);
    const int p2 = block_excl_scan(rem == 2, s_warp, &n2);
    const int p1 = block_excl_scan(rem == 1, s_warp, &n1);
    s_off[e] = off;
    // groups of four tokens first, then of three, two and one (largest first)
    for (int q = 0; q < full; ++q) {
        int32_t* g = groups + 3 * (pf + q);
        g[0] = e;
        g[1] = off + 4 * q;
        g[2] = 4;
    }
    if (rem) {
        const int pos = rem == 3 ? n_full + p3 : rem == 2 ? n_full + n3 + p2 : n_full + n3 + n2 + p1;
        int32_t* g = groups + 3 * pos;
        g[0] = e;
        g[1] = off + 4 * full;
        g[2] = rem;
    }
    if (tid == 0) *n_groups = n_full + n3 + n2 + n1;
    __syncthreads();
    if (warp < T && lane < k) {
        const int rank = __popc(mask[myidx] & ((1u << warp) - 1u));
        const int r = s_off[myidx] + rank;
        perm_t[r] = warp;
        perm_j[r] = lane;
    }
}

// ---- expert projections ---------------------------------------------------------

NVFP4_DEV float fma_f16hf(uint16_t a, uint16_t b, float c) {
    float d;
    asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
    return d;
}

// 32 code x activation products as two 16-element block partials.
NVFP4_DEV void dot32h(const uint4& wq, const uint32_t* xw, float& p0, float& p1) {
    const uint32_t w[4] = {wq.x, wq.y, wq.z, wq.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t h[4];
        e2m1x8_to_f16x2(w[j], h);
        float p = (j < 2) ? p0 : p1;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t xv = xw[4 * j + q];
            p = fma_f16hf((uint16_t)(h[q] & 0xFFFF), (uint16_t)(xv & 0xFFFF), p);
            p = fma_f16hf((uint16_t)(h[q] >> 16), (uint16_t)(xv >> 16), p);
        }
        if (j < 2) p0 = p; else p1 = p;
    }
}

// PHASE 0: gate/up + SwiGLU (K = H, 64 + 64 rows per tile, I / 64 tiles per
// group); PHASE 1: down + combine (K = I, 128 rows per tile, H / 128 tiles).
template <int PHASE, typename OutT>
__global__ void __launch_bounds__(moedec::kThreads, 1)
    moe_decode_kernel(const __grid_constant__ CUtensorMap cmap, const MoeDecArgs a) {
    using namespace moedec;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int K = PHASE == 0 ? a.H : a.I;
    const int nst = K / kStageK;
    const int tpg = PHASE == 0 ? a.I / 64 : a.H / 128;  // tiles per group
    uint8_t* s_codes = smem;
    uint8_t* s_scales = s_codes + kStages * kCodeBytes;
    __half* s_x = reinterpret_cast<__half*>(s_scales + kStages * kScaleBytes);  // [kMT][K]
    float* s_out = reinterpret_cast<float*>(s_x + kMT * K);                     // [128][kMT]
    float* s_max = s_out + 128 * kMT;                                            // [kMT][8]
    int* s_flag = reinterpret_cast<int*>(s_max + kMT * 8);                       // [kMT]
    uint64_t* full = reinterpret_cast<uint64_t*>(s_flag + 4);
    uint64_t* empty = full + kStages;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 8);  // one release per consumer warp
        }
        fence_barrier_init();
    }
    __syncthreads();
    griddep_launch_dependents();
    griddep_wait();  // routing tables (and, for down, a) are complete from here on
    const int n_units = __ldcg(a.n_groups) * tpg;

    if (warp == 8) {
        // ---------------- producer ----------------
        if (lane == 0) {
            prefetch_tensormap(&cmap);
            const uint64_t pol = l2_evict_first_policy();  // weights are read once per call
            int s = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
                const int g = u / tpg, p = u % tpg;
                const int e = __ldcg(a.groups + 3 * g);
                const uint8_t* sc_e = a.scales + (int64_t)e * a.sf_stride;
                for (int st = 0; st < nst; ++st, ++s) {
                    const int slot = s % kStages;
                    if (s >= kStages) {
                        if (!mbar_wait(&empty[slot], ((s / kStages) - 1) & 1, a.status)) {
                            ok = false;
                            break;
                        }
                        fence_proxy_async();  // consumers' generic reads before the async-proxy refill
                    }
                    uint8_t* cs = s_codes + slot * kCodeBytes;
                    uint8_t* ss = s_scales + slot * kScaleBytes;
                    if constexpr (PHASE == 0) {
                        mbar_expect_tx(&full[slot], kCodeBytes + 4096);
                        const int y0 = e * 2 * a.I + 64 * p;
                        tma_load_2d_hint(cs, &cmap, &full[slot], st * 128, y0, pol);
                        tma_load_2d_hint(cs + kCodeBytes / 2, &cmap, &full[slot], st * 128, y0 + a.I, pol);
                        bulk_load_hint(ss, sc_e + ((int64_t)(p >> 1) * a.cp4 + st * 4) * 512, 2048, &full[slot], pol);
                        bulk_load_hint(ss + 2048, sc_e + ((int64_t)((a.I >> 7) + (p >> 1)) * a.cp4 + st * 4) * 512,
                                       2048, &full[slot], pol);
                    } else {
                        mbar_expect_tx(&full[slot], kCodeBytes + 2048);
                        tma_load_2d_hint(cs, &cmap, &full[slot], st * 128, e * a.H + 128 * p, pol);
                        bulk_load_hint(ss, sc_e + ((int64_t)p * a.cp4 + st * 4) * 512, 2048, &full[slot], pol);
                    }
                }
            }
        }
        return;
    }

    // ---------------- consumers ----------------
    const int ctid = threadIdx.x;  // 0..255
    const int ch = lane & 7, rsub = lane >> 3;
    int s = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        const int g = u / tpg, p = u % tpg;
        const int e = __ldcg(a.groups + 3 * g), row0 = __ldcg(a.groups + 3 * g + 1);
        const int ntok = __ldcg(a.groups + 3 * g + 2);
        int tok[kMT], slt[kMT];
#pragma unroll
        for (int t = 0; t < kMT; ++t) {
            tok[t] = t < ntok ? __ldcg(a.perm_t + row0 + t) : 0;
            slt[t] = t < ntok ? __ldcg(a.perm_j + row0 + t) : 0;
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");  // the previous unit is done with s_x, s_out, s_flag
        // the group's activation rows -> shared memory, then fp16 * 2^p per token
        const int nv8 = K / 8;
        float mx[kMT];
#pragma unroll
        for (int t = 0; t < kMT; ++t) {
            mx[t] = 0.0f;
            if (t < ntok) {
                const int64_t xr = PHASE == 0 ? (int64_t)tok[t] : (int64_t)tok[t] * a.k + slt[t];
                const uint4* src = reinterpret_cast<const uint4*>(a.x + xr * K);
                for (int v = ctid; v < nv8; v += 256) {
                    const uint4 q4 = __ldcg(src + v);
                    reinterpret_cast<uint4*>(s_x + t * K)[v] = q4;
                    const uint32_t w4[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mx[t] = fmaxf(mx[t], fmaxf(fabsf(bf16lo_to_f32(w4[j])), fabsf(bf16hi_to_f32(w4[j]))));
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx[t] = fmaxf(mx[t], __shfl_xor_sync(0xffffffffu, mx[t], o));
            if (lane == 0) s_max[t * 8 + warp] = mx[t];
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        float inv_p[kMT];
#pragma unroll
        for (int t = 0; t < kMT; ++t) {
            float m = 0.0f;
#pragma unroll
            for (int w = 0; w < 8; ++w) m = fmaxf(m, s_max[t * 8 + w]);
            int pe = 0;
            if (m > 0.0f) pe = 141 - (int)((__float_as_uint(m) >> 23) & 0xFF);  // m * 2^pe in [2^14, 2^15)
            pe = pe < -126 ? -126 : (pe > 126 ? 126 : pe);
            const float sc = __uint_as_float((uint32_t)(127 + pe) << 23);
            inv_p[t] = __uint_as_float((uint32_t)(127 - pe) << 23);
            if (t < ntok)
                for (int v = ctid; v < nv8; v += 256) {  // the elements this thread loaded
                    uint4* qp = reinterpret_cast<uint4*>(s_x + t * K) + v;
                    const uint4 q4 = *qp;
                    const uint32_t w4[4] = {q4.x, q4.y, q4.z, q4.w};
                    uint32_t o[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const __half2 h2 = __floats2half2_rn(bf16lo_to_f32(w4[j]) * sc, bf16hi_to_f32(w4[j]) * sc);
                        o[j] = *reinterpret_cast<const uint32_t*>(&h2);
                    }
                    *qp = make_uint4(o[0], o[1], o[2], o[3]);
                }
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");

        float acc[4][kMT];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int t = 0; t < kMT; ++t) acc[i][t] = 0.0f;
        for (int st = 0; st < nst; ++st, ++s) {
            const int slot = s % kStages;
            if (ok) ok = mbar_wait(&full[slot], (s / kStages) & 1, a.status);
            if (!ok) continue;  // the producer stopped: keep the control flow, skip the work
            const uint8_t* cs = s_codes + slot * kCodeBytes;
            const uint8_t* ss = s_scales + slot * kScaleBytes;
            uint4 wq[4];
            uint32_t sc2[4];
            uint32_t dep = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = 16 * warp + rsub + 4 * i;  // row of the stage's 128
                wq[i] = *reinterpret_cast<const uint4*>(cs + r * 128 + ch * 16);
                // the row within its 128-row scale block
                const int rr = PHASE == 0 ? (r & 63) + 64 * (p & 1) : r;
                const uint8_t* sb = ss + ((PHASE == 0 && r >= 64) ? 2048 : 0);
                sc2[i] = *reinterpret_cast<const uint16_t*>(sb + (ch >> 1) * 512 + (rr & 31) * 16 + (rr >> 5) * 4 +
                                                            2 * (ch & 1));
                dep ^= wq[i].x ^ wq[i].y ^ wq[i].z ^ wq[i].w ^ sc2[i];
            }
            warp_release_after(&empty[slot], dep);
            float2 sd[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) sd[i] = f16x2_to_f32x2(e4m3x2_to_f16x2((uint16_t)sc2[i]));
#pragma unroll
            for (int t = 0; t < kMT; ++t) {
                if (t < ntok) {
                    uint32_t xw[16];
                    const uint4* xp = reinterpret_cast<const uint4*>(s_x + t * K + st * kStageK + ch * 32);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const uint4 xv = xp[v];
                        xw[4 * v] = xv.x; xw[4 * v + 1] = xv.y; xw[4 * v + 2] = xv.z; xw[4 * v + 3] = xv.w;
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float p0 = 0.0f, p1 = 0.0f;
                        dot32h(wq[i], xw, p0, p1);
                        acc[i][t] = fmaf(p0, sd[i].x, acc[i][t]);
                        acc[i][t] = fmaf(p1, sd[i].y, acc[i][t]);
                    }
                }
            }
        }
        // the 8 chunk columns of each row meet, then the rows go to shared memory
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int t = 0; t < kMT; ++t) {
                float v = acc[i][t];
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                acc[i][t] = v;
            }
        if (ch == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int t = 0; t < kMT; ++t) s_out[(16 * warp + rsub + 4 * i) * kMT + t] = acc[i][t] * inv_p[t];
        }
        ok = consumers_all(ok);  // also the barrier that makes s_out complete
        if (!ok) continue;       // a wait ran out (status recorded): no output from here on
        const float gsv = __ldg(a.gs + e);
        if constexpr (PHASE == 0) {
            for (int idx = ctid; idx < 64 * ntok; idx += 256) {
                const int c = idx & 63, t = idx >> 6;
                const float gg = s_out[c * kMT + t] * gsv;
                const float uu = s_out[(64 + c) * kMT + t] * gsv;
                a.a[((int64_t)tok[t] * a.k + slt[t]) * a.I + 64 * p + c] = __float2bfloat16_rn(gg / (1.0f + expf(-gg)) * uu);
            }
        } else {
            for (int idx = ctid; idx < 128 * ntok; idx += 256) {
                const int r = idx & 127, t = idx >> 7;
                a.d[((int64_t)tok[t] * a.k + slt[t]) * a.H + 128 * p + r] = s_out[r * kMT + t] * gsv;
            }
            __threadfence();  // the rows are visible device-wide before the arrival is counted
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (ctid < ntok) {
                const int old = atomicAdd(a.cnt + tok[ctid] * (a.H / 128) + p, 1);
                s_flag[ctid] = old == a.k - 1;  // this unit brought the count to k: it sums the slots
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            for (int idx = ctid; idx < 128 * ntok; idx += 256) {
                const int r = idx & 127, t = idx >> 7;
                if (!s_flag[t]) continue;
                __threadfence();
                const int64_t tt = tok[t];
                float acc_y = 0.0f;
                for (int j = 0; j < a.k; ++j)
                    acc_y = fmaf(__ldcg(a.topk_w + tt * a.k + j), __ldcg(a.d + (tt * a.k + j) * a.H + 128 * p + r), acc_y);
                store_out<OutT>(reinterpret_cast<OutT*>(a.y) + tt * a.H + 128 * p + r, acc_y);
            }
        }
    }
}

// ---- host ------------------------------------------------------------------

static int sm_count() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (!n) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

template <int PHASE, typename OutT>
static int launch_expert(const CUtensorMap& cm, const MoeDecArgs& a, cudaStream_t st) {
    auto kern = moe_decode_kernel<PHASE, OutT>;
    const size_t smem = moedec::smem_bytes(PHASE == 0 ? a.H : a.I);
    static std::once_flag once;
    std::call_once(once, [&] { cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024); });
    const int nsm = sm_count();
    if (nsm <= 0) return NVFP4_ERR_LAUNCH;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)nsm, 1, 1);  // persistent: one CTA per SM walks the units
    cfg.blockDim = dim3(moedec::kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    set_pdl_attr(attr[0]);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, cm, a) == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

size_t moe_decode_smem_bytes(int64_t H, int64_t I) { return moedec::smem_bytes((int)(H > I ? H : I)); }

int launch_moe_decode(const MoeDecodeLaunch& L, cudaStream_t st) {
    NVFP4_LAUNCH_TRY(launch_router_logits_small_pdl(L.h, L.w_router, L.logit_bias, L.T, L.H, L.E, L.logits, st));
    {
        const int per = (L.E + 31) / 32;
        const int ncnt = L.T * (L.H / 128);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(1, 1, 1);
        cfg.blockDim = dim3(1024, 1, 1);
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        set_pdl_attr(attr[0]);
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t r;
        if (per <= 8)
            r = cudaLaunchKernelEx(&cfg, moe_decode_route_kernel<8>, (const float*)L.logits, L.T, L.E, L.k, ncnt,
                                   L.topk_idx, L.topk_w, L.n_groups, L.groups, L.perm_t, L.perm_j, L.cnt);
        else if (per <= 16)
            r = cudaLaunchKernelEx(&cfg, moe_decode_route_kernel<16>, (const float*)L.logits, L.T, L.E, L.k, ncnt,
                                   L.topk_idx, L.topk_w, L.n_groups, L.groups, L.perm_t, L.perm_j, L.cnt);
        else
            r = cudaLaunchKernelEx(&cfg, moe_decode_route_kernel<32>, (const float*)L.logits, L.T, L.E, L.k, ncnt,
                                   L.topk_idx, L.topk_w, L.n_groups, L.groups, L.perm_t, L.perm_j, L.cnt);
        if (r != cudaSuccess) return NVFP4_ERR_LAUNCH;
    }
    MoeDecArgs a{};
    a.T = L.T;
    a.H = L.H;
    a.I = L.I;
    a.E = L.E;
    a.k = L.k;
    a.n_groups = L.n_groups;
    a.groups = L.groups;
    a.perm_t = L.perm_t;
    a.perm_j = L.perm_j;
    a.a = (__nv_bfloat16*)L.a;
    a.d = L.d;
    a.cnt = L.cnt;
    a.topk_w = L.topk_w;
    a.y = L.y;
    a.status = L.status;
    // gate/up + SwiGLU: stacked [E * 2I, H/2] codes, boxes of 64 rows
    CUtensorMap cm;
    if (!make_tmap_2d_u8(&cm, L.gu_codes, (uint64_t)(L.H / 2), (uint64_t)L.E * 2 * L.I, 128, 64))
        return NVFP4_ERR_LAUNCH;
    a.x = (const __nv_bfloat16*)L.h;
    a.scales = L.gu_scales;
    a.sf_stride = (int64_t)(2 * L.I) * (L.H / 16);  // TILED: rows already a multiple of 128, H/16 of 4
    a.cp4 = L.H / 64;
    a.gs = L.gu_gs;
    NVFP4_LAUNCH_TRY((launch_expert<0, float>(cm, a, st)));
    // down + combine: stacked [E * H, I/2] codes, boxes of 128 rows
    if (!make_tmap_2d_u8(&cm, L.dn_codes, (uint64_t)(L.I / 2), (uint64_t)L.E * L.H, 128, 128)) return NVFP4_ERR_LAUNCH;
    a.x = (const __nv_bfloat16*)L.a;
    a.scales = L.dn_scales;
    a.sf_stride = (int64_t)L.H * (L.I / 16);
    a.cp4 = L.I / 64;
    a.gs = L.dn_gs;
    if (L.y_dtype == NVFP4_DTYPE_BF16) return launch_expert<1, __nv_bfloat16>(cm, a, st);
    return launch_expert<1, float>(cm, a, st);
}

}  // namespace nvfp4
