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
//            (moe_decode_kernel<0>, moe_decode_kernel<1>, moe_decode_combine_kernel)
//
// The router is router_logits_tcs_kernel (router_tc.cu) for T <= 64.  The five
// kernels run as a programmatic-dependent chain: each one launches
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
// The producer also feeds each unit's activations: the route kernel writes h
// as fp16 scaled per token by a power of two, and the gate/up epilogue writes
// a both as bf16 (the layer's output) and as fp16 scaled per (row, 64-column
// block) for the down projection; the producer bulk-copies the unit's rows
// and their scales into a double-buffered slot together with the unit's
// routing metadata, so consumers never wait on a global load.  A last kernel
// sums the k fp32 rows d[t, j] of every token in slot order.
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
constexpr int kMaxBlk = 64;                       // 64-element prescale blocks per row (K <= 4096)

// Per-unit data the producer hands to the consumers with the activations.
struct UnitMeta {
    int e, p, ntok, pad;
    int tok[kMT], slt[kMT];
    float inv_tok[kMT];  // gate/up: 2^-p of each token's fp16 prescale
    float pad2[kMT];
};

constexpr size_t kRing = (size_t)kStages * (kCodeBytes + kScaleBytes);
size_t smem_bytes(int K) {
    return 1024 + kRing + 2 * (size_t)kMT * K * 2 + 128 * kMT * 4 + 2 * sizeof(UnitMeta) +
           2 * kMT * kMaxBlk * 4 + 8 * 4 + 8 * (2 * kStages + 4);
}
}  // namespace moedec

struct MoeDecArgs {
    int T, H, I, E, k;
    const __half* x16;        // prescaled fp16 activations: gate/up [T, H]; down [T * k, I]
    const float* inv_x;       // down: their 2^-p per (row, 64-block) [T * k][I / 64] (gate/up: in the records)
    const uint8_t* scales;    // per-expert TILED scale blocks, sf_stride bytes apart
    int64_t sf_stride;
    int64_t cp4;              // scale atoms along K (K / 64)
    const float* gs;          // [E]
    const int32_t* n_groups;  // routing tables (route kernel)
    const int32_t* groups;    // [max_groups] token-group records (kRecInts words)
    int max_groups;           // T * k: records that may exist
    __nv_bfloat16* a;         // gate/up output [T * k, I], row t * k + j
    __half* a16;              // the same prescaled for the down projection, and
    float* inv_a;             //   its 2^-p per (row, 64-block)
    float* d;                 // down output rows [T * k, H]
    int* status;
};

// ---- routing tables ----------------------------------------------------------

// Exclusive prefix sum over the 1024 threads of the CTA of four 16-bit
// counters packed in one 64-bit word (no field overflows: each total is at
// most T * k <= 1024); *total = the sum.
NVFP4_DEV uint64_t block_excl_scan4x16(uint64_t v, uint64_t* s_warp, uint64_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    uint64_t before = 0, tot = 0;
#pragma unroll 8
    for (int w = 0; w < 32; ++w) {
        const uint64_t t = s_warp[w];
        if (w < warp) before += t;
        tot += t;
    }
    *total = tot;
    return before + x - v;
}

// One CTA of 1024 threads: warp t takes token t's top-k; thread e takes
// expert e's token list.
// Power-of-two prescale of a row whose largest magnitude is m: m * 2^p lies in
// [2^14, 2^15), so fp16(v * 2^p) == v for every bf16 v within 2^28 of m.
NVFP4_DEV float prescale_of(float m, float* inv) {
    int pe = 0;
    if (m > 0.0f) pe = 141 - (int)((__float_as_uint(m) >> 23) & 0xFF);
    pe = pe < -126 ? -126 : (pe > 126 ? 126 : pe);
    *inv = __uint_as_float((uint32_t)(127 - pe) << 23);
    return __uint_as_float((uint32_t)(127 + pe) << 23);
}

// Token-group record written by the route kernel: {expert, tokens, the tokens
// (byte t of word 2), their slots (byte t of word 3), the tokens' 2^-p}.
constexpr int kRecInts = 8;

// Also prescales h for the gate/up projection: h16[t] = fp16(h[t] * 2^p_t)
// with p_t from the token's largest magnitude (2^-p_t goes into the records).
template <int PER>
__global__ void __launch_bounds__(1024) moe_decode_route_kernel(const float* __restrict__ logits,
                                                                const __nv_bfloat16* __restrict__ h, int T, int H,
                                                                int E, int k, int32_t* __restrict__ topk_idx,
                                                                float* __restrict__ topk_w, int32_t* __restrict__ n_groups,
                                                                int32_t* __restrict__ groups, __half* __restrict__ h16) {
    __shared__ uint32_t mask[moedec::kMaxE];            // bit t: token t chose expert e
    __shared__ uint8_t s_slot[32][moedec::kMaxE];       // slot in which token t chose expert e
    __shared__ unsigned s_tmax[32];                     // per token max |h| (float bits)
    __shared__ float s_inv[32];
    __shared__ uint64_t s_warp[32];
    griddep_launch_dependents();
    griddep_wait();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    mask[tid] = 0;
    if (tid < 32) s_tmax[tid] = 0u;
    __syncthreads();
    // h -> fp16 * 2^p_t: the [T, H] tensor in chunks of 8 x 1024 16-byte
    // pieces, every thread issuing its 8 loads of a chunk before using them; a
    // warp's 32 pieces lie in one token row (H % 256 == 0).  A single chunk
    // (T * H <= 65536) stays in registers between the max and the conversion.
    constexpr int kPer = 8;
    const int nv = T * (H / 8);
    const int rowv = H / 8;
    uint4 q4[kPer];
    for (int c0 = 0; c0 < nv; c0 += 1024 * kPer) {
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int v = c0 + tid + 1024 * i;
            if (v < nv) q4[i] = reinterpret_cast<const uint4*>(h)[v];
        }
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int v = c0 + tid + 1024 * i;
            if (c0 + 1024 * i >= nv) break;  // warp-uniform: nv is a multiple of 32
            float m = 0.0f;
            if (v < nv) {
                const uint32_t w4[4] = {q4[i].x, q4[i].y, q4[i].z, q4[i].w};
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    m = fmaxf(m, fmaxf(fabsf(bf16lo_to_f32(w4[j])), fabsf(bf16hi_to_f32(w4[j]))));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0 && v < nv) atomicMax(&s_tmax[v / rowv], __float_as_uint(m));
        }
    }
    __syncthreads();
    if (tid < T) prescale_of(__uint_as_float(s_tmax[tid]), &s_inv[tid]);
    __syncthreads();
    const bool kept = nv <= 1024 * kPer;
    for (int c0 = 0; c0 < nv; c0 += 1024 * kPer) {
        if (!kept) {
#pragma unroll
            for (int i = 0; i < kPer; ++i) {
                const int v = c0 + tid + 1024 * i;
                if (v < nv) q4[i] = reinterpret_cast<const uint4*>(h)[v];
            }
        }
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int v = c0 + tid + 1024 * i;
            if (v >= nv) break;
            const float sc = 1.0f / s_inv[v / rowv];  // a power of two: exact
            const uint32_t w4[4] = {q4[i].x, q4[i].y, q4[i].z, q4[i].w};
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const __half2 h2 = __floats2half2_rn(bf16lo_to_f32(w4[j]) * sc, bf16hi_to_f32(w4[j]) * sc);
                o[j] = *reinterpret_cast<const uint32_t*>(&h2);
            }
            reinterpret_cast<uint4*>(h16)[v] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
    int myidx = 0;
    float myw = 0.0f;
    if (warp < T) {
        warp_topk<PER>(logits + (int64_t)warp * E, E, k, lane, &myidx, &myw);
        if (lane < k) {
            topk_idx[warp * k + lane] = myidx;
            topk_w[warp * k + lane] = myw;
            atomicOr(&mask[myidx], 1u << warp);
            s_slot[warp][myidx] = (uint8_t)lane;
        }
    }
    __syncthreads();
    const int e = tid;
    const uint32_t me = e < E ? mask[e] : 0u;
    const int c = __popc(me);
    const int full = c >> 2, rem = c & 3;
    uint64_t tot;
    const uint64_t pre = block_excl_scan4x16((uint64_t)full | (uint64_t)(rem == 3) << 16 |
                                                 (uint64_t)(rem == 2) << 32 | (uint64_t)(rem == 1) << 48,
                                             s_warp, &tot);
    const int pf = (int)(pre & 0xFFFF), p3 = (int)((pre >> 16) & 0xFFFF), p2 = (int)((pre >> 32) & 0xFFFF),
              p1 = (int)(pre >> 48);
    const int n_full = (int)(tot & 0xFFFF), n3 = (int)((tot >> 16) & 0xFFFF), n2 = (int)((tot >> 32) & 0xFFFF),
              n1 = (int)(tot >> 48);
    // groups of four tokens first, then of three, two and one (largest first)
    uint32_t left = me;
    for (int q = 0; q * 4 < c; ++q) {
        const int nt = c - 4 * q < 4 ? c - 4 * q : 4;
        const int pos = nt == 4 ? pf + q : nt == 3 ? n_full + p3 : nt == 2 ? n_full + n3 + p2 : n_full + n3 + n2 + p1;
        uint32_t toks = 0, slots = 0;
        float inv[4] = {1.0f, 1.0f, 1.0f, 1.0f};
        for (int t = 0; t < nt; ++t) {
            const int tk = __ffs(left) - 1;  // tokens in ascending order
            left &= left - 1;
            toks |= (uint32_t)tk << (8 * t);
            slots |= (uint32_t)s_slot[tk][e] << (8 * t);
            inv[t] = s_inv[tk];
        }
        int4* rec = reinterpret_cast<int4*>(groups + kRecInts * pos);
        rec[0] = make_int4(e, nt, (int)toks, (int)slots);
        rec[1] = make_int4(__float_as_int(inv[0]), __float_as_int(inv[1]), __float_as_int(inv[2]),
                           __float_as_int(inv[3]));
    }
    if (tid == 0) *n_groups = n_full + n3 + n2 + n1;
}

// ---- expert projections ---------------------------------------------------------


// PHASE 0: gate/up + SwiGLU (K = H, 64 + 64 rows per tile, I / 64 tiles per
// group); PHASE 1: down (K = I, 128 rows per tile, H / 128 tiles per group).
template <int PHASE>
__global__ void __launch_bounds__(moedec::kThreads, 1)
    moe_decode_kernel(const __grid_constant__ CUtensorMap cmap, const MoeDecArgs a) {
    using namespace moedec;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int K = PHASE == 0 ? a.H : a.I;
    const int nst = K / kStageK;
    const int nblk = K / 64;
    const int tpg = PHASE == 0 ? a.I / 64 : a.H / 128;  // tiles per group
    uint8_t* s_codes = smem;
    uint8_t* s_scales = s_codes + kStages * kCodeBytes;
    __half* s_x = reinterpret_cast<__half*>(s_scales + kStages * kScaleBytes);   // [2][kMT][K]
    float* s_out = reinterpret_cast<float*>(s_x + 2 * kMT * K);                  // [128][kMT]
    UnitMeta* s_meta = reinterpret_cast<UnitMeta*>(s_out + 128 * kMT);           // [2]
    float* s_inv = reinterpret_cast<float*>(s_meta + 2);                         // [2][kMT][kMaxBlk]
    float* s_pmax = s_inv + 2 * kMT * kMaxBlk;                                   // [8]
    uint64_t* full = reinterpret_cast<uint64_t*>(s_pmax + 8);
    uint64_t* empty = full + kStages;
    uint64_t* xfull = empty + kStages;
    uint64_t* xempty = xfull + 2;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 8);  // one release per consumer warp
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&xfull[s], 1);
            mbar_init(&xempty[s], 8);
        }
        fence_barrier_init();
    }
    __syncthreads();
    griddep_launch_dependents();
    griddep_wait();  // the routing tables and activations are complete from here on
    const int n_units = __ldcg(a.n_groups) * tpg;

    if (warp == 8) {
        // ---------------- producer ----------------
        if (lane == 0) {
            prefetch_tensormap(&cmap);
            const uint64_t pol = l2_evict_first_policy();  // weights are read once per call
            int s = 0, n = 0;
            bool ok = true;
            // the next unit's group record is loaded one unit ahead
            auto load_rec = [&](int u, int4& r0, int4& r1) {
                const int g = u / tpg;
                if (g < a.max_groups) {
                    r0 = __ldcg(reinterpret_cast<const int4*>(a.groups + kRecInts * g));
                    r1 = __ldcg(reinterpret_cast<const int4*>(a.groups + kRecInts * g) + 1);
                }
            };
            int4 c0 = make_int4(0, 0, 0, 0), c1 = c0;
            load_rec(blockIdx.x, c0, c1);
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++n) {
                const int p = u % tpg;
                const int e = c0.x, ntok = c0.y;
                const uint32_t toks = (uint32_t)c0.z, slots = (uint32_t)c0.w;
                const int4 inv4 = c1;
                if (u + (int)gridDim.x < n_units) load_rec(u + gridDim.x, c0, c1);
                // the unit's activation rows and metadata (double-buffered by unit)
                const int xs = n & 1;
                if (n >= 2 && !mbar_wait(&xempty[xs], ((n >> 1) - 1) & 1, a.status)) {
                    ok = false;
                    break;
                }
                UnitMeta* m = s_meta + xs;
                m->e = e;
                m->p = p;
                m->ntok = ntok;
                uint32_t bytes = (uint32_t)(ntok * K * 2) + (PHASE == 1 ? (uint32_t)(ntok * nblk * 4) : 0u);
                int rows[kMT];
#pragma unroll
                for (int t = 0; t < kMT; ++t) {
                    const int tt = (toks >> (8 * t)) & 0xFF, jj = (slots >> (8 * t)) & 0xFF;
                    m->tok[t] = tt;
                    m->slt[t] = jj;
                    rows[t] = PHASE == 0 ? tt : tt * a.k + jj;
                }
                m->inv_tok[0] = __int_as_float(inv4.x);
                m->inv_tok[1] = __int_as_float(inv4.y);
                m->inv_tok[2] = __int_as_float(inv4.z);
                m->inv_tok[3] = __int_as_float(inv4.w);
                mbar_expect_tx(&xfull[xs], bytes);  // releases the metadata stores above
                __half* xd = s_x + xs * kMT * K;
                for (int t = 0; t < ntok; ++t) {
                    bulk_load(xd + t * K, a.x16 + (int64_t)rows[t] * K, (uint32_t)(K * 2), &xfull[xs]);
                    if (PHASE == 1)
                        bulk_load(s_inv + (xs * kMT + t) * kMaxBlk, a.inv_x + (int64_t)rows[t] * nblk,
                                  (uint32_t)(nblk * 4), &xfull[xs]);
                }
                // the unit's weight stages
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
    int s = 0, n = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++n) {
        const int xs = n & 1;
        if (ok) ok = mbar_wait(&xfull[xs], (n >> 1) & 1, a.status);
        const UnitMeta* m = s_meta + xs;
        const int e = ok ? m->e : 0, p = ok ? m->p : 0, ntok = ok ? m->ntok : 0;
        // the unit's token rows, read now: the slot is handed back to the producer before the epilogue
        int tok[kMT], slt[kMT];
#pragma unroll
        for (int t = 0; t < kMT; ++t) {
            tok[t] = ok ? m->tok[t] : 0;
            slt[t] = ok ? m->slt[t] : 0;
        }
        const __half* xb = s_x + xs * kMT * K;
        const float* ib = s_inv + xs * kMT * kMaxBlk;
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
                    // the chunk's prescale: per token (gate/up) or per 64-element block (down)
                    const float iv = PHASE == 0 ? m->inv_tok[t] : ib[t * kMaxBlk + st * 4 + (ch >> 1)];
                    uint32_t xw[16];
                    const uint4* xp = reinterpret_cast<const uint4*>(xb + t * K + st * kStageK + ch * 32);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const uint4 xv = xp[v];
                        xw[4 * v] = xv.x; xw[4 * v + 1] = xv.y; xw[4 * v + 2] = xv.z; xw[4 * v + 3] = xv.w;
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float p0 = 0.0f, p1 = 0.0f;
                        dot32_e2m1_f16(wq[i], xw, p0, p1);
                        acc[i][t] = fmaf(p0, sd[i].x * iv, acc[i][t]);
                        acc[i][t] = fmaf(p1, sd[i].y * iv, acc[i][t]);
                    }
                }
            }
        }
        // the 8 chunk columns of each row meet, then the rows go to shared memory
        uint32_t dep = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int t = 0; t < kMT; ++t) {
                float v = acc[i][t];
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                acc[i][t] = v;
                dep ^= __float_as_uint(v);
            }
        // every read of this unit's slot is done (the sums and the row indices depend on them)
#pragma unroll
        for (int t = 0; t < kMT; ++t) dep ^= (uint32_t)(tok[t] ^ (slt[t] << 8));
        dep ^= (uint32_t)(e ^ (p << 16) ^ (ntok << 24));
        warp_release_after(&xempty[xs], dep);
        if (ch == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int t = 0; t < kMT; ++t) s_out[(16 * warp + rsub + 4 * i) * kMT + t] = acc[i][t];
        }
        ok = consumers_all(ok);  // also the barrier that makes s_out complete
        const float gsv = __ldg(a.gs + e);
        if constexpr (PHASE == 0) {
            // a = bf16(silu(g) * u) for 64 columns of each token; then the same
            // values prescaled for the down projection (per row, this 64-block)
            float v = 0.0f;
            int t = ctid >> 6, c = ctid & 63;
            if (ok && ctid < 64 * ntok) {
                const float gg = s_out[c * kMT + t] * gsv;
                const float uu = s_out[(64 + c) * kMT + t] * gsv;
                const __nv_bfloat16 b = __float2bfloat16_rn(gg / (1.0f + expf(-gg)) * uu);
                a.a[((int64_t)tok[t] * a.k + slt[t]) * a.I + 64 * p + c] = b;
                v = __bfloat162float(b);
            }
            float mx = fabsf(v);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (lane == 0) s_pmax[warp] = mx;
            asm volatile("bar.sync 1, 256;" ::: "memory");
            mx = fmaxf(mx, s_pmax[warp ^ 1]);  // the row's 64 columns are warps 2t and 2t + 1
            if (ok && ctid < 64 * ntok) {
                float inv;
                const float sc = prescale_of(mx, &inv);
                const int64_t row = (int64_t)tok[t] * a.k + slt[t];
                a.a16[row * a.I + 64 * p + c] = __float2half_rn(v * sc);
                if (c == 0) a.inv_a[row * (a.I / 64) + p] = inv;
            }
        } else {
            if (ok)
                for (int idx = ctid; idx < 128 * ntok; idx += 256) {
                    const int r = idx & 127, t = idx >> 7;
                    a.d[((int64_t)tok[t] * a.k + slt[t]) * a.H + 128 * p + r] = s_out[r * kMT + t] * gsv;
                }
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");  // s_out and s_pmax free for the next unit
    }
}

// y[t, n] = sum_{j<k} topk_w[t, j] * d[t * k + j, n], j ascending, fp32.
template <typename OutT>
__global__ void __launch_bounds__(256) moe_decode_combine_kernel(const float* __restrict__ d,
                                                                 const float* __restrict__ w, int T, int k, int H,
                                                                 OutT* __restrict__ y) {
    griddep_launch_dependents();
    griddep_wait();
    const int n4 = H / 4;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= T * n4) return;
    const int t = i / n4, c = (i % n4) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
        const float wj = w[t * k + j];
        const float4 v = *reinterpret_cast<const float4*>(d + ((int64_t)t * k + j) * H + c);
        acc.x = fmaf(wj, v.x, acc.x);
        acc.y = fmaf(wj, v.y, acc.y);
        acc.z = fmaf(wj, v.z, acc.z);
        acc.w = fmaf(wj, v.w, acc.w);
    }
    OutT* yp = y + (int64_t)t * H + c;
    store_out<OutT>(yp, acc.x);
    store_out<OutT>(yp + 1, acc.y);
    store_out<OutT>(yp + 2, acc.z);
    store_out<OutT>(yp + 3, acc.w);
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

static void pdl_config(cudaLaunchConfig_t& cfg, cudaLaunchAttribute* attr, dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st) {
    cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    set_pdl_attr(attr[0]);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
}

template <int PHASE>
static int launch_expert(const CUtensorMap& cm, const MoeDecArgs& a, cudaStream_t st) {
    auto kern = moe_decode_kernel<PHASE>;
    const size_t smem = moedec::smem_bytes(PHASE == 0 ? a.H : a.I);
    static std::once_flag once;
    std::call_once(once, [&] { cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024); });
    const int nsm = sm_count();
    if (nsm <= 0) return NVFP4_ERR_LAUNCH;
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    // persistent: one CTA per SM walks the units
    pdl_config(cfg, attr, dim3((unsigned)nsm), dim3(moedec::kThreads), smem, st);
    return cudaLaunchKernelEx(&cfg, kern, cm, a) == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

size_t moe_decode_smem_bytes(int64_t H, int64_t I) { return moedec::smem_bytes((int)(H > I ? H : I)); }

int launch_moe_decode(const MoeDecodeLaunch& L, cudaStream_t st) {
    if (router_tcs_supported(L.h, L.w_router, L.T, L.H, L.E))
        NVFP4_LAUNCH_TRY(launch_router_logits_tcs(L.h, L.w_router, L.logit_bias, L.T, L.H, L.E, L.logits, L.status, st));
    else
        NVFP4_LAUNCH_TRY(launch_router_logits_small_pdl(L.h, L.w_router, L.logit_bias, L.T, L.H, L.E, L.logits, st));
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    {
        const int per = (L.E + 31) / 32;
        pdl_config(cfg, attr, dim3(1), dim3(1024), 0, st);
        const __nv_bfloat16* h = (const __nv_bfloat16*)L.h;
        cudaError_t r;
        if (per <= 8)
            r = cudaLaunchKernelEx(&cfg, moe_decode_route_kernel<8>, (const float*)L.logits, h, L.T, L.H, L.E, L.k,
                                   L.topk_idx, L.topk_w, L.n_groups, L.groups, (__half*)L.h16);
        else if (per <= 16)
            r = cudaLaunchKernelEx(&cfg, moe_decode_route_kernel<16>, (const float*)L.logits, h, L.T, L.H, L.E, L.k,
                                   L.topk_idx, L.topk_w, L.n_groups, L.groups, (__half*)L.h16);
        else
            r = cudaLaunchKernelEx(&cfg, moe_decode_route_kernel<32>, (const float*)L.logits, h, L.T, L.H, L.E, L.k,
                                   L.topk_idx, L.topk_w, L.n_groups, L.groups, (__half*)L.h16);
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
    a.max_groups = L.T * L.k;
    a.a = (__nv_bfloat16*)L.a;
    a.a16 = (__half*)L.a16;
    a.inv_a = L.inv_a;
    a.d = L.d;
    a.status = L.status;
    // gate/up + SwiGLU: stacked [E * 2I, H/2] codes, boxes of 64 rows
    CUtensorMap cm;
    if (!make_tmap_2d_u8(&cm, L.gu_codes, (uint64_t)(L.H / 2), (uint64_t)L.E * 2 * L.I, 128, 64))
        return NVFP4_ERR_LAUNCH;
    a.x16 = (const __half*)L.h16;
    a.inv_x = nullptr;
    a.scales = L.gu_scales;
    a.sf_stride = (int64_t)(2 * L.I) * (L.H / 16);  // TILED: rows a multiple of 128, H/16 of 4
    a.cp4 = L.H / 64;
    a.gs = L.gu_gs;
    NVFP4_LAUNCH_TRY(launch_expert<0>(cm, a, st));
    // down: stacked [E * H, I/2] codes, boxes of 128 rows
    if (!make_tmap_2d_u8(&cm, L.dn_codes, (uint64_t)(L.I / 2), (uint64_t)L.E * L.H, 128, 128)) return NVFP4_ERR_LAUNCH;
    a.x16 = (const __half*)L.a16;
    a.inv_x = L.inv_a;
    a.scales = L.dn_scales;
    a.sf_stride = (int64_t)L.H * (L.I / 16);
    a.cp4 = L.I / 64;
    a.gs = L.dn_gs;
    NVFP4_LAUNCH_TRY(launch_expert<1>(cm, a, st));
    // the weighted combine
    const int n = L.T * (L.H / 4);
    pdl_config(cfg, attr, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st);
    cudaError_t r;
    if (L.y_dtype == NVFP4_DTYPE_BF16)
        r = cudaLaunchKernelEx(&cfg, moe_decode_combine_kernel<__nv_bfloat16>, (const float*)L.d,
                               (const float*)L.topk_w, L.T, L.k, L.H, (__nv_bfloat16*)L.y);
    else
        r = cudaLaunchKernelEx(&cfg, moe_decode_combine_kernel<float>, (const float*)L.d, (const float*)L.topk_w, L.T,
                               L.k, L.H, (float*)L.y);
    return r == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

}  // namespace nvfp4
