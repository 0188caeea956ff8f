// K11: a chain of W4A16 decode linears in one persistent launch (Ignis
// README, "The decode round": a decode step streams every layer's weights at
// the card's bandwidth; "Credits": the decode chain runs as one replayed unit).
//
// A call runs a list of ops, each y_i = x_i W_i^T with W_i NVFP4 (TILED scales)
// and M <= 2 activation rows.  An op reads either a caller bf16 tensor or the
// output of an earlier op, through one of three transforms, every activation
// handed to a linear being rounded to bf16:
//   NONE      x = bf16(v)
//   RMS       x = bf16(v / sqrt(mean(v[:K]^2)))   (first K columns of v)
//   SILU_MUL  x[j] = bf16(silu(v[j]) * v[K + j])
// With those the 64-layer decode stack (q = QKV(x); o = O(rms(q[:, :5120]));
// g = GU(rms(o)); h = silu(g[:, :N/2]) * g[:, N/2:]; x' = rms(Down(h))) is one
// op list.
//
// Why one launch: a launch per linear pays, every time, the drain of the
// previous grid, the activation prologue, the tail of its slowest CTAs and the
// split-K reduction, while the HBM stream stalls (5-7 us per linear on B200
// against 2.3-15 us of weight streaming).  Here every CTA (two per SM, all
// resident) walks the ops in order.  Its producer warp streams weight stages
// (2D TMA of 128 rows x 128 bytes plus the 2 KB scale run, 4-deep ring) from
// one op into the next without stopping; only the consumers wait, at a grid
// barrier placed before an op that reads an earlier op's output.  The ring
// keeps the HBM busy through the barrier.
//
// Work of an op: 128-row tiles x QS K-splits (QS chosen so the op has about
// one unit per CTA; unit u goes to CTA u mod grid).  A unit writes its fp32
// partial sums (already scaled by gs) to the op's [QS][M][N] buffer in the
// workspace; readers add the QS partials in split order, so every result is
// deterministic.  Ops that return y to the caller are finalized after the
// launch's last barrier.  Consumer arithmetic is that of the dense decode
// kernel: the unit's activation slice as fp16 scaled by a power of two,
// cvt.rn.f16x2.e2m1x2 unpacking, fma.rn.f32.f16 accumulation, E4M3 block
// scales per 16 elements.
#include <cuda.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "internal.h"
#include "tma.cuh"

namespace nvfp4 {

namespace chain {
constexpr int kStages = 4;
constexpr int kStageK = 256;
constexpr int kCodeBytes = 128 * 128;
constexpr int kScaleBytes = 2048;
constexpr int kThreads = 288;
constexpr int kMaxOps = 12;
constexpr int kMaxMT = 2;
constexpr int kMaxQS = 12;        // K splits of an op
constexpr int kMaxSliceK = 6144;  // elements of an activation slice held in shared memory
constexpr long long kBarrierCycles = 4000000000LL;
static_assert(kMaxSliceK <= 3 * 8 * 256, "the activation prologue covers a slice in three passes of 256 threads");

constexpr size_t kSmemBytes =
    1024 + (size_t)kStages * (kCodeBytes + kScaleBytes) + (size_t)kMaxMT * kMaxSliceK * 2 + 128 * kMaxMT * 4 + 256;
}  // namespace chain

struct ChainOpDev {
    const uint8_t* scales;   // TILED
    const float* gs;
    const __nv_bfloat16* x;  // source: caller tensor (or null)
    const float* src_part;   // source: an earlier op's partials [src_qs][M][src_n]
    float* part;             // this op's partials [qs][M][N]
    void* y;                 // caller output (or null)
    int64_t x_ld;
    int N, K, nst, tiles, qs, units;
    int rot;                 // unit u runs on CTA (u + rot) mod grid: the ops' work spread over the CTAs
    int src_n, src_qs, xform;
    int barrier_before;      // grid barrier before this op's units
    int y_dtype, y_xform;
};

struct ChainArgs {
    int n_ops, M, grid;
    int n_final;             // ops with y to finalize at the end
    unsigned* counter;       // grid barrier arrivals (zeroed before the launch)
    int* status;
    ChainOpDev op[chain::kMaxOps];
};

struct ChainMaps {
    CUtensorMap m[chain::kMaxOps];
};


// Grid barrier among the consumer threads of every CTA: one thread per CTA
// counts its arrival after the CTA's writes, then polls (bounded) until all
// CTAs of this barrier have arrived.  Called by all 256 consumer threads.
NVFP4_DEV bool chain_barrier(unsigned* counter, unsigned target, int* status, bool ok) {
    asm volatile("bar.sync 1, 256;" ::: "memory");
    __shared__ int s_ok;
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(counter, 1u);
        bool good = ok;
        const long long t0 = clock64();
        while (good) {
            unsigned v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
            if (v >= target) break;
            if (clock64() - t0 > chain::kBarrierCycles) {
                atomicExch(status, NVFP4_ERR_DEVICE_TIMEOUT);
                good = false;
            }
        }
        __threadfence();
        s_ok = good;
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
    return s_ok != 0;
}

// Eight consecutive source elements (m, c..c+7) of an op's input before its
// transform: the sum of the source op's split partials, in split order.
struct SrcView {
    const float* part;  // [qs][M][n]
    int n, qs;
};

NVFP4_DEV void src_value8(const SrcView& sv, int M, int m, int c, float (&v)[8]) {
    // the splits' loads go out in groups of four before their adds
    const float* base = sv.part + (int64_t)m * sv.n + c;
    const int64_t qstride = (int64_t)M * sv.n;
    const int nq = sv.qs;
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = 0.0f;
    for (int q0 = 0; q0 < nq; q0 += 4) {
        float4 a0[4], a1[4];
#pragma unroll
        for (int d = 0; d < 4; ++d) {  // past the last split: re-read it, not added
            const int q = q0 + d < nq ? q0 + d : nq - 1;
            const float4* p = reinterpret_cast<const float4*>(base + q * qstride);
            a0[d] = __ldcg(p);
            a1[d] = __ldcg(p + 1);
        }
#pragma unroll
        for (int d = 0; d < 4; ++d)
            if (q0 + d < nq) {
                v[0] += a0[d].x; v[1] += a0[d].y; v[2] += a0[d].z; v[3] += a0[d].w;
                v[4] += a1[d].x; v[5] += a1[d].y; v[6] += a1[d].z; v[7] += a1[d].w;
            }
    }
}

// Row rms factors 1 / sqrt(mean(v[:n]^2)) of a source (n columns of the summed
// partials), computed by the 256 consumer threads; 0 for an all-zero row.
template <int MT>
NVFP4_DEV void row_rms(const SrcView& sv, int M, int n, float (*s_stat)[chain::kMaxMT], float* s_rms) {
    const int ctid = threadIdx.x, warp = ctid >> 5, lane = ctid & 31;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        float ss = 0.0f;
        if (m < M)
            for (int c = 8 * ctid; c < n; c += 8 * 256) {
                float v[8];
                src_value8(sv, M, m, c, v);
#pragma unroll
                for (int j = 0; j < 8; ++j) ss = fmaf(v[j], v[j], ss);
            }
        ss = warp_sum(ss);
        if (lane == 0) s_stat[warp][m] = ss;
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (ctid < MT) {
        float t = 0.0f;
        for (int w = 0; w < 8; ++w) t += s_stat[w][ctid];
        s_rms[ctid] = t > 0.0f ? 1.0f / sqrtf(t / (float)n) : 0.0f;
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
}

template <int MT>
__global__ void __launch_bounds__(chain::kThreads, 2)
    chain_kernel(const __grid_constant__ ChainMaps maps, const __grid_constant__ ChainArgs a) {
    using namespace chain;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* s_codes = smem;
    uint8_t* s_scales = s_codes + kStages * kCodeBytes;
    __half* s_x = reinterpret_cast<__half*>(s_scales + kStages * kScaleBytes);  // [kMaxMT][kMaxSliceK]
    uint64_t* full = reinterpret_cast<uint64_t*>(s_x + kMaxMT * kMaxSliceK);
    uint64_t* empty = full + kStages;
    __shared__ float s_stat[8][kMaxMT];
    __shared__ float s_rms[kMaxMT];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int M = a.M;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 8);
        }
        fence_barrier_init();
    }
    __syncthreads();
    griddep_launch_dependents();  // every CTA of this grid is resident by now

    if (warp == 8) {
        // ---------------- producer: weights of every unit of every op, in order ----------------
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            for (int i = 0; i < a.n_ops; ++i) prefetch_tensormap(&maps.m[i]);
            int s = 0;
            bool ok = true;
            for (int i = 0; i < a.n_ops && ok; ++i) {
                const ChainOpDev& o = a.op[i];
                const int64_t cp4 = o.K / 64;
                for (int u = ((int)blockIdx.x - o.rot + a.grid) % a.grid; u < o.units && ok; u += a.grid) {
                    const int tile = u / o.qs, q = u % o.qs;
                    const int st0 = (int)((int64_t)o.nst * q / o.qs), st1 = (int)((int64_t)o.nst * (q + 1) / o.qs);
                    for (int st = st0; st < st1; ++st, ++s) {
                        const int slot = s % kStages;
                        if (s >= kStages) {
                            if (!mbar_wait(&empty[slot], ((s / kStages) - 1) & 1, a.status)) {
                                ok = false;
                                break;
                            }
                            fence_proxy_async();  // consumers' generic reads before the async-proxy refill
                        }
                        mbar_expect_tx(&full[slot], kCodeBytes + kScaleBytes);
                        tma_load_2d_hint(s_codes + slot * kCodeBytes, &maps.m[i], &full[slot], st * 128, tile * 128,
                                         pol);
                        bulk_load_hint(s_scales + slot * kScaleBytes, o.scales + ((int64_t)tile * cp4 + st * 4) * 512,
                                       kScaleBytes, &full[slot], pol);
                    }
                }
            }
        }
        return;
    }

    // ---------------- consumers ----------------
    griddep_wait();  // caller inputs written by earlier kernels are visible from here on
    const int ctid = threadIdx.x, ch = lane & 7, rsub = lane >> 3;
    int s = 0;
    unsigned barriers = 0;
    bool ok = true;
    int rms_op = -1;  // op whose input rms factors are in s_rms
    for (int i = 0; i < a.n_ops; ++i) {
        const ChainOpDev& o = a.op[i];
        if (o.barrier_before) ok = chain_barrier(a.counter, (unsigned)a.grid * ++barriers, a.status, ok);
        for (int u = ((int)blockIdx.x - o.rot + a.grid) % a.grid; u < o.units; u += a.grid) {
            const int tile = u / o.qs, q = u % o.qs;
            const int st0 = (int)((int64_t)o.nst * q / o.qs), st1 = (int)((int64_t)o.nst * (q + 1) / o.qs);
            const int k0 = st0 * kStageK, kr = (st1 - st0) * kStageK;
            asm volatile("bar.sync 1, 256;" ::: "memory");  // the previous unit is done with s_x
            if (o.xform == NVFP4_CHAIN_XFORM_RMS && rms_op != i) {
                row_rms<MT>(SrcView{o.src_part, o.src_n, o.src_qs}, M, o.K, s_stat, s_rms);
                rms_op = i;
            }
            // the unit's activation slice: transform, round to bf16 (kept as bf16
            // bits in s_x), then fp16 * 2^p per row from the slice's largest value
            float mx[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                mx[m] = 0.0f;
                if (m >= M) continue;
                // a caller tensor: every piece of the thread is requested before the first is used
                uint4 pre[3];
                if (o.x)
#pragma unroll
                    for (int r = 0; r < 3; ++r) {
                        const int c = 8 * ctid + 8 * 256 * r;
                        if (c < kr) pre[r] = __ldcg(reinterpret_cast<const uint4*>(o.x + (int64_t)m * o.x_ld + k0 + c));
                    }
#pragma unroll
                for (int r = 0; r < 3; ++r) {
                    const int c = 8 * ctid + 8 * 256 * r;
                    if (c >= kr) break;
                    const int k = k0 + c;
                    uint4 b;
                    if (o.x) {
                        b = pre[r];
                    } else {
                        float v[8];
                        if (o.xform == NVFP4_CHAIN_XFORM_SILU_MUL) {
                            float up[8];
                            const SrcView sv{o.src_part, o.src_n, o.src_qs};
                            src_value8(sv, M, m, k, v);
                            src_value8(sv, M, m, o.K + k, up);
#pragma unroll
                            for (int j = 0; j < 8; ++j) v[j] = v[j] / (1.0f + expf(-v[j])) * up[j];
                        } else {
                            src_value8(SrcView{o.src_part, o.src_n, o.src_qs}, M, m, k, v);
                            if (o.xform == NVFP4_CHAIN_XFORM_RMS)
#pragma unroll
                                for (int j = 0; j < 8; ++j) v[j] *= s_rms[m];
                        }
                        uint32_t w4[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
                            w4[j] = *reinterpret_cast<const uint32_t*>(&h2);
                        }
                        b = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                    *reinterpret_cast<uint4*>(s_x + m * kMaxSliceK + c) = b;
                    const uint32_t w4[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mx[m] = fmaxf(mx[m], fmaxf(fabsf(bf16lo_to_f32(w4[j])), fabsf(bf16hi_to_f32(w4[j]))));
                }
                mx[m] = warp_max(mx[m]);
                if (lane == 0) s_stat[warp][m] = mx[m];
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            float inv_p[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                float mm = 0.0f;
                for (int w = 0; w < 8; ++w) mm = fmaxf(mm, s_stat[w][m]);
                int pe = 0;
                if (mm > 0.0f) pe = 141 - (int)((__float_as_uint(mm) >> 23) & 0xFF);  // mm * 2^pe in [2^14, 2^15)
                pe = pe < -126 ? -126 : (pe > 126 ? 126 : pe);
                const float sc = __uint_as_float((uint32_t)(127 + pe) << 23);
                inv_p[m] = __uint_as_float((uint32_t)(127 - pe) << 23);
                if (m < M)
                    for (int c = 8 * ctid; c < kr; c += 8 * 256) {  // the elements this thread wrote
                        uint4* qp = reinterpret_cast<uint4*>(s_x + m * kMaxSliceK + c);
                        const uint4 b = *qp;
                        const uint32_t w4[4] = {b.x, b.y, b.z, b.w};
                        uint32_t o4[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const __half2 h2 = __floats2half2_rn(bf16lo_to_f32(w4[j]) * sc, bf16hi_to_f32(w4[j]) * sc);
                            o4[j] = *reinterpret_cast<const uint32_t*>(&h2);
                        }
                        *qp = make_uint4(o4[0], o4[1], o4[2], o4[3]);
                    }
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");

            float acc[4][MT];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;
            for (int st = st0; st < st1; ++st, ++s) {
                const int slot = s % kStages;
                if (ok) ok = mbar_wait(&full[slot], (s / kStages) & 1, a.status);
                if (!ok) continue;  // the producer stopped: keep the control flow, skip the work
                const uint8_t* cs = s_codes + slot * kCodeBytes;
                const uint8_t* ss = s_scales + slot * kScaleBytes;
                uint32_t xw[MT][16];
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const uint4* xp = reinterpret_cast<const uint4*>(s_x + m * kMaxSliceK + (st - st0) * kStageK + ch * 32);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const uint4 xv = xp[v];
                        xw[m][4 * v] = xv.x; xw[m][4 * v + 1] = xv.y; xw[m][4 * v + 2] = xv.z; xw[m][4 * v + 3] = xv.w;
                    }
                }
                uint4 wq[4];
                uint32_t sc2[4];
                uint32_t dep = 0;
#pragma unroll
                for (int r4 = 0; r4 < 4; ++r4) {
                    const int r = 16 * warp + rsub + 4 * r4;
                    wq[r4] = *reinterpret_cast<const uint4*>(cs + r * 128 + ch * 16);
                    sc2[r4] = *reinterpret_cast<const uint16_t*>(ss + (ch >> 1) * 512 + (r & 31) * 16 + (r >> 5) * 4 +
                                                                 2 * (ch & 1));
                    dep ^= wq[r4].x ^ wq[r4].y ^ wq[r4].z ^ wq[r4].w ^ sc2[r4];
                }
                warp_release_after(&empty[slot], dep);
#pragma unroll
                for (int r4 = 0; r4 < 4; ++r4) {
                    const float2 sd = f16x2_to_f32x2(e4m3x2_to_f16x2((uint16_t)sc2[r4]));
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        float p0 = 0.0f, p1 = 0.0f;
                        dot32_e2m1_f16(wq[r4], xw[m], p0, p1);
                        acc[r4][m] = fmaf(p0, sd.x, acc[r4][m]);
                        acc[r4][m] = fmaf(p1, sd.y, acc[r4][m]);
                    }
                }
            }
            // the 8 chunk columns of each row meet; lane ch == 0 writes the split's partial
            const float g = __ldg(o.gs);
#pragma unroll
            for (int r4 = 0; r4 < 4; ++r4)
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    float v = acc[r4][m];
                    v += __shfl_xor_sync(0xffffffffu, v, 1);
                    v += __shfl_xor_sync(0xffffffffu, v, 2);
                    v += __shfl_xor_sync(0xffffffffu, v, 4);
                    const int row = tile * 128 + 16 * warp + rsub + 4 * r4;
                    if (ch == 0 && m < M && row < o.N) o.part[((int64_t)q * M + m) * o.N + row] = v * inv_p[m] * g;
                }
        }
    }
    if (a.n_final == 0) return;
    // ---------------- the ops that return y: sum the partials (in split order) ----------------
    ok = chain_barrier(a.counter, (unsigned)a.grid * ++barriers, a.status, ok);
    if (!ok) return;
    const int gtid = blockIdx.x * 256 + ctid, gthreads = a.grid * 256;
    for (int i = 0; i < a.n_ops; ++i) {
        const ChainOpDev& o = a.op[i];
        if (!o.y) continue;
        const SrcView rd{o.part, o.N, o.qs};  // op i's partials, read like a source
        if (o.y_xform == NVFP4_CHAIN_XFORM_RMS) row_rms<MT>(rd, M, o.N, s_stat, s_rms);
        for (int idx = gtid; idx < M * (o.N / 8); idx += gthreads) {
            const int m = idx / (o.N / 8), c = (idx % (o.N / 8)) * 8;
            float v[8];
            src_value8(rd, M, m, c, v);
            if (o.y_xform == NVFP4_CHAIN_XFORM_RMS)
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] *= s_rms[m];
            if (o.y_dtype == NVFP4_DTYPE_F32) {
                float4* yp = reinterpret_cast<float4*>(reinterpret_cast<float*>(o.y) + (int64_t)m * o.N + c);
                yp[0] = make_float4(v[0], v[1], v[2], v[3]);
                yp[1] = make_float4(v[4], v[5], v[6], v[7]);
            } else {
                uint32_t w4[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
                    w4[j] = *reinterpret_cast<const uint32_t*>(&h2);
                }
                *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(o.y) + (int64_t)m * o.N + c) =
                    make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
        }
    }
}

// ---- host: plan and launch -------------------------------------------------------

static size_t al256(size_t n) { return (n + 255) & ~(size_t)255; }

static int chain_grid() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    int g = cache[dev].load(std::memory_order_relaxed);
    if (!g) {
        int nsm = 0;
        if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        g = 2 * nsm;  // two resident CTAs per SM (checked against the occupancy at launch)
        cache[dev].store(g, std::memory_order_relaxed);
    }
    return g;
}

struct ChainPlan {
    std::vector<int> qs;          // per op
    std::vector<size_t> part_off; // per op, bytes into ws
    size_t counters_off = 0, bytes = 0;
    int n_launches = 0;
};

static ChainPlan plan_chain(const nvfp4_chain_op* ops, int n_ops, int64_t M, int grid) {
    ChainPlan p;
    p.qs.resize(n_ops);
    p.part_off.resize(n_ops);
    size_t off = 0;
    for (int i = 0; i < n_ops; ++i) {
        const int64_t tiles = (ops[i].N + 127) / 128, nst = ops[i].K / chain::kStageK;
        int64_t qs = grid / tiles;
        if (qs < 1) qs = 1;
        if (qs > chain::kMaxQS) qs = chain::kMaxQS;
        if (qs > nst) qs = nst;
        while (qs < nst && (nst + qs - 1) / qs * chain::kStageK > chain::kMaxSliceK) ++qs;  // slice fits in smem
        p.qs[i] = (int)qs;
        p.part_off[i] = off;
        off += al256((size_t)qs * (size_t)M * (size_t)ops[i].N * 4);
    }
    p.n_launches = (n_ops + chain::kMaxOps - 1) / chain::kMaxOps;
    p.counters_off = off;
    off += al256((size_t)p.n_launches * 4);
    p.bytes = off;
    return p;
}

int chain_validate(const nvfp4_chain_op* ops, int n_ops, int64_t M) {
    if (!ops) return NVFP4_ERR_NULL;
    if (n_ops < 1 || n_ops > 4096 || M < 1 || M > chain::kMaxMT) return NVFP4_ERR_SHAPE;
    for (int i = 0; i < n_ops; ++i) {
        const nvfp4_chain_op& o = ops[i];
        if (!o.w_codes || !o.w_scales || !o.w_gs) return NVFP4_ERR_NULL;
        if (o.N < 8 || o.N % 8 || o.K < chain::kStageK || o.K % chain::kStageK || o.N > (1 << 24) ||
            o.K > (1 << 20))
            return NVFP4_ERR_SHAPE;
        if (((uintptr_t)o.w_codes & 15) || ((uintptr_t)o.w_scales & 15)) return NVFP4_ERR_ALIGN;
        if (o.xform < NVFP4_CHAIN_XFORM_NONE || o.xform > NVFP4_CHAIN_XFORM_SILU_MUL) return NVFP4_ERR_MODE;
        if (o.y_xform != NVFP4_CHAIN_XFORM_NONE && o.y_xform != NVFP4_CHAIN_XFORM_RMS) return NVFP4_ERR_MODE;
        if (o.src == NVFP4_CHAIN_SRC_X) {
            if (!o.x) return NVFP4_ERR_NULL;
            if (o.xform != NVFP4_CHAIN_XFORM_NONE) return NVFP4_ERR_MODE;
            if (o.x_ld < o.K || o.x_ld % 8 || ((uintptr_t)o.x & 15)) return NVFP4_ERR_ALIGN;
        } else if (o.src == NVFP4_CHAIN_SRC_OP) {
            if (o.src_op < 0 || o.src_op >= i) return NVFP4_ERR_SHAPE;
            const int64_t sn = ops[o.src_op].N;
            if (o.xform == NVFP4_CHAIN_XFORM_SILU_MUL ? sn != 2 * o.K : sn < o.K) return NVFP4_ERR_SHAPE;
        } else {
            return NVFP4_ERR_MODE;
        }
        if (o.y) {
            if (o.y_dtype != NVFP4_DTYPE_F32 && o.y_dtype != NVFP4_DTYPE_BF16) return NVFP4_ERR_DTYPE;
            if ((uintptr_t)o.y & 15) return NVFP4_ERR_ALIGN;
        }
    }
    return NVFP4_OK;
}

size_t chain_workspace(const nvfp4_chain_op* ops, int n_ops, int64_t M) {
    if (chain_validate(ops, n_ops, M) != NVFP4_OK) return 0;
    return plan_chain(ops, n_ops, M, chain_grid() ? chain_grid() : 296).bytes;
}

template <int MT>
static int launch_chain_part(const ChainMaps& maps, const ChainArgs& args, cudaStream_t st) {
    auto kern = chain_kernel<MT>;
    static std::once_flag once;
    std::call_once(once, [&] {
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)chain::kSmemBytes);
    });
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)args.grid);
    cfg.blockDim = dim3(chain::kThreads);
    cfg.dynamicSmemBytes = chain::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    set_pdl_attr(attr[0]);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, maps, args) == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}

int launch_chain(const nvfp4_chain_op* ops, int n_ops, int64_t M, void* ws, size_t ws_bytes, int* status,
                 cudaStream_t st) {
    const int grid = chain_grid();
    if (grid <= 0) return NVFP4_ERR_LAUNCH;
    {
        // every CTA of the grid must be resident at once (grid barriers)
        int per_sm = 0, nsm = grid / 2;
        auto kern = M == 1 ? chain_kernel<1> : chain_kernel<2>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)chain::kSmemBytes);
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, chain::kThreads, chain::kSmemBytes) !=
                cudaSuccess ||
            per_sm * nsm < grid)
            return NVFP4_ERR_LAUNCH;
    }
    const ChainPlan p = plan_chain(ops, n_ops, M, grid);
    if (!ws || ws_bytes < p.bytes) return NVFP4_ERR_WORKSPACE;
    char* base = (char*)ws;
    unsigned* counters = (unsigned*)(base + p.counters_off);
    if (cudaMemsetAsync(counters, 0, (size_t)p.n_launches * 4, st) != cudaSuccess) return NVFP4_ERR_LAUNCH;
    for (int l = 0; l < p.n_launches; ++l) {
        const int i0 = l * chain::kMaxOps, i1 = (i0 + chain::kMaxOps < n_ops) ? i0 + chain::kMaxOps : n_ops;
        ChainMaps maps;
        ChainArgs args{};
        args.n_ops = i1 - i0;
        args.M = (int)M;
        args.grid = grid;
        args.counter = counters + l;
        args.status = status;
        int rot = 0;
        for (int i = i0; i < i1; ++i) {
            const nvfp4_chain_op& o = ops[i];
            if (!make_tmap_2d_u8(&maps.m[i - i0], o.w_codes, (uint64_t)(o.K / 2), (uint64_t)o.N, 128, 128))
                return NVFP4_ERR_LAUNCH;
            ChainOpDev& d = args.op[i - i0];
            d.scales = o.w_scales;
            d.gs = o.w_gs;
            d.N = (int)o.N;
            d.K = (int)o.K;
            d.nst = (int)(o.K / chain::kStageK);
            d.tiles = (int)((o.N + 127) / 128);
            d.qs = p.qs[i];
            d.units = d.tiles * d.qs;
            d.rot = rot;
            rot = (int)((rot + (int64_t)d.units) % grid);
            d.part = (float*)(base + p.part_off[i]);
            d.xform = o.xform;
            if (o.src == NVFP4_CHAIN_SRC_X) {
                d.x = (const __nv_bfloat16*)o.x;
                d.x_ld = o.x_ld;
            } else {
                d.src_part = (const float*)(base + p.part_off[o.src_op]);
                d.src_n = (int)ops[o.src_op].N;
                d.src_qs = p.qs[o.src_op];
                // an op of this launch: wait for it at a grid barrier (earlier launches have completed)
                d.barrier_before = o.src_op >= i0;
            }
            d.y = o.y;
            d.y_dtype = o.y_dtype;
            d.y_xform = o.y_xform;
            if (o.y) ++args.n_final;
        }
        // one barrier serves every op behind it: keep only the first after each op that is read
        int last_barrier_at = -1;
        for (int i = i0; i < i1; ++i) {
            ChainOpDev& d = args.op[i - i0];
            if (!d.barrier_before) continue;
            // the source op completed at an earlier barrier of this launch already?
            bool covered = last_barrier_at >= 0 && ops[i].src_op < last_barrier_at;
            if (covered) d.barrier_before = 0;
            else last_barrier_at = i;
        }
        const int r = M == 1 ? launch_chain_part<1>(maps, args, st) : launch_chain_part<2>(maps, args, st);
        if (r != NVFP4_OK) return r;
    }
    return NVFP4_OK;
}

}  // namespace nvfp4
