// Fused small-batch forward of a stack of MoE layers: every layer of the
// stack, for up to 64 tokens, in one persistent kernel (one CTA per SM).
//
// Method: the layer is the one of moe_layer_forward (Colibri-Nano model card,
// "Architecture": sigmoid+bias router, top-K, shared expert; colibri README,
// "What's implemented": DeepSeek-V3-style router with routed_scaling_factor,
// packed int4 with per-row scales and dequant-on-use, batch-union MoE).  The
// cross-layer expert prediction of the nanocolibri-engine README (knobs table,
// PREDICT: "future routers run on the current residual and readahead-hint
// their experts ... hint-only, output is bit-identical") and colibri's
// router-lookahead (README, "How it works": the next layer's experts are
// prefetched while the current one runs) become L2 prefetches here.
//
// Work of layer l, by phase (every CTA runs them in order):
//  A  router units.  Unit (g, cb) = token group g (8 tokens) x hidden block cb
//     (128 columns).  For l > 0 the unit first finishes layer l-1 for its
//     block: it waits until every CTA has finished layer l-1's down tasks,
//     combines the expert outputs (same order and rounding as the combine
//     kernel) into x_l, and writes x_l to layer l-1's output.  It then
//     computes the partial router logits of its block on the tensor cores
//     (bf16 x against the exact three-way bf16 split of the f32 router
//     weights, one f32 sum per 16-wide k step) for layer l and, for the
//     lookahead, for layer l+1 on the same x_l.  The unit that completes a
//     group (a counter per group) sums the blocks in order, selects every
//     token of the group, quantizes the group's x_l rows into the two int8
//     parts of the expert kernels, starts L2 prefetches of the selected
//     experts of layer l and of the predicted ones of layer l+1, and counts
//     the group done.
//  B  tables.  Once every group is done, every CTA builds the bucket list,
//     slot assignment and task lists of layer l in its shared memory from the
//     selections (the same tables in every CTA), and prefetches its share of
//     layer l+1's shared expert and routers into L2.
//  C  gate/up tasks (bucket, 16-token chunk, 64 gate + 64 up rows), as the
//     TMA-ring gate/up kernel computes them; each task counts itself done in
//     its expert's counter.
//  D  down tasks (bucket, chunk, 512-wide slice, row group), as the TMA-ring
//     down kernel computes them, each once its expert's gate/up tasks are
//     all done; the CTA then counts itself done with the layer.
// After the last layer a final round of units combines the last layer.
//
// A producer warp feeds the consumers' weight ring with TMA tiles across task
// and layer boundaries: a CTA whose first gate/up task of a layer belongs to
// the shared expert issues that task's weights before the layer's routing is
// known.  Every wait is bounded (~2 s) and gives up when any CTA aborts (a
// global flag); a timeout records ST_TIMEOUT.  After an abort the producer
// still waits (bounded, abort-agnostic) for every copy it issued.
//
// The launch is cooperative (all CTAs resident), which the cross-CTA
// counters need.  The counters are zeroed by the host before every launch.
#include <cuda.h>

#include "moe_common.cuh"
#include "moe_fused.h"
#include "moe_tc.h"
#include "stream_ops.cuh"

namespace moe {
namespace fused {

constexpr int kThreads = 288;  // 8 consumer warps + the producer warp
constexpr int kStages = 6;     // weight ring stages of 16 KB
constexpr int kChunk = kChunkTokens;
constexpr int kGroupTok = 8;
constexpr int kColBlk = 128;
constexpr int kMaxTasks = 32;  // task descriptors kept per kind; the rest are decoded on the fly
constexpr int kTab = kMaxE + 2;
constexpr int kMaxSlots = kDecodeMaxTokens * kMaxK;
constexpr int kXBytes = 2 * kChunk * kTmaXStride;  // activation rows of a gate/up stage
constexpr int kStride2 = kSliceK + kPadB;          // quantized h row of a down task
constexpr int kXs2Bytes = 2 * kChunk * kStride2;
constexpr int kRawBytes = kChunk * kSliceK * 4;    // f32 h slice of a down task
constexpr int kRsBytes = kMaxRows2 * 4;            // row scales of a down task
constexpr long long kDrainCycles = 200000000LL;

// Scratch of phase A inside the h staging area of the down tasks: the staged
// x block of a router unit, and the summed logits of a token group (this
// layer's and the lookahead's).
constexpr int kScrXb = 0;
constexpr int kScrLog = kScrXb + kGroupTok * kColBlk * 4;
constexpr int kScrEnd = kScrLog + 2 * kGroupTok * kMaxE * 4;
static_assert(kScrEnd <= kRawBytes, "phase A/B scratch fits the h staging");

struct TaskD {
    int e, n, off, rbk, sl, tok0, nc;  // e < 0: none; e == E: the shared expert
};

struct Sh {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tready;  // consumers -> producer: the layer's tables are built
    uint64_t pdone;   // producer -> consumers: every stage of the layer is issued
    int abort;        // this CTA gives up (volatile access)
    int never;        // nothing sets it (MOE_TEST_STALL)
    int bcast;        // thread 0 -> consumers: outcome of a counter wait
    int last;         // thread 0 -> consumers: this unit completed its token group
    int nb, ntask13, ntask2, my13, my2;
    int be[kTab], bn[kTab], boff[kTab], ts13[kTab], ts2[kTab];
    short slot_of[kMaxSlots];
    short tok_of_slot[kMaxSlots];
    float wts[kMaxSlots];
    int cnt[kMaxE];
    int off[kMaxE];
    TaskD td13[kMaxTasks], td2[kMaxTasks];
    float hm[2][8][kChunk];
    alignas(16) float hmr[kChunk][kSliceK / kTaskRows13];
    float xsc[kChunk];
    QScale qs[kChunk];
    float bias[2][kMaxE];  // router bias of layer l and l + 1 (router units)
    alignas(8) uint8_t cnt8[kMaxSlots / 32][kMaxE];  // table build: picks of each expert per 32-pick chunk
};

constexpr size_t kSmem = ((sizeof(Sh) + 1023) & ~size_t(1023)) + 1024 /* alignment slack */ +
                         (size_t)kStages * (kTmaWBytes + kXBytes) + kXs2Bytes + kRawBytes + kRsBytes;
static_assert(kSmem <= 227 * 1024, "fused decode shared memory");

__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// MOE_TRACE: thread 0 of the consumers stamps event `slot` of layer l.
__device__ __forceinline__ void stamp(const FArgs& a, int l, int slot, bool when = true) {
    if (a.trace && when && threadIdx.x == 0) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        a.trace[((size_t)blockIdx.x * (a.L + 1) + l) * kTraceSlots + slot] = t;
    }
}

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Bounded wait of thread 0 for *ctr >= target.  Gives up when the global
// abort flag is set; a timeout sets it and records ST_TIMEOUT.
__device__ bool wait_count(const FArgs& a, const int* ctr, int target) {
    if (ld_acquire(ctr) >= target) return true;
    const long long t0 = clock64();
    while (ld_acquire(ctr) < target) {
        if (*reinterpret_cast<volatile int*>(a.abort)) return false;
        if (clock64() - t0 > kBulkWaitCycles) {
            atomicOr(a.status, ST_TIMEOUT);
            atomicExch(a.abort, 1);
            return false;
        }
    }
    return true;
}

// One more round of a bounded wait that began at t0 (it: rounds so far)?
// False once this CTA aborts, the global abort flag is seen (read every 64
// rounds: it lives in L2) or the limit runs out (recorded as ST_TIMEOUT).
__device__ __forceinline__ bool keep_waiting(const FArgs& a, const Sh& sh, long long t0, int& it) {
    if (*reinterpret_cast<const volatile int*>(&sh.abort)) return false;
    if ((++it & 63) == 0) {
        if (*reinterpret_cast<const volatile int*>(a.abort)) return false;
        if (clock64() - t0 > kBulkWaitCycles) {
            atomicOr(a.status, ST_TIMEOUT);
            atomicExch(a.abort, 1);
            return false;
        }
    }
    return true;
}

// Pipeline wait of the fused kernel (an mbarrier phase); false on abort or timeout.
__device__ __forceinline__ bool ring_wait(const FArgs& a, Sh& sh, uint64_t* bar, uint32_t parity) {
    if (bar_try(bar, parity)) return true;
    const long long t0 = clock64();
    int it = 0;
    while (!bar_try(bar, parity))
        if (!keep_waiting(a, sh, t0, it)) return false;
    return true;
}

// This CTA gave up (its own flag; the global one is seen by the waits).
__device__ __forceinline__ bool aborted(const Sh& sh) { return *reinterpret_cast<const volatile int*>(&sh.abort); }

// ---------------------------------------------------------------------------
// Selection (one warp per token): lane l holds the logits of experts l + 32 j.
// key = sigmoid(L) + bias (NaN -> -inf), K rounds of a warp arg-max (ties to
// the lower index); the k-th pick's weight is scale * s_k / (s_0 + ... +
// s_{K-1}), the sum taken in pick order.  Lanes k < K return pick k.
__device__ __forceinline__ void select_warp(const float (&L)[kMaxE / 32], const float* bias, int E, int K, float scale,
                                            float topp, int lane, int& my_e, float& my_w) {
    float key[kMaxE / 32], sc[kMaxE / 32];
#pragma unroll
    for (int j = 0; j < kMaxE / 32; ++j) {
        const int e = lane + 32 * j;
        key[j] = -INFINITY;
        sc[j] = 0.f;
        if (e < E) {
            const float s = 1.0f / (1.0f + expf(-L[j]));
            const float kk = s + bias[e];
            key[j] = isnan(kk) ? -INFINITY : kk;
            sc[j] = s;
        }
    }
    unsigned taken = 0;
    my_e = -1;
    float my_s = 0.f, ssum = 0.f;
#pragma unroll 1
    for (int k = 0; k < K; ++k) {
        float bk = -INFINITY, bs = 0.f;
        int be = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < kMaxE / 32; ++j) {
            const int e = lane + 32 * j;
            if (e < E && !((taken >> j) & 1u) && (key[j] > bk || (key[j] == bk && e < be))) {
                bk = key[j]; be = e; bs = sc[j];
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            const float os = __shfl_xor_sync(0xffffffffu, bs, o);
            if (ok > bk || (ok == bk && oe < be)) { bk = ok; be = oe; bs = os; }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == k) { my_e = be; my_s = bs; }
        ssum += bs;
    }
    const int e_k = my_e;
    topp_picks(K, topp, scale, lane, e_k, my_s, ssum, my_e, my_w);
}

// Logits of the group's tokens t0 .. t0+nt-1 (all 256 consumer threads):
// dst[tt * kMaxE + e] = the partial logits of (t0 + tt, e) summed over the
// hidden blocks, block 0 first; with `look`, the lookahead's too, into
// dst[(kGroupTok + tt) * kMaxE + e].  Loads are issued eight blocks at a time,
// both routers' together.
__device__ __forceinline__ void sum_logits(const FArgs& a, int t0, int nt, bool look, float* dst) {
    const int n = nt * a.E;
    const size_t step = (size_t)a.T * a.E;
    for (int i = threadIdx.x; i < n; i += 256) {
        const int tt = i / a.E, e = i - tt * a.E;
        const float* src = a.lp + (size_t)(t0 + tt) * a.E + e;
        const float* srn = a.lpn + (size_t)(t0 + tt) * a.E + e;
        float acc = 0.f, acn = 0.f;
        int cb = 0;
        for (; cb + 8 <= a.NCB; cb += 8) {
            float v[8], w[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                v[u] = __ldcg(src + (cb + u) * step);
                w[u] = look ? __ldcg(srn + (cb + u) * step) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                acc += v[u];
                acn += w[u];
            }
        }
        for (; cb < a.NCB; ++cb) {
            acc += __ldcg(src + cb * step);
            if (look) acn += __ldcg(srn + cb * step);
        }
        dst[tt * kMaxE + e] = acc;
        if (look) dst[(kGroupTok + tt) * kMaxE + e] = acn;
    }
}

// x_l of token t as the input of layer l (the stack's input, or layer l-1's output).
__device__ __forceinline__ const __nv_bfloat16* layer_input(const FArgs& a, int l) {
    return l == 0 ? a.x : a.outs + (size_t)(l - 1) * a.T * a.H;
}

// Writes xq (both int8 parts) and xs of token t (one warp) from x_l.
__device__ void quantize_token(const FArgs& a, int l, int t, int lane) {
    const uint4* xr = reinterpret_cast<const uint4*>(layer_input(a, l) + (size_t)t * a.H);
    const int ng = a.H / 8;
    constexpr int kRegGroups = 8;  // rows up to 32 * 8 * 8 = 2048 elements stay in registers
    if (ng <= 32 * kRegGroups) {
        uint4 v[kRegGroups];
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < kRegGroups; ++i) {
            const int gi = lane + 32 * i;
            v[i] = gi < ng ? __ldcg(xr + gi) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < kRegGroups; ++i) {
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) m = nanmax(nanmax(m, fabsf(bf16lo(w[k]))), fabsf(bf16hi(w[k])));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = nanmax(m, __shfl_xor_sync(0xffffffffu, m, o));
        const QScale qs = qscale(m);
        uint2* q0 = reinterpret_cast<uint2*>(a.xq + (size_t)t * 2 * a.H);
        uint2* q1 = reinterpret_cast<uint2*>(a.xq + (size_t)t * 2 * a.H + a.H);
#pragma unroll
        for (int i = 0; i < kRegGroups; ++i) {
            const int gi = lane + 32 * i;
            if (gi >= ng) break;
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
            float f[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                f[2 * k] = bf16lo(w[k]);
                f[2 * k + 1] = bf16hi(w[k]);
            }
            uint2 p0, p1;
            quant2x8(f, qs, p0, p1);
            q0[gi] = p0;
            q1[gi] = p1;
        }
        if (lane == 0) a.xs[t] = qs.s;
        return;
    }
    float m = 0.f;
#pragma unroll 4
    for (int gi = lane; gi < ng; gi += 32) {
        const uint4 v = __ldcg(xr + gi);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) m = nanmax(nanmax(m, fabsf(bf16lo(w[i]))), fabsf(bf16hi(w[i])));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = nanmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    const QScale qs = qscale(m);
    uint2* q0 = reinterpret_cast<uint2*>(a.xq + (size_t)t * 2 * a.H);
    uint2* q1 = reinterpret_cast<uint2*>(a.xq + (size_t)t * 2 * a.H + a.H);
#pragma unroll 4
    for (int gi = lane; gi < ng; gi += 32) {
        const uint4 v = __ldcg(xr + gi);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        float f[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = bf16lo(w[i]);
            f[2 * i + 1] = bf16hi(w[i]);
        }
        uint2 p0, p1;
        quant2x8(f, qs, p0, p1);
        q0[gi] = p0;
        q1[gi] = p1;
    }
    if (lane == 0) a.xs[t] = qs.s;
}

// ---------------------------------------------------------------------------
// Router unit: partial logits of a block of 128 hidden columns for the
// group's tokens.  Thread (expert e = 64 b + tid / 4, quarter q = tid % 4)
// accumulates, for each token, the columns 16 i + 4 q .. 16 i + 4 q + 3 for
// i = 0..7 in that order with fused multiply-adds (the four quarters read
// neighbouring 16-byte chunks of a staged row: no bank conflict); the four
// quarters are then summed by an xor-butterfly (1, 2).  A job is (router,
// block b of 64 experts): this thread's 32 router weights of it.  A token's
// logit never depends on the other tokens of the batch.
struct WRow {
    float4 w[kColBlk / 4 / 4];
};

// Coherent (L2) loads, so that the compiler keeps them where they are: they
// are issued before the unit waits for the previous layer.
__device__ __forceinline__ void load_wrow(const FArgs& a, int layer, int eb, int col0, WRow& f) {
    const int e = eb * 64 + (threadIdx.x >> 2), q = threadIdx.x & 3;
    const float4* src = reinterpret_cast<const float4*>(a.rw + ((size_t)layer * a.E + min(e, a.E - 1)) * a.H + col0) + q;
#pragma unroll
    for (int i = 0; i < kColBlk / 16; ++i) f.w[i] = __ldcg(src + 4 * i);
}

// xf: the staged block, [kGroupTok][kColBlk] f32.
__device__ __forceinline__ void router_job(const FArgs& a, const float* xf, const WRow& f, int eb, int cb, int t0,
                                           int nt, float* part) {
    const int e = eb * 64 + (threadIdx.x >> 2), q = threadIdx.x & 3;
    float acc[kGroupTok];
#pragma unroll
    for (int t = 0; t < kGroupTok; ++t) acc[t] = 0.f;
#pragma unroll 1
    for (int i = 0; i < kColBlk / 16; ++i) {
#pragma unroll
        for (int t = 0; t < kGroupTok; ++t) {
            const float4 xv = *reinterpret_cast<const float4*>(xf + t * kColBlk + 16 * i + 4 * q);
            acc[t] = fmaf(xv.x, f.w[i].x, acc[t]);
            acc[t] = fmaf(xv.y, f.w[i].y, acc[t]);
            acc[t] = fmaf(xv.z, f.w[i].z, acc[t]);
            acc[t] = fmaf(xv.w, f.w[i].w, acc[t]);
        }
    }
#pragma unroll
    for (int t = 0; t < kGroupTok; ++t) {
        acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 1);
        acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 2);
    }
    // lane quarter q stores tokens q and q + 4
    if (e < a.E) {
#pragma unroll
        for (int t = 0; t < kGroupTok; ++t)
            if ((t & 3) == q && t < nt) part[((size_t)cb * a.T + t0 + t) * a.E + e] = acc[t];
    }
}

// Layer l-1's combined output (+ residual) of tokens t0..t0+nt-1 and columns
// col0..col0+127 (thread: token warp, 4 columns of lane) -> outs[l-1] and the
// staged router block.  Same order and rounding as the combine kernel: each
// routed pick's slices summed in ascending order, times its weight (fma, k
// ascending), then the shared expert's slices, then the residual, rounded
// once.
__device__ __forceinline__ void combine_block(const FArgs& a, const Sh& sh, int l, int t0, int nt, int col0,
                                              float* xf) {
    const int t = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (t >= nt) return;
    const int tok = t0 + t, j = col0 + 4 * lane;
    const size_t H = a.H, TK = (size_t)a.T * a.K;
    uint2 xv;
    if (l == 0) {
        xv = __ldg(reinterpret_cast<const uint2*>(a.x + (size_t)tok * H + j));
    } else {
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        for (int k = 0; k < a.K; ++k) {
            const int s = sh.slot_of[tok * a.K + k];
            if (s < 0) continue;  // a pick the top-p dropped
            const float w = sh.wts[tok * a.K + k];
            float4 v = __ldcg(reinterpret_cast<const float4*>(a.y + (size_t)s * H + j));
            for (int sl = 1; sl < a.nsl_r; ++sl) {
                const float4 u = __ldcg(reinterpret_cast<const float4*>(a.y + (sl * TK + s) * H + j));
                v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
            }
            a0 = fmaf(w, v.x, a0);
            a1 = fmaf(w, v.y, a1);
            a2 = fmaf(w, v.z, a2);
            a3 = fmaf(w, v.w, a3);
        }
        if (a.Is > 0) {
            const float* ys = a.y + TK * a.nsl_r * H;
            float4 v = __ldcg(reinterpret_cast<const float4*>(ys + (size_t)tok * H + j));
            for (int sl = 1; sl < a.nsl_s; ++sl) {
                const float4 u = __ldcg(reinterpret_cast<const float4*>(ys + ((size_t)sl * a.T + tok) * H + j));
                v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
            }
            a0 += v.x; a1 += v.y; a2 += v.z; a3 += v.w;
        }
        if (a.flags & kFlagResidual) {
            const uint2 pv = __ldcg(reinterpret_cast<const uint2*>(layer_input(a, l - 1) + (size_t)tok * H + j));
            a0 += bf16lo(pv.x); a1 += bf16hi(pv.x); a2 += bf16lo(pv.y); a3 += bf16hi(pv.y);
        }
        __nv_bfloat162 o01 = __floats2bfloat162_rn(a0, a1);
        __nv_bfloat162 o23 = __floats2bfloat162_rn(a2, a3);
        xv.x = *reinterpret_cast<uint32_t*>(&o01);
        xv.y = *reinterpret_cast<uint32_t*>(&o23);
        *reinterpret_cast<uint2*>(a.outs + ((size_t)(l - 1) * a.T + tok) * H + j) = xv;
    }
    if (xf)
        *reinterpret_cast<float4*>(xf + t * kColBlk + 4 * lane) =
            make_float4(bf16lo(xv.x), bf16hi(xv.x), bf16lo(xv.y), bf16hi(xv.y));
}

// ---------------------------------------------------------------------------
// Tables (consumers).  Bucket b < nb-1 (or < nb without a shared expert) is
// the b-th non-empty routed expert in ascending order; the shared expert is
// the last bucket.  Slots are expert-contiguous and in (t, k) order within an
// expert; the shared bucket's slots are T*K + t.
__device__ __forceinline__ int tasks13_of(const FArgs& a, int e, int n) {
    return (e == a.E ? a.r13_s : a.r13_r) * chunks_of(n, kChunk);
}

__device__ __forceinline__ int snake(int c, int r) {
    return (r & 1) ? (r + 1) * (int)gridDim.x - 1 - c : r * (int)gridDim.x + c;
}

// Task `lin` of the heaviest-first list of `kind` (0 gate/up, 1 down).
__device__ TaskD decode_task(const FArgs& a, const Sh& sh, int kind, int lin) {
    TaskD d;
    d.e = -1;
    d.n = d.off = d.rbk = d.sl = d.tok0 = d.nc = 0;
    const int ntask = kind == 0 ? sh.ntask13 : sh.ntask2;
    if (lin >= ntask) return d;
    const int task = ntask - 1 - lin;
    const int* ts = kind == 0 ? sh.ts13 : sh.ts2;
    int lo = 0, hi = sh.nb;  // ts[lo] <= task < ts[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (ts[mid] <= task) lo = mid; else hi = mid;
    }
    const int e = sh.be[lo], n = sh.bn[lo], local = task - ts[lo];
    const int irow = e == a.E ? a.Is : a.I;
    int c;
    if (kind == 0) {
        const int R = irow / kTaskRows13;
        c = local / R;
        d.rbk = local - c * R;
    } else {
        const int R = a.H / a.rows2, nsl = slices_of(irow);
        const int rest = local / R;
        d.rbk = local - rest * R;
        c = rest / nsl;
        d.sl = rest - c * nsl;
    }
    d.e = e;
    d.n = n;
    d.off = sh.boff[lo];
    d.tok0 = c * kChunk;
    d.nc = min(kChunk, n - d.tok0);
    return d;
}

__device__ __forceinline__ TaskD task_of(const FArgs& a, const Sh& sh, int kind, int r) {
    if (r < kMaxTasks) return kind == 0 ? sh.td13[r] : sh.td2[r];
    return decode_task(a, sh, kind, snake(blockIdx.x, r));
}

__device__ __forceinline__ int my_task_count(int ntask) {
    int r = 0;
    while (snake(blockIdx.x, r) < ntask) ++r;
    return r;
}

// Builds layer l's tables in shared memory from the selections (all 256
// consumer threads; the same result in every CTA).  cnt8: scratch of
// kMaxSlots / 32 x kMaxE bytes.
__device__ void build_tables(const FArgs& a, Sh& sh) {
    const int tid = threadIdx.x, lane = tid & 31;
    const int E = a.E, K = a.K, T = a.T, TK = T * K;
    constexpr int kChunks = kMaxSlots / 32;
    int my_e[2], my_rank[2];
    bool leader[2];
    // sh.cnt8 is all zero here (zeroed at the start, and after every use)
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int i = tid + 256 * u;
        int e = -1;
        if (i < TK) {
            e = __ldcg(a.idx + i);
            sh.wts[i] = __ldcg(a.wts + i);
            if (e == -1 && a.topp > 0.f && a.topp < 1.f) {
                // dropped by the top-p: no slot
            } else if (e < 0 || e >= E) {
                atomicOr(a.status, ST_BAD_EXPERT);
                e = -1;
            }
        }
        // picks of one warp are 32 consecutive (t, k): rank among equal experts
        const unsigned m = __match_any_sync(0xffffffffu, i < TK ? e : -2 - lane);
        my_e[u] = e;
        my_rank[u] = __popc(m & ((1u << lane) - 1u));
        leader[u] = e >= 0 && lane == __ffs(m) - 1;
        if (leader[u]) sh.cnt8[i >> 5][e] = (uint8_t)__popc(m);
    }
    consumers_sync();
    if (tid < 32) {
        // lane l owns experts 8l .. 8l+7: counts, buckets, gate/up and down tasks
        constexpr int kPer = kMaxE / 32;
        int c[kPer];
#pragma unroll
        for (int j = 0; j < kPer; ++j) c[j] = 0;
        for (int ch = 0; ch < (TK + 31) / 32; ++ch) {
            const uint2 w = *reinterpret_cast<const uint2*>(&sh.cnt8[ch][lane * kPer]);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                c[j] += (w.x >> (8 * j)) & 0xFF;
                c[4 + j] += (w.y >> (8 * j)) & 0xFF;
            }
        }
        int v[4] = {0, 0, 0, 0};
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int e = lane * kPer + j;
            if (e >= E) c[j] = 0;
            const int ch = (c[j] + kChunk - 1) / kChunk;
            v[0] += c[j];
            v[1] += c[j] > 0;
            v[2] += a.r13_r * ch;
            v[3] += a.r2_r * ch;
        }
        int inc[4] = {v[0], v[1], v[2], v[3]};
#pragma unroll
        for (int o = 1; o < 32; o <<= 1)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int s = __shfl_up_sync(0xffffffffu, inc[i], o);
                if (lane >= o) inc[i] += s;
            }
        int off = inc[0] - v[0], b = inc[1] - v[1], b13 = inc[2] - v[2], b2 = inc[3] - v[3];
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int e = lane * kPer + j;
            if (e < E) {
                sh.off[e] = off;
                if (c[j] > 0) {
                    const int ch = (c[j] + kChunk - 1) / kChunk;
                    sh.be[b] = e;
                    sh.bn[b] = c[j];
                    sh.boff[b] = off;
                    sh.ts13[b] = b13;
                    sh.ts2[b] = b2;
                    ++b;
                    b13 += a.r13_r * ch;
                    b2 += a.r2_r * ch;
                }
                off += c[j];
            }
        }
        const int total = __shfl_sync(0xffffffffu, inc[0], 31);
        int nb = __shfl_sync(0xffffffffu, inc[1], 31);
        int t13 = __shfl_sync(0xffffffffu, inc[2], 31), t2 = __shfl_sync(0xffffffffu, inc[3], 31);
        if (lane == 0) {
            const bool topp = a.topp > 0.f && a.topp < 1.f;  // dropped picks: fewer slots than T*K
            if (total != TK && !(topp && total < TK)) {  // inconsistent selections: flag them and run no routed task
                atomicOr(a.status, ST_BAD_COUNT);
                nb = t13 = t2 = 0;
            }
            if (a.Is > 0) {
                const int ch = (T + kChunk - 1) / kChunk;
                sh.be[nb] = E;
                sh.bn[nb] = T;
                sh.boff[nb] = TK;
                sh.ts13[nb] = t13;
                sh.ts2[nb] = t2;
                t13 += a.r13_s * ch;
                t2 += a.r2_s * ch;
                ++nb;
            }
            sh.ts13[nb] = t13;
            sh.ts2[nb] = t2;
            sh.nb = nb;
            sh.ntask13 = t13;
            sh.ntask2 = t2;
        }
    }
    consumers_sync();
    // slots; this CTA's task count and first task descriptors
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int i = tid + 256 * u;
        if (i >= TK) continue;
        const int e = my_e[u];
        int slot = -1;
        if (e >= 0) {
            int base = 0;
            for (int ch = 0; ch < (i >> 5); ++ch) base += sh.cnt8[ch][e];
            slot = sh.off[e] + base + my_rank[u];
        }
        if (slot < 0 || slot >= TK) {
            if (e >= 0) atomicOr(a.status, ST_BAD_SLOT);
            sh.slot_of[i] = e == -1 && a.topp > 0.f && a.topp < 1.f ? -1 : 0;
        } else {
            sh.slot_of[i] = (short)slot;
            sh.tok_of_slot[slot] = (short)(i / K);
        }
    }
    if (tid == 0) {
        sh.my13 = my_task_count(sh.ntask13);
        sh.my2 = my_task_count(sh.ntask2);
    }
    if (tid >= 64 && tid < 64 + kMaxTasks) sh.td13[tid - 64] = decode_task(a, sh, 0, snake(blockIdx.x, tid - 64));
    else if (tid >= 64 + kMaxTasks && tid < 64 + 2 * kMaxTasks)
        sh.td2[tid - 64 - kMaxTasks] = decode_task(a, sh, 1, snake(blockIdx.x, tid - 64 - kMaxTasks));
    consumers_sync();
    // back to zero for the next layer (only the leaders' entries are set)
#pragma unroll
    for (int u = 0; u < 2; ++u)
        if (leader[u]) sh.cnt8[(tid + 256 * u) >> 5][my_e[u]] = 0;
}

// ---------------------------------------------------------------------------
// Consumer main loops (as the TMA-ring kernels).
template <int NT>
__device__ __forceinline__ void consume13(const FArgs& a, Sh& sh, int nch, uint32_t& n, const uint8_t* wring,
                                          const uint8_t* xring, int (&acc)[4][4]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, q = lane & 3;
    constexpr int kSets = NT == 1 ? 2 : 1;
    int part[kSets][NT][4];
#pragma unroll
    for (int s = 0; s < kSets; ++s)
#pragma unroll
        for (int i = 0; i < NT; ++i) part[s][i][0] = part[s][i][1] = part[s][i][2] = part[s][i][3] = 0;
    const int wrow = (warp * 8 + g) * kTmaRowBytes;
    volatile int* abort = &sh.abort;
    for (int c = 0; c < nch; ++c, ++n) {
        const int s = n % kStages;
        if (!*abort && !ring_wait(a, sh, &sh.full[s], (n / kStages) & 1)) *abort = 1;
        const uint8_t* wt = wring + (size_t)s * kTmaWBytes + wrow;
        const uint8_t* xt = xring + (size_t)s * kXBytes + g * kTmaXStride + q * 32;
#pragma unroll
        for (int kb = 0; kb < kTmaChunk / 128; ++kb) {
            const int off = ((kb * 4 + q) ^ g) << 4;
            const uint4 wa = *reinterpret_cast<const uint4*>(wt + off);
            const uint4 wb = *reinterpret_cast<const uint4*>(wt + kTmaWBytes / 2 + off);
            kblock8<NT, kSets>(wa, wb, xt + kb * 128, 8 * kTmaXStride, part);
        }
        __syncwarp();
        if (lane == 0) bar_arrive(&sh.empty[s]);
    }
#pragma unroll
    for (int i = 0; i < NT; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][c] = part[0][i][c] + part[kSets - 1][i][c] * (kSets - 1);
}

template <int NT>
__device__ __forceinline__ void consume2(const FArgs& a, Sh& sh, const TaskD& d, int l, uint32_t& n,
                                         const uint8_t* wring, const uint8_t* xs2, const float* rs) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, q = lane & 3;
    constexpr int kSets = NT == 1 ? 2 : 1;
    const bool shd = d.e == a.E;
    const int irow = shd ? a.Is : a.I;
    const size_t TK = (size_t)a.T * a.K;
    const size_t yrow0 = shd ? TK * a.nsl_r + (size_t)d.sl * a.T + d.tok0 : (size_t)d.sl * TK + d.off + d.tok0;
    const int klen = min(kSliceK, irow - d.sl * kSliceK);
    const int nkc = klen / kTmaChunk, ng = a.rows2 / kTaskRows2;
    const int row0 = d.rbk * a.rows2;
    const int wa_row = (warp * 16 + g) * kTmaRowBytes, wb_row = wa_row + 8 * kTmaRowBytes;
    volatile int* abort = &sh.abort;
    for (int m = 0; m < ng; ++m) {
        int part[kSets][NT][4];
#pragma unroll
        for (int s = 0; s < kSets; ++s)
#pragma unroll
            for (int i = 0; i < NT; ++i) part[s][i][0] = part[s][i][1] = part[s][i][2] = part[s][i][3] = 0;
        for (int c = 0; c < nkc; ++c, ++n) {
            const int s = n % kStages;
            if (!*abort && !ring_wait(a, sh, &sh.full[s], (n / kStages) & 1)) *abort = 1;
            const uint8_t* wt = wring + (size_t)s * kTmaWBytes;
            const uint8_t* xt = xs2 + g * kStride2 + q * 32 + c * kTmaChunk;
#pragma unroll
            for (int kb = 0; kb < kTmaChunk / 128; ++kb) {
                const int off = ((kb * 4 + q) ^ g) << 4;
                const uint4 wa = *reinterpret_cast<const uint4*>(wt + wa_row + off);
                const uint4 wb = *reinterpret_cast<const uint4*>(wt + wb_row + off);
                kblock8<NT, kSets>(wa, wb, xt + kb * 128, 8 * kStride2, part);
            }
            __syncwarp();
            if (lane == 0) bar_arrive(&sh.empty[s]);
        }
        const int jr = m * kTaskRows2 + warp * 16 + g;
        const float s_lo = rs[jr], s_hi = rs[jr + 8];
        float* y0 = a.y + yrow0 * a.H + row0 + jr;
#pragma unroll
        for (int i = 0; i < NT; ++i) {
            const int j = 4 * i + q;
            if (j < d.nc) {
                const int a0 = part[0][i][0] + part[kSets - 1][i][0] * (kSets - 1);
                const int a1 = part[0][i][1] + part[kSets - 1][i][1] * (kSets - 1);
                const int a2 = part[0][i][2] + part[kSets - 1][i][2] * (kSets - 1);
                const int a3 = part[0][i][3] + part[kSets - 1][i][3] * (kSets - 1);
                const float xsc = sh.xsc[j];
                float* yr = y0 + (size_t)j * a.H;
                yr[0] = join(a0, a1) * (s_lo * xsc);
                yr[8] = join(a2, a3) * (s_hi * xsc);
            }
        }
    }
}

__device__ __forceinline__ bool task_ok(const FArgs& a, const TaskD& d) {
    return d.e >= 0 && d.e <= a.E && !(d.e == a.E && a.Is == 0) && d.nc > 0;
}

// L2 prefetch by the producer warp (bulk prefetches through the CTA's copy
// engine, lanes in parallel), every CTA its 1/grid share of each region: what
// layer `n1` reads first -- the experts its router picked when run on the
// previous layer's input (the lookahead), its shared expert and router, and
// the router after it (which the next lookahead reads).
__device__ __forceinline__ void prefetch_bulk_share(const void* p, size_t n) {
    const size_t per = ((n + gridDim.x - 1) / gridDim.x + 15) & ~size_t(15);
    const size_t o = (size_t)blockIdx.x * per;
    if (o >= n) return;
    const size_t len = n - o < per ? n - o : per;
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(static_cast<const char*>(p) + o), "r"((uint32_t)len)
                 : "memory");
}

__device__ void prefetch_layer(const FArgs& a, int n1, bool experts, int lane) {
    if (!(a.flags & kFlagLookahead) || n1 >= a.L) return;
    if (experts) {
        unsigned pred[kMaxE / 32];
#pragma unroll
        for (int w = 0; w < kMaxE / 32; ++w) pred[w] = __ldcg(a.pred_bits + n1 * 8 + w);
        // lane j takes the j-th, (j+32)-th, ... predicted expert
        int k = 0;
#pragma unroll
        for (int w = 0; w < kMaxE / 32; ++w) {
            unsigned bits = pred[w];
            while (bits) {
                const int e = 32 * w + __ffs(bits) - 1;
                bits &= bits - 1;
                if ((k++ & 31) == lane) {
                    const size_t le = (size_t)n1 * a.E + e;
                    prefetch_bulk_share(a.w13 + le * (size_t)a.I * a.H, (size_t)a.I * a.H);
                    prefetch_bulk_share(a.w2 + le * (size_t)a.H * (a.I / 2), (size_t)a.H * (a.I / 2));
                    prefetch_bulk_share(a.s13 + le * 2 * a.I, (size_t)2 * a.I * 4);
                    prefetch_bulk_share(a.s2 + le * a.H, (size_t)a.H * 4);
                }
            }
        }
    }
    if (a.Is > 0) {
        if (lane == 0) prefetch_bulk_share(a.sh_w13 + (size_t)n1 * a.Is * a.H, (size_t)a.Is * a.H);
        if (lane == 1) prefetch_bulk_share(a.sh_w2 + (size_t)n1 * a.H * (a.Is / 2), (size_t)a.H * (a.Is / 2));
        if (lane == 2) prefetch_bulk_share(a.sh_s13 + (size_t)n1 * 2 * a.Is, (size_t)2 * a.Is * 4);
        if (lane == 3) prefetch_bulk_share(a.sh_s2 + (size_t)n1 * a.H, (size_t)a.H * 4);
    }
    if (lane == 4) prefetch_bulk_share(a.rw + (size_t)n1 * a.E * a.H, (size_t)a.E * a.H * 4);
    if (lane == 5 && n1 + 1 < a.L) prefetch_bulk_share(a.rw + (size_t)(n1 + 1) * a.E * a.H, (size_t)a.E * a.H * 4);
}

// ---------------------------------------------------------------------------
// Producer warp.
__device__ void producer(const FArgs& a, Sh& sh, uint8_t* wring, uint8_t* xring, const CUtensorMap* tm13,
                         const CUtensorMap* tms13, const CUtensorMap* tm2, const CUtensorMap* tms2) {
    const int lane = threadIdx.x & 31;
    const int H = a.H, nch = H / kTmaChunk;
    volatile int* abort = &sh.abort;
    uint32_t n = 0;
    int last_round[kStages];
    bool act_missing[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) last_round[s] = -1, act_missing[s] = false;
    if (lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm13)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tms13)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm2)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tms2)) : "memory");
    }
    const int Rs = a.Is / kTaskRows13;
    const int ns = a.Is > 0 ? Rs * chunks_of(a.T, kChunk) : 0;
    bool ok = true;
    prefetch_layer(a, 0, false, lane);
    // next free stage: waits for its slot (round > 0); false on abort / timeout
    auto acquire = [&](int& s, int& round) -> bool {
        s = (int)(n % kStages);
        round = (int)(n / kStages);
        if (round > 0 && !ring_wait(a, sh, &sh.empty[s], (round - 1) & 1)) return false;
        return true;
    };
    for (int l = 0; ok && l < a.L; ++l) {
        // (a) the first gate/up task of this CTA, when it belongs to the shared
        // expert, does not depend on the routing: issue its weights now
        const bool pre = (int)blockIdx.x < ns;
        int npre = 0, pre_rbk = 0, pre_tok0 = 0;
        const uint32_t n_pre0 = n;
        if (pre) {
            const int local = ns - 1 - (int)blockIdx.x;
            pre_rbk = local % Rs;
            pre_tok0 = (local / Rs) * kChunk;
            const int want = min(nch, kStages);
            const int rg = l * 2 * a.Is + pre_rbk * kTaskRows13;
            for (; npre < want; ++npre) {
                int s, round;
                if (!acquire(s, round)) { ok = false; break; }
                if (lane == 0) {
                    bar_expect_tx(&sh.full[s], kTmaWBytes);
                    tma_tile(wring + (size_t)s * kTmaWBytes, tms13, &sh.full[s], npre * kTmaRowBytes, rg);
                    tma_tile(wring + (size_t)s * kTmaWBytes + kTmaWBytes / 2, tms13, &sh.full[s], npre * kTmaRowBytes,
                             rg + a.Is);
                }
                last_round[s] = round;
                act_missing[s] = true;
                ++n;
            }
            if (!ok) break;
        }
        // the layer's predicted experts, shared expert and routers (MOE_LOOKAHEAD),
        // behind its first weights and ahead of its routing
        if (l > 0) prefetch_layer(a, l, true, lane);
        // (b) the layer's tables
        const bool got = ring_wait(a, sh, &sh.tready, l & 1);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        const int my13 = sh.my13, my2 = sh.my2;
        // (c) gate/up tasks: weights (TMA) and the tokens' activation rows
        for (int r = 0; ok && r < my13; ++r) {
            const TaskD d = task_of(a, sh, 0, r);
            if (!task_ok(a, d) || (r == 0 && pre && !(d.e == a.E && d.rbk == pre_rbk && d.tok0 == pre_tok0))) {
                if (lane == 0) atomicOr(a.status, ST_BAD_TASK);
                ok = false;
                break;
            }
            const bool shd = d.e == a.E;
            const int irow = shd ? a.Is : a.I;
            const int rg = (shd ? l * 2 * a.Is : (l * a.E + d.e) * 2 * a.I) + d.rbk * kTaskRows13;
            const CUtensorMap* map = shd ? tms13 : tm13;
            // lane l copies activation row l (part l & 1 of the chunk's token l >> 1)
            const int8_t* src = nullptr;
            if (lane < 2 * d.nc) {
                const int tok = shd ? d.tok0 + (lane >> 1) : sh.tok_of_slot[d.off + d.tok0 + (lane >> 1)];
                if (tok >= 0 && tok < a.T) src = a.xq + (size_t)tok * 2 * H + (lane & 1) * H;
            }
            for (int c = 0; c < nch; ++c) {
                int s;
                if (r == 0 && c < npre) {
                    s = (int)((n_pre0 + c) % kStages);
                } else {
                    int round;
                    if (!acquire(s, round)) { ok = false; break; }
                    if (lane == 0) {
                        bar_expect_tx(&sh.full[s], kTmaWBytes);
                        tma_tile(wring + (size_t)s * kTmaWBytes, map, &sh.full[s], c * kTmaRowBytes, rg);
                        tma_tile(wring + (size_t)s * kTmaWBytes + kTmaWBytes / 2, map, &sh.full[s], c * kTmaRowBytes,
                                 rg + irow);
                    }
                    last_round[s] = round;
                    ++n;
                }
                if (src) {
                    uint8_t* dst = xring + (size_t)s * kXBytes + lane * kTmaXStride;
#pragma unroll
                    for (int j = 0; j < kTmaChunk / 16; ++j) cp_async16(dst + j * 16, src + c * kTmaChunk + j * 16);
                }
                cp_async_arrive(&sh.full[s]);
                act_missing[s] = false;
            }
        }
        if (!ok) break;
        // (d) down tasks: weights only
        for (int r = 0; ok && r < my2; ++r) {
            const TaskD d = task_of(a, sh, 1, r);
            if (!task_ok(a, d)) {
                if (lane == 0) atomicOr(a.status, ST_BAD_TASK);
                ok = false;
                break;
            }
            const bool shd = d.e == a.E;
            const int irow = shd ? a.Is : a.I;
            const int k0 = d.sl * kSliceK, nkc = min(kSliceK, irow - k0) / kTmaChunk;
            const int row0 = (shd ? l * H : (l * a.E + d.e) * H) + d.rbk * a.rows2;
            const CUtensorMap* map = shd ? tms2 : tm2;
            const int ng = a.rows2 / kTaskRows2;
            for (int m = 0; ok && m < ng; ++m)
                for (int c = 0; c < nkc; ++c) {
                    int s, round;
                    if (!acquire(s, round)) { ok = false; break; }
                    if (lane == 0) {
                        bar_expect_tx(&sh.full[s], kW2Bytes);
                        tma_tile(wring + (size_t)s * kTmaWBytes, map, &sh.full[s], (k0 + c * kTmaChunk) / 2,
                                 row0 + m * kTaskRows2);
                    }
                    bar_arrive(&sh.full[s]);
                    last_round[s] = round;
                    ++n;
                }
        }
        __syncwarp();
        if (ok && lane == 0) bar_arrive(&sh.pdone);
    }
    if (!ok) *abort = 1;
    // Before the CTA exits, every copy issued into the ring has landed (waits
    // that ignore the abort, bounded).  Stages whose weights were issued early
    // but never got their activations first get their arrivals.  After a
    // normal run every stage was consumed and these waits return at once.
#pragma unroll
    for (int s = 0; s < kStages; ++s)
        if (act_missing[s]) cp_async_arrive(&sh.full[s]);
#pragma unroll
    for (int s = 0; s < kStages; ++s)
        if (last_round[s] >= 0) bar_wait(&sh.full[s], last_round[s] & 1, kDrainCycles);
    cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// Consumers.
struct Smem {
    uint8_t* wring;
    uint8_t* xring;
    uint8_t* xs2;
    float* raw;
    float* rs;
};

// Phase A of layer l (l == L: the final combine only).  False on abort.
__device__ bool phase_units(const FArgs& a, Sh& sh, const Smem& m, int l) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = a.G, U = G * a.NCB;
    const int first = (int)gridDim.x - 1 - (int)blockIdx.x;
    stamp(a, l, 0);
    if (first >= U) {
        stamp(a, l, 2);
        return true;
    }
    const bool final = l == a.L;
    const bool look = !final && l + 1 < a.L && (a.flags & kFlagLookahead);
    float* xf = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(m.raw) + kScrXb);
    const int per = (a.E + 63) / 64;  // expert blocks per router
    const int jobs = final ? 0 : per * (look ? 2 : 1);
    // job k: router k / per (0 = layer l, 1 = layer l + 1), expert block k % per
    WRow wr[2];
    auto load_job = [&](int k, int col0, WRow& f) {
        if (k < jobs) load_wrow(a, l + k / per, k % per, col0, f);
    };
    // nothing of this depends on the wait below: the first unit's first two
    // jobs' router weights, and the routers' biases
    load_job(0, (first % a.NCB) * kColBlk, wr[0]);
    load_job(1, (first % a.NCB) * kColBlk, wr[1]);
    if (!final)
        for (int i = tid; i < 2 * a.E; i += 256) {
            const int r = i / a.E, e = i - r * a.E;
            if (r == 0 || look) sh.bias[r][e] = __ldcg(a.rb + (size_t)(l + r) * a.E + e);
        }
    if (l > 0) {
        if (tid == 0) sh.bcast = wait_count(a, a.down_done + (l - 1), (int)gridDim.x);
        consumers_sync();
        if (!sh.bcast) return false;
    }
    stamp(a, l, 1);
    for (int u = first; u < U; u += gridDim.x) {
        const int g = u / a.NCB, cb = u - g * a.NCB;
        const int t0 = g * kGroupTok, nt = min(kGroupTok, a.T - t0), col0 = cb * kColBlk;
        if (u != first) {
            consumers_sync();  // the previous unit is done with xf
            load_job(0, col0, wr[0]);
            load_job(1, col0, wr[1]);
        }
        combine_block(a, sh, l, t0, nt, col0, final ? nullptr : xf);
        if (final) continue;
        consumers_sync();  // xf staged
        stamp(a, l, 7, u == first);
        for (int k = 0; k < jobs; k += 2) {  // two jobs per round: wr is indexed statically
            router_job(a, xf, wr[0], k % per, cb, t0, nt, k / per == 0 ? a.lp : a.lpn);
            load_job(k + 2, col0, wr[0]);
            if (k + 1 < jobs) {
                router_job(a, xf, wr[1], (k + 1) % per, cb, t0, nt, (k + 1) / per == 0 ? a.lp : a.lpn);
                load_job(k + 3, col0, wr[1]);
            }
        }
        consumers_sync();  // every partial logit and output of the unit written
        stamp(a, l, 8, u == first);
        if (tid == 0) {
            __threadfence();  // this unit's writes before its count
            const int old = atomicAdd(a.grp_cnt + l * kMaxGroupsF + g, 1);
            __threadfence();  // the other units' writes after their counts
            sh.last = old == a.NCB - 1;
        }
        consumers_sync();
        stamp(a, l, 9, u == first);
        if (!sh.last) continue;
        // the last unit of group g: select its tokens and quantize their rows
        float* lg = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(m.raw) + kScrLog);
        sum_logits(a, t0, nt, look, lg);
        consumers_sync();
        if (warp < nt) {
            const int t = t0 + warp;
            float L[kMaxE / 32];
#pragma unroll
            for (int j = 0; j < kMaxE / 32; ++j) L[j] = lg[warp * kMaxE + lane + 32 * j];
            int e;
            float w;
            select_warp(L, sh.bias[0], a.E, a.K, a.scale, a.topp, lane, e, w);
            if ((a.flags & kFlagTestBadIndex) && t == 0 && lane == 0) e = a.E;  // test hook: an out-of-range pick
            if (lane < a.K) {
                const size_t o = (size_t)t * a.K + lane;
                a.idx[o] = e;
                a.wts[o] = w;
                if (a.topk_idx) a.topk_idx[(size_t)l * a.T * a.K + o] = e;
                if (a.topk_w) a.topk_w[(size_t)l * a.T * a.K + o] = w;
            }
            if (look) {
                // the next layer's router on this layer's input: the experts it
                // predicts are prefetched (by every CTA, its share) in the tables phase
#pragma unroll
                for (int j = 0; j < kMaxE / 32; ++j) L[j] = lg[(kGroupTok + warp) * kMaxE + lane + 32 * j];
                int pe;
                float pw;
                select_warp(L, sh.bias[1], a.E, a.K, a.scale, a.topp, lane, pe, pw);
                if (lane < a.K && pe >= 0 && pe < a.E) atomicOr(a.pred_bits + (l + 1) * 8 + (pe >> 5), 1u << (pe & 31));
            }
            if (warp == 0) stamp(a, l, 10);
            quantize_token(a, l, t, lane);
        }
        consumers_sync();
        stamp(a, l, 11);
        if (tid == 0) {
            __threadfence();
            atomicAdd(a.groups_done + l, 1);
        }
    }
    stamp(a, l, 2);
    return !aborted(sh);
}

// Phase B of layer l.  False on abort.
__device__ bool phase_tables(const FArgs& a, Sh& sh, const Smem& m, int l) {
    if (threadIdx.x == 0) {
        sh.bcast = wait_count(a, a.groups_done + l, a.G);
        // the producer has issued every stage of layer l-1 and reads the old
        // tables no more (this also keeps the two barriers' phases in step:
        // neither side gets a layer ahead of the other)
        if (sh.bcast && l > 0) sh.bcast = ring_wait(a, sh, &sh.pdone, (l - 1) & 1);
    }
    consumers_sync();
    if (!sh.bcast) return false;
    stamp(a, l, 3);
    build_tables(a, sh);
    if (threadIdx.x == 0) bar_arrive(&sh.tready);  // the producer may start
    stamp(a, l, 4);
    stamp(a, l, 12);
    return true;
}

// Phase C of layer l: this CTA's gate/up tasks.
__device__ bool phase_gate_up(const FArgs& a, Sh& sh, const Smem& m, int l, uint32_t& n) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, q = lane & 3;
    const int nch = a.H / kTmaChunk;
    for (int r = 0; r < sh.my13; ++r) {
        const TaskD d = task_of(a, sh, 0, r);
        if (!task_ok(a, d)) {
            if (tid == 0) atomicOr(a.status, ST_BAD_TASK);
            sh.abort = 1;
            return false;
        }
        const bool shd = d.e == a.E;
        const int irow = shd ? a.Is : a.I;
        const int r0 = d.rbk * kTaskRows13 + warp * 8;
        const float* S = shd ? a.sh_s13 + (size_t)l * 2 * a.Is : a.s13 + ((size_t)l * a.E + d.e) * 2 * a.I;
        const float gs = __ldg(S + r0 + g), us = __ldg(S + irow + r0 + g);
        const int NTt = (2 * d.nc + 7) >> 3;
        float xsc[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int j = 4 * i + q;
            xsc[i] = 0.f;
            if (i < NTt && j < d.nc) {
                const int tok = shd ? d.tok0 + j : sh.tok_of_slot[d.off + d.tok0 + j];
                xsc[i] = (tok >= 0 && tok < a.T) ? __ldcg(a.xs + tok) * 0.0625f : 0.f;
            }
        }
        int acc[4][4];
        if (r == 0 && a.trace) {  // MOE_TRACE: when the first stage lands
            ring_wait(a, sh, &sh.full[n % kStages], (n / kStages) & 1);
            stamp(a, l, 13);
        }
        switch (NTt) {
            case 1: consume13<1>(a, sh, nch, n, m.wring, m.xring, acc); break;
            case 2: consume13<2>(a, sh, nch, n, m.wring, m.xring, acc); break;
            case 3: consume13<3>(a, sh, nch, n, m.wring, m.xring, acc); break;
            default: consume13<4>(a, sh, nch, n, m.wring, m.xring, acc); break;
        }
        const int slot0 = (shd ? 0 : d.off) + d.tok0;
        float* hrow0 = (shd ? a.h32_s : a.h32_r) + (size_t)slot0 * irow + r0 + g;
        float(*hm)[kChunk] = sh.hm[r & 1];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (i >= NTt) break;
            const int j = 4 * i + q;
            float hmv = 0.f;
            if (j < d.nc) {
                const float gv = join(acc[i][0], acc[i][1]) * (gs * xsc[i]);
                const float uv = join(acc[i][2], acc[i][3]) * (us * xsc[i]);
                const float h = silu_mul(gv, uv);
                hrow0[(size_t)j * irow] = h;
                hmv = fabsf(h);
            }
            hmv = nanmax(hmv, __shfl_xor_sync(0xffffffffu, hmv, 4));
            hmv = nanmax(hmv, __shfl_xor_sync(0xffffffffu, hmv, 8));
            hmv = nanmax(hmv, __shfl_xor_sync(0xffffffffu, hmv, 16));
            if (g == 0 && j < d.nc) hm[warp][j] = hmv;
        }
        consumers_sync();  // h rows and the warps' maxima are written
        if (tid == 0) {
            const int nrb = irow / kTaskRows13;
            float* hmax = shd ? a.hmax_s : a.hmax_r;
            for (int j = 0; j < d.nc; ++j) {
                float mx = 0.f;
#pragma unroll
                for (int w = 0; w < 8; ++w) mx = nanmax(mx, hm[w][j]);
                hmax[(size_t)(slot0 + j) * nrb + d.rbk] = mx;
            }
            __threadfence();
            atomicAdd(a.ready + l * (kMaxE + 1) + d.e, 1);
        }
        if (aborted(sh)) return false;
    }
    stamp(a, l, 5);
    return true;
}

// Phase D of layer l: this CTA's down tasks; then the CTA counts itself done.
__device__ bool phase_down(const FArgs& a, Sh& sh, const Smem& m, int l, uint32_t& n) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int r = 0; r < sh.my2; ++r) {
        const TaskD d = task_of(a, sh, 1, r);
        if (!task_ok(a, d)) {
            if (tid == 0) atomicOr(a.status, ST_BAD_TASK);
            sh.abort = 1;
            return false;
        }
        const bool shd = d.e == a.E;
        const int irow = shd ? a.Is : a.I;
        const int k0 = d.sl * kSliceK, klen = min(kSliceK, irow - k0);
        // every gate/up task of the expert is done
        if (tid == 0) sh.bcast = wait_count(a, a.ready + l * (kMaxE + 1) + d.e, tasks13_of(a, d.e, d.n));
        consumers_sync();
        if (!sh.bcast) return false;
        stamp(a, l, 14, r == 0);
        // the slice of h, its per-64-row maxima and the task's row scales
        const float* S = (shd ? a.sh_s2 + (size_t)l * a.H : a.s2 + ((size_t)l * a.E + d.e) * a.H) + d.rbk * a.rows2;
        for (int c = tid; c < a.rows2 / 4; c += 256) cp_async16(m.rs + 4 * c, S + 4 * c);
        const float* hb = shd ? a.h32_s : a.h32_r;
        const float* hmb = shd ? a.hmax_s : a.hmax_r;
        const int nrb = irow / kTaskRows13;
        const int slot0 = (shd ? 0 : d.off) + d.tok0;
        const int per = klen / 4;
        for (int c = tid; c < d.nc * per; c += 256) {
            const int j = c / per, k4 = c - j * per;
            cp_async16(m.raw + j * kSliceK + k4 * 4, hb + (size_t)(slot0 + j) * irow + k0 + k4 * 4);
        }
        const int nb4 = klen / kTaskRows13 / 4;  // 16-byte groups of the slice's maxima
        for (int c = tid; c < d.nc * nb4; c += 256) {
            const int j = c / nb4, r4 = c - j * nb4;
            cp_async16(&sh.hmr[j][4 * r4], hmb + (size_t)(slot0 + j) * nrb + k0 / kTaskRows13 + 4 * r4);
        }
        cp_async_commit();
        cp_async_wait<0>();
        consumers_sync();
        if (tid < d.nc) {
            float mx = 0.f;
            for (int b = 0; b < klen / kTaskRows13; ++b) mx = nanmax(mx, sh.hmr[tid][b]);
            const QScale qs = qscale(mx);
            sh.qs[tid] = qs;
            sh.xsc[tid] = qs.s * 0.0625f;
        }
        consumers_sync();
        for (int j = warp; j < d.nc; j += 8) {
            const QScale qs = sh.qs[j];
            const float* src = m.raw + j * kSliceK;
            for (int gi = lane; gi < klen / 8; gi += 32) {
                const float4 v0 = *reinterpret_cast<const float4*>(src + 8 * gi);
                const float4 v1 = *reinterpret_cast<const float4*>(src + 8 * gi + 4);
                const float f[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                uint2 p0, p1;
                quant2x8(f, qs, p0, p1);
                *reinterpret_cast<uint2*>(m.xs2 + (2 * j) * kStride2 + 8 * gi) = p0;
                *reinterpret_cast<uint2*>(m.xs2 + (2 * j + 1) * kStride2 + 8 * gi) = p1;
            }
        }
        consumers_sync();  // staged
        stamp(a, l, 15, r == 0);
        switch ((2 * d.nc + 7) >> 3) {
            case 1: consume2<1>(a, sh, d, l, n, m.wring, m.xs2, m.rs); break;
            case 2: consume2<2>(a, sh, d, l, n, m.wring, m.xs2, m.rs); break;
            case 3: consume2<3>(a, sh, d, l, n, m.wring, m.xs2, m.rs); break;
            default: consume2<4>(a, sh, d, l, n, m.wring, m.xs2, m.rs); break;
        }
        consumers_sync();  // every warp is done with xs2, raw and rs
        if (aborted(sh)) return false;
    }
    consumers_sync();
    stamp(a, l, 6);
    if (tid == 0) {
        __threadfence();
        atomicAdd(a.down_done + l, 1);
    }
    return true;
}

__global__ void __launch_bounds__(kThreads, 1)
    decode_stack_kernel(const __grid_constant__ CUtensorMap tm13, const __grid_constant__ CUtensorMap tms13,
                        const __grid_constant__ CUtensorMap tm2, const __grid_constant__ CUtensorMap tms2,
                        const FArgs a) {
    extern __shared__ __align__(128) uint8_t dsm[];
    Sh& sh = *reinterpret_cast<Sh*>(dsm);
    const uint32_t base_s = smem_addr(dsm);
    const uint32_t ring_s = (base_s + (uint32_t)sizeof(Sh) + 1023u) & ~1023u;
    Smem m;
    m.wring = dsm + (ring_s - base_s);
    m.xring = m.wring + (size_t)kStages * kTmaWBytes;
    m.xs2 = m.xring + (size_t)kStages * kXBytes;
    m.raw = reinterpret_cast<float*>(m.xs2 + kXs2Bytes);
    m.rs = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(m.raw) + kRawBytes);
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            bar_init(&sh.full[s], 1 + 32);  // the TMA arrival + one arrival per producer lane
            bar_init(&sh.empty[s], 8);      // one arrival per consumer warp
        }
        bar_init(&sh.tready, 1);
        bar_init(&sh.pdone, 1);
        sh.abort = 0;
        sh.never = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (warp == 8) {
        producer(a, sh, m.wring, m.xring, &tm13, &tms13, &tm2, &tms2);
        return;
    }
    // consumers
    if ((a.flags & kFlagTestStall) && threadIdx.x == 0) {  // a wait that runs out: take the timeout path
        stall_on_unset_flag(&sh.never, kStallCycles);
        atomicOr(a.status, ST_TIMEOUT);
        atomicExch(a.abort, 1);
    }
    for (int i = threadIdx.x; i < (int)sizeof(sh.cnt8) / 4; i += 256) reinterpret_cast<int*>(sh.cnt8)[i] = 0;
    consumers_sync();
    uint32_t n = 0;
    bool ok = true;
    for (int l = 0; ok && l < a.L; ++l) {
        ok = phase_units(a, sh, m, l) && phase_tables(a, sh, m, l) && phase_gate_up(a, sh, m, l, n) &&
             phase_down(a, sh, m, l, n);
    }
    if (ok) ok = phase_units(a, sh, m, a.L);
    if (!ok) sh.abort = 1;  // the producer stops and drains
    cp_async_wait<0>();
}

}  // namespace fused

size_t fused_smem_bytes() { return fused::kSmem; }

bool fused_supported(int H, int E, int K, int I, int Is, int T, int L) {
    return T >= 1 && T <= kDecodeMaxTokens && L >= 1 && L <= kMaxFusedLayers && H % kTmaChunk == 0 &&
           H <= 16384 && I % kTmaChunk == 0 && Is % kTmaChunk == 0 && E >= 1 && E <= kMaxE && K >= 1 &&
           K <= kMaxK && K <= E;
}

// Rows of one down task: 128 x rg, rg up to max(4, H/1024) dividing H/128, as
// long as the down tasks (counted from the upper bound of the routed buckets)
// still give every SM one.
int fused_rows2(int H, int E, int K, int I, int Is, int T, int sms) {
    const long long TK = (long long)T * K;
    const long long slices = (E < TK ? E : TK) * slices_of(I) + (Is > 0 ? (long long)chunks_of(T, kChunkTokens) * slices_of(Is) : 0);
    const int groups = H / kTaskRows2, want = H / 1024 > 4 ? H / 1024 : 4;
    for (int c : {8, 6, 4, 3, 2})
        if (c <= want && groups % c == 0 && (long long)(groups / c) * slices >= sms) return kTaskRows2 * c;
    return kTaskRows2;
}

cudaError_t launch_decode_stack(const FArgs& a, int grid, cudaStream_t stream) {
    static int attr_set[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (!attr_set[dev]) {
        const cudaError_t e = cudaFuncSetAttribute(fused::decode_stack_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)fused::kSmem);
        if (e != cudaSuccess) return e;
        attr_set[dev] = 1;
    }
    const int H = a.H, E = a.E, I = a.I, L = a.L;
    const int Is = a.Is > 0 ? a.Is : kTaskRows13;  // any valid map when there is no shared expert
    CUtensorMap tm13, tms13, tm2, tms2;
    const bool ok =
        encode_tensor_map_2d(&tm13, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.w13, H / 2, (uint64_t)L * E * 2 * I,
                             kTmaRowBytes, kTaskRows13, CU_TENSOR_MAP_SWIZZLE_128B) &&
        encode_tensor_map_2d(&tms13, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.Is > 0 ? (const void*)a.sh_w13 : (const void*)a.w13,
                             H / 2, a.Is > 0 ? (uint64_t)L * 2 * Is : 2 * (uint64_t)kTaskRows13, kTmaRowBytes,
                             kTaskRows13, CU_TENSOR_MAP_SWIZZLE_128B) &&
        encode_tensor_map_2d(&tm2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.w2, I / 2, (uint64_t)L * E * H, kTmaRowBytes,
                             kTaskRows2, CU_TENSOR_MAP_SWIZZLE_128B) &&
        encode_tensor_map_2d(&tms2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.Is > 0 ? (const void*)a.sh_w2 : (const void*)a.w2,
                             a.Is > 0 ? Is / 2 : I / 2, a.Is > 0 ? (uint64_t)L * H : (uint64_t)H, kTmaRowBytes,
                             kTaskRows2, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(fused::kThreads);
    cfg.dynamicSmemBytes = fused::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fused::decode_stack_kernel, tm13, tms13, tm2, tms2, a);
}

int fused_grid() {
    static int cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (cache[dev] == 0) {
        cudaFuncSetAttribute(fused::decode_stack_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fused::kSmem);
        int per_sm = 0, sms = 0;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fused::decode_stack_kernel, fused::kThreads, fused::kSmem);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cache[dev] = per_sm >= 1 && sms > 0 ? sms : -1;
    }
    return cache[dev];
}

}  // namespace moe
