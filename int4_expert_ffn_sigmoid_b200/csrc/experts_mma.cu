// Weight-streaming expert kernels (gate/up + SwiGLU, then down) for the
// int4 per-row-symmetric SwiGLU experts and the shared expert.
//
// Method: colibri README (project listing), "What's implemented": packed int4
// with per-row scales, dequant-on-use, batch-union MoE (each expert touched
// by the batch is read once and applied to all of its tokens);
// nanocolibri-engine README, "Converting a checkpoint yourself": per-row
// symmetric int4, f32 row scales.
//
// Design.  One CTA (8 compute warps) owns one task and walks the reduction
// dimension in 128-wide k blocks.  Gate/up task = (bucket, chunk of up to 16
// of its tokens (32 on large batches), 64 gate rows + the same 64 up rows);
// down task = (bucket, chunk, 512-wide slice of the intermediate dimension,
// a group of 128-row blocks).  The grid is persistent; CTA c takes tasks in
// snake order counted from the heaviest end of the task list (the shared
// expert's tasks are at that end).  Three ways to bring the weights in:
//  - TMA ring (H >= 1024, multiples of 256; experts_w13_tma_kernel,
//    experts_w2_tma_kernel): a producer warp keeps 6-8 stages of 16 KB of
//    swizzled weight tiles in flight per SM across task boundaries; the
//    compute warps read their fragments from shared memory.
//  - Bulk copies (H < 1024, experts_w13_bulk_kernel): each warp's 16 rows of
//    a task are two contiguous blocks fetched with cp.async.bulk two tasks
//    ahead.
//  - Register ring (other shapes): every thread streams 16 contiguous bytes
//    (32 codes) of two rows per k block with non-allocating 128-bit loads,
//    kept 4 k blocks ahead in registers.
//  - The codes become int8 operands 16*c with three logic operations per
//    eight weights (lo8 / hi8), and feed mma.sync m16n8k32 (s8 x s8 -> s32).
//    Thread q's 16-byte chunk of a row is exactly its A fragments of four
//    mma k steps: word m gives the even elements (lo8) and the odd ones (hi8)
//    of one k step.
//  - Activations are two int8 parts per token (v ~= s (q0 + q1/256), see
//    quant2); the two parts of token j are mma columns 2j and 2j+1, so a
//    thread's accumulators hold both parts of the same (row, token) and the
//    products accumulate exactly in int32.  The chunk's activation rows are
//    staged in shared memory, padded by 16 bytes so that the per-thread
//    16-byte fragment reads are conflict-free: the gate/up kernels copy the
//    router's quantized x with cp.async (the TMA-ring kernel into each stage,
//    256-wide; the bulk kernel whole rows into a second buffer while the
//    previous task computes; the register-ring kernel whole rows, or for
//    H > 2048 a 4-deep ring of 128-wide slices); the down kernels prefetch
//    the next task's f32 slice of h and its per-64-row maxima of |h| (from
//    the gate/up epilogue) while the current task computes, then quantize it
//    with one scale per (token, slice).
//  - Latency: the weight ring runs on across task boundaries (the last
//    blocks of a task are replaced by the first blocks of the CTA's next
//    task), and a CTA whose first task belongs to the shared expert fills its
//    ring before the router has finished.
//  - Gate/up: the 16 mma rows are 8 gate rows and the same 8 up rows, so each
//    thread ends with gate and up of the same (row, token) and applies SwiGLU
//    in registers; h is stored in f32.  Row and activation scales are applied
//    to the integer result (they factor out of the row's dot product).
//  - Down: every slice writes its own partial output row; the combine adds
//    the slices.
//  - Small-batch path: each gate/up CTA derives the bucket list, its task
//    list and the token of every slot from the router's per-group pick counts
//    and ranks in its prologue; its CTA 0 also writes them to the workspace
//    for the down kernel and the combine (on the large-batch path the large
//    router writes them).
#include <cuda.h>

#include "moe_common.cuh"
#include "moe_launch.h"
#include "moe_tc.h"
#include "stream_ops.cuh"

namespace moe {

namespace {

constexpr int kRows13 = kTaskRows13;  // gate (and up) rows per gate/up task
constexpr int kRows2 = kTaskRows2;    // down rows per down task
constexpr int kRing = 4;      // weight k blocks in flight per thread
constexpr int kXRing = 4;     // staged activation slices (ring mode)
constexpr int kStageRows = 2 * kChunkTokens;  // two int8 rows (parts) per token
constexpr int kTab = kMaxE + 2;               // entries of each table
constexpr int kMaxSlots = kDecodeMaxTokens * kMaxK;
// Register-ring gate/up activation staging: one whole-row buffer up to
// kWholeMaxK, a ring of slices beyond.
constexpr int kWholeMaxK = 2048;

struct Tables {
    int n_buckets, ntask;
    int e[kTab], n[kTab], off[kTab], ts[kTab];
};

// Per-CTA shared state, ahead of the staging areas.
// One task of the CTA's task sequence, decoded once (see precompute_tasks).
struct TaskDesc {
    int e, off, rbk, sl, tok0, nc;  // e < 0: no task
};
constexpr int kMaxCtaTasks = 32;

struct Shm {
    Tables tb;
    TaskDesc td[kMaxCtaTasks];                    // the first tasks of this CTA, in its order
    int tok[kMaxSlots];                           // token of each routed slot (T*K <= kMaxSlots)
    float xsr[2][kChunkTokens];                   // gate/up: activation scale of each token (per buffer)
    float hmr[kMaxChunk][kSliceK / kRows13];      // down: the slice's per-64-row maxima of |h|
    float xsc[kMaxChunk];                         // down: activation scale / 16 of each token
    QScale qs[kMaxChunk];                         // down: activation scale of each token
    float hm[8][kChunkTokens];                    // gate/up: per-warp max |h| of each token
};
constexpr size_t kShmBytes = (sizeof(Shm) + 127) & ~size_t(127);

// scratch of the small-batch table build, in the staging area
constexpr size_t kBuildBytes = (size_t)(kDecodeGroups + 2) * kMaxE * 4;
static_assert(kBuildBytes <= (size_t)kStageRows * (kXRing * 128 + kPadB), "table build scratch fits the staging area");
// Mode 2 stages whole rows too when a task's rows fit in this many bytes.
constexpr size_t kRingWholeBytes = 100 * 1024;
constexpr size_t kSmem13[3] = {0 /* no mode 0 */, kShmBytes + (size_t)kStageRows * (kWholeMaxK + kPadB),
                               kShmBytes + kRingWholeBytes};
static_assert(kRingWholeBytes >= (size_t)kStageRows * (kXRing * 128 + kPadB), "ring staging fits");
// down: int8 staging of one slice + the next task's f32 slice
constexpr int kStride2 = kSliceK + kPadB;
constexpr size_t kRaw2Off = (size_t)kStageRows * kStride2;
constexpr size_t kRs2Off = kRaw2Off + (size_t)kChunkTokens * kSliceK * 4;  // row scales [2][kMaxRows2]
constexpr size_t kSmem2 = kShmBytes + kRs2Off + (size_t)2 * kMaxRows2 * 4;

// The bucket list and task prefix that the router wrote to the workspace,
// and (for at most kMaxSlots routed slots) the token of every slot.
__device__ __forceinline__ void load_tables(const Params& p, const int32_t* ts, const int* ntask, Tables& tb,
                                            int* tok) {
    const int TK = p.T * p.K;
    if (tok && TK <= kMaxSlots)
        for (int i = threadIdx.x; i < TK; i += blockDim.x) tok[i] = __ldcg(p.tok_of_slot + i);
    const int nb = __ldcg(&p.ctrl->n_buckets);
    for (int i = threadIdx.x; i <= nb && i < kTab; i += blockDim.x) {
        tb.ts[i] = __ldcg(ts + i);
        if (i < nb) {
            tb.e[i] = __ldcg(p.bucket_e + i);
            tb.n[i] = __ldcg(p.bucket_n + i);
            tb.off[i] = __ldcg(p.bucket_off + i);
        }
    }
    if (threadIdx.x == 0) {
        tb.n_buckets = nb < kTab ? nb : 0;
        tb.ntask = nb < kTab ? __ldcg(ntask) : 0;
        if (nb >= kTab) atomicOr(&p.ctrl->status, ST_BAD_COUNT);
    }
    __syncthreads();
}

// Small-batch path, from the router's per-group pick counts (hist), picks
// (idx) and ranks.  kind 0 (gate/up kernel): the bucket list, the gate/up
// task prefix and the token of every routed slot; the slot of pick (t, k) of
// expert e is offset[e] + (picks of e in the groups before t's) + rank[t, k],
// and CTA 0 also writes the bucket list, the down-task prefix, slot_of and
// tok_of_slot to the workspace.  kind 1 (down kernel): the bucket list and
// the down-task prefix only, with no write to global memory.
__device__ void build_tables_small(const Params& p, Shm& sh, int* scratch, int kind = 0) {
    int* s_base = scratch;  // [kDecodeGroups][kMaxE]
    int* s_cnt = scratch + kDecodeGroups * kMaxE;
    int* s_off = s_cnt + kMaxE;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = p.E, K = p.K, T = p.T, TK = T * K, G = p.decode_groups;
    const bool writer = kind == 0 && blockIdx.x == 0;
    Tables& tb = sh.tb;
    int my_e[2], my_rank[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {  // threads 0..255 cover the T*K <= 512 picks
        const int i = tid < 256 && kind == 0 ? tid + 256 * u : TK;
        my_e[u] = i < TK ? __ldcg(p.idx + i) : -1;
        my_rank[u] = i < TK ? __ldcg(p.rank + i) : 0;
    }
    if (tid < E) {
        int h[kDecodeGroups];
#pragma unroll
        for (int g = 0; g < kDecodeGroups; ++g) h[g] = g < G ? __ldcg(p.hist + (size_t)g * E + tid) : 0;
        int run = 0;
#pragma unroll
        for (int g = 0; g < kDecodeGroups; ++g) {
            s_base[g * kMaxE + tid] = run;
            run += h[g];
        }
        s_cnt[tid] = run;
    }
    if (kind == 0)
        for (int i = tid; i < kMaxSlots; i += blockDim.x) sh.tok[i] = -1;
    __syncthreads();
    if (warp == 0) {
        // lane l owns experts 8l .. 8l+7: counts, non-empty buckets, gate/up
        // and down tasks, scanned across the warp in one pass
        constexpr int kPer = kMaxE / 32;
        const int R13 = p.I / kTaskRows13, R2 = (p.H / p.rows2) * slices_of(p.I);
        int c[kPer];
        int v[4] = {0, 0, 0, 0};  // slots, buckets, gate/up tasks, down tasks
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int e = lane * kPer + j;
            c[j] = e < E ? s_cnt[e] : 0;
            v[0] += c[j];
            v[1] += c[j] > 0;
            v[2] += R13 * chunks_of(c[j], p.chunk);
            v[3] += R2 * chunks_of(c[j], p.chunk);
        }
        int inc[4] = {v[0], v[1], v[2], v[3]};
#pragma unroll
        for (int o = 1; o < 32; o <<= 1)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int a = __shfl_up_sync(0xffffffffu, inc[i], o);
                if (lane >= o) inc[i] += a;
            }
        int off = inc[0] - v[0], b = inc[1] - v[1], b13 = inc[2] - v[2], b2 = inc[3] - v[3];
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int e = lane * kPer + j;
            if (e < E) {
                s_off[e] = off;
                if (c[j] > 0) {
                    tb.e[b] = e;
                    tb.n[b] = c[j];
                    tb.off[b] = off;
                    tb.ts[b] = kind == 0 ? b13 : b2;
                    if (writer) {
                        p.bucket_e[b] = e;
                        p.bucket_n[b] = c[j];
                        p.bucket_off[b] = off;
                        p.ts2[b] = b2;
                    }
                    ++b;
                }
                off += c[j];
                b13 += R13 * chunks_of(c[j], p.chunk);
                b2 += R2 * chunks_of(c[j], p.chunk);
            }
        }
        const int total = __shfl_sync(0xffffffffu, inc[0], 31);
        int nb = __shfl_sync(0xffffffffu, inc[1], 31);
        int t13 = __shfl_sync(0xffffffffu, inc[2], 31), t2 = __shfl_sync(0xffffffffu, inc[3], 31);
        __syncwarp();
        if (lane == 0) {
            const bool topp = p.topp > 0.f && p.topp < 1.f;  // dropped picks: fewer slots than T*K
            if (total != TK && !(topp && total < TK)) {  // inconsistent counts: flag them and run no routed task
                atomicOr(&p.ctrl->status, ST_BAD_COUNT);
                nb = t13 = t2 = 0;
            }
            if (p.Is > 0) {  // the shared expert: last bucket, slots TK .. TK+T-1
                tb.e[nb] = E;
                tb.n[nb] = T;
                tb.off[nb] = TK;
                tb.ts[nb] = kind == 0 ? t13 : t2;
                if (writer) {
                    p.bucket_e[nb] = E;
                    p.bucket_n[nb] = T;
                    p.bucket_off[nb] = TK;
                    p.ts2[nb] = t2;
                }
                t13 += (p.Is / kTaskRows13) * chunks_of(T, p.chunk);
                t2 += (p.H / p.rows2) * slices_of(p.Is) * chunks_of(T, p.chunk);
                ++nb;
            }
            tb.ts[nb] = kind == 0 ? t13 : t2;
            tb.n_buckets = nb;
            tb.ntask = kind == 0 ? t13 : t2;
            if (writer) {
                p.ts2[nb] = t2;
                p.ctrl->n_buckets = nb;
                p.ctrl->tasks2 = t2;
            }
        }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 2; ++u) {  // the slots (kind 0)
        const int i = tid < 256 && kind == 0 ? tid + 256 * u : TK;
        if (i >= TK) continue;
        const int e = my_e[u], t = i / K;
        if (e == -1 && p.topp > 0.f && p.topp < 1.f) {  // dropped by the top-p: no slot
            if (writer) p.slot_of[i] = -1;
            continue;
        }
        int slot = -1;
        if (e >= 0 && e < E) slot = s_off[e] + s_base[(t / kDecodeRouterTok) * kMaxE + e] + my_rank[u];
        else atomicOr(&p.ctrl->status, ST_BAD_EXPERT);
        if (slot < 0 || slot >= TK) {
            atomicOr(&p.ctrl->status, ST_BAD_SLOT);
            slot = -1;
        } else {
            sh.tok[slot] = t;
            if (writer) p.tok_of_slot[slot] = t;
        }
        if (writer) p.slot_of[i] = slot < 0 ? 0 : slot;
    }
    __syncthreads();
}


__device__ __forceinline__ int find_bucket(const Tables& tb, int task) {
    int lo = 0, hi = tb.n_buckets;  // ts[lo] <= task < ts[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tb.ts[mid] <= task) lo = mid; else hi = mid;
    }
    return lo;
}

// Token of slot s of a bucket starting at slot `off` (from shared memory
// when load_tables copied the slot tokens there).
__device__ __forceinline__ int slot_token(const Params& p, const Shm& sh, bool shared, int off, int s) {
    if (shared) return s;
    if (p.T * p.K <= kMaxSlots) return off + s < kMaxSlots ? sh.tok[off + s] : -1;
    return __ldcg(p.tok_of_slot + off + s);
}

// One k block: this thread's 16 bytes of weight rows a (mma row g) and b (mma
// row g + 8) against NT n-tiles of staged activations; xrow points at staged
// row g, byte q*32 of the k block, and n-tile i is 8*i rows further.
// This thread's weight stream of one task: 16 bytes of rows a (mma row g)
// and b (mma row g + 8) per k block, nkb blocks 64 bytes apart (nkb = 0: no
// task).
struct WStream {
    const uint8_t* ra;
    const uint8_t* rb;
    int nkb;
};

// Register ring of weight blocks in flight (block kb of a task in slot
// kb % kRing).
struct Ring {
    uint4 a[kRing], b[kRing];
};

__device__ __forceinline__ void prime(Ring& r, const WStream& s) {
#pragma unroll
    for (int i = 0; i < kRing; ++i) {
        r.a[i] = i < s.nkb ? ld_stream_v4(s.ra + i * 64) : make_uint4(0, 0, 0, 0);
        r.b[i] = i < s.nkb ? ld_stream_v4(s.rb + i * 64) : make_uint4(0, 0, 0, 0);
    }
}

// Main loop of both projections.  On entry the ring holds the first blocks
// of `cur` and (whole modes) every k block of its activations is staged and
// visible at byte 128*kb of its rows.  Ring mode: stage_slice(kb) issues the
// cp.async of block kb into slot kb % kXRing, driven from here.  While the
// last blocks of `cur` are consumed, the freed ring slots are refilled with
// the first blocks of `nxt` (when cur.nkb is a multiple of kRing, so that
// they land in their own slots); returns whether it did.
template <int NT, bool kRingMode, typename StageSlice>
__device__ __forceinline__ bool stream8(Ring& ring, const WStream& cur, const WStream& nxt, const uint8_t* xs,
                                        int stride, StageSlice&& stage_slice, int (&acc)[NT][4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int nkb = cur.nkb;
    const bool cont = nxt.nkb > 0 && nkb % kRing == 0;
    // two accumulator sets break the chain of dependent mma when there is one tile
    constexpr int kSets = NT == 1 ? 2 : 1;
    int part[kSets][NT][4];
#pragma unroll
    for (int s = 0; s < kSets; ++s)
#pragma unroll
        for (int i = 0; i < NT; ++i) part[s][i][0] = part[s][i][1] = part[s][i][2] = part[s][i][3] = 0;
    if (kRingMode) {
#pragma unroll
        for (int i = 0; i < kXRing - 1; ++i) {
            if (i < nkb) stage_slice(i);
            cp_async_commit();
        }
    }
    const uint8_t* xrow = xs + g * stride + q * 32;
    for (int kb0 = 0; kb0 < nkb; kb0 += kRing) {
#pragma unroll
        for (int rr = 0; rr < kRing; ++rr) {
            const int kb = kb0 + rr;
            if (kb < nkb) {
                if (kRingMode) {
                    cp_async_wait<kXRing - 2>();
                    __syncthreads();  // block kb visible to all; block kb-1's readers are done
                    if (kb + kXRing - 1 < nkb) stage_slice(kb + kXRing - 1);
                    cp_async_commit();
                }
                const uint4 wa = ring.a[rr], wb = ring.b[rr];
                const int nb = kb + kRing;
                if (nb < nkb) {
                    ring.a[rr] = ld_stream_v4(cur.ra + nb * 64);
                    ring.b[rr] = ld_stream_v4(cur.rb + nb * 64);
                } else if (cont && nb - nkb < nxt.nkb) {
                    ring.a[rr] = ld_stream_v4(nxt.ra + (nb - nkb) * 64);
                    ring.b[rr] = ld_stream_v4(nxt.rb + (nb - nkb) * 64);
                }
                kblock8<NT, kSets>(wa, wb, xrow + (kRingMode ? kb % kXRing : kb) * 128, 8 * stride, part);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NT; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][c] = part[0][i][c] + part[kSets - 1][i][c] * (kSets - 1);
    return cont;
}

// One gate/up task as this thread sees it.
struct Task13 {
    WStream w;  // gate row r0 + g and up row r0 + g
    bool ok;    // false: no task, or a table entry out of range
    bool shared;
    int e, off, irow, rbk, tok0, nc, r0;
};

// Gate/up task `local` of bucket (e, n, off).
__device__ __forceinline__ Task13 make13(const Params& p, int e, int n, int off, int local) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, q = lane & 3;
    Task13 t;
    t.ok = !(e < 0 || e > p.E || (e == p.E && p.Is == 0));
    t.shared = e == p.E;
    t.e = e;
    t.off = off;
    t.irow = t.shared ? p.Is : p.I;
    const int R = t.irow / kRows13;
    const int c = local / R;
    t.rbk = local - c * R;
    t.tok0 = c * p.chunk;
    t.nc = min(p.chunk, n - t.tok0);
    t.r0 = t.rbk * kRows13 + warp * 8;
    const int row_bytes = p.H / 2;
    const uint8_t* W = t.shared ? p.sh_w13 : p.w13 + (size_t)(t.ok ? e : 0) * 2 * p.I * row_bytes;
    t.w.ra = W + (size_t)(t.r0 + g) * row_bytes + q * 16;
    t.w.rb = W + (size_t)(t.irow + t.r0 + g) * row_bytes + q * 16;
    t.w.nkb = t.ok ? p.H / 128 : 0;
    return t;
}

// The r-th task of CTA c in snake order over the heaviest-first task list:
// even rounds go up the CTAs, odd rounds come back down, so that a CTA whose
// first task was one of the heaviest gets one of the lightest next.
__device__ __forceinline__ int snake(int c, int r) {
    return (r & 1) ? (r + 1) * (int)gridDim.x - 1 - c : r * (int)gridDim.x + c;
}

// Task `lin` of the heaviest-first list: its bucket and coordinates.  kind
// 0: gate/up (rows, chunk), 1: down (rows, slice, chunk).
__device__ __forceinline__ TaskDesc decode_task(const Params& p, const Tables& tb, int kind, int lin) {
    TaskDesc d;
    d.e = -1;
    d.off = d.rbk = d.sl = d.tok0 = d.nc = 0;
    if (lin >= tb.ntask) return d;
    const int task = tb.ntask - 1 - lin;
    const int b = find_bucket(tb, task);
    const int e = tb.e[b], n = tb.n[b], local = task - tb.ts[b];
    const int irow = e == p.E ? p.Is : p.I;
    int c;
    if (kind == 0) {
        const int R = irow / kRows13;
        c = local / R;
        d.rbk = local - c * R;
    } else {
        const int R = p.H / p.rows2, nsl = slices_of(irow);
        const int rest = local / R;
        d.rbk = local - rest * R;
        c = rest / nsl;
        d.sl = rest - c * nsl;
    }
    d.e = e;
    d.off = tb.off[b];
    d.tok0 = c * p.chunk;
    d.nc = min(p.chunk, n - d.tok0);
    return d;
}

// Decodes the CTA's first kMaxCtaTasks tasks (in snake order) into shared
// memory, so that the task loop does not repeat the search and divisions.
__device__ __forceinline__ void precompute_tasks(const Params& p, Shm& sh, int kind) {
    if (threadIdx.x < kMaxCtaTasks) sh.td[threadIdx.x] = decode_task(p, sh.tb, kind, snake(blockIdx.x, threadIdx.x));
    __syncthreads();
}

__device__ __forceinline__ TaskDesc task_desc(const Params& p, const Shm& sh, int kind, int r) {
    return r < kMaxCtaTasks ? sh.td[r] : decode_task(p, sh.tb, kind, snake(blockIdx.x, r));
}

// Gate/up task from its descriptor (no task: ok = false).
__device__ __forceinline__ Task13 task13_from(const Params& p, const TaskDesc& d) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, q = lane & 3;
    Task13 t{};
    if (d.e < 0) return t;
    t.ok = !(d.e > p.E || (d.e == p.E && p.Is == 0));
    t.shared = d.e == p.E;
    t.e = d.e;
    t.off = d.off;
    t.irow = t.shared ? p.Is : p.I;
    t.rbk = d.rbk;
    t.tok0 = d.tok0;
    t.nc = d.nc;
    t.r0 = d.rbk * kRows13 + warp * 8;
    const int row_bytes = p.H / 2;
    const uint8_t* W = t.shared ? p.sh_w13 : p.w13 + (size_t)(t.ok ? d.e : 0) * 2 * p.I * row_bytes;
    t.w.ra = W + (size_t)(t.r0 + g) * row_bytes + q * 16;
    t.w.rb = W + (size_t)(t.irow + t.r0 + g) * row_bytes + q * 16;
    t.w.nkb = t.ok ? p.H / 128 : 0;
    return t;
}

__device__ __forceinline__ Task13 task13_r(const Params& p, const Shm& sh, int r) {
    return task13_from(p, task_desc(p, sh, 0, r));
}

// Issues the cp.async of task t's activation rows (both parts of each token)
// into `buf` and of its tokens' activation scales into xsr, as one group.
__device__ __forceinline__ void stage13(const Params& p, const Shm& sh, const Task13& t, uint8_t* buf, int stride,
                                        float* xsr) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int H = p.H;
    for (int r = warp; r < 2 * t.nc; r += blockDim.x / 32) {
        const int tok = slot_token(p, sh, t.shared, t.off, t.tok0 + (r >> 1));
        if (tok < 0 || tok >= p.T) continue;
        const int8_t* src = p.xq + (size_t)tok * 2 * H + (r & 1) * H;
        for (int c16 = lane; c16 < H / 16; c16 += 32) cp_async16(buf + r * stride + c16 * 16, src + c16 * 16);
    }
    if (threadIdx.x < t.nc) {
        const int tok = slot_token(p, sh, t.shared, t.off, t.tok0 + threadIdx.x);
        if (tok >= 0 && tok < p.T) {
            cp_async4(xsr + threadIdx.x, p.xs + tok);
        } else {
            xsr[threadIdx.x] = 0.f;
            atomicOr(&p.ctrl->status, ST_BAD_SLOT);
        }
    }
    cp_async_commit();
}

template <int NT, bool kRingMode, typename StageSlice>
__device__ __forceinline__ bool run13(Ring& ring, const Task13& tk, const WStream& nx, float gs, float us,
                                      const Params& p, const uint8_t* xs, int stride, Shm& sh, const float* xsr,
                                      StageSlice&& stage_slice) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, q = lane & 3;
    int acc[NT][4];
    const bool cont = stream8<NT, kRingMode>(ring, tk.w, nx, xs, stride, stage_slice, acc);
    const int slot0 = (tk.shared ? 0 : tk.off) + tk.tok0;
    float* hrow0 = (tk.shared ? p.h32_s : p.h32_r) + (size_t)slot0 * tk.irow + tk.r0 + g;
#pragma unroll
    for (int i = 0; i < NT; ++i) {
        const int j = 4 * i + q;
        float hm = 0.f;
        if (j < tk.nc) {
            const float xsc = xsr[j] * 0.0625f;
            const float gv = join(acc[i][0], acc[i][1]) * (gs * xsc);
            const float uv = join(acc[i][2], acc[i][3]) * (us * xsc);
            const float h = silu_mul(gv, uv);
            hrow0[(size_t)j * tk.irow] = h;
            hm = fabsf(h);
        }
        hm = nanmax(hm, __shfl_xor_sync(0xffffffffu, hm, 4));
        hm = nanmax(hm, __shfl_xor_sync(0xffffffffu, hm, 8));
        hm = nanmax(hm, __shfl_xor_sync(0xffffffffu, hm, 16));
        if (g == 0 && j < tk.nc) sh.hm[warp][j] = hm;
    }
    __syncthreads();  // also: every warp is past its main loop
    if (threadIdx.x < tk.nc) {
        const int j = threadIdx.x;
        const int nrb = tk.irow / kRows13;
        float m = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) m = nanmax(m, sh.hm[w][j]);
        (tk.shared ? p.hmax_s : p.hmax_r)[(size_t)(slot0 + j) * nrb + tk.rbk] = m;
    }
    return cont;
}

// kMode: 1 one whole-row buffer (H <= kWholeMaxK), 2 (larger H) one
// whole-row buffer for tasks whose rows fit in kRingWholeBytes, else a ring of
// 128-wide slices.  Serves hidden sizes above 1024 that the TMA-ring kernel
// does not (not a multiple of 256).
template <int kMode>
__global__ void __launch_bounds__(256, 2) experts_w13_kernel(Params p) {
    extern __shared__ __align__(128) uint8_t dsm[];
    Shm& sh = *reinterpret_cast<Shm*>(dsm);
    uint8_t* xs = dsm + kShmBytes;
    const int g = (threadIdx.x & 31) >> 2;
    const int H = p.H;
    static_assert(kMode == 1 || kMode == 2, "staging mode");
    const int stride = (kMode == 2 ? kXRing * 128 : H) + kPadB;
    Ring ring;
    // The shared expert's tasks come first in every CTA's order and do not
    // depend on the routing: a CTA whose first task is one starts its weight
    // stream before the router has finished; the rest of the shared expert
    // is warmed in L2.
    const int ns = p.Is > 0 ? (p.Is / kRows13) * chunks_of(p.T, p.chunk) : 0;
    bool primed = false;
    const uint8_t* primed_ra = nullptr;
    if ((int)blockIdx.x < ns) {
        const Task13 t = make13(p, p.E, p.T, p.T * p.K, ns - 1 - (int)blockIdx.x);
        prime(ring, t.w);
        primed = true;
        primed_ra = t.w.ra;
    }
    if (p.Is > 0) prefetch_l2_slice(p.sh_w13, (size_t)p.Is * p.H);
    pdl_wait();
    pdl_release();
    if (p.decode_groups > 0) build_tables_small(p, sh, reinterpret_cast<int*>(xs));
    else load_tables(p, p.ts13, &p.ctrl->tasks13, sh.tb, sh.tok);
    precompute_tasks(p, sh, 0);
    const Tables& tb = sh.tb;
    Task13 cur = task13_r(p, sh, 0);
    if (primed && cur.w.ra != primed_ra) primed = false;
    // activations first: they are L2 hits that should not queue behind the weight stream
    if (kMode != 2 && cur.ok) stage13(p, sh, cur, xs, stride, sh.xsr[0]);
    const float* S = cur.shared ? p.sh_s13 : p.s13 + (size_t)cur.e * 2 * p.I;
    float gs = cur.ok ? __ldg(S + cur.r0 + g) : 0.f, us = cur.ok ? __ldg(S + cur.irow + cur.r0 + g) : 0.f;
    for (int r = 0, lin = blockIdx.x; lin < tb.ntask; lin = snake(blockIdx.x, ++r)) {
        const Task13 nx = task13_r(p, sh, r + 1);
        if (!cur.ok) {  // a table entry out of range: flag it and stop
            if (threadIdx.x == 0) atomicOr(&p.ctrl->status, ST_BAD_TASK);
            break;
        }
        if (!primed) prime(ring, cur.w);
        // large H: whole rows when every row the mma tiles read (8 per n-tile) fits,
        // else slices staged in the main loop
        const bool whole2 = kMode == 2 && (size_t)8 * ((2 * cur.nc + 7) >> 3) * (H + kPadB) <= kRingWholeBytes;
        if (whole2) {
            stage13(p, sh, cur, xs, H + kPadB, sh.xsr[0]);
            cp_async_wait<0>();
        } else if (kMode == 2 && threadIdx.x < cur.nc) {  // the scales only
            const int tok = slot_token(p, sh, cur.shared, cur.off, cur.tok0 + threadIdx.x);
            if (tok >= 0 && tok < p.T) cp_async4(sh.xsr[0] + threadIdx.x, p.xs + tok);
            else sh.xsr[0][threadIdx.x] = 0.f;
        }
        if (kMode != 2) cp_async_wait<0>();
        __syncthreads();  // cur's activations are visible; the previous task is done with every buffer
        float gs_n = 0.f, us_n = 0.f;
        if (nx.ok) {
            const float* Sn = nx.shared ? p.sh_s13 : p.s13 + (size_t)nx.e * 2 * p.I;
            gs_n = __ldg(Sn + nx.r0 + g);
            us_n = __ldg(Sn + nx.irow + nx.r0 + g);
        }
        const int nc = cur.nc;
        const Task13& c = cur;
        auto stage_slice = [&](int kb) {
            const int r = threadIdx.x >> 3, part = threadIdx.x & 7;
            if (r < 2 * nc) {
                const int tok = slot_token(p, sh, c.shared, c.off, c.tok0 + (r >> 1));
                if (tok >= 0 && tok < p.T)
                    cp_async16(xs + r * stride + (kb % kXRing) * 128 + part * 16,
                               p.xq + (size_t)tok * 2 * H + (r & 1) * H + kb * 128 + part * 16);
            }
        };
        const uint8_t* xb = xs;
        const float* xsr = sh.xsr[0];
        if (kMode == 2 && whole2) {
            switch ((2 * nc + 7) >> 3) {
                case 1: primed = run13<1, false>(ring, cur, nx.w, gs, us, p, xb, H + kPadB, sh, xsr, stage_slice); break;
                case 2: primed = run13<2, false>(ring, cur, nx.w, gs, us, p, xb, H + kPadB, sh, xsr, stage_slice); break;
                case 3: primed = run13<3, false>(ring, cur, nx.w, gs, us, p, xb, H + kPadB, sh, xsr, stage_slice); break;
                default: primed = run13<4, false>(ring, cur, nx.w, gs, us, p, xb, H + kPadB, sh, xsr, stage_slice); break;
            }
        } else {
            switch ((2 * nc + 7) >> 3) {
                case 1: primed = run13<1, kMode == 2>(ring, cur, nx.w, gs, us, p, xb, stride, sh, xsr, stage_slice); break;
                case 2: primed = run13<2, kMode == 2>(ring, cur, nx.w, gs, us, p, xb, stride, sh, xsr, stage_slice); break;
                case 3: primed = run13<3, kMode == 2>(ring, cur, nx.w, gs, us, p, xb, stride, sh, xsr, stage_slice); break;
                default: primed = run13<4, kMode == 2>(ring, cur, nx.w, gs, us, p, xb, stride, sh, xsr, stage_slice); break;
            }
        }
        if (kMode == 1 && nx.ok) stage13(p, sh, nx, xs, stride, sh.xsr[0]);
        cur = nx;
        gs = gs_n;
        us = us_n;
    }
}

// ---------------------------------------------------------------------------
// Gate/up for H <= kBulkMaxK: one CTA per SM.  Each warp's 8 gate rows and 8
// up rows of a task are two contiguous blocks of the weight matrix; the
// warp's lane 0 fetches them with two bulk copies (cp.async.bulk, completion
// counted on an mbarrier) into the warp's own two-slot ring in shared memory,
// two tasks ahead, so that every SM keeps 128 KB of weights in flight, and
// the warp reads its fragments from there.  Activations are staged per task
// as in the kernel above (two cp.async buffers).  Every wait is bounded: on
// a timeout the CTA flags ST_TIMEOUT, stops issuing, and still waits (again
// bounded) for the copies it issued before it exits.
// ---------------------------------------------------------------------------
constexpr int kBulkMaxK = 1024;
constexpr int kBulkSlots = 2;
constexpr size_t kBulkWarpSlot = 16 * (kBulkMaxK / 2);  // 8 gate + 8 up rows
constexpr size_t kBulkBarBytes = 128;
constexpr size_t kSmem13Bulk = kShmBytes + kBulkBarBytes + 8 * kBulkSlots * kBulkWarpSlot +
                               (size_t)2 * kStageRows * (kBulkMaxK + kPadB);

// Lane 0 of the calling warp issues the warp's 8 gate + 8 up rows of task t
// into `slot`.
__device__ __forceinline__ void issue13(const Params& p, const Task13& t, uint8_t* slot, uint64_t* bar) {
    if ((threadIdx.x & 31) != 0 || !t.ok) return;
    const size_t rb = (size_t)p.H / 2;
    const uint8_t* W = t.shared ? p.sh_w13 : p.w13 + (size_t)t.e * 2 * p.I * rb;
    const int r0 = t.r0;  // this warp's first row (r0 is per warp)
    bar_expect_tx(bar, (uint32_t)(16 * rb));
    bulk_g2s(slot, W + (size_t)r0 * rb, (uint32_t)(8 * rb), bar);
    bulk_g2s(slot + 8 * rb, W + (size_t)(t.irow + r0) * rb, (uint32_t)(8 * rb), bar);
}

template <int NT>
__device__ __forceinline__ void run13b(const Task13& tk, const uint8_t* wslot, float gs, float us, const Params& p,
                                       const uint8_t* xs, int stride, Shm& sh, const float* xsr) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, q = lane & 3;
    const int rb = p.H / 2, nkb = p.H / 128;
    constexpr int kSets = NT == 1 ? 2 : 1;
    int part[kSets][NT][4];
#pragma unroll
    for (int s = 0; s < kSets; ++s)
#pragma unroll
        for (int i = 0; i < NT; ++i) part[s][i][0] = part[s][i][1] = part[s][i][2] = part[s][i][3] = 0;
    const uint8_t* ga = wslot + g * rb + q * 16;
    const uint8_t* ua = wslot + (8 + g) * rb + q * 16;
    const uint8_t* xrow = xs + g * stride + q * 32;
#pragma unroll 2
    for (int kb = 0; kb < nkb; ++kb) {
        const uint4 wa = *reinterpret_cast<const uint4*>(ga + kb * 64);
        const uint4 wb = *reinterpret_cast<const uint4*>(ua + kb * 64);
        kblock8<NT, kSets>(wa, wb, xrow + kb * 128, 8 * stride, part);
    }
    int acc[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][c] = part[0][i][c] + part[kSets - 1][i][c] * (kSets - 1);
    const int slot0 = (tk.shared ? 0 : tk.off) + tk.tok0;
    float* hrow0 = (tk.shared ? p.h32_s : p.h32_r) + (size_t)slot0 * tk.irow + tk.r0 + g;
#pragma unroll
    for (int i = 0; i < NT; ++i) {
        const int j = 4 * i + q;
        float hm = 0.f;
        if (j < tk.nc) {
            const float xsc = xsr[j] * 0.0625f;
            const float gv = join(acc[i][0], acc[i][1]) * (gs * xsc);
            const float uv = join(acc[i][2], acc[i][3]) * (us * xsc);
            const float h = silu_mul(gv, uv);
            hrow0[(size_t)j * tk.irow] = h;
            hm = fabsf(h);
        }
        hm = nanmax(hm, __shfl_xor_sync(0xffffffffu, hm, 4));
        hm = nanmax(hm, __shfl_xor_sync(0xffffffffu, hm, 8));
        hm = nanmax(hm, __shfl_xor_sync(0xffffffffu, hm, 16));
        if (g == 0 && j < tk.nc) sh.hm[warp][j] = hm;
    }
    __syncthreads();
    if (threadIdx.x < tk.nc) {
        const int j = threadIdx.x;
        const int nrb = tk.irow / kRows13;
        float m = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) m = nanmax(m, sh.hm[w][j]);
        (tk.shared ? p.hmax_s : p.hmax_r)[(size_t)(slot0 + j) * nrb + tk.rbk] = m;
    }
}

__global__ void __launch_bounds__(256, 1) experts_w13_bulk_kernel(Params p) {
    extern __shared__ __align__(128) uint8_t dsm[];
    Shm& sh = *reinterpret_cast<Shm*>(dsm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(dsm + kShmBytes);  // [warp][slot]
    uint8_t* wring = dsm + kShmBytes + kBulkBarBytes;
    uint8_t* xs = wring + 8 * kBulkSlots * kBulkWarpSlot;
    const int warp = threadIdx.x >> 5, g = (threadIdx.x & 31) >> 2;
    const int H = p.H;
    const int stride = H + kPadB;
    const int bufbytes = kStageRows * stride;
    const size_t wslot_bytes = (size_t)16 * (H / 2);
    auto slot_ptr = [&](int s) { return wring + ((size_t)warp * kBulkSlots + s) * kBulkWarpSlot; };
    auto bar_of = [&](int s) { return bars + warp * kBulkSlots + s; };
    if (threadIdx.x == 0) {
        for (int i = 0; i < 8 * kBulkSlots; ++i) bar_init(bars + i, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    (void)wslot_bytes;
    // A CTA whose first task belongs to the shared expert fetches its weights
    // before the router has finished.
    const int ns = p.Is > 0 ? (p.Is / kRows13) * chunks_of(p.T, p.chunk) : 0;
    bool pre = false;
    const uint8_t* pre_ra = nullptr;
    if ((int)blockIdx.x < ns) {
        const Task13 t = make13(p, p.E, p.T, p.T * p.K, ns - 1 - (int)blockIdx.x);
        issue13(p, t, slot_ptr(0), bar_of(0));
        pre = true;
        pre_ra = t.w.ra;
    }
    if (p.Is > 0) prefetch_l2_slice(p.sh_w13, (size_t)p.Is * p.H);
    pdl_wait();
    pdl_release();
    if (p.decode_groups > 0) build_tables_small(p, sh, reinterpret_cast<int*>(xs));
    else load_tables(p, p.ts13, &p.ctrl->tasks13, sh.tb, sh.tok);
    precompute_tasks(p, sh, 0);
    Task13 cur = task13_r(p, sh, 0);
    bool abort = false;
    if (pre && cur.w.ra != pre_ra) {  // cannot happen with consistent tables
        if (threadIdx.x == 0) atomicOr(&p.ctrl->status, ST_BAD_TASK);
        abort = true;
    }
    bool issued[kBulkSlots] = {pre, false};
    uint32_t ph[kBulkSlots] = {0u, 0u};
    if (!abort) {
        if (!pre && cur.ok) { issue13(p, cur, slot_ptr(0), bar_of(0)); issued[0] = true; }
        const Task13 t1 = task13_r(p, sh, 1);
        if (t1.ok) { issue13(p, t1, slot_ptr(1), bar_of(1)); issued[1] = true; }
        // activations first in the memory queues of this SM's first task
        if (cur.ok) stage13(p, sh, cur, xs, stride, sh.xsr[0]);
    }
    const float* S = cur.shared ? p.sh_s13 : p.s13 + (size_t)cur.e * 2 * p.I;
    float gs = cur.ok ? __ldg(S + cur.r0 + g) : 0.f, us = cur.ok ? __ldg(S + cur.irow + cur.r0 + g) : 0.f;
    for (int r = 0; !abort && cur.ok; ++r) {
        const int s = r & 1;
        const Task13 nx = task13_r(p, sh, r + 1);
        cp_async_wait<0>();
        __syncthreads();  // cur's activations are visible; the previous task is done with the other buffer
        if (nx.ok) stage13(p, sh, nx, xs + (s ^ 1) * bufbytes, stride, sh.xsr[s ^ 1]);
        float gs_n = 0.f, us_n = 0.f;
        if (nx.ok) {
            const float* Sn = nx.shared ? p.sh_s13 : p.s13 + (size_t)nx.e * 2 * p.I;
            gs_n = __ldg(Sn + nx.r0 + g);
            us_n = __ldg(Sn + nx.irow + nx.r0 + g);
        }
        // this warp's weights of cur (slot s); a timeout flags the CTA, whose
        // warps then stop issuing and leave the loop together below
        const bool got = bar_wait(bar_of(s), ph[s], kBulkWaitCycles);
        if (got) ph[s] ^= 1u, issued[s] = false;
        if (!got && (threadIdx.x & 31) == 0) atomicOr(&p.ctrl->status, ST_TIMEOUT);
        if (__syncthreads_or(!got)) {
            abort = true;
            break;
        }
        const uint8_t* wslot = slot_ptr(s);
        const uint8_t* xb = xs + s * bufbytes;
        const float* xsr = sh.xsr[s];
        switch ((2 * cur.nc + 7) >> 3) {
            case 1: run13b<1>(cur, wslot, gs, us, p, xb, stride, sh, xsr); break;
            case 2: run13b<2>(cur, wslot, gs, us, p, xb, stride, sh, xsr); break;
            case 3: run13b<3>(cur, wslot, gs, us, p, xb, stride, sh, xsr); break;
            default: run13b<4>(cur, wslot, gs, us, p, xb, stride, sh, xsr); break;
        }
        // the slot is free (the epilogue's barrier follows every warp's reads): refill it two tasks ahead
        const Task13 t2 = task13_r(p, sh, r + 2);
        if (t2.ok) { issue13(p, t2, slot_ptr(s), bar_of(s)); issued[s] = true; }
        cur = nx;
        gs = gs_n;
        us = us_n;
    }
    // every copy this warp issued has landed before the CTA's shared memory goes away
    for (int s = 0; s < kBulkSlots; ++s)
        if (issued[s]) bar_wait(bar_of(s), ph[s], kBulkWaitCycles);
    cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// Gate/up for H > kBulkMaxK with H a multiple of 256: one CTA per SM, a
// producer warp and 8 consumer warps around a ring of kTmaStages stages.  A
// stage is one 256-wide k chunk of a task: its 64 gate rows and 64 up rows
// (two TMA tile loads of 64 rows x 128 bytes with the 128-byte swizzle) and
// the chunk's activations (both int8 parts of each of the task's tokens,
// 256 bytes each), which the producer lanes copy with cp.async and whose
// completion counts on the same mbarrier as the tile loads.  The consumers
// read their mma fragments from the stage and release it; the producer runs
// ahead across task boundaries, so the weight stream does not pause between
// tasks, and a CTA whose first task belongs to the shared expert issues that
// task's first stages of weights before the router has finished.  Every wait
// is bounded: a timeout flags ST_TIMEOUT and sets the CTA's abort flag, after
// which nobody waits any more, the tasks run to their end on whatever the
// stages hold, and the producer waits (bounded) for its last copies before
// it exits.
// ---------------------------------------------------------------------------
constexpr int kTmaThreads = 288;                               // 8 consumer warps + the producer warp
// Ring geometry for tasks of kChunk tokens and WB-bit codes: the activation
// part of a stage holds 2 kChunk rows, the weight part the 256-wide k chunk of
// 64 gate and 64 up rows (16 KiB of int4, 32 KiB of int8: the 128-byte rows
// of four tiles, gate k 0..127, gate k 128..255, then up), and the ring is
// as deep as shared memory allows (int4: 8 stages for 16 tokens, 6 for 32;
// int8: 5 and 4), or, for two CTAs per SM (kOcc = 2: int4, 16-token tasks),
// 4 stages each.
template <int kChunk, int WB, int kOcc = 1>
struct Tma13 {
    static_assert(kOcc == 1 || (kOcc == 2 && WB == 4 && kChunk == kChunkTokens), "two CTAs per SM: int4, 16 tokens");
    static constexpr int kWBytes = kTmaWBytes * WB / 4;
    static constexpr int kStages = kOcc == 2 ? 4 : WB == 4 ? (kChunk == kChunkTokens ? 8 : 6) : (kChunk == kChunkTokens ? 5 : 4);
    static constexpr int kXBytes = 2 * kChunk * kTmaXStride;
    static constexpr size_t kMisc = 256 + 2 * 8 * kChunk * 4;  // barriers, flag, per-warp maxima
    static constexpr size_t kSmem = kShmBytes + kMisc + 1024 /* alignment */ + (size_t)kStages * (kWBytes + kXBytes);
    static_assert(kSmem <= 227 * 1024 / kOcc, "TMA gate/up shared memory");
    static_assert((size_t)kStages * kXBytes >= kBuildBytes, "table build scratch fits the activation ring");
};

// The weights of k chunk c of a task whose gate rows start at row rg and up
// rows at ru of `map`: expect the bytes, then the tile loads (64 rows x 128
// bytes each: two for int4, four for int8).
template <int WB>
__device__ __forceinline__ void issue_w13_chunk(const CUtensorMap* map, uint64_t* bar, uint8_t* dst, int c, int rg,
                                                int ru) {
    constexpr int kTile = kRows13 * kTmaRowBytes;
    bar_expect_tx(bar, kTmaWBytes * WB / 4);
    if (WB == 4) {
        tma_tile(dst, map, bar, c * kTmaRowBytes, rg);
        tma_tile(dst + kTile, map, bar, c * kTmaRowBytes, ru);
    } else {
        tma_tile(dst, map, bar, c * kTmaChunk, rg);
        tma_tile(dst + kTile, map, bar, c * kTmaChunk + kTmaRowBytes, rg);
        tma_tile(dst + 2 * kTile, map, bar, c * kTmaChunk, ru);
        tma_tile(dst + 3 * kTile, map, bar, c * kTmaChunk + kTmaRowBytes, ru);
    }
}

// Consumer main loop of one task: nch stages from stage counter n on.
template <int NT, int kStages, int kXBytes, int WB>
__device__ __forceinline__ void consume13(int nch, uint32_t& n, uint64_t* full, uint64_t* empty, const uint8_t* wring,
                                          const uint8_t* xring, volatile int* abort, unsigned* status,
                                          int (&acc)[NT][4]) {
    constexpr int kWBytes = kTmaWBytes * WB / 4, kTile = kRows13 * kTmaRowBytes;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, q = lane & 3;
    constexpr int kSets = NT == 1 ? 2 : 1;
    int part[kSets][NT][4];
#pragma unroll
    for (int s = 0; s < kSets; ++s)
#pragma unroll
        for (int i = 0; i < NT; ++i) part[s][i][0] = part[s][i][1] = part[s][i][2] = part[s][i][3] = 0;
    // row warp*8 + g of a 1024-byte aligned tile: its 16-byte chunk j sits at j ^ g
    const int wrow = (warp * 8 + g) * kTmaRowBytes;
    for (int c = 0; c < nch; ++c, ++n) {
        const int s = n % kStages;
        if (!*abort && !bar_wait_or_abort(full + s, (n / kStages) & 1, kBulkWaitCycles, abort)) {
            *abort = 1;
            if (lane == 0) atomicOr(status, ST_TIMEOUT);
        }
        const uint8_t* wt = wring + (size_t)s * kWBytes + wrow;
        const uint8_t* xt = xring + (size_t)s * kXBytes + g * kTmaXStride + q * 32;
#pragma unroll
        for (int kb = 0; kb < kTmaChunk / 128; ++kb) {
            if (WB == 4) {
                const int off = ((kb * 4 + q) ^ g) << 4;
                const uint4 wa = *reinterpret_cast<const uint4*>(wt + off);
                const uint4 wb = *reinterpret_cast<const uint4*>(wt + kTile + off);
                kblock8<NT, kSets>(wa, wb, xt + kb * 128, 8 * kTmaXStride, part);
            } else {  // codes 32q .. 32q + 31 of block kb: 16-byte chunks 2q, 2q + 1 of tile kb
                const uint8_t* ga = wt + kb * kTile;
                const uint8_t* ub = wt + (2 + kb) * kTile;
                const int o0 = ((2 * q) ^ g) << 4, o1 = ((2 * q + 1) ^ g) << 4;
                kblock8_i8<NT, kSets>(*reinterpret_cast<const uint4*>(ga + o0), *reinterpret_cast<const uint4*>(ga + o1),
                                      *reinterpret_cast<const uint4*>(ub + o0), *reinterpret_cast<const uint4*>(ub + o1),
                                      xt + kb * 128, 8 * kTmaXStride, part);
            }
        }
        __syncwarp();
        if (lane == 0) bar_arrive(empty + s);
    }
#pragma unroll
    for (int i = 0; i < NT; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][c] = part[0][i][c] + part[kSets - 1][i][c] * (kSets - 1);
}

template <int kChunk, int WB, int kOcc = 1>
__global__ void __launch_bounds__(kTmaThreads, kOcc)
    experts_w13_tma_kernel(const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_s, Params p) {
    using Cfg = Tma13<kChunk, WB, kOcc>;
    constexpr int kStages = Cfg::kStages, kXBytes = Cfg::kXBytes, kWBytes = Cfg::kWBytes;
    extern __shared__ __align__(128) uint8_t dsm[];
    Shm& sh = *reinterpret_cast<Shm*>(dsm);
    uint64_t* full = reinterpret_cast<uint64_t*>(dsm + kShmBytes);
    uint64_t* empty = full + kStages;
    volatile int* abort = reinterpret_cast<volatile int*>(empty + kStages);
    volatile int* never = abort + 1;  // nothing sets it (MOE_TEST_STALL)
    float(*hm2)[8][kChunk] = reinterpret_cast<float(*)[8][kChunk]>(dsm + kShmBytes + 256);
    const uint32_t base_s = static_cast<uint32_t>(__cvta_generic_to_shared(dsm));
    const uint32_t ring_s = (base_s + (uint32_t)(kShmBytes + Cfg::kMisc) + 1023u) & ~1023u;
    uint8_t* wring = dsm + (ring_s - base_s);
    uint8_t* xring = wring + (size_t)kStages * kWBytes;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const bool producer = warp == 8;
    const int H = p.H, nch = H / kTmaChunk;
    unsigned* status = &p.ctrl->status;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            bar_init(full + i, 1 + 32);  // the tile loads' arrival + one cp.async arrival per producer lane
            bar_init(empty + i, 8);      // one arrival per consumer warp
        }
        *abort = 0;
        *never = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    // the shared expert's first task of this CTA, if its first task is one
    const int ns = p.Is > 0 ? (p.Is / kRows13) * chunks_of(p.T, p.chunk) : 0;
    const bool pre = (int)blockIdx.x < ns;
    const int npre = pre ? min(kStages, nch) : 0;
    int pre_rbk = 0, pre_tok0 = 0;
    if (pre) {
        const int R = p.Is / kRows13, local = ns - 1 - (int)blockIdx.x;
        pre_rbk = local % R;
        pre_tok0 = (local / R) * p.chunk;
        if (producer && lane == 0)
            for (int c = 0; c < npre; ++c)
                issue_w13_chunk<WB>(&tm_s, full + c, wring + (size_t)c * kWBytes, c, pre_rbk * kRows13,
                                    p.Is + pre_rbk * kRows13);
    }
    if (p.Is > 0) prefetch_l2_slice(p.sh_w13, (size_t)p.Is * p.H * WB / 4);
    pdl_wait();
    pdl_release();
    if (p.decode_groups > 0) build_tables_small(p, sh, reinterpret_cast<int*>(xring));
    else load_tables(p, p.ts13, &p.ctrl->tasks13, sh.tb, sh.tok);
    precompute_tasks(p, sh, 0);
    if (threadIdx.x == 0 && pre) {  // cannot fail with consistent tables
        const TaskDesc d = sh.td[0];
        if (!(d.e == p.E && d.rbk == pre_rbk && d.tok0 == pre_tok0 && sh.tb.ntask > (int)blockIdx.x)) {
            *abort = 1;
            atomicOr(status, ST_BAD_TASK);
        }
    }
    __syncthreads();
    const int ntask = sh.tb.ntask;
    if (!producer && *abort) return;
    if (producer) {
        uint32_t n = 0;
        int last_round[kStages];
#pragma unroll
        for (int s = 0; s < kStages; ++s) last_round[s] = s < npre ? 0 : -1;
        for (int r = 0; !*abort && snake(blockIdx.x, r) < ntask; ++r) {
            const TaskDesc d = task_desc(p, sh, 0, r);
            if (d.e < 0 || d.e > p.E || (d.e == p.E && p.Is == 0)) break;  // the consumers flag it
            const bool shared = d.e == p.E;
            const int irow = shared ? p.Is : p.I;
            const int rg = (shared ? 0 : d.e * 2 * p.I) + d.rbk * kRows13, ru = rg + irow;
            // lane l copies activation rows l and l + 32 (row r: part r & 1 of the
            // chunk's token r >> 1)
            const int8_t* src[2] = {nullptr, nullptr};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = lane + 32 * h;
                if (row < 2 * d.nc) {
                    const int tok = slot_token(p, sh, shared, d.off, d.tok0 + (row >> 1));
                    if (tok >= 0 && tok < p.T) src[h] = p.xq + (size_t)tok * 2 * H + (row & 1) * H;
                }
            }
            for (int c = 0; c < nch; ++c, ++n) {
                const int s = n % kStages;
                const int round = (int)(n / kStages);
                const bool issued = r == 0 && c < npre;  // weights issued before the wait
                if (round > 0) {
                    bool ok = *abort == 0 && bar_wait_or_abort(empty + s, (round - 1) & 1, kBulkWaitCycles, abort);
                    if (__any_sync(0xffffffffu, !ok)) {
                        if (lane == 0 && !*abort) atomicOr(status, ST_TIMEOUT);
                        *abort = 1;
                        break;
                    }
                }
                if (lane == 0 && !issued)
                    issue_w13_chunk<WB>(shared ? &tm_s : &tm_r, full + s, wring + (size_t)s * kWBytes, c, rg, ru);
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    if (src[h]) {
                        uint8_t* dst = xring + (size_t)s * kXBytes + (lane + 32 * h) * kTmaXStride;
#pragma unroll
                        for (int j = 0; j < kTmaChunk / 16; ++j)
                            cp_async16(dst + j * 16, src[h] + c * kTmaChunk + j * 16);
                    }
                cp_async_arrive(full + s);
                last_round[s] = round;
            }
        }
        // stages issued before an abort that nobody consumed: their arrivals
        // (pre-issued weights) and their copies land before the CTA exits
        if (*abort) {
            for (int s = 0; s < npre; ++s)
                if (last_round[s] == 0 && n <= (uint32_t)s) cp_async_arrive(full + s);
            for (int s = 0; s < kStages; ++s)
                if (last_round[s] >= 0) bar_wait(full + s, last_round[s] & 1, kBulkWaitCycles);
        }
        cp_async_wait<0>();
        return;
    }
    // consumers
    if ((p.flags & kFlagTestStall) && threadIdx.x == 0) {  // a wait that runs out: take the timeout path
        stall_on_unset_flag(never, kStallCycles);
        *abort = 1;
        atomicOr(status, ST_TIMEOUT);
    }
    uint32_t n = 0;
    for (int r = 0; snake(blockIdx.x, r) < ntask; ++r) {
        const Task13 t = task13_r(p, sh, r);
        if (!t.ok) {
            if (threadIdx.x == 0) atomicOr(status, ST_BAD_TASK);
            break;
        }
        const float* S = t.shared ? p.sh_s13 : p.s13 + (size_t)t.e * 2 * p.I;
        const float gs = __ldg(S + t.r0 + g), us = __ldg(S + t.irow + t.r0 + g);
        const int NTt = (2 * t.nc + 7) >> 3;
        constexpr int kMaxNT = kChunk / 4;
        float xsc[kMaxNT];
#pragma unroll
        for (int i = 0; i < kMaxNT; ++i) {
            const int j = 4 * i + q;
            xsc[i] = 0.f;
            if (i < NTt && j < t.nc) {
                const int tok = slot_token(p, sh, t.shared, t.off, t.tok0 + j);
                xsc[i] = (tok >= 0 && tok < p.T) ? __ldcg(p.xs + tok) * code_unit<WB>() : 0.f;
            }
        }
        int acc[kMaxNT][4];
#define MOE_CONSUME13(N)                                                                                        \
    consume13<N, kStages, kXBytes, WB>(nch, n, full, empty, wring, xring, abort, status,                      \
                                   reinterpret_cast<int(&)[N][4]>(acc))
        switch (NTt) {
            case 1: MOE_CONSUME13(1); break;
            case 2: MOE_CONSUME13(2); break;
            case 3: MOE_CONSUME13(3); break;
            case 4: MOE_CONSUME13(4); break;
            case 5: MOE_CONSUME13((kMaxNT > 4 ? 5 : 1)); break;
            case 6: MOE_CONSUME13((kMaxNT > 4 ? 6 : 1)); break;
            case 7: MOE_CONSUME13((kMaxNT > 4 ? 7 : 1)); break;
            default: MOE_CONSUME13(kMaxNT); break;
        }
#undef MOE_CONSUME13
        const int slot0 = (t.shared ? 0 : t.off) + t.tok0;
        float* hrow0 = (t.shared ? p.h32_s : p.h32_r) + (size_t)slot0 * t.irow + t.r0 + g;
        float(*hm)[kChunk] = hm2[r & 1];
#pragma unroll
        for (int i = 0; i < kMaxNT; ++i) {
            if (i >= NTt) break;
            const int j = 4 * i + q;
            float hmv = 0.f;
            if (j < t.nc) {
                const float gv = join(acc[i][0], acc[i][1]) * (gs * xsc[i]);
                const float uv = join(acc[i][2], acc[i][3]) * (us * xsc[i]);
                const float h = silu_mul(gv, uv);
                hrow0[(size_t)j * t.irow] = h;
                hmv = fabsf(h);
            }
            hmv = nanmax(hmv, __shfl_xor_sync(0xffffffffu, hmv, 4));
            hmv = nanmax(hmv, __shfl_xor_sync(0xffffffffu, hmv, 8));
            hmv = nanmax(hmv, __shfl_xor_sync(0xffffffffu, hmv, 16));
            if (g == 0 && j < t.nc) hm[warp][j] = hmv;
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");  // the consumer warps' maxima are in
        if (threadIdx.x < t.nc) {
            const int j = threadIdx.x;
            const int nrb = t.irow / kRows13;
            float m = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) m = nanmax(m, hm[w][j]);
            (t.shared ? p.hmax_s : p.hmax_r)[(size_t)(slot0 + j) * nrb + t.rbk] = m;
        }
    }
}

// ---------------------------------------------------------------------------
// Gate/up on the 5th-generation tensor cores (tcgen05.mma kind::i8), for H a
// multiple of 256 on the large-batch weight-streaming sequence.  Two rings
// per 256-wide k chunk of a task: a weight ring (two 64-row TMA tiles of the
// codes, issued by one producer thread) and an activation ring (both int8
// parts of every token of the task, copied with cp.async by a second
// producer warp into the 128-byte swizzled K-major layout of the MMA's B
// operand: N = 2 * chunk rows, token j's parts are rows 2j and 2j+1).  The 8 converter warps turn a
// weight stage's int4 codes into int8 16*c (lo8 / hi8, the activations' byte
// order) and write them into a tensor-memory A stage (row 2i is gate row i
// of the task, row 2i + 1 up row i), which frees the weight stage at once:
// the weight ring refills without waiting for the MMAs.  One thread issues the
// MMAs (M = 128, N, K = 32; int32 accumulators in tensor memory), and 4
// epilogue warps join the two parts of each token, apply the row and
// activation scales and SwiGLU (a lane and its neighbour hold gate and up of
// one feature), store h in f32 and the per-(token, 64-row block) maxima of
// |h|.  Every wait is bounded and gives up when the CTA aborts; the producer
// waits for its copies and the MMA thread for its MMAs before the CTA exits.
// ---------------------------------------------------------------------------
constexpr int kTc8Threads = 480;  // converters 0-7, weight producer 8, MMA 9, epilogue 10-13, activations 14
constexpr int kTc8AStages = 4;    // int8 A stages in tensor memory (64 columns each)
constexpr int kTc8ACols = kTmaChunk / 4;

template <int kChunk>
struct Tc8 {
    static constexpr int kN = 2 * kChunk;      // MMA N
    static constexpr int kStages = 5;          // weight stages
    static constexpr int kXStages = 8;         // activation stages
    static constexpr int kXBytes = 2 * kN * 128;  // two 128-byte K blocks of kN rows
    static constexpr int kTmemCols = 512;         // accumulators at 0 and kN, A stages from 128
    static constexpr int kACol0 = 128;
    static constexpr size_t kMisc = 512 + 4 * kChunk * 4;  // barriers, flags, per-warp maxima
    static constexpr size_t kSmem = kShmBytes + kMisc + 1024 + (size_t)kStages * kTmaWBytes + (size_t)kXStages * kXBytes;
    static_assert(2 * kN <= kACol0 && kACol0 + kTc8AStages * kTc8ACols <= kTmemCols, "tensor memory layout");
    static_assert(kSmem <= 227 * 1024, "tcgen05 gate/up shared memory");
    static_assert((size_t)kXStages * kXBytes >= kBuildBytes, "table build scratch fits the activation ring");
};

__device__ __forceinline__ uint64_t tc8_desc_sw128(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// kind::i8: signed 8-bit A and B, s32 accumulate, both K-major.
__host__ __device__ constexpr uint32_t tc8_idesc(int M, int N) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void tc8_mma(uint32_t d, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void tc8_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}
__device__ __forceinline__ void tc8_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc8_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Every lane waits; the warp goes on only if every lane's wait succeeded.
__device__ __forceinline__ bool tc8_warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
    const bool ok = *abort == 0 && bar_wait_or_abort(bar, parity, kBulkWaitCycles, abort);
    return __all_sync(0xffffffffu, ok) != 0;
}

template <int kChunk>
__global__ void __launch_bounds__(kTc8Threads, 1)
    experts_w13_tc8_kernel(const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_s, Params p) {
    using Cfg = Tc8<kChunk>;
    constexpr int kStages = Cfg::kStages, kXStages = Cfg::kXStages, kXBytes = Cfg::kXBytes, kN = Cfg::kN;
    extern __shared__ __align__(128) uint8_t dsm[];
    Shm& sh = *reinterpret_cast<Shm*>(dsm);
    uint64_t* full = reinterpret_cast<uint64_t*>(dsm + kShmBytes);  // weight stage landed
    uint64_t* empty = full + kStages;                                // weight stage converted
    uint64_t* xfull = empty + kStages;                               // activation stage landed
    uint64_t* xempty = xfull + kXStages;                             // activation stage consumed by the MMAs
    uint64_t* a_full = xempty + kXStages;
    uint64_t* a_empty = a_full + kTc8AStages;
    uint64_t* acc_full = a_empty + kTc8AStages;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* never = abort + 1;  // nothing sets it (MOE_TEST_STALL)
    volatile int* ep_ok = abort + 2;  // [4] per epilogue warp: its accumulator wait succeeded
    float(*hmx)[kChunk] = reinterpret_cast<float(*)[kChunk]>(dsm + kShmBytes + 512);
    static_assert((2 * kStages + 2 * kXStages + 2 * kTc8AStages + 5) * 8 + 4 * 7 <= 512, "barrier area");
    const uint32_t base_s = smem_addr(dsm);
    const uint32_t ring_s = (base_s + (uint32_t)(kShmBytes + Cfg::kMisc) + 1023u) & ~1023u;
    uint8_t* wring = dsm + (ring_s - base_s);
    uint8_t* xring = wring + (size_t)kStages * kTmaWBytes;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = p.H, nch = H / kTmaChunk;
    unsigned* status = &p.ctrl->status;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            bar_init(full + i, 1);   // the tile loads' arrival
            bar_init(empty + i, 8);  // one arrival per converter warp
        }
        for (int i = 0; i < kXStages; ++i) {
            bar_init(xfull + i, 32);  // one cp.async arrival per lane of the activation warp
            bar_init(xempty + i, 1);  // the MMAs' commit
        }
        for (int i = 0; i < kTc8AStages; ++i) {
            bar_init(a_full + i, 8);
            bar_init(a_empty + i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            bar_init(acc_full + i, 1);
            bar_init(acc_empty + i, 4);
        }
        bar_init(drain, 1);
        *abort = 0;
        *never = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 9) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                     "r"(Cfg::kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc8_fence_before();
    __syncthreads();
    tc8_fence_after();
    const uint32_t tmem = *tmem_slot;
    // the shared expert's first task of this CTA, if its first task is one
    const int ns = p.Is > 0 ? (p.Is / kRows13) * chunks_of(p.T, p.chunk) : 0;
    const bool pre = (int)blockIdx.x < ns;
    const int npre = pre ? min(kStages, nch) : 0;
    int pre_rbk = 0, pre_tok0 = 0;
    if (pre) {
        const int R = p.Is / kRows13, local = ns - 1 - (int)blockIdx.x;
        pre_rbk = local % R;
        pre_tok0 = (local / R) * p.chunk;
        if (warp == 8 && lane == 0)
            for (int c = 0; c < npre; ++c)
                issue_w13_chunk<4>(&tm_s, full + c, wring + (size_t)c * kTmaWBytes, c, pre_rbk * kRows13,
                                   p.Is + pre_rbk * kRows13);
    }
    if (p.Is > 0) prefetch_l2_slice(p.sh_w13, (size_t)p.Is * p.H);
    pdl_wait();
    pdl_release();
    if (p.decode_groups > 0) build_tables_small(p, sh, reinterpret_cast<int*>(xring));
    else load_tables(p, p.ts13, &p.ctrl->tasks13, sh.tb, sh.tok);
    precompute_tasks(p, sh, 0);
    if (threadIdx.x == 0 && pre) {  // cannot fail with consistent tables
        const TaskDesc d = sh.td[0];
        if (!(d.e == p.E && d.rbk == pre_rbk && d.tok0 == pre_tok0 && sh.tb.ntask > (int)blockIdx.x)) {
            *abort = 1;
            atomicOr(status, ST_BAD_TASK);
        }
    }
    __syncthreads();
    const int ntask = sh.tb.ntask;
    auto task_ok = [&](const TaskDesc& d) { return !(d.e < 0 || d.e > p.E || (d.e == p.E && p.Is == 0)); };

    if (warp == 8) {
        // ---------------- weight producer: two TMA tiles per k chunk ----------------
        if (lane == 0) {
            uint32_t n = 0;
            int last_round[kStages];
#pragma unroll
            for (int s = 0; s < kStages; ++s) last_round[s] = s < npre ? 0 : -1;
            for (int r = 0; !*abort && snake(blockIdx.x, r) < ntask; ++r) {
                const TaskDesc d = task_desc(p, sh, 0, r);
                if (!task_ok(d)) break;  // the epilogue flags it
                const bool shared = d.e == p.E;
                const int irow = shared ? p.Is : p.I;
                const int rg = (shared ? 0 : d.e * 2 * p.I) + d.rbk * kRows13, ru = rg + irow;
                bool ok = true;
                for (int c = 0; c < nch; ++c, ++n) {
                    const int s = n % kStages;
                    const int round = (int)(n / kStages);
                    if (round > 0 && !(*abort == 0 && bar_wait_or_abort(empty + s, (round - 1) & 1, kBulkWaitCycles, abort))) {
                        if (!*abort) atomicOr(status, ST_TIMEOUT);
                        *abort = 1;
                        ok = false;
                        break;
                    }
                    if (!(r == 0 && c < npre))  // else issued before the tables were read
                        issue_w13_chunk<4>(shared ? &tm_s : &tm_r, full + s, wring + (size_t)s * kTmaWBytes, c, rg, ru);
                    last_round[s] = round;
                }
                if (!ok) break;
            }
            // every tile load issued lands before the CTA exits
            for (int s = 0; s < kStages; ++s)
                if (last_round[s] >= 0) bar_wait(full + s, last_round[s] & 1, kBulkWaitCycles);
        }
    } else if (warp == 14) {
        // ---------------- activation producer: both int8 parts of the task's tokens ----------------
        uint32_t n = 0;
        for (int r = 0; !*abort && snake(blockIdx.x, r) < ntask; ++r) {
            const TaskDesc d = task_desc(p, sh, 0, r);
            if (!task_ok(d)) break;
            const bool shared = d.e == p.E;
            // lane l copies rows l and l + 32 (row r: part r & 1 of the task's token
            // r >> 1) into the swizzled B layout
            const int8_t* src[2] = {nullptr, nullptr};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = lane + 32 * h;
                if (row < 2 * d.nc) {
                    const int tok = slot_token(p, sh, shared, d.off, d.tok0 + (row >> 1));
                    if (tok >= 0 && tok < p.T) src[h] = p.xq + (size_t)tok * 2 * H + (row & 1) * H;
                }
            }
            bool ok = true;
            for (int c = 0; c < nch; ++c, ++n) {
                const int s = n % kXStages;
                const int round = (int)(n / kXStages);
                if (round > 0) {
                    const bool w = *abort == 0 && bar_wait_or_abort(xempty + s, (round - 1) & 1, kBulkWaitCycles, abort);
                    if (__any_sync(0xffffffffu, !w)) {
                        if (lane == 0 && !*abort) atomicOr(status, ST_TIMEOUT);
                        *abort = 1;
                        ok = false;
                        break;
                    }
                }
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    if (src[h]) {
                        const int row = lane + 32 * h;
                        uint8_t* dst = xring + (size_t)s * kXBytes + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
                        for (int j = 0; j < kTmaChunk / 16; ++j)
                            cp_async16(dst + (j >> 3) * (kN * 128) + (((j & 7) ^ (row & 7)) << 4),
                                       src[h] + c * kTmaChunk + j * 16);
                    }
                cp_async_arrive(xfull + s);
            }
            if (!ok) break;
        }
        cp_async_wait<0>();  // every copy issued lands before the CTA exits
    } else if (warp == 9) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idesc = tc8_idesc(128, kN);
            uint32_t n = 0, acc_ph[2] = {0, 0};
            int buf = 0;
            bool any = false, ok = true;
            for (int r = 0; ok && snake(blockIdx.x, r) < ntask; ++r) {
                if (!task_ok(task_desc(p, sh, 0, r))) break;
                if (!(*abort == 0 && bar_wait_or_abort(acc_empty + buf, acc_ph[buf] ^ 1u, kBulkWaitCycles, abort))) {
                    ok = false;
                    break;
                }
                tc8_fence_after();
                const uint32_t d = tmem + buf * kN;
                for (int c = 0; c < nch; ++c, ++n) {
                    const int s = n % kXStages, sa = n % kTc8AStages;
                    if (!(*abort == 0 && bar_wait_or_abort(xfull + s, (n / kXStages) & 1, kBulkWaitCycles, abort) &&
                          bar_wait_or_abort(a_full + sa, (n / kTc8AStages) & 1, kBulkWaitCycles, abort))) {
                        ok = false;
                        break;
                    }
                    tc8_fence_after();
                    const uint32_t xs = smem_addr(xring + (size_t)s * kXBytes);
                    const uint32_t acol = tmem + Cfg::kACol0 + sa * kTc8ACols;
#pragma unroll
                    for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc8_mma(d, acol + kb * 32 + kk * 8, tc8_desc_sw128(xs + kb * (kN * 128) + kk * 32), idesc,
                                    (c | kb | kk) != 0);
                    any = true;
                    tc8_commit(xempty + s);
                    tc8_commit(a_empty + sa);
                }
                if (!ok) break;
                tc8_commit(acc_full + buf);
                acc_ph[buf] ^= 1u;
                buf ^= 1;
            }
            if (!ok && !*abort) *abort = 1;
            if (any) {  // every MMA issued is complete before tensor memory is freed
                tc8_commit(drain);
                bar_wait(drain, 0, kBulkWaitCycles);
            }
        }
    } else if (warp < 8) {
        // ---------------- converters: int4 codes -> int8 A rows in tensor memory ----------------
        // warp w writes TMEM lanes 32 (w % 4) .. + 31, the K half w / 4 of the
        // 256-wide chunk (32 columns of 4 bytes); lane l's row m = 32 (w % 4) + l
        // is gate row m / 2 (m even) or up row m / 2 (m odd) of the task
        const int quarter = warp & 3, kh = warp >> 2;
        const int m = quarter * 32 + lane, i = m >> 1;
        const uint32_t roff = (uint32_t)((m & 1) ? kTmaWBytes / 2 : 0) + (uint32_t)i * kTmaRowBytes;
        const uint32_t tlane = tmem + ((uint32_t)(quarter * 32) << 16) + Cfg::kACol0 + kh * 32;
        uint32_t n = 0;
        for (int r = 0; snake(blockIdx.x, r) < ntask; ++r) {
            if (!task_ok(task_desc(p, sh, 0, r))) break;
            bool ok = true;
            for (int c = 0; c < nch; ++c, ++n) {
                const int s = n % kStages, sa = n % kTc8AStages;
                if (!tc8_warp_wait(full + s, (n / kStages) & 1, abort) ||
                    !tc8_warp_wait(a_empty + sa, ((n / kTc8AStages) & 1) ^ 1u, abort)) {
                    ok = false;
                    break;
                }
                tc8_fence_after();
                const uint32_t wrow = smem_addr(wring + (size_t)s * kTmaWBytes) + roff;
                uint32_t o[32];
#pragma unroll
                for (int j = 0; j < 4; ++j) {  // 16-byte chunk 4 kh + j of the row (swizzled)
                    uint4 w;
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w)
                                 : "r"(wrow + ((((uint32_t)(4 * kh + j)) ^ (uint32_t)(i & 7)) << 4)));
                    o[8 * j + 0] = lo8(w.x); o[8 * j + 1] = hi8(w.x);
                    o[8 * j + 2] = lo8(w.y); o[8 * j + 3] = hi8(w.y);
                    o[8 * j + 4] = lo8(w.z); o[8 * j + 5] = hi8(w.z);
                    o[8 * j + 6] = lo8(w.w); o[8 * j + 7] = hi8(w.w);
                }
                asm volatile(
                    "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
                    "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n"
                    "tcgen05.wait::st.sync.aligned;\n" ::"r"(tlane + sa * kTc8ACols),
                    "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3]), "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7]), "r"(o[8]),
                    "r"(o[9]), "r"(o[10]), "r"(o[11]), "r"(o[12]), "r"(o[13]), "r"(o[14]), "r"(o[15]), "r"(o[16]),
                    "r"(o[17]), "r"(o[18]), "r"(o[19]), "r"(o[20]), "r"(o[21]), "r"(o[22]), "r"(o[23]), "r"(o[24]),
                    "r"(o[25]), "r"(o[26]), "r"(o[27]), "r"(o[28]), "r"(o[29]), "r"(o[30]), "r"(o[31])
                    : "memory");
                tc8_fence_before();
                __syncwarp();
                if (lane == 0) {
                    bar_arrive(a_full + sa);
                    bar_arrive(empty + s);  // this warp is done with the stage's weights
                }
            }
            if (!ok) break;
        }
    } else {
        // ---------------- epilogue: a lane quarter each (rows 32 q .. 32 q + 31) ----------------
        const int quarter = warp & 3;
        const int m = quarter * 32 + lane, i = m >> 1;
        const bool up = m & 1;
        if ((p.flags & kFlagTestStall) && warp == 10 && lane == 0) {  // a wait that runs out: the timeout path
            stall_on_unset_flag(never, kStallCycles);
            *abort = 1;
            atomicOr(status, ST_TIMEOUT);
        }
        uint32_t acc_ph[2] = {0, 0};
        int buf = 0;
        for (int r = 0; snake(blockIdx.x, r) < ntask; ++r) {
            const TaskDesc d = task_desc(p, sh, 0, r);
            if (!task_ok(d)) {
                if (warp == 10 && lane == 0) atomicOr(status, ST_BAD_TASK);
                break;
            }
            const bool shared = d.e == p.E;
            const int irow = shared ? p.Is : p.I;
            const float* S = shared ? p.sh_s13 : p.s13 + (size_t)d.e * 2 * p.I;
            const float rs = __ldg(S + (up ? irow : 0) + d.rbk * kRows13 + i);
            // token j's activation scale / 16 (the weights are 16 c), on lane j
            float xsc_l = 0.f;
            if (lane < d.nc) {
                const int tok = slot_token(p, sh, shared, d.off, d.tok0 + lane);
                xsc_l = (tok >= 0 && tok < p.T) ? __ldcg(p.xs + tok) * 0.0625f : 0.f;
            }
            const bool got = tc8_warp_wait(acc_full + buf, acc_ph[buf], abort);
            if (lane == 0) ep_ok[quarter] = got;
            asm volatile("bar.sync 2, 128;" ::: "memory");  // every epilogue warp's outcome is known
            if (!(ep_ok[0] && ep_ok[1] && ep_ok[2] && ep_ok[3])) break;
            tc8_fence_after();
            const int slot0 = (shared ? 0 : d.off) + d.tok0;
            float* hcol = (shared ? p.h32_s : p.h32_r) + (size_t)slot0 * irow + d.rbk * kRows13 + i;
            const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + buf * kN;
#pragma unroll
            for (int c0 = 0; c0 < kN; c0 += 32) {  // tokens c0 / 2 .. c0 / 2 + 15
                uint32_t v[32];
                asm volatile(
                    "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                    "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
                    "tcgen05.wait::ld.sync.aligned;\n"
                    : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                      "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
                      "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
                      "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
                      "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
                    : "r"(tbase + c0)
                    : "memory");
#pragma unroll
                for (int jj = 0; jj < 16; jj += 2) {  // tokens j0 = c0/2 + jj and j0 + 1
                    const int j0 = c0 / 2 + jj;
                    const float x0 = __shfl_sync(0xffffffffu, xsc_l, j0 & 31);
                    const float x1 = __shfl_sync(0xffffffffu, xsc_l, (j0 + 1) & 31);
                    const float e0 = join((int)v[2 * jj], (int)v[2 * jj + 1]) * (rs * x0);
                    const float e1 = join((int)v[2 * jj + 2], (int)v[2 * jj + 3]) * (rs * x1);
                    // the gate lane takes token j0, the up lane token j0 + 1
                    const float recv = __shfl_xor_sync(0xffffffffu, up ? e0 : e1, 1);
                    const float gv = up ? recv : e0, uv = up ? e1 : recv;
                    const int j = up ? j0 + 1 : j0;
                    const float h = silu_mul(gv, uv);
                    float hm = 0.f;
                    if (j < d.nc) {
                        hcol[(size_t)j * irow] = h;
                        hm = fabsf(h);
                    }
                    // max over the warp's 16 features (lanes of the same parity)
                    hm = nanmax(hm, __shfl_xor_sync(0xffffffffu, hm, 2));
                    hm = nanmax(hm, __shfl_xor_sync(0xffffffffu, hm, 4));
                    hm = nanmax(hm, __shfl_xor_sync(0xffffffffu, hm, 8));
                    hm = nanmax(hm, __shfl_xor_sync(0xffffffffu, hm, 16));
                    if (lane < 2 && j < d.nc) hmx[quarter][j] = hm;
                }
            }
            tc8_fence_before();
            asm volatile("bar.sync 2, 128;" ::: "memory");  // the four warps' maxima are in
            if (warp == 10 && lane < d.nc) {
                const int nrb = irow / kRows13;
                const float mx = nanmax(nanmax(hmx[0][lane], hmx[1][lane]), nanmax(hmx[2][lane], hmx[3][lane]));
                (shared ? p.hmax_s : p.hmax_r)[(size_t)(slot0 + lane) * nrb + d.rbk] = mx;
            }
            __syncwarp();
            if (lane == 0) bar_arrive(acc_empty + buf);
            asm volatile("bar.sync 2, 128;" ::: "memory");  // hmx and ep_ok are read before the next task writes them
            acc_ph[buf] ^= 1u;
            buf ^= 1;
        }
    }
    __syncthreads();
    if (warp == 9) {
        tc8_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(Cfg::kTmemCols) : "memory");
    }
}

// One down task as this thread sees it: ng row groups of 128 rows starting
// at row0; in group m this thread streams rows row0 + 128 m + j0 + g and + 8.
struct Task2 {
    WStream w;  // this thread's rows of group 0, from the slice's first k block
    bool ok, shared;
    int e, off, irow, sl, k0, klen, tok0, nc, j0, row0, ng;
};

// Down task `local` of bucket (e, n, off).
__device__ __forceinline__ Task2 make2(const Params& p, int e, int n, int off, int local) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, q = lane & 3;
    Task2 t;
    t.ok = !(e < 0 || e > p.E || (e == p.E && p.Is == 0));
    t.shared = e == p.E;
    t.e = e;
    t.off = off;
    t.irow = t.shared ? p.Is : p.I;
    const int R = p.H / p.rows2, nsl = slices_of(t.irow);
    const int rbk = local % R, rest = local / R;
    t.sl = rest % nsl;
    const int c = rest / nsl;
    t.k0 = t.sl * kSliceK;
    t.klen = min(kSliceK, t.irow - t.k0);
    t.tok0 = c * p.chunk;
    t.nc = min(p.chunk, n - t.tok0);
    t.row0 = rbk * p.rows2;
    t.ng = p.rows2 / kRows2;
    t.j0 = warp * 16;
    const int row_bytes = t.irow / 2;
    const uint8_t* W = t.shared ? p.sh_w2 : p.w2 + (size_t)(t.ok ? e : 0) * p.H * row_bytes;
    t.w.ra = W + (size_t)(t.row0 + t.j0 + g) * row_bytes + t.k0 / 2 + q * 16;
    t.w.rb = W + (size_t)(t.row0 + t.j0 + g + 8) * row_bytes + t.k0 / 2 + q * 16;
    t.w.nkb = t.ok ? t.klen / 128 : 0;
    return t;
}

// Down task from its descriptor (no task: ok = false).
__device__ __forceinline__ Task2 task2_from(const Params& p, const TaskDesc& d) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, q = lane & 3;
    Task2 t{};
    if (d.e < 0) return t;
    t.ok = !(d.e > p.E || (d.e == p.E && p.Is == 0));
    t.shared = d.e == p.E;
    t.e = d.e;
    t.off = d.off;
    t.irow = t.shared ? p.Is : p.I;
    t.sl = d.sl;
    t.k0 = d.sl * kSliceK;
    t.klen = min(kSliceK, t.irow - t.k0);
    t.tok0 = d.tok0;
    t.nc = d.nc;
    t.row0 = d.rbk * p.rows2;
    t.ng = p.rows2 / kRows2;
    t.j0 = warp * 16;
    const int row_bytes = t.irow / 2;
    const uint8_t* W = t.shared ? p.sh_w2 : p.w2 + (size_t)(t.ok ? d.e : 0) * p.H * row_bytes;
    t.w.ra = W + (size_t)(t.row0 + t.j0 + g) * row_bytes + t.k0 / 2 + q * 16;
    t.w.rb = W + (size_t)(t.row0 + t.j0 + g + 8) * row_bytes + t.k0 / 2 + q * 16;
    t.w.nkb = t.ok ? t.klen / 128 : 0;
    return t;
}

__device__ __forceinline__ Task2 task2_r(const Params& p, const Shm& sh, int r) {
    return task2_from(p, task_desc(p, sh, 1, r));
}

// Issues the cp.async of task t's f32 slice of h (raw[j][k], k < klen), of
// its per-64-row maxima of |h| (sh.hmr) and of its row scales (rs), as one
// group.
__device__ __forceinline__ void fetch2(const Params& p, Shm& sh, const Task2& t, float* raw, float* rs) {
    const float* S = (t.shared ? p.sh_s2 : p.s2 + (size_t)t.e * p.H) + t.row0;
    for (int c = threadIdx.x; c < p.rows2 / 4; c += blockDim.x) cp_async16(rs + 4 * c, S + 4 * c);
    const float* hb = t.shared ? p.h32_s : p.h32_r;
    const float* hmb = t.shared ? p.hmax_s : p.hmax_r;
    const int nrb = t.irow / kRows13;
    const int slot0 = (t.shared ? 0 : t.off) + t.tok0;
    const int per = t.klen / 4;  // 16-byte chunks per token
    for (int c = threadIdx.x; c < t.nc * per; c += blockDim.x) {
        const int j = c / per, k4 = c - j * per;
        cp_async16(raw + j * kSliceK + k4 * 4, hb + (size_t)(slot0 + j) * t.irow + t.k0 + k4 * 4);
    }
    const int nb = t.klen / kRows13;
    for (int c = threadIdx.x; c < t.nc * nb; c += blockDim.x) {
        const int j = c / nb, r = c - j * nb;
        cp_async4(&sh.hmr[j][r], hmb + (size_t)(slot0 + j) * nrb + t.k0 / kRows13 + r);
    }
    cp_async_commit();
}

template <int NT>
__device__ __forceinline__ bool run2(Ring& ring, const Task2& tk, const WStream& nx, const float* rs, const Params& p,
                                     const uint8_t* xs, const Shm& sh) {
    const int g = (threadIdx.x & 31) >> 2, q = (threadIdx.x & 31) & 3;
    const size_t TK = (size_t)p.T * p.K;
    const size_t yrow0 = tk.shared ? TK * p.nsl_r + (size_t)tk.sl * p.T + tk.tok0 : (size_t)tk.sl * TK + tk.off + tk.tok0;
    const size_t group_bytes = (size_t)kRows2 * (tk.irow / 2);
    bool cont = false;
    for (int m = 0; m < tk.ng; ++m) {
        WStream cur = tk.w;
        cur.ra += m * group_bytes;
        cur.rb += m * group_bytes;
        WStream nxt = nx;
        if (m + 1 < tk.ng) {
            nxt = tk.w;
            nxt.ra += (m + 1) * group_bytes;
            nxt.rb += (m + 1) * group_bytes;
        }
        int acc[NT][4];
        cont = stream8<NT, false>(ring, cur, nxt, xs, kStride2, [](int) {}, acc);
        if (!cont && m + 1 < tk.ng) prime(ring, nxt);
        const int jr = m * kRows2 + tk.j0 + g;  // row of this thread within the task
        const float s_lo = rs[jr], s_hi = rs[jr + 8];
        float* y0 = p.y + yrow0 * p.H + tk.row0 + jr;
#pragma unroll
        for (int i = 0; i < NT; ++i) {
            const int j = 4 * i + q;
            if (j < tk.nc) {
                const float xsc = sh.xsc[j];
                float* yr = y0 + (size_t)j * p.H;
                yr[0] = join(acc[i][0], acc[i][1]) * (s_lo * xsc);
                yr[8] = join(acc[i][2], acc[i][3]) * (s_hi * xsc);
            }
        }
    }
    return cont;
}

__global__ void __launch_bounds__(256, 2) experts_w2_kernel(Params p) {
    extern __shared__ __align__(128) uint8_t dsm[];
    Shm& sh = *reinterpret_cast<Shm*>(dsm);
    uint8_t* xs = dsm + kShmBytes;
    float* raw = reinterpret_cast<float*>(xs + kRaw2Off);
    float* rs2 = reinterpret_cast<float*>(xs + kRs2Off);  // [task parity][row of the task]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    Ring ring;
    const int ns = p.Is > 0 ? (p.H / p.rows2) * chunks_of(p.T, p.chunk) * slices_of(p.Is) : 0;
    bool primed = false;
    const uint8_t* primed_ra = nullptr;
    if ((int)blockIdx.x < ns) {
        const Task2 t = make2(p, p.E, p.T, p.T * p.K, ns - 1 - (int)blockIdx.x);
        prime(ring, t.w);
        primed = true;
        primed_ra = t.w.ra;
    }
    if (p.Is > 0) prefetch_l2_slice(p.sh_w2, (size_t)p.H * p.Is / 2);
    pdl_wait();
    pdl_release();
    load_tables(p, p.ts2, &p.ctrl->tasks2, sh.tb, nullptr);
    precompute_tasks(p, sh, 1);
    const Tables& tb = sh.tb;
    Task2 cur = task2_r(p, sh, 0);
    if (primed && cur.w.ra != primed_ra) primed = false;
    if (cur.ok) fetch2(p, sh, cur, raw, rs2);
    for (int r = 0, lin = blockIdx.x; lin < tb.ntask; lin = snake(blockIdx.x, ++r)) {
        const Task2 nx = task2_r(p, sh, r + 1);
        if (!cur.ok) {  // a table entry out of range: flag it and stop
            if (threadIdx.x == 0) atomicOr(&p.ctrl->status, ST_BAD_TASK);
            break;
        }
        if (!primed) prime(ring, cur.w);
        const int nc = cur.nc, klen = cur.klen;
        cp_async_wait<0>();
        __syncthreads();  // cur's h slice and maxima are visible; the previous task is done with xs
        if (threadIdx.x < nc) {
            const int j = threadIdx.x;
            float m = 0.f;
            for (int r = 0; r < klen / kRows13; ++r) m = nanmax(m, sh.hmr[j][r]);
            const QScale qs = qscale(m);
            sh.qs[j] = qs;
            sh.xsc[j] = qs.s * 0.0625f;
        }
        __syncthreads();
        for (int j = warp; j < nc; j += 8) {
            const QScale qs = sh.qs[j];
            const float* src = raw + j * kSliceK;
            for (int gi = lane; gi < klen / 8; gi += 32) {
                const float4 a = *reinterpret_cast<const float4*>(src + 8 * gi);
                const float4 b2 = *reinterpret_cast<const float4*>(src + 8 * gi + 4);
                const float f[8] = {a.x, a.y, a.z, a.w, b2.x, b2.y, b2.z, b2.w};
                uint2 p0, p1;
                quant2x8(f, qs, p0, p1);
                *reinterpret_cast<uint2*>(xs + (2 * j) * kStride2 + 8 * gi) = p0;
                *reinterpret_cast<uint2*>(xs + (2 * j + 1) * kStride2 + 8 * gi) = p1;
            }
        }
        __syncthreads();  // staged; raw and hmr are free for the next task
        if (nx.ok) fetch2(p, sh, nx, raw, rs2 + ((r + 1) & 1) * kMaxRows2);
        const float* rs = rs2 + (r & 1) * kMaxRows2;
        switch ((2 * nc + 7) >> 3) {
            case 1: primed = run2<1>(ring, cur, nx.w, rs, p, xs, sh); break;
            case 2: primed = run2<2>(ring, cur, nx.w, rs, p, xs, sh); break;
            case 3: primed = run2<3>(ring, cur, nx.w, rs, p, xs, sh); break;
            default: primed = run2<4>(ring, cur, nx.w, rs, p, xs, sh); break;
        }
        cur = nx;
    }
}

// ---------------------------------------------------------------------------
// Down projection with a TMA weight ring (large H; I and Is multiples of 256):
// one CTA per SM, a producer warp and 8 consumer warps, as the TMA gate/up
// kernel.  A stage is one 256-wide k chunk of one 128-row group of the task
// (one TMA tile load of 128 rows x 128 bytes, 128-byte swizzle).  The
// consumers prefetch the next task's f32 h slice, maxima and row scales with
// cp.async and quantize the current task's slice in shared memory while the
// producer keeps the ring full.
// ---------------------------------------------------------------------------
constexpr size_t kW2MiscBytes = 256;
// Ring and staging for tasks of kChunk tokens (offsets from the ring's start).
// Down ring geometry for tasks of kChunk tokens and WB-bit codes: a stage is
// the 256-wide k chunk of 128 down rows (16 KiB of int4; 32 KiB of int8, two
// 128-byte-row tiles for k 0..127 and 128..255).
template <int kChunk, int WB>
struct Tma2 {
    static constexpr int kWBytes = kW2Bytes * WB / 4;
    static constexpr int kStages = WB == 4 ? (kChunk == kChunkTokens ? 8 : 6) : (kChunk == kChunkTokens ? 4 : 3);
    static constexpr size_t kXOff = (size_t)kStages * kWBytes;
    static constexpr size_t kRawOff = kXOff + (size_t)2 * kChunk * kStride2;
    static constexpr size_t kRsOff = kRawOff + (size_t)kChunk * kSliceK * 4;
    static constexpr size_t kSmem = kShmBytes + kW2MiscBytes + 1024 /* alignment */ + kRsOff + (size_t)2 * kMaxRows2 * 4;
    static_assert(kSmem <= 227 * 1024, "TMA down shared memory");
    static_assert(kRsOff - kXOff >= kBuildBytes, "table build scratch fits the activation and h staging");
};

__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// fetch2 for the 256 consumer threads.
__device__ __forceinline__ void fetch2c(const Params& p, Shm& sh, const Task2& t, float* raw, float* rs) {
    const int tid = threadIdx.x;
    const float* S = (t.shared ? p.sh_s2 : p.s2 + (size_t)t.e * p.H) + t.row0;
    for (int c = tid; c < p.rows2 / 4; c += 256) cp_async16(rs + 4 * c, S + 4 * c);
    const float* hb = t.shared ? p.h32_s : p.h32_r;
    const float* hmb = t.shared ? p.hmax_s : p.hmax_r;
    const int nrb = t.irow / kRows13;
    const int slot0 = (t.shared ? 0 : t.off) + t.tok0;
    const int per = t.klen / 4;
    for (int c = tid; c < t.nc * per; c += 256) {
        const int j = c / per, k4 = c - j * per;
        cp_async16(raw + j * kSliceK + k4 * 4, hb + (size_t)(slot0 + j) * t.irow + t.k0 + k4 * 4);
    }
    const int nb = t.klen / kRows13;
    for (int c = tid; c < t.nc * nb; c += 256) {
        const int j = c / nb, r = c - j * nb;
        cp_async4(&sh.hmr[j][r], hmb + (size_t)(slot0 + j) * nrb + t.k0 / kRows13 + r);
    }
    cp_async_commit();
}

template <int NT, int kStages, int WB>
__device__ __forceinline__ void consume2(const Task2& tk, uint32_t& n, uint64_t* full, uint64_t* empty,
                                         const uint8_t* wring, const uint8_t* xs, const float* rs, const Params& p,
                                         const Shm& sh, volatile int* abort, unsigned* status) {
    constexpr int kWBytes = kW2Bytes * WB / 4;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, q = lane & 3;
    constexpr int kSets = NT == 1 ? 2 : 1;
    const size_t TK = (size_t)p.T * p.K;
    const size_t yrow0 = tk.shared ? TK * p.nsl_r + (size_t)tk.sl * p.T + tk.tok0 : (size_t)tk.sl * TK + tk.off + tk.tok0;
    const int nkc = tk.klen / kTmaChunk;
    // rows warp*16 + g and + 8 of a 1024-byte aligned tile: 16-byte chunk j sits at j ^ g
    const int wa_row = (warp * 16 + g) * kTmaRowBytes, wb_row = wa_row + 8 * kTmaRowBytes;
    for (int m = 0; m < tk.ng; ++m) {
        int part[kSets][NT][4];
#pragma unroll
        for (int s = 0; s < kSets; ++s)
#pragma unroll
            for (int i = 0; i < NT; ++i) part[s][i][0] = part[s][i][1] = part[s][i][2] = part[s][i][3] = 0;
        for (int c = 0; c < nkc; ++c, ++n) {
            const int s = n % kStages;
            if (!*abort && !bar_wait_or_abort(full + s, (n / kStages) & 1, kBulkWaitCycles, abort)) {
                *abort = 1;
                if (lane == 0) atomicOr(status, ST_TIMEOUT);
            }
            const uint8_t* wt = wring + (size_t)s * kWBytes;
            const uint8_t* xt = xs + g * kStride2 + q * 32 + c * kTmaChunk;
#pragma unroll
            for (int kb = 0; kb < kTmaChunk / 128; ++kb) {
                if (WB == 4) {
                    const int off = ((kb * 4 + q) ^ g) << 4;
                    const uint4 wa = *reinterpret_cast<const uint4*>(wt + wa_row + off);
                    const uint4 wb = *reinterpret_cast<const uint4*>(wt + wb_row + off);
                    kblock8<NT, kSets>(wa, wb, xt + kb * 128, 8 * kStride2, part);
                } else {  // codes 32q .. 32q + 31 of block kb: 16-byte chunks 2q, 2q + 1 of tile kb
                    const uint8_t* tb = wt + kb * kW2Bytes;
                    const int o0 = ((2 * q) ^ g) << 4, o1 = ((2 * q + 1) ^ g) << 4;
                    kblock8_i8<NT, kSets>(*reinterpret_cast<const uint4*>(tb + wa_row + o0),
                                          *reinterpret_cast<const uint4*>(tb + wa_row + o1),
                                          *reinterpret_cast<const uint4*>(tb + wb_row + o0),
                                          *reinterpret_cast<const uint4*>(tb + wb_row + o1), xt + kb * 128, 8 * kStride2,
                                          part);
                }
            }
            __syncwarp();
            if (lane == 0) bar_arrive(empty + s);
        }
        const int jr = m * kRows2 + warp * 16 + g;  // row of this thread within the task
        const float s_lo = rs[jr], s_hi = rs[jr + 8];
        float* y0 = p.y + yrow0 * p.H + tk.row0 + jr;
#pragma unroll
        for (int i = 0; i < NT; ++i) {
            const int j = 4 * i + q;
            if (j < tk.nc) {
                const int a0 = part[0][i][0] + part[kSets - 1][i][0] * (kSets - 1);
                const int a1 = part[0][i][1] + part[kSets - 1][i][1] * (kSets - 1);
                const int a2 = part[0][i][2] + part[kSets - 1][i][2] * (kSets - 1);
                const int a3 = part[0][i][3] + part[kSets - 1][i][3] * (kSets - 1);
                const float xsc = sh.xsc[j];
                float* yr = y0 + (size_t)j * p.H;
                yr[0] = join(a0, a1) * (s_lo * xsc);
                yr[8] = join(a2, a3) * (s_hi * xsc);
            }
        }
    }
}

// The down weights of k chunk c (k0 the chunk's first code) of the 128 rows from
// `row` of `map`: expect the bytes, then the tile load(s): one 128 x 128-byte
// tile of int4, two of int8.
template <int WB>
__device__ __forceinline__ void issue_w2_chunk(const CUtensorMap* map, uint64_t* bar, uint8_t* dst, int k0, int row) {
    bar_expect_tx(bar, kW2Bytes * WB / 4);
    if (WB == 4) {
        tma_tile(dst, map, bar, k0 / 2, row);
    } else {
        tma_tile(dst, map, bar, k0, row);
        tma_tile(dst + kW2Bytes, map, bar, k0 + kTmaRowBytes, row);
    }
}

template <int kChunk, int WB>
__global__ void __launch_bounds__(kTmaThreads, 1)
    experts_w2_tma_kernel(const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_s, Params p) {
    using Cfg = Tma2<kChunk, WB>;
    constexpr int kStages = Cfg::kStages, kWBytes = Cfg::kWBytes;
    extern __shared__ __align__(128) uint8_t dsm[];
    Shm& sh = *reinterpret_cast<Shm*>(dsm);
    uint64_t* full = reinterpret_cast<uint64_t*>(dsm + kShmBytes);
    uint64_t* empty = full + kStages;
    volatile int* abort = reinterpret_cast<volatile int*>(empty + kStages);
    volatile int* never = abort + 1;  // nothing sets it (MOE_TEST_STALL)
    const uint32_t base_s = static_cast<uint32_t>(__cvta_generic_to_shared(dsm));
    const uint32_t ring_s = (base_s + (uint32_t)(kShmBytes + kW2MiscBytes) + 1023u) & ~1023u;
    uint8_t* wring = dsm + (ring_s - base_s);
    uint8_t* xs = wring + Cfg::kXOff;
    float* raw = reinterpret_cast<float*>(wring + Cfg::kRawOff);
    float* rs2 = reinterpret_cast<float*>(wring + Cfg::kRsOff);  // [task parity][row of the task]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool producer = warp == 8;
    unsigned* status = &p.ctrl->status;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            bar_init(full + i, 1);   // the tile load's arrival
            bar_init(empty + i, 8);  // one arrival per consumer warp
        }
        *abort = 0;
        *never = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    const int R = p.H / p.rows2, ng = p.rows2 / kRows2;
    // the shared expert's first task of this CTA, if its first task is one
    const int nsl_s = p.Is > 0 ? slices_of(p.Is) : 0;
    const int ns = p.Is > 0 ? R * chunks_of(p.T, p.chunk) * nsl_s : 0;
    const bool pre = (int)blockIdx.x < ns;
    int pre_rbk = 0, pre_sl = 0, pre_tok0 = 0, npre = 0;
    if (pre) {
        const int local = ns - 1 - (int)blockIdx.x, rest = local / R;
        pre_rbk = local % R;
        pre_sl = rest % nsl_s;
        pre_tok0 = (rest / nsl_s) * p.chunk;
        const int k0 = pre_sl * kSliceK, nkc = min(kSliceK, p.Is - k0) / kTmaChunk;
        npre = min(kStages, ng * nkc);
        if (producer && lane == 0)
            for (int i = 0; i < npre; ++i) {
                const int m = i / nkc, c = i - m * nkc;
                issue_w2_chunk<WB>(&tm_s, full + i, wring + (size_t)i * kWBytes, k0 + c * kTmaChunk,
                                   pre_rbk * p.rows2 + m * kRows2);
            }
    }
    if (p.Is > 0) prefetch_l2_slice(p.sh_w2, (size_t)p.H * p.Is * WB / 8);
    // Small batches can build the down tables from the router's outputs before
    // the wait: the router completed before the gate/up kernel that this one
    // waits for released it (scratch: the activation and h staging areas,
    // unused until the first task).
    const bool early = p.decode_groups > 0 && p.w2_tables_early;
    if (early) {
        build_tables_small(p, sh, reinterpret_cast<int*>(xs), 1);
        precompute_tasks(p, sh, 1);
    }
    pdl_wait();
    pdl_release();
    if (!early) {
        load_tables(p, p.ts2, &p.ctrl->tasks2, sh.tb, nullptr);
        precompute_tasks(p, sh, 1);
    }
    if (threadIdx.x == 0 && pre) {  // cannot fail with consistent tables
        const TaskDesc d = sh.td[0];
        if (!(d.e == p.E && d.rbk == pre_rbk && d.sl == pre_sl && d.tok0 == pre_tok0 &&
              sh.tb.ntask > (int)blockIdx.x)) {
            *abort = 1;
            atomicOr(status, ST_BAD_TASK);
        }
    }
    __syncthreads();
    const int ntask = sh.tb.ntask;
    if (!producer && *abort) return;
    if (producer) {
        uint32_t n = 0;
        int last_round[kStages];
#pragma unroll
        for (int s = 0; s < kStages; ++s) last_round[s] = s < npre ? 0 : -1;
        for (int r = 0; !*abort && snake(blockIdx.x, r) < ntask; ++r) {
            const TaskDesc d = task_desc(p, sh, 1, r);
            if (d.e < 0 || d.e > p.E || (d.e == p.E && p.Is == 0)) break;  // the consumers flag it
            const bool shared = d.e == p.E;
            const int irow = shared ? p.Is : p.I;
            const int k0 = d.sl * kSliceK, nkc = min(kSliceK, irow - k0) / kTmaChunk;
            const int row0 = (shared ? 0 : d.e * p.H) + d.rbk * p.rows2;
            const CUtensorMap* map = shared ? &tm_s : &tm_r;
            bool stop = false;
            for (int m = 0; m < ng && !stop; ++m)
                for (int c = 0; c < nkc; ++c, ++n) {
                    const int s = n % kStages;
                    const int round = (int)(n / kStages);
                    if (round > 0) {
                        const bool ok =
                            *abort == 0 && bar_wait_or_abort(empty + s, (round - 1) & 1, kBulkWaitCycles, abort);
                        if (__any_sync(0xffffffffu, !ok)) {
                            if (lane == 0 && !*abort) atomicOr(status, ST_TIMEOUT);
                            *abort = 1;
                            stop = true;
                            break;
                        }
                    }
                    if (lane == 0 && !(r == 0 && (int)n < npre))
                        issue_w2_chunk<WB>(map, full + s, wring + (size_t)s * kWBytes, k0 + c * kTmaChunk, row0 + m * kRows2);
                    last_round[s] = round;
                }
        }
        // copies nobody will consume land before the CTA exits
        if (*abort && lane == 0)
            for (int s = 0; s < kStages; ++s)
                if (last_round[s] >= 0) bar_wait(full + s, last_round[s] & 1, kBulkWaitCycles);
        __syncwarp();
        return;
    }
    // consumers
    if ((p.flags & kFlagTestStall) && threadIdx.x == 0) {  // a wait that runs out: take the timeout path
        stall_on_unset_flag(never, kStallCycles);
        *abort = 1;
        atomicOr(status, ST_TIMEOUT);
    }
    uint32_t n = 0;
    Task2 cur = task2_r(p, sh, 0);
    if (cur.ok) fetch2c(p, sh, cur, raw, rs2);
    for (int r = 0; snake(blockIdx.x, r) < ntask; ++r) {
        const Task2 nx = task2_r(p, sh, r + 1);
        if (!cur.ok) {
            if (threadIdx.x == 0) atomicOr(status, ST_BAD_TASK);
            break;
        }
        const int nc = cur.nc, klen = cur.klen;
        cp_async_wait<0>();
        consumers_sync();  // cur's h slice and maxima are visible; the previous task is done with xs
        if (threadIdx.x < nc) {
            const int j = threadIdx.x;
            float m = 0.f;
            for (int b = 0; b < klen / kRows13; ++b) m = nanmax(m, sh.hmr[j][b]);
            const QScale qs = qscale(m);
            sh.qs[j] = qs;
            sh.xsc[j] = qs.s * code_unit<WB>();
        }
        consumers_sync();
        for (int j = warp; j < nc; j += 8) {
            const QScale qs = sh.qs[j];
            const float* src = raw + j * kSliceK;
            for (int gi = lane; gi < klen / 8; gi += 32) {
                const float4 a = *reinterpret_cast<const float4*>(src + 8 * gi);
                const float4 b2 = *reinterpret_cast<const float4*>(src + 8 * gi + 4);
                const float f[8] = {a.x, a.y, a.z, a.w, b2.x, b2.y, b2.z, b2.w};
                uint2 p0, p1;
                quant2x8(f, qs, p0, p1);
                *reinterpret_cast<uint2*>(xs + (2 * j) * kStride2 + 8 * gi) = p0;
                *reinterpret_cast<uint2*>(xs + (2 * j + 1) * kStride2 + 8 * gi) = p1;
            }
        }
        consumers_sync();  // staged; raw and hmr are free for the next task
        if (nx.ok) fetch2c(p, sh, nx, raw, rs2 + ((r + 1) & 1) * kMaxRows2);
        const float* rs = rs2 + (r & 1) * kMaxRows2;
        constexpr int kMaxNT = kChunk / 4;
#define MOE_CONSUME2(N) consume2<N, kStages, WB>(cur, n, full, empty, wring, xs, rs, p, sh, abort, status)
        switch ((2 * nc + 7) >> 3) {
            case 1: MOE_CONSUME2(1); break;
            case 2: MOE_CONSUME2(2); break;
            case 3: MOE_CONSUME2(3); break;
            case 4: MOE_CONSUME2(4); break;
            case 5: MOE_CONSUME2((kMaxNT > 4 ? 5 : 1)); break;
            case 6: MOE_CONSUME2((kMaxNT > 4 ? 6 : 1)); break;
            case 7: MOE_CONSUME2((kMaxNT > 4 ? 7 : 1)); break;
            default: MOE_CONSUME2(kMaxNT); break;
        }
#undef MOE_CONSUME2
        cur = nx;
    }
    cp_async_wait<0>();
}

// The TMA-ring kernels serve hidden sizes from kTmaMinH on (measured faster
// than the bulk-copy gate/up and the register-ring down kernel there).
constexpr int kTmaMinH = 1024;
bool w13_tma(int H) { return H >= kTmaMinH && H % kTmaChunk == 0; }

template <typename Kern>
int resident(Kern kern, size_t smem, int which, int threads = 256) {
    static int cache[16][64];  // by kernel (`which`) and device
    static_assert(kSmem13Bulk <= 227 * 1024, "bulk gate/up shared memory");
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    int& c = cache[which][dev];
    if (c == 0) {
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        int per_sm = 0, sms = 0;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        c = (per_sm > 0 ? per_sm : 1) * (sms > 0 ? sms : 148);
    }
    return c;
}

}  // namespace

// Persistent grid of the weight-streaming kernels: the CTAs that fit at once
// (which: 0 gate/up, 1 down; int8w: int8 codes, TMA-ring kernels only).  Also
// sets the kernels' shared-memory limits.
int experts_resident_ctas(int which, int H, bool w2_tma, int chunk, bool int8w, bool occ2) {
    if (int8w) {
        if (which == 1)
            return chunk == kMaxChunk
                       ? resident(experts_w2_tma_kernel<kMaxChunk, 8>, Tma2<kMaxChunk, 8>::kSmem, 13, kTmaThreads)
                       : resident(experts_w2_tma_kernel<kChunkTokens, 8>, Tma2<kChunkTokens, 8>::kSmem, 12, kTmaThreads);
        return chunk == kMaxChunk
                   ? resident(experts_w13_tma_kernel<kMaxChunk, 8>, Tma13<kMaxChunk, 8>::kSmem, 11, kTmaThreads)
                   : resident(experts_w13_tma_kernel<kChunkTokens, 8>, Tma13<kChunkTokens, 8>::kSmem, 10, kTmaThreads);
    }
    if (which == 1) {
        if (!w2_tma) return resident(experts_w2_kernel, kSmem2, 3);
        return chunk == kMaxChunk ? resident(experts_w2_tma_kernel<kMaxChunk, 4>, Tma2<kMaxChunk, 4>::kSmem, 7, kTmaThreads)
                                  : resident(experts_w2_tma_kernel<kChunkTokens, 4>, Tma2<kChunkTokens, 4>::kSmem, 6,
                                             kTmaThreads);
    }
    if (w13_tma(H) && occ2 && chunk == kChunkTokens)
        return resident(experts_w13_tma_kernel<kChunkTokens, 4, 2>, Tma13<kChunkTokens, 4, 2>::kSmem, 14, kTmaThreads);
    if (w13_tma(H))
        return chunk == kMaxChunk
                   ? resident(experts_w13_tma_kernel<kMaxChunk, 4>, Tma13<kMaxChunk, 4>::kSmem, 8, kTmaThreads)
                   : resident(experts_w13_tma_kernel<kChunkTokens, 4>, Tma13<kChunkTokens, 4>::kSmem, 5, kTmaThreads);
    if (H <= kBulkMaxK) return resident(experts_w13_bulk_kernel, kSmem13Bulk, 4);
    return H <= kWholeMaxK ? resident(experts_w13_kernel<1>, kSmem13[1], 1)
                           : resident(experts_w13_kernel<2>, kSmem13[2], 2);
}

cudaError_t launch_experts_w13(const Params& p, int grid, cudaStream_t stream) {
    const dim3 g(grid), b(256);
    const bool int8w = (p.flags & kFlagWeightsInt8) != 0;
    if (int8w && !w13_tma(p.H)) return cudaErrorInvalidValue;  // the host routes such shapes elsewhere
    if (w13_tma(p.H)) {
        // routed gate/up rows [E*2I][H/2] (int8: [H]) and the shared expert's
        // [2Is][H/2] ([H]), tiles of 64 rows x 128 bytes (any valid map when
        // there is no shared expert)
        const int per = int8w ? 1 : 2;  // code elements per byte
        CUtensorMap tm_r, tm_s;
        const bool ok =
            encode_tensor_map_2d(&tm_r, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.w13, p.H / per, (uint64_t)p.E * 2 * p.I,
                                 kTmaRowBytes, kRows13, CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_tensor_map_2d(&tm_s, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.Is > 0 ? (const void*)p.sh_w13 : (const void*)p.w13,
                                 p.H / per, p.Is > 0 ? 2 * (uint64_t)p.Is : 2 * (uint64_t)kRows13, kTmaRowBytes, kRows13,
                                 CU_TENSOR_MAP_SWIZZLE_128B);
        if (!ok) return cudaErrorInvalidValue;
        if (int8w) {
            if (p.chunk == kMaxChunk)
                return launch_pdl(experts_w13_tma_kernel<kMaxChunk, 8>, g, dim3(kTmaThreads), Tma13<kMaxChunk, 8>::kSmem,
                                  stream, tm_r, tm_s, p);
            return launch_pdl(experts_w13_tma_kernel<kChunkTokens, 8>, g, dim3(kTmaThreads),
                              Tma13<kChunkTokens, 8>::kSmem, stream, tm_r, tm_s, p);
        }
        if (p.chunk == kMaxChunk && experts_w13_tc8(p.H, p.I, p.Is, p.T, p.K, p.E)) {
            // one CTA per SM, like the mma.sync kernel whose residency sized the grid
            // (this call also sets the kernel's shared-memory limit)
            if (resident(experts_w13_tc8_kernel<kMaxChunk>, Tc8<kMaxChunk>::kSmem, 9, kTc8Threads) < grid)
                return cudaErrorInvalidConfiguration;
            return launch_pdl(experts_w13_tc8_kernel<kMaxChunk>, g, dim3(kTc8Threads), Tc8<kMaxChunk>::kSmem, stream,
                              tm_r, tm_s, p);
        }
        if (p.chunk == kMaxChunk)
            return launch_pdl(experts_w13_tma_kernel<kMaxChunk, 4>, g, dim3(kTmaThreads), Tma13<kMaxChunk, 4>::kSmem,
                              stream, tm_r, tm_s, p);
        if (p.w13_occ2)
            return launch_pdl(experts_w13_tma_kernel<kChunkTokens, 4, 2>, g, dim3(kTmaThreads),
                              Tma13<kChunkTokens, 4, 2>::kSmem, stream, tm_r, tm_s, p);
        return launch_pdl(experts_w13_tma_kernel<kChunkTokens, 4>, g, dim3(kTmaThreads), Tma13<kChunkTokens, 4>::kSmem,
                          stream, tm_r, tm_s, p);
    }
    if (p.H <= kBulkMaxK) return launch_pdl(experts_w13_bulk_kernel, g, b, kSmem13Bulk, stream, p);
    if (p.H <= kWholeMaxK) return launch_pdl(experts_w13_kernel<1>, g, b, kSmem13[1], stream, p);
    return launch_pdl(experts_w13_kernel<2>, g, b, kSmem13[2], stream, p);
}

bool experts_w13_tma(int H) { return w13_tma(H); }

// Picks per routed expert (T*K/E, on average) from which the tcgen05 gate/up
// kernel runs on the large-batch streaming sequence: measured on the
// 6144-hidden 256-expert layer, it takes 1.06-1.10 ms at 16 picks per expert
// against 1.22 ms for the mma.sync kernel, and 0.72 / 0.61 ms at 6 and 2.5
// (against 0.64 / 0.38 ms).
constexpr int kTc8MinPicksPerExpert = 12;

bool experts_w13_tc8(int H, int I, int Is, int T, int K, int E) {
    return w13_tma(H) && experts_w2_tma(H, I, Is) && (long long)T * K >= (long long)kTc8MinPicksPerExpert * E;
}

bool experts_w2_tma(int H, int I, int Is) { return H >= kTmaMinH && I % kTmaChunk == 0 && Is % kTmaChunk == 0; }

cudaError_t launch_experts_w2(const Params& p, int grid, cudaStream_t stream) {
    const bool int8w = (p.flags & kFlagWeightsInt8) != 0;
    if (int8w && !experts_w2_tma(p.H, p.I, p.Is)) return cudaErrorInvalidValue;  // routed elsewhere by the host
    if (experts_w2_tma(p.H, p.I, p.Is)) {
        // routed down rows [E*H][I/2] (int8: [I]) and the shared expert's
        // [H][Is/2] ([Is]), tiles of 128 rows x 128 bytes (any valid map when
        // there is no shared expert)
        const int per = int8w ? 1 : 2;  // code elements per byte
        CUtensorMap tm_r, tm_s;
        const bool ok =
            encode_tensor_map_2d(&tm_r, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.w2, p.I / per, (uint64_t)p.E * p.H,
                                 kTmaRowBytes, kRows2, CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_tensor_map_2d(&tm_s, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.Is > 0 ? (const void*)p.sh_w2 : (const void*)p.w2,
                                 p.Is > 0 ? p.Is / per : p.I / per, p.H, kTmaRowBytes, kRows2, CU_TENSOR_MAP_SWIZZLE_128B);
        if (!ok) return cudaErrorInvalidValue;
        const dim3 g(grid), b(kTmaThreads);
        if (int8w)
            return p.chunk == kMaxChunk
                       ? launch_pdl(experts_w2_tma_kernel<kMaxChunk, 8>, g, b, Tma2<kMaxChunk, 8>::kSmem, stream, tm_r, tm_s, p)
                       : launch_pdl(experts_w2_tma_kernel<kChunkTokens, 8>, g, b, Tma2<kChunkTokens, 8>::kSmem, stream,
                                    tm_r, tm_s, p);
        return p.chunk == kMaxChunk
                   ? launch_pdl(experts_w2_tma_kernel<kMaxChunk, 4>, g, b, Tma2<kMaxChunk, 4>::kSmem, stream, tm_r, tm_s, p)
                   : launch_pdl(experts_w2_tma_kernel<kChunkTokens, 4>, g, b, Tma2<kChunkTokens, 4>::kSmem, stream, tm_r,
                                tm_s, p);
    }
    return launch_pdl(experts_w2_kernel, dim3(grid), dim3(256), kSmem2, stream, p);
}

}  // namespace moe
