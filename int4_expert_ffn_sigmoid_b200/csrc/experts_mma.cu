// Weight-streaming expert kernels (gate/up + SwiGLU, then down) for the
// int4 per-row-symmetric SwiGLU experts and the shared expert.
//
// Method: colibri README (project listing), "What's implemented": packed int4
// with per-row scales, dequant-on-use, batch-union MoE (each expert touched
// by the batch is read once and applied to all of its tokens);
// nanocolibri-engine README, "Converting a checkpoint yourself": per-row
// symmetric int4, f32 row scales.
//
// Design.  One CTA (8 warps) owns one task = (bucket, chunk of up to 16 of the
// bucket's tokens, block of rows: 64 gate rows + the same 64 up rows, or 128
// down rows) and walks the reduction dimension in 128-wide k blocks.  The
// grid is persistent; CTA c takes tasks c, c + grid, ... counted from the
// heaviest end of the task list (the shared expert's tasks come last in it).
// The bucket and task tables are copied to shared memory once per CTA.
//  - Weights go HBM -> registers: every thread streams 16 contiguous bytes
//    (32 codes) of two rows per k block with non-allocating 128-bit loads,
//    kept 4 k blocks ahead in a register ring.  They never touch shared
//    memory.
//  - The chunk's activations (x rows, or h rows for the down projection) are
//    staged in shared memory with cp.async: the whole reduction range at once
//    when it fits (one barrier per task), else through a 4-deep ring of
//    128-wide slices.  Rows are padded by 16 bytes so that the per-thread
//    16-byte fragment reads are conflict-free.
//  - Codes are unpacked to exact 16-bit integers in natural order and feed
//    mma.sync m16n8k16 with the tokens as the n dimension; thread q's 16-byte
//    chunk is exactly its A fragments over two k steps, and the matching
//    activation chunk is exactly its B fragments.  The four 32-bit words of a
//    chunk accumulate into four independent accumulator sets (summed at the
//    end), so consecutive mma never wait on each other.  The row scale is
//    applied to the f32 result (it factors out of the row's dot product).
//  - Gate/up: the 16 mma rows are 8 gate rows and the same 8 up rows, so each
//    thread ends with gate and up of the same (row, token) and applies SwiGLU
//    in registers.
#include "moe_common.cuh"
#include "moe_launch.h"

namespace moe {

namespace {

constexpr int kRows13 = 64;  // gate (and up) rows per CTA task
constexpr int kRows2 = 128;  // down rows per CTA task
constexpr int kRing = 4;     // weight k blocks in flight per thread
constexpr int kXRing = 4;    // staged activation slices (ring mode)
constexpr int kPad = 8;      // 16-bit elements of padding per staged row
constexpr int kTiles = kChunkTokens / 8;
constexpr int kTab = kMaxE + 2;  // entries of each shared-memory table

// Activation staging capacity of the whole-range mode (elements per row).
constexpr int kWholeMaxK = 2048;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
                 "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Shared-memory copy of the bucket and task lists of one kernel.
struct Tables {
    int n_buckets, ntask;
    int e[kTab], n[kTab], off[kTab], ts[kTab];
};

__device__ __forceinline__ void load_tables(const Params& p, const int32_t* ts, int ntask_field, Tables& tb) {
    const int nb = p.ctrl->n_buckets;
    for (int i = threadIdx.x; i <= nb; i += blockDim.x) {
        tb.ts[i] = ts[i];
        if (i < nb) {
            tb.e[i] = p.bucket_e[i];
            tb.n[i] = p.bucket_n[i];
            tb.off[i] = p.bucket_off[i];
        }
    }
    if (threadIdx.x == 0) {
        tb.n_buckets = nb;
        tb.ntask = ntask_field;
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

// Stage k blocks [kb_lo, kb_hi) of the chunk's rows (row j at xs + j*stride).
// Ring mode keeps slice kb at column (kb % kXRing) * 128, whole mode at kb * 128.
template <bool kWhole>
__device__ __forceinline__ void stage(uint16_t* xs, int stride, const uint16_t* const* rows, int n, int kb_lo,
                                      int kb_hi) {
    const int per_row = (kb_hi - kb_lo) * 16;  // 16-byte chunks per row
    for (int c = threadIdx.x; c < n * per_row; c += blockDim.x) {
        const int j = c / per_row, r = c - j * per_row;
        const int kb = kb_lo + (r >> 4), part = r & 15;
        const uint16_t* src = rows[j];
        const int col = (kWhole ? kb : kb % kXRing) * 128 + part * 8;
        if (src) cp_async16(xs + j * stride + col, src + kb * 128 + part * 8);
    }
}

// One k block: unpack this thread's 16 bytes of rows a and b, multiply with
// the staged activations of every n-tile.
template <bool kBf16>
__device__ __forceinline__ void kblock(const uint4& wa, const uint4& wb, const uint16_t* xs, int stride, int col0,
                                       int ntiles, float (&part)[4][kTiles][4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const uint32_t aw[4] = {wa.x, wa.y, wa.z, wa.w};
    const uint32_t bw[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        uint32_t PA[4], PB[4];
        int4x8_to_16<kBf16>(aw[w], PA);
        int4x8_to_16<kBf16>(bw[w], PB);
        const uint32_t s0[4] = {PA[0], PB[0], PA[1], PB[1]};
        const uint32_t s1[4] = {PA[2], PB[2], PA[3], PB[3]};
#pragma unroll
        for (int i = 0; i < kTiles; ++i) {
            if (i < ntiles) {
                const uint4 xv = *reinterpret_cast<const uint4*>(xs + (8 * i + g) * stride + col0 + q * 32 + w * 8);
                if (kBf16) {
                    mma_bf16(part[w][i], s0, xv.x, xv.y);
                    mma_bf16(part[w][i], s1, xv.z, xv.w);
                } else {
                    mma_f16(part[w][i], s0, xv.x, xv.y);
                    mma_f16(part[w][i], s1, xv.z, xv.w);
                }
            }
        }
    }
}

// Main loop of both projections: this thread streams 16 bytes of rows ra
// (mma row g) and rb (mma row g + 8) per k block; on return acc[i] holds
// weights x activations of n-tile i.
template <bool kBf16, bool kWhole>
__device__ __forceinline__ void stream_rows(const uint8_t* ra, const uint8_t* rb, int nkb, uint16_t* xs, int stride,
                                            const uint16_t* const* rows, int nc, int ntiles,
                                            float (&acc)[kTiles][4]) {
    float part[4][kTiles][4];
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
        for (int i = 0; i < kTiles; ++i) part[w][i][0] = part[w][i][1] = part[w][i][2] = part[w][i][3] = 0.f;
    uint4 ring_a[kRing], ring_b[kRing];
#pragma unroll
    for (int i = 0; i < kRing; ++i) {
        ring_a[i] = i < nkb ? ld_stream_v4(ra + i * 64) : make_uint4(0, 0, 0, 0);
        ring_b[i] = i < nkb ? ld_stream_v4(rb + i * 64) : make_uint4(0, 0, 0, 0);
    }
    if (kWhole) {
        stage<true>(xs, stride, rows, nc, 0, nkb);
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
    } else {
#pragma unroll
        for (int i = 0; i < kXRing - 1; ++i) {
            if (i < nkb) stage<false>(xs, stride, rows, nc, i, i + 1);
            cp_async_commit();
        }
    }
    for (int kb0 = 0; kb0 < nkb; kb0 += kRing) {
#pragma unroll
        for (int rr = 0; rr < kRing; ++rr) {
            const int kb = kb0 + rr;
            if (kb < nkb) {
                if (!kWhole) {
                    cp_async_wait<kXRing - 2>();
                    __syncthreads();  // slice kb visible to all; slice kb-1's readers are done
                    if (kb + kXRing - 1 < nkb) stage<false>(xs, stride, rows, nc, kb + kXRing - 1, kb + kXRing);
                    cp_async_commit();
                }
                const uint4 wa = ring_a[rr], wb = ring_b[rr];
                if (kb + kRing < nkb) {
                    ring_a[rr] = ld_stream_v4(ra + (kb + kRing) * 64);
                    ring_b[rr] = ld_stream_v4(rb + (kb + kRing) * 64);
                }
                kblock<kBf16>(wa, wb, xs, stride, (kWhole ? kb : kb % kXRing) * 128, ntiles, part);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kTiles; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][c] = (part[0][i][c] + part[1][i][c]) + (part[2][i][c] + part[3][i][c]);
}

// Per-task data of the epilogue, loaded before the main loop: the h-scale
// exponent of each token column this thread owns.
__device__ __forceinline__ void load_hexp(const Params& p, bool shared, int off, int tok0, int n,
                                          int (&hx)[2 * kTiles]) {
    const int q = (threadIdx.x & 31) & 3;
#pragma unroll
    for (int i = 0; i < kTiles; ++i)
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int s = tok0 + 8 * i + 2 * q + cc;
            int t = -1;
            if (s < n) t = shared ? s : __ldg(p.tok_of_slot + off + s);
            hx[2 * i + cc] = (t >= 0 && t < p.T) ? __ldg(p.hexp + t) : 0;
        }
}

constexpr size_t kTabBytes = (sizeof(Tables) + 15) & ~size_t(15);

template <bool kWhole>
__global__ void __launch_bounds__(256, 2) experts_w13_kernel(Params p) {
    extern __shared__ __align__(16) uint8_t dsm[];
    Tables& tb = *reinterpret_cast<Tables*>(dsm);
    uint16_t* xs = reinterpret_cast<uint16_t*>(dsm + kTabBytes);
    __shared__ const uint16_t* rows[kChunkTokens];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int H = p.H, E = p.E;
    const int row_bytes = H / 2;
    const int nkb = H / 128;
    const int stride = (kWhole ? H : kXRing * 128) + kPad;
    // the shared expert's weights are needed whatever the routing: warm L2
    // while the router finishes
    if (p.Is > 0) prefetch_l2_slice(p.sh_w13, (size_t)p.Is * p.H);
    pdl_wait();
    pdl_release();
    load_tables(p, p.ts13, p.ctrl->tasks13, tb);
    for (int lin = blockIdx.x; lin < tb.ntask; lin += gridDim.x) {
        const int task = tb.ntask - 1 - lin;
        const int b = find_bucket(tb, task);
        const int e = tb.e[b], n = tb.n[b], off = tb.off[b];
        if (e < 0 || e > E || (e == E && p.Is == 0)) {
            if (threadIdx.x == 0) atomicOr(&p.ctrl->status, ST_BAD_TASK);
            continue;
        }
        const bool shared = (e == E);
        const int irow = shared ? p.Is : p.I;
        const int R = irow / kRows13;
        const int local = task - tb.ts[b];
        const int c = local / R, rbk = local - c * R;
        const int tok0 = c * kChunkTokens;
        const int nc = min(kChunkTokens, n - tok0);
        const int ntiles = (nc + 7) >> 3;
        const int r0 = rbk * kRows13 + warp * 8;
        const uint8_t* W = shared ? p.sh_w13 : p.w13 + (size_t)e * 2 * p.I * row_bytes;
        const float* S = shared ? p.sh_s13 : p.s13 + (size_t)e * 2 * p.I;
        const uint8_t* grow = W + (size_t)(r0 + g) * row_bytes + q * 16;
        const uint8_t* urow = W + (size_t)(irow + r0 + g) * row_bytes + q * 16;

        __syncthreads();  // the previous task is done with rows[] and xs
        for (int j = threadIdx.x; j < nc; j += blockDim.x) {
            const int t = shared ? tok0 + j : __ldg(p.tok_of_slot + off + tok0 + j);
            const bool ok = t >= 0 && t < p.T;
            if (!ok) atomicOr(&p.ctrl->status, ST_BAD_SLOT);
            rows[j] = ok ? reinterpret_cast<const uint16_t*>(p.x + (size_t)t * H) : nullptr;
        }
        int hx[2 * kTiles];
        load_hexp(p, shared, off, tok0, n, hx);
        const float gs = __ldg(S + r0 + g), us = __ldg(S + irow + r0 + g);
        __syncthreads();
        float acc[kTiles][4];
        stream_rows<true, kWhole>(grow, urow, nkb, xs, stride, rows, nc, ntiles, acc);

        __half* hb = shared ? p.h_s : p.h_r;
        const size_t hbase = shared ? 0 : (size_t)off;
#pragma unroll
        for (int i = 0; i < kTiles; ++i) {
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int s = tok0 + 8 * i + 2 * q + cc;
                if (i < ntiles && s < n) {
                    const float sc = ldexpf(1.0f, -hx[2 * i + cc]);
                    const float gv = acc[i][cc] * gs, uv = acc[i][2 + cc] * us;
                    hb[(hbase + s) * irow + r0 + g] = __float2half_rn(silu_mul(gv, uv) * sc);
                }
            }
        }
    }
}

template <bool kWhole>
__global__ void __launch_bounds__(256, 2) experts_w2_kernel(Params p) {
    extern __shared__ __align__(16) uint8_t dsm[];
    Tables& tb = *reinterpret_cast<Tables*>(dsm);
    uint16_t* hs = reinterpret_cast<uint16_t*>(dsm + kTabBytes);
    __shared__ const uint16_t* rows[kChunkTokens];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int H = p.H, E = p.E;
    const int R = H / kRows2;
    const int stride = (kWhole ? max(p.I, p.Is) : kXRing * 128) + kPad;
    if (p.Is > 0) prefetch_l2_slice(p.sh_w2, (size_t)p.H * p.Is / 2);
    pdl_wait();
    pdl_release();
    load_tables(p, p.ts2, p.ctrl->tasks2, tb);
    for (int lin = blockIdx.x; lin < tb.ntask; lin += gridDim.x) {
        const int task = tb.ntask - 1 - lin;
        const int b = find_bucket(tb, task);
        const int e = tb.e[b], n = tb.n[b], off = tb.off[b];
        if (e < 0 || e > E || (e == E && p.Is == 0)) {
            if (threadIdx.x == 0) atomicOr(&p.ctrl->status, ST_BAD_TASK);
            continue;
        }
        const bool shared = (e == E);
        const int irow = shared ? p.Is : p.I;
        const int row_bytes = irow / 2;
        const int nkb = irow / 128;
        const int local = task - tb.ts[b];
        const int c = local / R, rbk = local - c * R;
        const int tok0 = c * kChunkTokens;
        const int nc = min(kChunkTokens, n - tok0);
        const int ntiles = (nc + 7) >> 3;
        const int j0 = rbk * kRows2 + warp * 16;
        const uint8_t* W = shared ? p.sh_w2 : p.w2 + (size_t)e * H * row_bytes;
        const float* S = shared ? p.sh_s2 : p.s2 + (size_t)e * H;
        const uint8_t* lrow = W + (size_t)(j0 + g) * row_bytes + q * 16;
        const uint8_t* hrow8 = W + (size_t)(j0 + g + 8) * row_bytes + q * 16;
        const __half* hb = shared ? p.h_s : p.h_r;
        const size_t hbase = shared ? 0 : (size_t)off;

        __syncthreads();
        for (int j = threadIdx.x; j < nc; j += blockDim.x)
            rows[j] = reinterpret_cast<const uint16_t*>(hb + (hbase + tok0 + j) * irow);
        int hx[2 * kTiles];
        load_hexp(p, shared, off, tok0, n, hx);
        const float sl = __ldg(S + j0 + g), sh = __ldg(S + j0 + g + 8);
        __syncthreads();
        float acc[kTiles][4];
        stream_rows<false, kWhole>(lrow, hrow8, nkb, hs, stride, rows, nc, ntiles, acc);

#pragma unroll
        for (int i = 0; i < kTiles; ++i) {
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int s = tok0 + 8 * i + 2 * q + cc;
                if (i < ntiles && s < n) {
                    const float inv = ldexpf(1.0f, hx[2 * i + cc]);
                    const size_t ys = shared ? (size_t)p.T * p.K + s : (size_t)off + s;
                    float* yr = p.y + ys * H + j0 + g;
                    yr[0] = acc[i][cc] * (sl * inv);
                    yr[8] = acc[i][2 + cc] * (sh * inv);
                }
            }
        }
    }
}

template <typename Kern>
int resident(Kern kern, size_t smem, int which) {
    static int cache[4][64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    int& c = cache[which][dev];
    if (c == 0) {
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        int per_sm = 0, sms = 0;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        c = (per_sm > 0 ? per_sm : 1) * (sms > 0 ? sms : 148);
    }
    return c;
}

constexpr size_t kWholeSmem = kTabBytes + (size_t)kChunkTokens * (kWholeMaxK + kPad) * 2;
constexpr size_t kRingSmem = kTabBytes + (size_t)kChunkTokens * (kXRing * 128 + kPad) * 2;

}  // namespace

// Persistent grid of the weight-streaming kernels: the CTAs that fit at once
// (which: 0 gate/up, 1 down; kdim: its longest reduction range).
int experts_resident_ctas(int which, int kdim) {
    const bool whole = kdim <= kWholeMaxK;
    if (which == 0)
        return whole ? resident(experts_w13_kernel<true>, kWholeSmem, 0)
                     : resident(experts_w13_kernel<false>, kRingSmem, 1);
    return whole ? resident(experts_w2_kernel<true>, kWholeSmem, 2) : resident(experts_w2_kernel<false>, kRingSmem, 3);
}

cudaError_t launch_experts_w13(const Params& p, int grid, cudaStream_t stream) {
    if (p.H <= kWholeMaxK) return launch_pdl(experts_w13_kernel<true>, dim3(grid), dim3(256), kWholeSmem, stream, p);
    return launch_pdl(experts_w13_kernel<false>, dim3(grid), dim3(256), kRingSmem, stream, p);
}

cudaError_t launch_experts_w2(const Params& p, int grid, cudaStream_t stream) {
    if (max(p.I, p.Is) <= kWholeMaxK)
        return launch_pdl(experts_w2_kernel<true>, dim3(grid), dim3(256), kWholeSmem, stream, p);
    return launch_pdl(experts_w2_kernel<false>, dim3(grid), dim3(256), kRingSmem, stream, p);
}

}  // namespace moe
