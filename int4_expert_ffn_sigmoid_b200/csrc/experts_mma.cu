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
// down rows) and walks the reduction dimension in 128-wide k blocks.  CTAs
// are persistent and claim tasks from an atomic counter, heaviest (shared
// expert) first.
//  - Weights go HBM -> registers: every thread streams 16 contiguous bytes
//    (32 codes) of two rows per k block with non-allocating 128-bit loads,
//    kept 4 k blocks ahead in a register ring.  They never touch shared
//    memory.
//  - The chunk's activations (x rows, or h rows for the down projection) are
//    staged per k block in shared memory through a 4-deep cp.async ring,
//    padded so that the per-thread 16-byte fragment reads are conflict-free.
//  - Codes are unpacked to biased 16-bit integers 2^m + 8 + c (two
//    instructions per pair) and feed mma.sync m16n8k16 with the tokens as the
//    n dimension; thread q's 16-byte chunk is exactly its A fragments over two
//    k steps, and the matching activation chunk is exactly its B fragments.
//    Warp 0 also multiplies a ones matrix by the same fragments, which gives
//    each token's activation sum S; the epilogue removes the bias,
//    dot = acc - (2^m + 8) * S, then applies the row scale (the scale factors
//    out of the row's dot product).
//  - Gate/up: the 16 mma rows are 8 gate rows and the same 8 up rows, so each
//    thread ends with gate and up of the same (row, token) and applies SwiGLU
//    in registers.
#include "moe_common.cuh"
#include "moe_launch.h"

namespace moe {

namespace {

constexpr int kRows13 = 64;    // gate (and up) rows per CTA task
constexpr int kRows2 = 128;    // down rows per CTA task
constexpr int kRing = 4;       // weight k blocks in flight per thread
constexpr int kXRing = 4;      // staged activation k blocks (cp.async ring)
constexpr int kXStride = 136;  // 16-bit elements per staged row: 128 + 8 (16 bytes of padding)
constexpr int kTiles = kChunkTokens / 8;

__device__ __forceinline__ int find_bucket(const int32_t* ts, int nb, int task) {
    int lo = 0, hi = nb;  // ts[lo] <= task < ts[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(ts + mid) <= task) lo = mid; else hi = mid;
    }
    return lo;
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
                 "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_ring() {
    asm volatile("cp.async.wait_group %0;" ::"n"(kXRing - 2) : "memory");
}

// Claim the next task (thread 0 of the CTA, broadcast).  Tasks are handed out
// from the highest index down, so the shared expert's (last) tasks go first.
__device__ __forceinline__ int claim_task(int* counter, int ntask, int* s_task) {
    __syncthreads();  // everyone is done with the previous task's shared state
    if (threadIdx.x == 0) *s_task = ntask - 1 - atomicAdd(counter, 1);
    __syncthreads();
    return *s_task;
}

// Copy k block kb (128 elements) of the chunk's rows into a staging buffer.
// rows[j] points at row j's element 0 (null: not staged, left as is).
__device__ __forceinline__ void stage_slice(uint16_t (*buf)[kXStride], const uint16_t* const* rows, int n, int kb) {
    for (int c = threadIdx.x; c < n * 16; c += blockDim.x) {
        const int j = c >> 4, part = c & 15;
        const uint16_t* src = rows[j];
        if (src) cp_async16(&buf[j][part * 8], src + kb * 128 + part * 8);
    }
}

// The token of slot s of a bucket (shared bucket: slot index = token).
__device__ __forceinline__ int token_of(const Params& p, bool shared, int off, int s) {
    return shared ? s : __ldg(p.tok_of_slot + off + s);
}

// Main loop of both projections.  This thread streams 16 bytes of rows ra
// (mma row g) and rb (mma row g + 8) per k block; the CTA stages the chunk's
// activations.  acc[i] += biased weights x activations of n-tile i; warp 0
// also accumulates accS[i] += ones x activations.
template <bool kBf16>
__device__ __forceinline__ void stream_rows(const uint8_t* ra, const uint8_t* rb, int nkb,
                                            uint16_t (*xs)[kChunkTokens][kXStride],
                                            const uint16_t* const* rows, int nc, int ntiles, bool warp0,
                                            float (&acc)[kTiles][4], float (&accS)[kTiles][4]) {
    constexpr uint32_t kMagic = kBf16 ? kMagicBf16 : kMagicF16;
    constexpr uint32_t kOnes = kBf16 ? kOnesBf16 : kOnesF16;
    const uint32_t ones[4] = {kOnes, kOnes, kOnes, kOnes};
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int i = 0; i < kTiles; ++i) {
        acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
        accS[i][0] = accS[i][1] = accS[i][2] = accS[i][3] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < kXRing - 1; ++i) {
        if (i < nkb) stage_slice(xs[i], rows, nc, i);
        cp_async_commit();
    }
    uint4 ring_a[kRing], ring_b[kRing];
#pragma unroll
    for (int i = 0; i < kRing; ++i) {
        ring_a[i] = i < nkb ? ld_stream_v4(ra + i * 64) : make_uint4(0, 0, 0, 0);
        ring_b[i] = i < nkb ? ld_stream_v4(rb + i * 64) : make_uint4(0, 0, 0, 0);
    }
    for (int kb0 = 0; kb0 < nkb; kb0 += kRing) {
#pragma unroll
        for (int rr = 0; rr < kRing; ++rr) {
            const int kb = kb0 + rr;
            if (kb < nkb) {
                cp_async_wait_ring();
                __syncthreads();  // slice kb visible to all; slice kb-1's readers are done
                if (kb + kXRing - 1 < nkb) stage_slice(xs[(kb + kXRing - 1) % kXRing], rows, nc, kb + kXRing - 1);
                cp_async_commit();
                const uint4 wa = ring_a[rr], wb = ring_b[rr];
                if (kb + kRing < nkb) {
                    ring_a[rr] = ld_stream_v4(ra + (kb + kRing) * 64);
                    ring_b[rr] = ld_stream_v4(rb + (kb + kRing) * 64);
                }
                const uint32_t aw[4] = {wa.x, wa.y, wa.z, wa.w};
                const uint32_t bw[4] = {wb.x, wb.y, wb.z, wb.w};
                const uint16_t (*buf)[kXStride] = xs[kb % kXRing];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    uint32_t PA[4], PB[4];
                    int4x8_biased<kMagic>(aw[w], PA);
                    int4x8_biased<kMagic>(bw[w], PB);
                    const uint32_t s0[4] = {PA[0], PB[0], PA[1], PB[1]};
                    const uint32_t s1[4] = {PA[2], PB[2], PA[3], PB[3]};
#pragma unroll
                    for (int i = 0; i < kTiles; ++i) {
                        if (i < ntiles) {
                            const uint4 xv = *reinterpret_cast<const uint4*>(&buf[8 * i + g][q * 32 + w * 8]);
                            if (kBf16) {
                                mma_bf16(acc[i], s0, xv.x, xv.y);
                                mma_bf16(acc[i], s1, xv.z, xv.w);
                                if (warp0) {
                                    mma_bf16(accS[i], ones, xv.x, xv.y);
                                    mma_bf16(accS[i], ones, xv.z, xv.w);
                                }
                            } else {
                                mma_f16(acc[i], s0, xv.x, xv.y);
                                mma_f16(acc[i], s1, xv.z, xv.w);
                                if (warp0) {
                                    mma_f16(accS[i], ones, xv.x, xv.y);
                                    mma_f16(accS[i], ones, xv.z, xv.w);
                                }
                            }
                        }
                    }
                }
            }
        }
    }
}

// Warp 0 publishes the per-token activation sums of its accS (every row of
// the ones product holds them; lanes 0..3 own row 0).
__device__ __forceinline__ void publish_sums(const float (&accS)[kTiles][4], float* s_sum, bool warp0) {
    const int lane = threadIdx.x & 31;
    if (warp0 && lane < 4) {
#pragma unroll
        for (int i = 0; i < kTiles; ++i) {
            s_sum[8 * i + 2 * lane] = accS[i][0];
            s_sum[8 * i + 2 * lane + 1] = accS[i][1];
        }
    }
    __syncthreads();
}

}  // namespace

__global__ void __launch_bounds__(256, 3) experts_w13_kernel(Params p) {
    __shared__ __align__(16) uint16_t xs[kXRing][kChunkTokens][kXStride];
    __shared__ const uint16_t* rows[kChunkTokens];
    __shared__ float s_sum[kChunkTokens];
    __shared__ int s_task;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int ntask = p.ctrl->tasks13;
    const int nb = p.ctrl->n_buckets;
    const int H = p.H, E = p.E;
    const int row_bytes = H / 2;
    const int nkb = H / 128;
    for (int task = claim_task(&p.ctrl->claim13, ntask, &s_task); task >= 0;
         task = claim_task(&p.ctrl->claim13, ntask, &s_task)) {
        const int b = find_bucket(p.ts13, nb, task);
        const int e = __ldg(p.bucket_e + b);
        const int n = __ldg(p.bucket_n + b);
        const int off = __ldg(p.bucket_off + b);
        if (e < 0 || e > E || (e == E && p.Is == 0)) {
            if (threadIdx.x == 0) atomicOr(&p.ctrl->status, ST_BAD_TASK);
            continue;
        }
        const bool shared = (e == E);
        const int irow = shared ? p.Is : p.I;
        const int R = irow / kRows13;
        const int local = task - __ldg(p.ts13 + b);
        const int c = local / R, rbk = local - c * R;
        const int tok0 = c * kChunkTokens;
        const int nc = min(kChunkTokens, n - tok0);
        const int ntiles = (nc + 7) >> 3;
        const int r0 = rbk * kRows13 + warp * 8;
        const uint8_t* W = shared ? p.sh_w13 : p.w13 + (size_t)e * 2 * p.I * row_bytes;
        const float* S = shared ? p.sh_s13 : p.s13 + (size_t)e * 2 * p.I;
        const uint8_t* grow = W + (size_t)(r0 + g) * row_bytes + q * 16;
        const uint8_t* urow = W + (size_t)(irow + r0 + g) * row_bytes + q * 16;

        for (int j = threadIdx.x; j < nc; j += blockDim.x) {
            const int t = token_of(p, shared, off, tok0 + j);
            const bool ok = t >= 0 && t < p.T;
            if (!ok) atomicOr(&p.ctrl->status, ST_BAD_SLOT);
            rows[j] = ok ? reinterpret_cast<const uint16_t*>(p.x + (size_t)t * H) : nullptr;
        }
        __syncthreads();
        float acc[kTiles][4], accS[kTiles][4];
        stream_rows<true>(grow, urow, nkb, xs, rows, nc, ntiles, warp == 0, acc, accS);
        publish_sums(accS, s_sum, warp == 0);

        const float gs = __ldg(S + r0 + g), us = __ldg(S + irow + r0 + g);
        __half* hb = shared ? p.h_s : p.h_r;
        const size_t hbase = shared ? 0 : (size_t)off;
#pragma unroll
        for (int i = 0; i < kTiles; ++i) {
            if (i < ntiles) {
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int j = 8 * i + 2 * q + cc;  // token of the chunk
                    const int s = tok0 + j;
                    if (s < n) {
                        const int t = token_of(p, shared, off, s);
                        const float sc = ldexpf(1.0f, -__ldg(p.hexp + t));
                        const float sx = s_sum[j];
                        const float gv = fmaf(-kBiasBf16, sx, acc[i][cc]) * gs;
                        const float uv = fmaf(-kBiasBf16, sx, acc[i][2 + cc]) * us;
                        hb[(hbase + s) * irow + r0 + g] = __float2half_rn(silu_mul(gv, uv) * sc);
                    }
                }
            }
        }
    }
}

__global__ void __launch_bounds__(256, 3) experts_w2_kernel(Params p) {
    __shared__ __align__(16) uint16_t hs[kXRing][kChunkTokens][kXStride];
    __shared__ const uint16_t* rows[kChunkTokens];
    __shared__ float s_sum[kChunkTokens];
    __shared__ int s_task;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int ntask = p.ctrl->tasks2;
    const int nb = p.ctrl->n_buckets;
    const int H = p.H, E = p.E;
    const int R = H / kRows2;
    for (int task = claim_task(&p.ctrl->claim2, ntask, &s_task); task >= 0;
         task = claim_task(&p.ctrl->claim2, ntask, &s_task)) {
        const int b = find_bucket(p.ts2, nb, task);
        const int e = __ldg(p.bucket_e + b);
        const int n = __ldg(p.bucket_n + b);
        const int off = __ldg(p.bucket_off + b);
        if (e < 0 || e > E || (e == E && p.Is == 0)) {
            if (threadIdx.x == 0) atomicOr(&p.ctrl->status, ST_BAD_TASK);
            continue;
        }
        const bool shared = (e == E);
        const int irow = shared ? p.Is : p.I;
        const int row_bytes = irow / 2;
        const int nkb = irow / 128;
        const int local = task - __ldg(p.ts2 + b);
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

        for (int j = threadIdx.x; j < nc; j += blockDim.x)
            rows[j] = reinterpret_cast<const uint16_t*>(hb + (hbase + tok0 + j) * irow);
        __syncthreads();
        float acc[kTiles][4], accS[kTiles][4];
        stream_rows<false>(lrow, hrow8, nkb, hs, rows, nc, ntiles, warp == 0, acc, accS);
        publish_sums(accS, s_sum, warp == 0);

        const float sl = __ldg(S + j0 + g), sh = __ldg(S + j0 + g + 8);
#pragma unroll
        for (int i = 0; i < kTiles; ++i) {
            if (i < ntiles) {
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int j = 8 * i + 2 * q + cc;
                    const int s = tok0 + j;
                    if (s < n) {
                        const int t = token_of(p, shared, off, s);
                        const float inv = ldexpf(1.0f, __ldg(p.hexp + t));
                        const float hsum = s_sum[j];
                        const size_t ys = shared ? (size_t)p.T * p.K + s : (size_t)off + s;
                        float* yr = p.y + ys * H + j0 + g;
                        yr[0] = fmaf(-kBiasF16, hsum, acc[i][cc]) * (sl * inv);
                        yr[8] = fmaf(-kBiasF16, hsum, acc[i][2 + cc]) * (sh * inv);
                    }
                }
            }
        }
    }
}

int experts_resident_ctas(int which) {
    static int cache[2][64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    int& c = cache[which][dev];
    if (c == 0) {
        int per_sm = 0, sms = 0;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &per_sm, which == 0 ? (const void*)experts_w13_kernel : (const void*)experts_w2_kernel, 256, 0);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        c = (per_sm > 0 ? per_sm : 1) * (sms > 0 ? sms : 148);
    }
    return c;
}

cudaError_t launch_experts_w13(const Params& p, int grid, cudaStream_t stream) {
    experts_w13_kernel<<<grid, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_experts_w2(const Params& p, int grid, cudaStream_t stream) {
    experts_w2_kernel<<<grid, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace moe
