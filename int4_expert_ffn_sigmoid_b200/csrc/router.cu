// Router: logits x.W^T (f32), sigmoid scores, bias-for-selection top-k with
// normalised, scaled weights; then bucketing of the (token, k) slots by expert
// and the work lists of the expert kernels.
//
// Method: Colibri-Nano model card, "Architecture" (sigmoid+bias router,
// top-2 of 64 plus a shared expert); colibri README (project listing), "What's
// implemented" (DeepSeek-V3-style sigmoid router with routed_scaling_factor;
// batch-union MoE: every expert touched by the batch is read once for all of
// its tokens).
//
// Every logit is computed with one fixed arithmetic order whatever the batch
// size: lane l of a warp accumulates, with fused multiply-adds, the elements
// 128*i + 4*l + j (i ascending, then j = 0..3), and the 32 lane partials are
// summed by an xor-butterfly (16, 8, 4, 2, 1).  A token therefore gets the
// same bits from the small-batch and the large-batch router.
#include "moe_common.cuh"
#include "moe_launch.h"

namespace moe {

__device__ __forceinline__ float dot_step(float acc, uint2 xv, float4 wv) {
    acc = fmaf(bf16lo(xv.x), wv.x, acc);
    acc = fmaf(bf16hi(xv.x), wv.y, acc);
    acc = fmaf(bf16lo(xv.y), wv.z, acc);
    acc = fmaf(bf16hi(xv.y), wv.w, acc);
    return acc;
}

__device__ __forceinline__ float warp_sum_tree(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 16);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    return v;
}

// Exponent k_t of the token's h storage scale 2^-k_t (one warp):
// k_t = 8 + floor(log2(mean_h x[t,h]^2)), the mean square summed in the same
// lane order as the router logits.
__device__ __forceinline__ void token_hexp(const Params& p, int t, int lane) {
    const __nv_bfloat16* xr = p.x + (size_t)t * p.H;
    float acc = 0.f;
    for (int i = 0; i < p.H / 128; ++i) {
        const uint2 xv = __ldg(reinterpret_cast<const uint2*>(xr + i * 128 + lane * 4));
        const float a = bf16lo(xv.x), b = bf16hi(xv.x), c = bf16lo(xv.y), d = bf16hi(xv.y);
        acc = fmaf(a, a, acc);
        acc = fmaf(b, b, acc);
        acc = fmaf(c, c, acc);
        acc = fmaf(d, d, acc);
    }
    const float ms = warp_sum_tree(acc) / (float)p.H;
    const int e = (ms > 0.f && isfinite(ms)) ? ilogbf(ms) : 0;
    if (lane == 0) p.hexp[t] = min(max(kHExpBase + e, kHExpMin), kHExpMax);
}

// Top-K of one token (one warp).  Lane l holds experts l, l+32, ...  The key
// is sigmoid(L) + bias (NaN -> -inf); ties go to the lower expert index.  The
// weight of the k-th pick is scale * s_k / (s_0 + ... + s_{K-1}).
// Returns, on lanes k < K, the k-th selected expert (else -1).
template <bool kGlobalLogits>
__device__ int select_token(const Params& p, int t, const float* lg, int lane) {
    const int E = p.E, K = p.K;
    float key[kMaxE / 32], sc[kMaxE / 32];
#pragma unroll
    for (int j = 0; j < kMaxE / 32; ++j) {
        const int e = lane + 32 * j;
        key[j] = -INFINITY;
        sc[j] = 0.f;
        if (e < E) {
            const float L = kGlobalLogits ? __ldcg(lg + e) : lg[e];
            const float s = 1.0f / (1.0f + expf(-L));
            const float kk = s + __ldg(p.rb + e);
            key[j] = isnan(kk) ? -INFINITY : kk;
            sc[j] = s;
        }
    }
    unsigned taken = 0;
    int my_e = -1;
    float my_s = 0.f, ssum = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxK; ++k) {
        if (k >= K) break;
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
    if (lane < K) {
        const float w = p.scale * my_s / ssum;
        const size_t o = (size_t)t * K + lane;
        p.idx[o] = my_e;
        p.wts[o] = w;
        if (p.topk_idx_out) p.topk_idx_out[o] = my_e;
        if (p.topk_w_out) p.topk_w_out[o] = w;
    }
    return lane < K ? my_e : -1;
}

// Bucket list and task prefixes from the per-expert slot counts (one CTA of
// 256 threads).  s_off receives the first slot of every expert's bucket.
__device__ void finalize_buckets(const Params& p, const int* s_cnt, int* s_off) {
    __shared__ int s_nb, s_total;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int E = p.E;
    if (warp == 0) {
        int c[kMaxE / 32];
        int sum = 0, nz = 0;
#pragma unroll
        for (int j = 0; j < kMaxE / 32; ++j) {
            const int e = lane * (kMaxE / 32) + j;
            c[j] = e < E ? s_cnt[e] : 0;
            sum += c[j];
            nz += c[j] > 0;
        }
        int isum = sum, inz = nz;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int a = __shfl_up_sync(0xffffffffu, isum, o);
            const int b = __shfl_up_sync(0xffffffffu, inz, o);
            if (lane >= o) { isum += a; inz += b; }
        }
        int off = isum - sum, b = inz - nz;
#pragma unroll
        for (int j = 0; j < kMaxE / 32; ++j) {
            const int e = lane * (kMaxE / 32) + j;
            if (e < E) {
                s_off[e] = off;
                p.offsets[e] = off;
                p.counts[e] = c[j];
                if (c[j] > 0) {
                    p.bucket_e[b] = e;
                    p.bucket_n[b] = c[j];
                    p.bucket_off[b] = off;
                    ++b;
                }
                off += c[j];
            }
        }
        if (lane == 31) { s_total = isum; s_nb = inz; }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (s_total != p.T * p.K) atomicOr(&p.ctrl->status, ST_BAD_COUNT);
        int nb = s_nb;
        if (p.Is > 0) {
            p.bucket_e[nb] = E;
            p.bucket_n[nb] = p.T;
            p.bucket_off[nb] = p.T * p.K;
            ++nb;
        }
        s_nb = nb;
    }
    __syncthreads();
    if (warp == 0) {
        const int nb = s_nb;
        int base13 = 0, base2 = 0, baset1 = 0, baset2 = 0;
        for (int b0 = 0; b0 < nb; b0 += 32) {
            const int b = b0 + lane;
            int n13 = 0, n2 = 0, nt1 = 0, nt2 = 0;
            if (b < nb) {
                const int e = p.bucket_e[b];
                const int irow = (e == E) ? p.Is : p.I;
                const int n = p.bucket_n[b];
                const int ch = chunks_of(n);
                n13 = (irow / 64) * ch;   // CTA tasks: 64 gate/up rows x 64 tokens
                n2 = (p.H / 128) * ch;    // CTA tasks: 128 down rows x 64 tokens
                if (e != E) {  // tensor-core tiles: 128 tokens x 128 features / 256 columns
                    const int mt = (n + 127) / 128;
                    nt1 = mt * (p.I / 128);
                    nt2 = mt * (p.H / 256);
                }
            }
            int i13 = n13, i2 = n2, it1 = nt1, it2 = nt2;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int a = __shfl_up_sync(0xffffffffu, i13, o);
                const int c2 = __shfl_up_sync(0xffffffffu, i2, o);
                const int d1 = __shfl_up_sync(0xffffffffu, it1, o);
                const int d2 = __shfl_up_sync(0xffffffffu, it2, o);
                if (lane >= o) { i13 += a; i2 += c2; it1 += d1; it2 += d2; }
            }
            if (b < nb) {
                p.ts13[b] = base13 + i13 - n13;
                p.ts2[b] = base2 + i2 - n2;
                p.tcs1[b] = baset1 + it1 - nt1;
                p.tcs2[b] = baset2 + it2 - nt2;
            }
            base13 += __shfl_sync(0xffffffffu, i13, 31);
            base2 += __shfl_sync(0xffffffffu, i2, 31);
            baset1 += __shfl_sync(0xffffffffu, it1, 31);
            baset2 += __shfl_sync(0xffffffffu, it2, 31);
        }
        if (lane == 0) {
            p.ts13[nb] = base13;
            p.ts2[nb] = base2;
            p.tcs1[nb] = baset1;
            p.tcs2[nb] = baset2;
            p.ctrl->n_buckets = nb;
            p.ctrl->tasks13 = base13;
            p.ctrl->tasks2 = base2;
            p.ctrl->tc_tiles1 = baset1;
            p.ctrl->tc_tiles2 = baset2;
        }
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// Small batch (T <= kDecodeMaxTokens): grid (ceil(T/8), ceil(E/8)); warp w of
// CTA (bx, by) computes the logits of expert 8*by + w for tokens 8*bx ...
// 8*bx + 7.  The last CTA of each token block selects that block's tokens
// (one warp per token); the last of those counts, scans and scatters.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) router_small_kernel(Params p) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t0 = blockIdx.x * kDecodeRouterTok;
    const int e = blockIdx.y * kDecodeRouterExp + warp;
    const int nt = min(kDecodeRouterTok, p.T - t0);
    if (blockIdx.y == 0 && warp < nt) token_hexp(p, t0 + warp, lane);
    if (e < p.E) {
        float acc[kDecodeRouterTok];
#pragma unroll
        for (int tt = 0; tt < kDecodeRouterTok; ++tt) acc[tt] = 0.f;
        const float4* W = reinterpret_cast<const float4*>(p.rw + (size_t)e * p.H);
        const int nblk = p.H / 128;  // processed 4 blocks per batch of loads
        for (int i0 = 0; i0 < nblk; i0 += 4) {
            float4 wv[4];
            uint2 xv[4][kDecodeRouterTok];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u;
                wv[u] = i < nblk ? __ldg(W + i * 32 + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int tt = 0; tt < kDecodeRouterTok; ++tt)
                    xv[u][tt] = (i < nblk && tt < nt)
                                    ? __ldg(reinterpret_cast<const uint2*>(p.x + (size_t)(t0 + tt) * p.H + i * 128 + lane * 4))
                                    : make_uint2(0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (i0 + u < nblk) {
#pragma unroll
                    for (int tt = 0; tt < kDecodeRouterTok; ++tt) acc[tt] = dot_step(acc[tt], xv[u][tt], wv[u]);
                }
            }
        }
#pragma unroll
        for (int tt = 0; tt < kDecodeRouterTok; ++tt) {
            const float v = warp_sum_tree(acc[tt]);
            if (lane == 0 && tt < nt) p.logits[(size_t)(t0 + tt) * p.E + e] = v;
        }
    }

    // ---- last CTA of this token block: selection of its tokens
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(&p.ctrl->blk_done[blockIdx.x], 1u) == gridDim.y - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    __shared__ float s_lg[kDecodeRouterTok * kMaxE];
    for (int i = threadIdx.x; i < nt * p.E; i += blockDim.x) s_lg[i] = __ldcg(p.logits + (size_t)t0 * p.E + i);
    __syncthreads();
    if (warp < nt) {
        const int sel = select_token<false>(p, t0 + warp, s_lg + warp * p.E, lane);
        if (lane < p.K && (sel < 0 || sel >= p.E)) atomicOr(&p.ctrl->status, ST_BAD_EXPERT);
    }

    // ---- last token block: counts, scan, bucket and task lists, slots
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(&p.ctrl->sel_done, 1u) == gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    __shared__ int s_idx[kDecodeMaxTokens * kMaxK];
    __shared__ int s_cnt[kMaxE];
    __shared__ int s_off[kMaxE];
    const int TK = p.T * p.K;
    for (int i = threadIdx.x; i < p.E; i += blockDim.x) s_cnt[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < TK; i += blockDim.x) {
        int ex = __ldcg(p.idx + i);
        if (ex < 0 || ex >= p.E) ex = 0;  // reported above; keep every index in range
        s_idx[i] = ex;
        atomicAdd(&s_cnt[ex], 1);
    }
    __syncthreads();
    finalize_buckets(p, s_cnt, s_off);
    for (int i = threadIdx.x; i < TK; i += blockDim.x) {
        const int ex = s_idx[i];
        int rank = 0;
        for (int j = 0; j < i; ++j) rank += (s_idx[j] == ex);
        const int slot = s_off[ex] + rank;
        if (slot < 0 || slot >= TK) {
            atomicOr(&p.ctrl->status, ST_BAD_SLOT);
            p.slot_of[i] = 0;
            continue;
        }
        p.slot_of[i] = slot;
        p.tok_of_slot[slot] = i / p.K;
    }
}

// ---------------------------------------------------------------------------
// Large batch: router_blocks CTAs walk tiles of 16 tokens (tile = block,
// block + grid, ...).  Each tile's logits stay in shared memory; one warp per
// token selects; every CTA records its per-expert slot counts in hist.  The
// last CTA sums them, scans and builds the bucket and task lists.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) router_large_kernel(Params p) {
    __shared__ float s_logit[kRouterTileTokens][kMaxE];
    __shared__ int s_cnt[kMaxE];
    __shared__ int s_off[kMaxE];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int E = p.E, H = p.H;
    for (int i = threadIdx.x; i < E; i += blockDim.x) s_cnt[i] = 0;
    __syncthreads();
    const int ntiles = (p.T + kRouterTileTokens - 1) / kRouterTileTokens;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int t0 = tile * kRouterTileTokens;
        const int nt = min(kRouterTileTokens, p.T - t0);
        for (int tt = warp; tt < nt; tt += 8) token_hexp(p, t0 + tt, lane);
        for (int e0 = warp; e0 < E; e0 += 16) {
            const int e1 = e0 + 8;
            const bool has1 = e1 < E;
            float a0[kRouterTileTokens], a1[kRouterTileTokens];
#pragma unroll
            for (int tt = 0; tt < kRouterTileTokens; ++tt) { a0[tt] = 0.f; a1[tt] = 0.f; }
            const float4* W0 = reinterpret_cast<const float4*>(p.rw + (size_t)e0 * H);
            const float4* W1 = reinterpret_cast<const float4*>(p.rw + (size_t)(has1 ? e1 : e0) * H);
            for (int i = 0; i < H / 128; ++i) {
                const float4 w0 = __ldg(W0 + i * 32 + lane);
                const float4 w1 = __ldg(W1 + i * 32 + lane);
#pragma unroll
                for (int tt = 0; tt < kRouterTileTokens; ++tt) {
                    if (tt < nt) {
                        const uint2 xv = __ldg(reinterpret_cast<const uint2*>(
                            p.x + (size_t)(t0 + tt) * H + i * 128 + lane * 4));
                        a0[tt] = dot_step(a0[tt], xv, w0);
                        a1[tt] = dot_step(a1[tt], xv, w1);
                    }
                }
            }
#pragma unroll
            for (int tt = 0; tt < kRouterTileTokens; ++tt) {
                const float v0 = warp_sum_tree(a0[tt]);
                const float v1 = warp_sum_tree(a1[tt]);
                if (lane == 0 && tt < nt) {
                    s_logit[tt][e0] = v0;
                    if (has1) s_logit[tt][e1] = v1;
                }
            }
        }
        __syncthreads();
        for (int tt = warp; tt < nt; tt += 8) {
            const int sel = select_token<false>(p, t0 + tt, s_logit[tt], lane);
            if (lane < p.K) {
                if (sel >= 0 && sel < E) atomicAdd(&s_cnt[sel], 1);
                else atomicOr(&p.ctrl->status, ST_BAD_EXPERT);
            }
        }
        __syncthreads();
    }
    for (int i = threadIdx.x; i < E; i += blockDim.x) p.hist[(size_t)blockIdx.x * E + i] = s_cnt[i];

    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(&p.ctrl->done, 1u) == gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int c = 0;
        for (int b = 0; b < (int)gridDim.x; ++b) c += __ldcg(p.hist + (size_t)b * E + e);
        s_cnt[e] = c;
    }
    __syncthreads();
    finalize_buckets(p, s_cnt, s_off);
    if (threadIdx.x == 0) p.ctrl->done = 0;
}

// Large batch, second pass: CTA c walks the same tiles as router CTA c and
// assigns slots in (tile, token, k) order, after the slots of CTAs 0..c-1.
__global__ void __launch_bounds__(256) scatter_large_kernel(Params p) {
    __shared__ int s_base[kMaxE];
    __shared__ int s_idx[kRouterTileTokens * kMaxK];
    const int E = p.E, K = p.K;
    const int TK = p.T * K;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int b = p.offsets[e];
        for (int c = 0; c < (int)blockIdx.x; ++c) b += p.hist[(size_t)c * E + e];
        s_base[e] = b;
    }
    __syncthreads();
    const int ntiles = (p.T + kRouterTileTokens - 1) / kRouterTileTokens;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int t0 = tile * kRouterTileTokens;
        const int n = min(kRouterTileTokens, p.T - t0) * K;
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            int e = p.idx[(size_t)t0 * K + i];
            if (e < 0 || e >= E) {
                atomicOr(&p.ctrl->status, ST_BAD_EXPERT);
                e = -1;
            }
            s_idx[i] = e;
        }
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const int e = s_idx[i];
            int slot = -1;
            if (e >= 0) {
                int rank = 0;
                for (int j = 0; j < i; ++j) rank += (s_idx[j] == e);
                slot = s_base[e] + rank;
            }
            if (slot < 0 || slot >= TK) {
                atomicOr(&p.ctrl->status, ST_BAD_SLOT);
                p.slot_of[(size_t)t0 * K + i] = 0;
                continue;
            }
            p.slot_of[(size_t)t0 * K + i] = slot;
            p.tok_of_slot[slot] = t0 + i / K;
        }
        __syncthreads();
        if (p.x_perm) {  // copy each token row to its slots (one warp per slot)
            const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
            for (int i = warp; i < n; i += blockDim.x / 32) {
                if (s_idx[i] < 0) continue;
                const int slot = p.slot_of[(size_t)t0 * K + i];
                const uint4* src = reinterpret_cast<const uint4*>(p.x + (size_t)(t0 + i / K) * p.H);
                uint4* dst = reinterpret_cast<uint4*>(p.x_perm + (size_t)slot * p.H);
                for (int c = lane; c < p.H / 8; c += 32) dst[c] = __ldg(src + c);
            }
        }
        for (int e = threadIdx.x; e < E; e += blockDim.x) {
            int c = 0;
            for (int j = 0; j < n; ++j) c += (s_idx[j] == e);
            s_base[e] += c;
        }
        __syncthreads();
    }
}

cudaError_t launch_router(const Params& p, bool small_path, cudaStream_t stream) {
    if (small_path) {
        dim3 grid((p.T + kDecodeRouterTok - 1) / kDecodeRouterTok, (p.E + kDecodeRouterExp - 1) / kDecodeRouterExp);
        router_small_kernel<<<grid, 256, 0, stream>>>(p);
        return cudaGetLastError();
    }
    router_large_kernel<<<p.router_blocks, 256, 0, stream>>>(p);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    scatter_large_kernel<<<p.router_blocks, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace moe
