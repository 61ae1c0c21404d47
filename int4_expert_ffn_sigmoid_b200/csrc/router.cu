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
// Each router computes a logit with one fixed arithmetic order that does not
// depend on the other tokens of the batch, so a token gets the same routing
// whatever it is batched with (within one path).  The small-batch router
// accumulates, in lane l of a warp, the elements 128*i + 4*l + j (i ascending,
// then j = 0..3) with fused multiply-adds and sums the 32 lane partials by an
// xor-butterfly (16, 8, 4, 2, 1); the large-batch routers are described above
// router_large_kernel and in router_tc.cu.
#include <cooperative_groups.h>

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

__device__ __forceinline__ float sq_step(float acc, uint2 xv) {
    const float a = bf16lo(xv.x), b = bf16hi(xv.x), c = bf16lo(xv.y), d = bf16hi(xv.y);
    acc = fmaf(a, a, acc);
    acc = fmaf(b, b, acc);
    acc = fmaf(c, c, acc);
    acc = fmaf(d, d, acc);
    return acc;
}

// k_t = 8 + floor(log2(mean_h x[t,h]^2)), clamped: the exponent of the
// token's h storage scale 2^-k_t.  `lane_sq` is the lane's share of the sum of
// squares in the router's lane order (see dot_step).
__device__ __forceinline__ void store_hexp(const Params& p, int t, float lane_sq, int lane) {
    const float ms = warp_sum_tree(lane_sq) / (float)p.H;
    const int e = (ms > 0.f && isfinite(ms)) ? ilogbf(ms) : 0;
    if (lane == 0) p.hexp[t] = min(max(kHExpBase + e, kHExpMin), kHExpMax);
}

// k_t of the tokens warp, warp + 8, warp + 16, warp + 24 of a tile (nt
// tokens from t0): lane l sums the squares of elements 128 i + 4 l .. + 3 of
// each 128-block i in ascending order, with the four tokens' loads of four
// 128-blocks in flight together.
__device__ __forceinline__ void tile_hexp(const Params& p, int t0, int nt, int warp, int lane) {
    const int nblk = p.H / 128;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i0 = 0; i0 < nblk; i0 += 4) {
        uint2 xv[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int tt = warp + 8 * j;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                xv[j][u] = (tt < nt && i0 + u < nblk)
                               ? __ldg(reinterpret_cast<const uint2*>(p.x + (size_t)(t0 + tt) * p.H + (i0 + u) * 128 +
                                                                      lane * 4))
                               : make_uint2(0u, 0u);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (i0 + u < nblk) acc[j] = sq_step(acc[j], xv[j][u]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
        if (warp + 8 * j < nt) store_hexp(p, t0 + warp + 8 * j, acc[j], lane);
}

// Top-K of one token (one warp).  Lane l holds the logits L[j] of experts
// l + 32 j (entries of experts >= E are ignored).  The key is sigmoid(L) +
// bias (NaN -> -inf); ties go to the lower expert index.  The weight of the
// k-th pick is scale * s_k / (s_0 + ... + s_{K-1}).  Writes idx / wts (and
// the optional user outputs) of token t; returns, on lanes k < K, the k-th
// selected expert (else -1).
// kKUnroll: unrolling of the loop over the K picks (1 where the selection
// runs once per launch, its code cold in the instruction cache: a short
// rolled loop is fetched once).
template <int kKUnroll = kMaxK>
__device__ int select_from_logits(const Params& p, int t, const float (&L)[kMaxE / 32], const float* bias, int lane) {
    const int E = p.E, K = p.K;
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
    int my_e = -1;
    float my_s = 0.f, ssum = 0.f;
#pragma unroll kKUnroll
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
    int out_e;
    float w;
    topp_picks(K, p.topp, p.scale, lane, my_e, my_s, ssum, out_e, w);
    if ((p.flags & kFlagTestBadIndex) && t == 0 && lane == 0) out_e = E;  // test hook: an out-of-range pick
    if (lane < K) {
        const size_t o = (size_t)t * K + lane;
        p.idx[o] = out_e;
        p.wts[o] = w;
        if (p.topk_idx_out) p.topk_idx_out[o] = out_e;
        if (p.topk_w_out) p.topk_w_out[o] = w;
    }
    return lane < K ? out_e : -1;
}

// select_from_logits with the token's logits and the router bias in shared
// memory (a bias read from global memory per token put a round trip on every
// selection).
__device__ int select_token(const Params& p, int t, const float* lg, const float* s_bias, int lane) {
    float L[kMaxE / 32];
#pragma unroll
    for (int j = 0; j < kMaxE / 32; ++j) {
        const int e = lane + 32 * j;
        L[j] = e < p.E ? lg[e] : 0.f;
    }
    return select_from_logits(p, t, L, s_bias, lane);
}

// Writes xq (both int8 parts, see quant2) and xs of token t (one warp) from
// its bf16 row xrow (global or shared memory).
__device__ void quantize_x_row(const Params& p, int t, const __nv_bfloat16* xrow, int lane) {
    const uint4* xr = reinterpret_cast<const uint4*>(xrow);
    const int ng = p.H / 8;
    float m = 0.f;
    for (int gi = lane; gi < ng; gi += 32) {
        const uint4 v = xr[gi];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) m = nanmax(nanmax(m, fabsf(bf16lo(w[i]))), fabsf(bf16hi(w[i])));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = nanmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    const QScale qs = qscale(m);
    uint2* q0 = reinterpret_cast<uint2*>(p.xq + (size_t)t * 2 * p.H);
    uint2* q1 = reinterpret_cast<uint2*>(p.xq + (size_t)t * 2 * p.H + p.H);
    for (int gi = lane; gi < ng; gi += 32) {
        const uint4 v = xr[gi];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        float f[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = bf16lo(w[i]);
            f[2 * i + 1] = bf16hi(w[i]);
        }
        uint2 a, b;
        quant2x8(f, qs, a, b);
        q0[gi] = a;
        q1[gi] = b;
    }
    if (lane == 0) p.xs[t] = qs.s;
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
        // (under the top-p, dropped picks make fewer slots than T*K)
        const bool topp = p.topp > 0.f && p.topp < 1.f;
        if (s_total != p.T * p.K && !(topp && s_total < p.T * p.K)) atomicOr(&p.ctrl->status, ST_BAD_COUNT);
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
                const int ch = chunks_of(n, p.chunk);
                n13 = (irow / kTaskRows13) * ch;                    // gate/up rows x a token chunk
                n2 = (p.H / p.rows2) * ch * slices_of(irow);        // down rows x a chunk x a slice
                if (e != E) {  // tensor-core tiles: 128 tokens x 128 features / 256 output features
                    const int mt = (n + kTcTokens - 1) / kTcTokens;
                    nt1 = mt * (p.I / kTcFeat1);
                    nt2 = mt * (p.H / kTcFeat2);
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
// Small batch (T <= kDecodeMaxTokens): one kernel, a cluster of
// kDecodeRouterCtas CTAs per group of kDecodeRouterTok tokens (grid
// (groups, kDecodeRouterCtas)).  CTA r computes the logits of the experts
// [r*epc, (r+1)*epc), epc = ceil(E / kDecodeRouterCtas), for the group's
// tokens into its shared memory (the group's activations are staged there
// with one round of cp.async); after a cluster barrier CTA 0 reads every
// token's logits through distributed shared memory, selects (one warp per
// token), and writes the group's per-expert pick counts (hist[group][e]) and
// the rank of every pick among the group's picks of the same expert, in
// (token, k) order.  The other CTAs quantize the group's activations (xq,
// xs) from their shared copy.  The gate/up kernel derives the bucket and
// task tables from hist, idx and rank.  The expert kernels derive the buckets and slots from hist, idx and
// rank themselves: the slot of pick (t, k) of expert e is offset[e] + (picks
// of e in earlier groups) + rank, i.e. buckets list their tokens in (t, k)
// order.
// ---------------------------------------------------------------------------
// The group's activations are staged in (dynamic) shared memory up to this
// hidden size.
constexpr int kRouterXMaxH = 12288;
constexpr int kRouterWarps = 16;
constexpr int kRouterBatch = 8;  // router-weight blocks per batch of loads
// The small-batch logits are computed by a separate kernel spread over many
// SMs (router_logits_kernel) when a warp of the cluster router would stream
// more than kRouterWarpMaxBytes of router weights (its ceil(epc /
// kRouterWarps) rows of H f32 each).  On the large-batch path the router
// weights (E * H f32) are read by every CTA of router_large_kernel up to
// kRouterLargeMaxBytes; above that the tensor-core logits of router_tc.cu
// compute the logits in hidden slices.
constexpr size_t kRouterWarpMaxBytes = 8192;
constexpr size_t kRouterLargeMaxBytes = (size_t)512 << 10;

bool router_large_uses_tc(int E, int H) { return (size_t)E * H * 4 > kRouterLargeMaxBytes; }
constexpr int kLogitSliceBlocks = 3;   // 128-element blocks of the hidden dimension per slice
constexpr int kLogitCtaExperts = 32;   // experts per CTA (4 per warp)
constexpr int kLogitTileTokens = 64;   // tokens per CTA

int router_split_slices(int E, int H) {
    const int epc = (E + kDecodeRouterCtas - 1) / kDecodeRouterCtas;
    const size_t warp_bytes = (size_t)((epc + kRouterWarps - 1) / kRouterWarps) * H * 4;
    if (warp_bytes <= kRouterWarpMaxBytes) return 0;
    return (H / 128 + kLogitSliceBlocks - 1) / kLogitSliceBlocks;
}

size_t router_decode_smem(int H) {
    return H <= kRouterXMaxH ? (size_t)kDecodeRouterTok * H * sizeof(__nv_bfloat16) : 0;
}

// Split router, first kernel: CTA (s, b, z) computes, for tokens [64 z,
// 64 z + 64), the partial logits over hidden slice s (blocks
// s*kLogitSliceBlocks onwards, 128 elements each) of experts [32 b, 32 b +
// 32): warp w takes experts 32 b + 4 w .. + 3 and holds their weights of the
// slice in registers (loaded before waiting on the previous kernel); the
// tokens' activations of the slice are staged in shared memory.  Lane l
// accumulates the elements 128 i + 4 l + j of the slice (i ascending, then j)
// and the lanes are summed by the xor-butterfly; the selecting kernel (the
// cluster router) adds the slices in ascending order.
// The logit of a token therefore does not depend on the other tokens of the
// batch.
__global__ void __launch_bounds__(256) router_logits_kernel(Params p) {
    extern __shared__ __align__(16) __nv_bfloat16 s_xl[];  // [tile tokens][kLogitSliceBlocks * 128]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int E = p.E, H = p.H, T = p.T;
    const int t0 = blockIdx.z * kLogitTileTokens, nt = min(kLogitTileTokens, T - t0);
    const int s = blockIdx.x;
    const int b0 = s * kLogitSliceBlocks, nb = min(kLogitSliceBlocks, H / 128 - b0);
    const int e0 = blockIdx.y * kLogitCtaExperts + warp * 4;
    constexpr int kW = kLogitSliceBlocks * 128;
    float4 w[4][kLogitSliceBlocks];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int i = 0; i < kLogitSliceBlocks; ++i)
            w[u][i] = (e0 + u < E && i < nb)
                          ? __ldg(reinterpret_cast<const float4*>(p.rw + (size_t)(e0 + u) * H + (b0 + i) * 128) + lane)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
    pdl_wait();
    pdl_release();
    const int per = nb * 16;  // 16-byte chunks of a token's slice
    for (int c = threadIdx.x; c < nt * per; c += blockDim.x) {
        const int t = c / per, k = c - t * per;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(
                         __cvta_generic_to_shared(s_xl + (size_t)t * kW + k * 8))),
                     "l"(p.x + (size_t)(t0 + t) * H + b0 * 128 + k * 8)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    if (e0 >= E) return;
    for (int t = 0; t < nt; ++t) {
        uint2 xv[kLogitSliceBlocks];
#pragma unroll
        for (int i = 0; i < kLogitSliceBlocks; ++i)
            xv[i] = i < nb ? *reinterpret_cast<const uint2*>(s_xl + (size_t)t * kW + i * 128 + lane * 4)
                           : make_uint2(0u, 0u);
        float v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < kLogitSliceBlocks; ++i)
                if (i < nb) acc = dot_step(acc, xv[i], w[u][i]);
            v[u] = warp_sum_tree(acc);
        }
        if (lane < 4 && e0 + lane < E) {
            const float r = lane == 0 ? v[0] : lane == 1 ? v[1] : lane == 2 ? v[2] : v[3];
            p.lpart[((size_t)s * T + t0 + t) * E + e0 + lane] = r;
        }
    }
}

size_t router_logits_smem(int T) {
    return (size_t)min(T, kLogitTileTokens) * kLogitSliceBlocks * 128 * sizeof(__nv_bfloat16);
}

__global__ void __cluster_dims__(1, kDecodeRouterCtas, 1) __launch_bounds__(32 * kRouterWarps, 1)
    router_decode_kernel(Params p) {
    namespace cg = cooperative_groups;
    constexpr int kEpcMax = kMaxE / kDecodeRouterCtas;
    extern __shared__ __align__(16) __nv_bfloat16 s_xd[];  // [kDecodeRouterTok][H] when staged
    __shared__ float s_logit[kDecodeRouterTok][kEpcMax];
    __shared__ float s_bias[kMaxE];
    __shared__ int s_pick[kDecodeRouterTok * kMaxK];
    cg::cluster_group cluster = cg::this_cluster();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r = blockIdx.y;  // rank in the cluster
    const int t0 = blockIdx.x * kDecodeRouterTok;
    const int nt = min(kDecodeRouterTok, p.T - t0);
    const int E = p.E, H = p.H, K = p.K;
    const int nblk = H / 128;
    const int epc = (E + kDecodeRouterCtas - 1) / kDecodeRouterCtas;
    const int e_lo = r * epc, e_hi = min(E, e_lo + epc);
    const bool staged = H <= kRouterXMaxH;
    const bool split = p.lslices > 0;  // the logits kernel ran first
    // Nothing below depends on the previous kernel until pdl_wait: the bias,
    // the first batch of this warp's first router row (registers) and the
    // rest of the CTA's rows (L2).
    if (r == 0)
        for (int e = threadIdx.x; e < E; e += blockDim.x) s_bias[e] = __ldg(p.rb + e);
    float4 wpre[kRouterBatch];
    if (!split) {
        const int e = e_lo + warp;
        const float4* W = reinterpret_cast<const float4*>(p.rw + (size_t)min(e, E - 1) * H);
#pragma unroll
        for (int i = 0; i < kRouterBatch; ++i)
            wpre[i] = (e < e_hi && i < nblk) ? __ldg(W + i * 32 + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int e = e_lo + warp; !split && e < e_hi; e += kRouterWarps) {
        const char* wrow = reinterpret_cast<const char*>(p.rw + (size_t)e * H);
        for (int l = lane; l < H * 4 / 128; l += 32) asm volatile("prefetch.global.L2 [%0];" ::"l"(wrow + l * 128));
    }
    pdl_wait();
    reset_ctrl(p);
    pdl_release();
    if (staged) {
        const int per = H / 8;  // 16-byte chunks per row
        for (int c = threadIdx.x; c < nt * per; c += blockDim.x) {
            const int tt = c / per, k = c - tt * per;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(
                             __cvta_generic_to_shared(s_xd + (size_t)tt * H + k * 8))),
                         "l"(p.x + (size_t)(t0 + tt) * H + k * 8)
                         : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
    }
    auto xblock = [&](int tt, int i) -> uint2 {
        if (tt >= nt) return make_uint2(0u, 0u);
        if (staged) return *reinterpret_cast<const uint2*>(s_xd + (size_t)tt * H + i * 128 + lane * 4);
        return __ldg(reinterpret_cast<const uint2*>(p.x + (size_t)(t0 + tt) * H + i * 128 + lane * 4));
    };
    if (split) {  // this CTA's experts: the sum of the slices' partial logits, slice 0 first
        const int ne = e_hi - e_lo;
        for (int i = threadIdx.x; i < nt * ne; i += blockDim.x) {
            const int tt = i / ne, e = e_lo + (i - tt * ne);
            const float* src = p.lpart + (size_t)(t0 + tt) * E + e;
            float v = 0.f;
            for (int sl = 0; sl < p.lslices; ++sl) v += __ldcg(src + (size_t)sl * p.T * E);
            s_logit[tt][e - e_lo] = v;
        }
    }
    // Each warp's one expert row in registers (wpre): a rolled loop over the
    // group's tokens, each in the block order of the general loop below.  The
    // kernel runs once per layer with its code cold in the instruction cache;
    // the rolled loop is a short stretch of code, fetched once (measured:
    // Nano stack T = 16 0.760 -> 0.741 ms, T = 64 0.955 -> 0.944 ms).
    const bool w_in_regs = !split && nblk <= kRouterBatch && epc <= kRouterWarps;
    if (w_in_regs) {
        const int e = e_lo + warp;
        if (e < e_hi) {
#pragma unroll 1
            for (int tt = 0; tt < nt; ++tt) {
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < kRouterBatch; ++i)
                    if (i < nblk) acc = dot_step(acc, xblock(tt, i), wpre[i]);
                const float v = warp_sum_tree(acc);
                if (lane == 0) s_logit[tt][e - e_lo] = v;
            }
        }
    }
    for (int e = e_lo + warp, j = 0; !split && !w_in_regs && e < e_hi; e += kRouterWarps, ++j) {
        float acc[kDecodeRouterTok];
#pragma unroll
        for (int tt = 0; tt < kDecodeRouterTok; ++tt) acc[tt] = 0.f;
        const float4* W = reinterpret_cast<const float4*>(p.rw + (size_t)e * H);
        // batches of kRouterBatch blocks; the next batch is in flight while this one is used
        float4 cur[kRouterBatch], nxt[kRouterBatch];
#pragma unroll
        for (int u = 0; u < kRouterBatch; ++u)
            cur[u] = j == 0 ? wpre[u] : (u < nblk ? __ldg(W + u * 32 + lane) : make_float4(0.f, 0.f, 0.f, 0.f));
        for (int i0 = 0; i0 < nblk; i0 += kRouterBatch) {
#pragma unroll
            for (int u = 0; u < kRouterBatch; ++u) {
                const int i = i0 + kRouterBatch + u;
                nxt[u] = i < nblk ? __ldg(W + i * 32 + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < kRouterBatch; ++u)
                if (i0 + u < nblk)
#pragma unroll
                    for (int tt = 0; tt < kDecodeRouterTok; ++tt) acc[tt] = dot_step(acc[tt], xblock(tt, i0 + u), cur[u]);
#pragma unroll
            for (int u = 0; u < kRouterBatch; ++u) cur[u] = nxt[u];
        }
#pragma unroll
        for (int tt = 0; tt < kDecodeRouterTok; ++tt) {
            const float v = warp_sum_tree(acc[tt]);
            if (lane == 0) s_logit[tt][e - e_lo] = v;
        }
    }
    cluster.sync();  // every logit of the group is in some CTA's shared memory
    if (r == 0) {
        if (warp < nt) {
            float L[kMaxE / 32];
#pragma unroll
            for (int jj = 0; jj < kMaxE / 32; ++jj) {
                const int e = lane + 32 * jj;
                L[jj] = 0.f;
                if (e < E) {
                    const int src = e / epc;
                    L[jj] = *cluster.map_shared_rank(&s_logit[warp][e - src * epc], src);
                }
            }
            const int sel = select_from_logits<1>(p, t0 + warp, L, s_bias, lane);
            if (lane < K) s_pick[warp * K + lane] = sel;
        }
        __syncthreads();
        const int n = nt * K;
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const int e = s_pick[i];
            int rk = 0;
            for (int jj = 0; jj < i; ++jj) rk += (s_pick[jj] == e);
            p.rank[(size_t)t0 * K + i] = rk;
        }
        for (int e = threadIdx.x; e < E; e += blockDim.x) {
            int c = 0;
            for (int jj = 0; jj < n; ++jj) c += (s_pick[jj] == e);
            p.hist[(size_t)blockIdx.x * E + e] = c;
        }
    } else {
        // token tt of the group is quantized by CTA max(tt, 1), warp (tt == 0)
        for (int tt = 0; tt < nt; ++tt)
            if (r == max(tt, 1) && warp == (tt == 0 ? 1 : 0))
                quantize_x_row(p, t0 + tt, staged ? s_xd + (size_t)tt * H : p.x + (size_t)(t0 + tt) * H, lane);
    }
    cluster.sync();  // the remote reads of CTA 0 are done before any CTA exits
}

// ---------------------------------------------------------------------------
// Large batch, two kernels.
// router_large_kernel (router weights up to kRouterLargeMaxBytes) or, after
// the tensor-core router logits of router_tc.cu (larger router weights),
// router_select_kernel: router_blocks CTAs walk tiles of kRouterTileTokens
// tokens (tile = block, block + grid, ...); each tile's logits stay in shared
// memory (router_select_kernel: the hidden slices' partial logits added in
// ascending order), one warp per token selects, and every CTA records its
// per-expert pick counts.  scatter_large_kernel: every CTA derives the bucket
// offsets and its own slot bases from those counts (CTA 0 also writes the
// bucket and task lists), then the slots, and the gathered activation rows of
// the tensor-core path.  The int8 activations of the weight-streaming kernels
// come from extra CTAs past the router's (one warp per token, every token in
// flight at once), or, when the grid has no room for them, from the router's.
// ---------------------------------------------------------------------------
// Tensor-core router logits for a tile of kRouterTileTokens tokens and every
// expert.  x is exactly bf16; each f32 router weight w is split exactly into
// three bf16 terms w = hi + mid + lo (hi = bf16(w), mid = bf16(w - hi),
// lo = bf16(w - hi - mid); together they hold w's 24-bit mantissa), and
// x.w = x.lo + x.mid + x.hi is accumulated in f32 by mma.sync m16n8k16
// (A = tokens, B = experts).  Every 16-wide k step is accumulated from zero
// by the tensor cores (16 products per instruction) and added to the running
// f32 sum with ordinary IEEE adds, so the logits carry f32 rounding only.  The activations are staged in shared memory
// with cp.async (chunks of kRouterKC along the hidden dimension, double-
// buffered) and read with ldmatrix.
constexpr int kRouterKC = 128;                // hidden elements per staged chunk (H % 128 == 0)
constexpr int kRouterXS = kRouterKC + 8;      // padded row (bf16 elements)
constexpr int kRouterMT = kRouterTileTokens / 16;
constexpr int kRouterXStages = 4;             // staged chunks in flight


__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* smem_row) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_row))));
}

__global__ void __launch_bounds__(256, 2) router_large_kernel(Params p) {
    // the staged activations and, after the k loop, the tile's logits share one buffer
    constexpr int kXBytes = kRouterXStages * kRouterTileTokens * kRouterXS * 2;
    constexpr int kLBytes = kRouterTileTokens * kMaxE * 4;
    __shared__ __align__(16) uint8_t s_buf[kXBytes > kLBytes ? kXBytes : kLBytes];
    __shared__ int s_cnt[kMaxE];
    __shared__ float s_bias[kMaxE];
    auto s_x = reinterpret_cast<uint16_t (*)[kRouterTileTokens][kRouterXS]>(s_buf);
    auto s_logit = reinterpret_cast<float (*)[kMaxE]>(s_buf);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int E = p.E, H = p.H;
    const int n_ntiles = (E + 7) / 8;
    // B fragments of this warp's first n-tile for one chunk: w[k + 2q, +1] and
    // w[k + 2q + 8, +9] of every k step, loaded together one chunk ahead (the
    // first before waiting on the previous kernel: they do not depend on it)
    float2 wpre[kRouterKC / 16][2];
    auto load_w0 = [&](int c) {
        const float* wrow = p.rw + (size_t)min(warp * 8 + g, E - 1) * H + c * kRouterKC;
#pragma unroll
        for (int k = 0; k < kRouterKC / 16; ++k) {
            wpre[k][0] = __ldg(reinterpret_cast<const float2*>(wrow + k * 16 + 2 * q));
            wpre[k][1] = __ldg(reinterpret_cast<const float2*>(wrow + k * 16 + 2 * q + 8));
        }
    };
    if (warp < n_ntiles) load_w0(0);
    pdl_wait();
    reset_ctrl(p);
    pdl_release();
    for (int i = threadIdx.x; i < E; i += blockDim.x) {
        s_cnt[i] = 0;
        s_bias[i] = __ldg(p.rb + i);
    }
    __syncthreads();
    const int ntiles_tok = (p.T + kRouterTileTokens - 1) / kRouterTileTokens;
    const int nchunks = H / kRouterKC;
    for (int tile = blockIdx.x; tile < ntiles_tok; tile += gridDim.x) {
        const int t0 = tile * kRouterTileTokens;
        const int nt = min(kRouterTileTokens, p.T - t0);
        auto stage_chunk = [&](int c, int buf) {
            for (int i = threadIdx.x; i < kRouterTileTokens * (kRouterKC / 8); i += blockDim.x) {
                const int r = i / (kRouterKC / 8), part = i % (kRouterKC / 8);
                uint16_t* dst = &s_x[buf][r][part * 8];
                if (r < nt) {
                    const void* src = p.x + (size_t)(t0 + r) * H + c * kRouterKC + part * 8;
                    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                                     static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                                 "l"(src)
                                 : "memory");
                } else {
                    *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        };

        // this warp's expert n-tiles: warp, warp + 8, ... (at most kMaxE / 64)
        float acc[kMaxE / 64][kRouterMT][4];
#pragma unroll
        for (int j = 0; j < kMaxE / 64; ++j)
#pragma unroll
            for (int m = 0; m < kRouterMT; ++m) acc[j][m][0] = acc[j][m][1] = acc[j][m][2] = acc[j][m][3] = 0.f;

        // sum of squares of the tile's tokens from the staged chunks (k_t of the
        // h scale): thread 8 r + u takes elements 16 u .. 16 u + 15 of row r of
        // every chunk, and the 8 partial sums are added by an xor-butterfly
        float sq = 0.f;
        const int sq_row = threadIdx.x >> 3, sq_col = (threadIdx.x & 7) * 16;
        __syncthreads();  // s_x is free (previous tile done)
#pragma unroll
        for (int i = 0; i < kRouterXStages - 1; ++i) {
            if (i < nchunks) stage_chunk(i, i);
            else asm volatile("cp.async.commit_group;" ::: "memory");
        }
        for (int c = 0; c < nchunks; ++c) {
            const int cn = c + kRouterXStages - 1;  // into the buffer chunk c - 1 used
            if (cn < nchunks) stage_chunk(cn, cn % kRouterXStages);
            else asm volatile("cp.async.commit_group;" ::: "memory");
            asm volatile("cp.async.wait_group %0;" ::"n"(kRouterXStages - 1) : "memory");
            __syncthreads();
            const uint16_t (*xs)[kRouterXS] = s_x[c % kRouterXStages];
            {
                const uint4 a = *reinterpret_cast<const uint4*>(&xs[sq_row][sq_col]);
                const uint4 b = *reinterpret_cast<const uint4*>(&xs[sq_row][sq_col + 8]);
                sq = sq_step(sq, make_uint2(a.x, a.y));
                sq = sq_step(sq, make_uint2(a.z, a.w));
                sq = sq_step(sq, make_uint2(b.x, b.y));
                sq = sq_step(sq, make_uint2(b.z, b.w));
            }
#pragma unroll
            for (int j = 0; j < kMaxE / 64; ++j) {
                const int ntile = warp + 8 * j;
                if (ntile < n_ntiles) {
                    const int e = ntile * 8 + g;
                    float2 wall[kRouterKC / 16][2];
                    if (j == 0) {  // prefetched; fetch the next chunk's (or the next tile's first)
#pragma unroll
                        for (int k = 0; k < kRouterKC / 16; ++k) {
                            wall[k][0] = wpre[k][0];
                            wall[k][1] = wpre[k][1];
                        }
                        if (c + 1 < nchunks) load_w0(c + 1);
                        else if (tile + (int)gridDim.x < ntiles_tok) load_w0(0);
                    } else {  // every k step of the chunk loaded together (one round trip)
                        const float* wrow = p.rw + (size_t)min(e, E - 1) * H + c * kRouterKC;
#pragma unroll
                        for (int k = 0; k < kRouterKC / 16; ++k) {
                            wall[k][0] = __ldg(reinterpret_cast<const float2*>(wrow + k * 16 + 2 * q));
                            wall[k][1] = __ldg(reinterpret_cast<const float2*>(wrow + k * 16 + 2 * q + 8));
                        }
                    }
#pragma unroll
                    for (int ks = 0; ks < kRouterKC / 16; ks += 2) {
                        const float2(*wv)[2] = &wall[ks];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            uint32_t bh[2], bm[2], bl[2];
#pragma unroll
                            for (int v = 0; v < 2; ++v) {
                                const float w0 = e < E ? wv[u][v].x : 0.f, w1 = e < E ? wv[u][v].y : 0.f;
                                uint16_t h0, m0, l0, h1, m1, l1;
                                split3(w0, h0, m0, l0);
                                split3(w1, h1, m1, l1);
                                bh[v] = (uint32_t)h0 | ((uint32_t)h1 << 16);
                                bm[v] = (uint32_t)m0 | ((uint32_t)m1 << 16);
                                bl[v] = (uint32_t)l0 | ((uint32_t)l1 << 16);
                            }
#pragma unroll
                            for (int m = 0; m < kRouterMT; ++m) {
                                uint32_t a[4];
                                ldmatrix_x4(a, &xs[m * 16 + (lane & 15)][(ks + u) * 16 + (lane >> 4) * 8]);
                                float t[4] = {0.f, 0.f, 0.f, 0.f};
                                mma_bf16(t, a, bl[0], bl[1]);
                                mma_bf16(t, a, bm[0], bm[1]);
                                mma_bf16(t, a, bh[0], bh[1]);
#pragma unroll
                                for (int v = 0; v < 4; ++v) acc[j][m][v] += t[v];
                            }
                        }
                    }
                }
            }
            __syncthreads();  // chunk c's readers are done before it is overwritten
        }
        sq += __shfl_xor_sync(0xffffffffu, sq, 1);
        sq += __shfl_xor_sync(0xffffffffu, sq, 2);
        sq += __shfl_xor_sync(0xffffffffu, sq, 4);
        if ((threadIdx.x & 7) == 0 && sq_row < nt) {
            const float ms = sq / (float)H;
            const int ex = (ms > 0.f && isfinite(ms)) ? ilogbf(ms) : 0;
            p.hexp[t0 + sq_row] = min(max(kHExpBase + ex, kHExpMin), kHExpMax);
        }
#pragma unroll
        for (int j = 0; j < kMaxE / 64; ++j) {
            const int ntile = warp + 8 * j;
            if (ntile < n_ntiles) {
                const int e = ntile * 8 + 2 * q;
#pragma unroll
                for (int m = 0; m < kRouterMT; ++m) {
                    const int r = m * 16 + g;
                    if (e < E) { s_logit[r][e] = acc[j][m][0]; s_logit[r + 8][e] = acc[j][m][2]; }
                    if (e + 1 < E) { s_logit[r][e + 1] = acc[j][m][1]; s_logit[r + 8][e + 1] = acc[j][m][3]; }
                }
            }
        }
        __syncthreads();
        for (int tt = warp; tt < nt; tt += 8) {
            const int sel = select_token(p, t0 + tt, s_logit[tt], s_bias, lane);
            // an index outside [0, E) cannot occur; it is counted nowhere and
            // reported by the scatter kernel's range check
            if (lane < p.K && sel >= 0 && sel < E) atomicAdd(&s_cnt[sel], 1);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += blockDim.x) p.hist[(size_t)blockIdx.x * E + i] = s_cnt[i];
}

// 512 threads: the selections of a tile's 32 tokens run two per warp.
constexpr int kSelectThreads = 512;
__global__ void __launch_bounds__(kSelectThreads) router_select_kernel(Params p) {
    __shared__ __align__(16) float s_logit[kRouterTileTokens][kMaxE];
    __shared__ int s_cnt[kMaxE];
    __shared__ float s_bias[kMaxE];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int E = p.E;
    pdl_wait();  // the weight split, the call's first kernel, zeroed the status word
    pdl_release();
    for (int i = threadIdx.x; i < E; i += blockDim.x) {
        s_cnt[i] = 0;
        s_bias[i] = __ldg(p.rb + i);
    }
    __syncthreads();
    const int ntiles_tok = (p.T + kRouterTileTokens - 1) / kRouterTileTokens;
    for (int tile = blockIdx.x; tile < ntiles_tok; tile += gridDim.x) {
        const int t0 = tile * kRouterTileTokens;
        const int nt = min(kRouterTileTokens, p.T - t0);
        static_assert(kRouterTileTokens == 32, "four tokens per warp in tile_hexp");
        // the h-scale exponents serve the tensor-core sequence's fp16 h only
        // (the streaming sequences keep h in f32): a pass over x skipped there
        if (p.x_perm && warp < 8) tile_hexp(p, t0, nt, warp, lane);
        __syncthreads();  // s_logit is free (previous tile done)
        // four elements per thread, each summed over the slices in ascending
        // order, with up to eight slices' loads of all four in flight
        for (int i0 = threadIdx.x; i0 < nt * E; i0 += 4 * blockDim.x) {
            float v[4] = {0.f, 0.f, 0.f, 0.f};
            for (int sl0 = 0; sl0 < p.lslices; sl0 += 8) {
                float part[8][4];
#pragma unroll
                for (int sl = 0; sl < 8; ++sl)
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int i = i0 + u * blockDim.x;
                        part[sl][u] = (sl0 + sl < p.lslices && i < nt * E)
                                          ? __ldcg(p.lpart + ((size_t)(sl0 + sl) * p.T + t0 + i / E) * E + i % E)
                                          : 0.f;
                    }
#pragma unroll
                for (int sl = 0; sl < 8; ++sl)
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (sl0 + sl < p.lslices) v[u] += part[sl][u];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * blockDim.x;
                if (i < nt * E) s_logit[i / E][i % E] = v[u];
            }
        }
        __syncthreads();
        for (int tt = warp; tt < nt; tt += (int)blockDim.x / 32) {
            const int sel = select_token(p, t0 + tt, s_logit[tt], s_bias, lane);
            // an index outside [0, E) cannot occur; it is counted nowhere and
            // reported by the scatter kernel's range check
            if (lane < p.K && sel >= 0 && sel < E) atomicAdd(&s_cnt[sel], 1);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += blockDim.x) p.hist[(size_t)blockIdx.x * E + i] = s_cnt[i];
}

// Exclusive prefix of s_tot[0..E) into s_off (warp 0; the caller synchronises).
__device__ void expert_offsets(const int* s_tot, int* s_off, int E) {
    const int lane = threadIdx.x & 31;
    if (threadIdx.x >= 32) return;
    constexpr int kPer = kMaxE / 32;
    int c[kPer], sum = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int e = lane * kPer + j;
        c[j] = e < E ? s_tot[e] : 0;
        sum += c[j];
    }
    int inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += u;
    }
    int off = inc - sum;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int e = lane * kPer + j;
        if (e < E) s_off[e] = off;
        off += c[j];
    }
}

// CTA c walks the same tiles as router CTA c and assigns slots in (tile,
// token, k) order, after the slots of CTAs 0..c-1: from the router CTAs'
// per-expert counts it takes every expert's total (the bucket offsets) and
// the picks of CTAs 0..c-1.  CTA 0 also builds the bucket and task lists.
__global__ void __launch_bounds__(256) scatter_large_kernel(Params p) {
    __shared__ int s_base[kMaxE];
    __shared__ int s_tot[kMaxE];
    __shared__ int s_off[kMaxE];
    __shared__ int s_idx[kRouterTileTokens * kMaxK];
    __shared__ int s_slot[kRouterTileTokens * kMaxK];  // -1: not copied
    const int E = p.E, K = p.K;
    const int TK = p.T * K;
    const int nblk = p.router_blocks;
    pdl_wait();
    pdl_release();
    if ((int)blockIdx.x >= nblk) {
        // quantizer CTAs (weight-streaming sequence, launched past the router's
        // CTAs): the int8 activations, one warp per token, all tokens in flight
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
        const int nq = (int)gridDim.x - nblk;
        for (int t = ((int)blockIdx.x - nblk) * nw + warp; t < p.T; t += nq * nw)
            quantize_x_row(p, t, p.x + (size_t)t * p.H, lane);
        return;
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_tot[e] = s_base[e] = 0;
    __syncthreads();
    {  // the whole [nblk][E] count matrix: G = blockDim / E threads per expert
       // (E <= kMaxE = blockDim) sum the blocks g, g + G, ... of their expert
       // with eight loads in flight, then add their partial sums
        const int G = (int)blockDim.x / E, e = (int)threadIdx.x % E, g = (int)threadIdx.x / E;
        if (g < G) {
            int tot = 0, base = 0;
            for (int b0 = g; b0 < nblk; b0 += 8 * G) {
                int v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int b = b0 + u * G;
                    v[u] = b < nblk ? __ldcg(p.hist + (size_t)b * E + e) : 0;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    tot += v[u];
                    if (b0 + u * G < (int)blockIdx.x) base += v[u];
                }
            }
            atomicAdd(&s_tot[e], tot);
            atomicAdd(&s_base[e], base);
        }
    }
    __syncthreads();
    if (blockIdx.x == 0) {
        finalize_buckets(p, s_tot, s_off);  // the tables (and s_off); synchronises the CTA
    } else {
        expert_offsets(s_tot, s_off, E);
        __syncthreads();
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_base[e] += s_off[e];
    __syncthreads();
    const int ntiles = (p.T + kRouterTileTokens - 1) / kRouterTileTokens;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int t0 = tile * kRouterTileTokens;
        const int n = min(kRouterTileTokens, p.T - t0) * K;
        const bool topp = p.topp > 0.f && p.topp < 1.f;
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            int e = p.idx[(size_t)t0 * K + i];
            if (e == -1 && topp) {
                e = -2;  // dropped by the top-p: no slot
            } else if (e < 0 || e >= E) {
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
            if (e == -2) {  // dropped by the top-p
                p.slot_of[(size_t)t0 * K + i] = -1;
                s_slot[i] = -1;
                continue;
            }
            if (slot < 0 || slot >= TK) {
                atomicOr(&p.ctrl->status, ST_BAD_SLOT);
                p.slot_of[(size_t)t0 * K + i] = 0;
                s_slot[i] = -1;
                continue;
            }
            s_slot[i] = slot;
            p.slot_of[(size_t)t0 * K + i] = slot;
            p.tok_of_slot[slot] = t0 + i / K;
        }
        __syncthreads();
        if (p.x_perm) {  // copy each token row to its slots (one warp per slot)
            const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
            for (int i = warp; i < n; i += blockDim.x / 32) {
                const int slot = s_slot[i];
                if (slot < 0) continue;
                const uint4* src = reinterpret_cast<const uint4*>(p.x + (size_t)(t0 + i / K) * p.H);
                uint4* dst = reinterpret_cast<uint4*>(p.x_perm + (size_t)slot * p.H);
                for (int c = lane; c < p.H / 8; c += 32) dst[c] = __ldg(src + c);
            }
        }
        if (p.xq && (int)gridDim.x == nblk) {  // int8 activations (no quantizer CTAs): one warp per token
            const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
            for (int tt = warp; tt < n / K; tt += blockDim.x / 32)
                quantize_x_row(p, t0 + tt, p.x + (size_t)(t0 + tt) * p.H, lane);
        }
        for (int e = threadIdx.x; e < E; e += blockDim.x) {
            int c = 0;
            for (int j = 0; j < n; ++j) c += (s_idx[j] == e);
            s_base[e] += c;
        }
        __syncthreads();
    }
}

cudaError_t launch_router_logits(const Params& p, cudaStream_t stream) {
    const dim3 grid(p.lslices, (p.E + kLogitCtaExperts - 1) / kLogitCtaExperts,
                    (p.T + kLogitTileTokens - 1) / kLogitTileTokens);
    return launch_pdl(router_logits_kernel, grid, dim3(256), router_logits_smem(p.T), stream, p);
}

cudaError_t launch_router(const Params& p, bool small_path, cudaStream_t stream) {
    cudaError_t err;
    if (small_path) {
        const size_t smem = router_decode_smem(p.H);
        static int attr_set[64];
        int dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64 && !attr_set[dev]) {
            const cudaError_t e = cudaFuncSetAttribute(router_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)router_decode_smem(kRouterXMaxH));
            if (e != cudaSuccess) return e;
            attr_set[dev] = 1;
        }
        if (p.lslices > 0) {
            const cudaError_t e = launch_router_logits(p, stream);
            if (e != cudaSuccess) return e;
        }
        return launch_pdl(router_decode_kernel, dim3(p.decode_groups, kDecodeRouterCtas), dim3(32 * kRouterWarps),
                          smem, stream, p);
    }
    if (p.tc_router) {
        if (p.lslices <= 0) return cudaErrorInvalidValue;
        err = launch_router_tc(p, stream);
        if (err == cudaSuccess)
            err = launch_pdl(router_select_kernel, dim3(p.router_blocks), dim3(kSelectThreads), 0, stream, p);
    } else {
        err = launch_pdl(router_large_kernel, dim3(p.router_blocks), dim3(256), 0, stream, p);
    }
    if (err != cudaSuccess) return err;
    // the weight-streaming sequence's int8 activations: quantizer CTAs past the
    // router's, one warp per token (up to kRouterMaxBlocks CTAs in all)
    int quant_ctas = 0;
    if (p.xq) {
        const int want = (p.T + 7) / 8, room = kRouterMaxBlocks - p.router_blocks;
        quant_ctas = want < room ? want : room;
    }
    if (err == cudaSuccess)
        err = launch_pdl(scatter_large_kernel, dim3(p.router_blocks + quant_ctas), dim3(256), 0, stream, p);
    return err;
}

}  // namespace moe
