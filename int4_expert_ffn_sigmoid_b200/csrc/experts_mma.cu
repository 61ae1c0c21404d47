// Weight-streaming expert kernels (gate/up + SwiGLU, then down) for the
// int4 per-row-symmetric SwiGLU experts and the shared expert.
//
// Method: colibri README (project listing), "What's implemented": packed int4
// with per-row scales, dequant-on-use, batch-union MoE (each expert touched
// by the batch is read once and applied to all of its tokens);
// nanocolibri-engine README, "Converting a checkpoint yourself": per-row
// symmetric int4, f32 row scales.
//
// Design.  One warp owns one task = (bucket, 8 gate/up rows or 16 down rows,
// chunk of up to 64 of the bucket's tokens) and walks the whole reduction
// dimension.  Weights go HBM -> registers with 128-bit streaming loads (each
// thread reads 16 contiguous bytes = 32 codes of a row per 128-wide k block),
// are turned into exact 16-bit integers (the row scale is applied to the f32
// result, since it factors out of the row's dot product), and feed mma.sync
// m16n8k16 with the tokens as the n dimension.  The reduction index is
// permuted identically for weights and activations (pairs (e, e+4) of every
// group of 8), which leaves each dot product unchanged.  For gate/up the 16
// mma rows are 8 gate rows and the same 8 up rows, so each thread ends with
// gate and up of the same (row, token) and applies SwiGLU in registers.
#include "moe_common.cuh"
#include "moe_launch.h"

namespace moe {

__device__ __forceinline__ int find_bucket(const int32_t* ts, int nb, int task) {
    int lo = 0, hi = nb;  // ts[lo] <= task < ts[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(ts + mid) <= task) lo = mid; else hi = mid;
    }
    return lo;
}

__global__ void __launch_bounds__(256) experts_w13_kernel(Params p) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int ntask = p.ctrl->tasks13;
    const int nb = p.ctrl->n_buckets;
    const int H = p.H, E = p.E;
    const int row_bytes = H / 2;
    const int nkb = H / 128;
    for (int task = blockIdx.x * 8 + warp; task < ntask; task += gridDim.x * 8) {
        const int b = find_bucket(p.ts13, nb, task);
        const int e = __ldg(p.bucket_e + b);
        const int n = __ldg(p.bucket_n + b);
        const int off = __ldg(p.bucket_off + b);
        if (e < 0 || e > E || (e == E && p.Is == 0)) {
            if (lane == 0) atomicOr(&p.ctrl->status, ST_BAD_TASK);
            continue;
        }
        const bool shared = (e == E);
        const int irow = shared ? p.Is : p.I;
        const int R = irow / 8;
        const int local = task - __ldg(p.ts13 + b);
        const int c = local / R, rg = local - c * R;
        const int r0 = rg * 8, tok0 = c * kChunkTokens;
        const int nt = min(kChunkTokens, n - tok0);
        const int ntiles = (nt + 7) >> 3;
        const uint8_t* W = shared ? p.sh_w13 : p.w13 + (size_t)e * 2 * p.I * row_bytes;
        const float* S = shared ? p.sh_s13 : p.s13 + (size_t)e * 2 * p.I;
        const uint8_t* grow = W + (size_t)(r0 + g) * row_bytes + q * 16;
        const uint8_t* urow = W + (size_t)(irow + r0 + g) * row_bytes + q * 16;

        const __nv_bfloat16* xr[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int s = tok0 + 8 * i + g;
            xr[i] = nullptr;
            if (i < ntiles && s < n) {
                const int t = shared ? s : __ldg(p.tok_of_slot + off + s);
                if (t >= 0 && t < p.T) xr[i] = p.x + (size_t)t * H + q * 32;
                else atomicOr(&p.ctrl->status, ST_BAD_SLOT);
            }
        }

        float acc[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

        uint4 wg = ld_stream_v4(grow), wu = ld_stream_v4(urow);
        for (int kb = 0; kb < nkb; ++kb) {
            uint4 ng = make_uint4(0, 0, 0, 0), nu = ng;
            if (kb + 1 < nkb) {
                ng = ld_stream_v4(grow + (kb + 1) * 64);
                nu = ld_stream_v4(urow + (kb + 1) * 64);
            }
            const uint32_t gw[4] = {wg.x, wg.y, wg.z, wg.w};
            const uint32_t uw[4] = {wu.x, wu.y, wu.z, wu.w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                uint32_t G[4], U[4];
                int4x8_to_bf16x2(gw[w], G);
                int4x8_to_bf16x2(uw[w], U);
                const uint32_t aA[4] = {G[0], U[0], G[1], U[1]};
                const uint32_t aB[4] = {G[2], U[2], G[3], U[3]};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (i < ntiles) {
                        uint4 xv = make_uint4(0, 0, 0, 0);
                        if (xr[i]) xv = ld_v4(xr[i] + kb * 128 + w * 8);
                        uint32_t X[4];
                        pair8(xv, X);
                        mma_bf16(acc[i], aA, X[0], X[1]);
                        mma_bf16(acc[i], aB, X[2], X[3]);
                    }
                }
            }
            wg = ng;
            wu = nu;
        }

        const float gs = __ldg(S + r0 + g), us = __ldg(S + irow + r0 + g);
        __half* hb = shared ? p.h_s : p.h_r;
        const size_t hbase = shared ? 0 : (size_t)off;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i < ntiles) {
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int s = tok0 + 8 * i + 2 * q + cc;
                    if (s < n) {
                        const float gv = acc[i][cc] * gs, uv = acc[i][2 + cc] * us;
                        hb[(hbase + s) * irow + r0 + g] = __float2half_rn(silu_mul(gv, uv));
                    }
                }
            }
        }
    }
}

__global__ void __launch_bounds__(256) experts_w2_kernel(Params p) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int ntask = p.ctrl->tasks2;
    const int nb = p.ctrl->n_buckets;
    const int H = p.H, E = p.E;
    const int R = H / 16;
    for (int task = blockIdx.x * 8 + warp; task < ntask; task += gridDim.x * 8) {
        const int b = find_bucket(p.ts2, nb, task);
        const int e = __ldg(p.bucket_e + b);
        const int n = __ldg(p.bucket_n + b);
        const int off = __ldg(p.bucket_off + b);
        if (e < 0 || e > E || (e == E && p.Is == 0)) {
            if (lane == 0) atomicOr(&p.ctrl->status, ST_BAD_TASK);
            continue;
        }
        const bool shared = (e == E);
        const int irow = shared ? p.Is : p.I;
        const int row_bytes = irow / 2;
        const int nkb = irow / 128;
        const int local = task - __ldg(p.ts2 + b);
        const int c = local / R, rg = local - c * R;
        const int j0 = rg * 16, tok0 = c * kChunkTokens;
        const int nt = min(kChunkTokens, n - tok0);
        const int ntiles = (nt + 7) >> 3;
        const uint8_t* W = shared ? p.sh_w2 : p.w2 + (size_t)e * H * row_bytes;
        const float* S = shared ? p.sh_s2 : p.s2 + (size_t)e * H;
        const uint8_t* lrow = W + (size_t)(j0 + g) * row_bytes + q * 16;
        const uint8_t* hrow8 = W + (size_t)(j0 + g + 8) * row_bytes + q * 16;
        const __half* hb = shared ? p.h_s : p.h_r;
        const size_t hbase = shared ? 0 : (size_t)off;

        const __half* hr[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int s = tok0 + 8 * i + g;
            hr[i] = (i < ntiles && s < n) ? hb + (hbase + s) * irow + q * 32 : nullptr;
        }

        float acc[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

        uint4 wl = ld_stream_v4(lrow), wh = ld_stream_v4(hrow8);
        for (int kb = 0; kb < nkb; ++kb) {
            uint4 nl = make_uint4(0, 0, 0, 0), nh = nl;
            if (kb + 1 < nkb) {
                nl = ld_stream_v4(lrow + (kb + 1) * 64);
                nh = ld_stream_v4(hrow8 + (kb + 1) * 64);
            }
            const uint32_t lw[4] = {wl.x, wl.y, wl.z, wl.w};
            const uint32_t hw[4] = {wh.x, wh.y, wh.z, wh.w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                uint32_t Lo[4], Hi[4];
                int4x8_to_f16x2(lw[w], Lo);
                int4x8_to_f16x2(hw[w], Hi);
                const uint32_t aA[4] = {Lo[0], Hi[0], Lo[1], Hi[1]};
                const uint32_t aB[4] = {Lo[2], Hi[2], Lo[3], Hi[3]};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (i < ntiles) {
                        uint4 hv = make_uint4(0, 0, 0, 0);
                        if (hr[i]) hv = ld_v4(hr[i] + kb * 128 + w * 8);
                        uint32_t X[4];
                        pair8(hv, X);
                        mma_f16(acc[i], aA, X[0], X[1]);
                        mma_f16(acc[i], aB, X[2], X[3]);
                    }
                }
            }
            wl = nl;
            wh = nh;
        }

        const float sl = __ldg(S + j0 + g), sh = __ldg(S + j0 + g + 8);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i < ntiles) {
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int s = tok0 + 8 * i + 2 * q + cc;
                    if (s < n) {
                        const size_t ys = shared ? (size_t)p.T * p.K + s : (size_t)off + s;
                        float* yr = p.y + ys * H + j0 + g;
                        yr[0] = acc[i][cc] * sl;
                        yr[8] = acc[i][2 + cc] * sh;
                    }
                }
            }
        }
    }
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
