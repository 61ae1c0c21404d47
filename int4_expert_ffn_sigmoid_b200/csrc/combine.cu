// Weighted combine: out[t] = sum_k w[t,k] y[slot(t,k)] + y_shared[t] (+ x[t]),
// summed in f32 (k ascending, then the shared expert, then the residual) and
// rounded once to bf16 (round to nearest even).  An expert output that the
// weight-streaming down projection wrote as partial rows, one per slice of
// its reduction, is first summed over the slices (ascending).
//
// Method: colibri README (project listing), "What's implemented" (shared
// expert; routed experts weighted by the sigmoid router); Colibri-Nano model
// card, "Architecture" (the always-resident shared expert is added for every
// token).
#include "moe_common.cuh"
#include "moe_launch.h"

namespace moe {

__global__ void __launch_bounds__(256) combine_kernel(Params p) {
    __shared__ int s_slot[kMaxK];
    __shared__ float s_w[kMaxK];
    const int t = blockIdx.x;
    const int j = (blockIdx.y * blockDim.x + threadIdx.x) * 4;
    const int K = p.K, H = p.H;
    // The token's slots and routing weights, and its residual row, are final
    // before this kernel starts: the kernel it waits for (the down
    // projection) started only after the one before it had completed, and
    // those were written there or earlier (the bucket tables, the router, the
    // caller).  Small batches, bound by the latency of this chain, read them
    // before the wait (measured: Nano stack T = 64 0.924 -> 0.907 ms); large
    // ones, with thousands of CTAs in flight, read them in the loop (the
    // staging barrier made the T = 16384 combine 72 -> 86 us).
    const bool early = p.decode_groups > 0;
    if (early && threadIdx.x < K) {
        s_slot[threadIdx.x] = __ldcg(p.slot_of + (size_t)t * K + threadIdx.x);
        s_w[threadIdx.x] = __ldcg(p.wts + (size_t)t * K + threadIdx.x);
    }
    const bool res = (p.flags & kFlagResidual) && j < H;
    uint2 xv = early && res ? __ldg(reinterpret_cast<const uint2*>(p.x + (size_t)t * H + j)) : make_uint2(0u, 0u);
    pdl_wait();
    pdl_release();
    if (early) __syncthreads();
    if (j >= H) return;
    if (!early && res) xv = __ldg(reinterpret_cast<const uint2*>(p.x + (size_t)t * H + j));
    const size_t TK = (size_t)p.T * K;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    for (int k = 0; k < K; ++k) {
        const int s = early ? s_slot[k] : __ldcg(p.slot_of + (size_t)t * K + k);
        if (s < 0) continue;  // a pick the top-p dropped
        const float w = early ? s_w[k] : __ldcg(p.wts + (size_t)t * K + k);
        float4 v = __ldcg(reinterpret_cast<const float4*>(p.y + (size_t)s * H + j));
        for (int sl = 1; sl < p.nsl_r; ++sl) {
            const float4 u = __ldcg(reinterpret_cast<const float4*>(p.y + (sl * TK + s) * H + j));
            v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
        }
        a0 = fmaf(w, v.x, a0);
        a1 = fmaf(w, v.y, a1);
        a2 = fmaf(w, v.z, a2);
        a3 = fmaf(w, v.w, a3);
    }
    if (p.Is > 0) {
        const float* ys = p.y + TK * p.nsl_r * H;
        float4 v = __ldcg(reinterpret_cast<const float4*>(ys + (size_t)t * H + j));
        for (int sl = 1; sl < p.nsl_s; ++sl) {
            const float4 u = __ldcg(reinterpret_cast<const float4*>(ys + ((size_t)sl * p.T + t) * H + j));
            v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
        }
        a0 += v.x; a1 += v.y; a2 += v.z; a3 += v.w;
    }
    if (res) {
        a0 += bf16lo(xv.x); a1 += bf16hi(xv.x); a2 += bf16lo(xv.y); a3 += bf16hi(xv.y);
    }
    if (p.flags & kFlagOutF32) {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + (size_t)t * H + j) = make_float4(a0, a1, a2, a3);
        return;
    }
    __nv_bfloat162 o01 = __floats2bfloat162_rn(a0, a1);
    __nv_bfloat162 o23 = __floats2bfloat162_rn(a2, a3);
    uint2 ov;
    ov.x = *reinterpret_cast<uint32_t*>(&o01);
    ov.y = *reinterpret_cast<uint32_t*>(&o23);
    *reinterpret_cast<uint2*>(p.out + (size_t)t * H + j) = ov;
}

cudaError_t launch_combine(const Params& p, cudaStream_t stream) {
    return launch_pdl(combine_kernel, dim3(p.T, (p.H + 1023) / 1024), dim3(256), 0, stream, p);
}

}  // namespace moe
