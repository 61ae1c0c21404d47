// Router logits of the large-batch sequences on the 5th-generation tensor
// cores (tcgen05, accumulators in tensor memory).
//
// Method: colibri README (project listing), "What's implemented": the
// sigmoid+bias router with f32 router weights (nanocolibri-engine README,
// "Converting a checkpoint yourself": the router stays f32).  The logit of
// token t and expert e is L[t][e] = sum_h x[t][h] * W[e][h].
//
// Arithmetic.  x is exactly bf16.  Each f32 weight splits exactly into three
// bf16 terms, w = hi + mid + lo (hi = bf16(w), mid = bf16(w - hi),
// lo = bf16(w - hi - mid): together they hold w's 24-bit significand), so the
// products x*hi, x*mid, x*lo are exact in f32.  Every 16-wide k step is one
// accumulation chain on the tensor cores that starts from zero (the 16
// products of lo, then of mid, then of hi), written to a tensor-memory buffer
// of its own; the epilogue adds the step sums to its registers with ordinary
// f32 adds in k order.  The logits therefore carry f32 rounding only.  Each
// CTA covers one hidden slice; the selecting kernel adds the slices' partial
// logits in ascending order, so a token's logit does not depend on the other
// tokens of the batch.
//
// Kernels:
//   router_wsplit_kernel     W [E][H] f32 -> Wsplit [3][E][H] bf16 (hi, mid, lo);
//                            the first kernel of the call (it zeroes the status word)
//   router_logits_tc_kernel  CTA (128-token tile, expert tile of N <= 128, hidden
//                            slice) -> lpart[slice][T][E]
// Roles of router_logits_tc_kernel (576 threads):
//   warp 0      TMA producer (token tile 128 x 64, and the three weight terms'
//               N x 64 tiles, 128-byte swizzle) and TMEM owner
//   warp 1      MMA issuer (three tcgen05.mma kind::f16 per 16-wide k step,
//               M=128, N, K=16, into a fresh buffer)
//   warps 2-17  epilogue: the warp of lane quarter q and column quarter c adds
//               the step sums of tokens 32q..32q+31, experts c*N/4.. of the tile
// Every wait is bounded (clock64); on timeout the CTA records ST_TIMEOUT,
// drains its copies and MMAs (bounded waits that ignore the abort), frees
// tensor memory and exits.
#include <cuda.h>

#include "moe_common.cuh"
#include "moe_launch.h"
#include "moe_tc.h"
#include "stream_ops.cuh"

namespace moe {
namespace rtc {

constexpr int BM = 128;  // tokens per tile
constexpr int BK = 64;   // hidden elements per stage
constexpr int STAGES = 3;
constexpr int X_BYTES = BM * BK * 2;
constexpr int EPI_WARPS = 16;
constexpr int NUM_THREADS = 64 + 32 * EPI_WARPS;
constexpr int kMaxN = 128;
// Hidden slices: at least kMinSliceKb k blocks each, at most kMaxSlices of
// them.  The slicing depends on H only, so a token's logit is summed in the
// same order whatever the rest of the batch.
constexpr int kMinSliceKb = 4;
constexpr int kMaxSlices = 8;
constexpr long long kTimeoutCycles = 4000000000LL;
constexpr long long kDrainCycles = 200000000LL;

template <int N>
struct Geo {
    static constexpr int W_BYTES = N * BK * 2;  // one weight term's tile
    static constexpr int STAGE_BYTES = X_BYTES + 3 * W_BYTES;
    static constexpr int NBUF = (512 / N) < 8 ? 512 / N : 8;  // tensor-memory step buffers
    static constexpr int TMEM_COLS = NBUF * N < 32 ? 32 : NBUF * N;
    static constexpr int CPW = N / 4;  // columns per epilogue warp
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256;
    static_assert(STAGE_BYTES % 1024 == 0, "stages stay 1024-byte aligned");
    static_assert((TMEM_COLS & (TMEM_COLS - 1)) == 0 && TMEM_COLS <= 512, "tensor memory allocation");
};

struct Bars {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t bfull[8];
    uint64_t bempty[8];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Bars* b) {
    if (bar_try(bar, parity)) return true;
    const long long t0 = clock64();
    while (!bar_try(bar, parity)) {
        if (*reinterpret_cast<volatile int*>(&b->abort_flag)) return false;
        if (clock64() - t0 > kTimeoutCycles) {
            *reinterpret_cast<volatile int*>(&b->abort_flag) = 1;
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// kind::f16, bf16 operands, f32 accumulate, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// CPW consecutive f32 columns of this thread's TMEM lane, added to acc.
template <int CPW>
__device__ __forceinline__ void tmem_add(uint32_t taddr, float (&acc)[CPW]) {
    uint32_t v[CPW];
    if constexpr (CPW == 4) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];\n"
            "tcgen05.wait::ld.sync.aligned;\n"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
            : "r"(taddr)
            : "memory");
    } else if constexpr (CPW == 8) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
            "tcgen05.wait::ld.sync.aligned;\n"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
            : "r"(taddr)
            : "memory");
    } else if constexpr (CPW == 16) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
            "tcgen05.wait::ld.sync.aligned;\n"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
            : "r"(taddr)
            : "memory");
    } else {
        static_assert(CPW == 32, "column count of an epilogue warp");
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
            "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
            "tcgen05.wait::ld.sync.aligned;\n"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
              "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
              "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
            : "r"(taddr)
            : "memory");
    }
#pragma unroll
    for (int i = 0; i < CPW; ++i) acc[i] += __uint_as_float(v[i]);
}

struct Geom {
    int N, ntile_e, slices, kb_per;  // expert tile width, expert tiles, hidden slices, k blocks per slice
};

__host__ __device__ inline Geom geometry(int E, int H) {
    Geom g;
    int n = 16;
    while (n < E && n < kMaxN) n <<= 1;
    g.N = n;
    g.ntile_e = (E + n - 1) / n;
    const int nkb = H / BK;
    const int per = (nkb + kMaxSlices - 1) / kMaxSlices;
    g.kb_per = per < kMinSliceKb ? kMinSliceKb : per;
    g.slices = (nkb + g.kb_per - 1) / g.kb_per;
    return g;
}

}  // namespace rtc

// W [E][H] f32 -> Wsplit [3][E][H] bf16 (hi, mid, lo), 8 weights per thread step.
__global__ void __launch_bounds__(256) router_wsplit_kernel(Params p) {
    pdl_wait();  // the previous call's kernels are done with the workspace
    reset_ctrl(p);
    pdl_release();
    const size_t n8 = (size_t)p.E * p.H / 8, plane = (size_t)p.E * p.H;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(p.rw) + 2 * i);
        const float4 b = __ldg(reinterpret_cast<const float4*>(p.rw) + 2 * i + 1);
        const float w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint16_t hi[8], mid[8], lo[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) split3(w[j], hi[j], mid[j], lo[j]);
        auto pack = [](const uint16_t* v) {
            return make_uint4((uint32_t)v[0] | ((uint32_t)v[1] << 16), (uint32_t)v[2] | ((uint32_t)v[3] << 16),
                              (uint32_t)v[4] | ((uint32_t)v[5] << 16), (uint32_t)v[6] | ((uint32_t)v[7] << 16));
        };
        uint4* dst = reinterpret_cast<uint4*>(p.wsplit);
        dst[i] = pack(hi);
        dst[plane / 8 + i] = pack(mid);
        dst[2 * (plane / 8) + i] = pack(lo);
    }
}

template <int N>
__global__ void __launch_bounds__(rtc::NUM_THREADS, 1)
router_logits_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, const Params p,
                        const rtc::Geom geo) {
    using G = rtc::Geo<N>;
    using namespace rtc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + STAGES * G::STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int slice = blockIdx.x % geo.slices;
    const int rest = blockIdx.x / geo.slices;
    const int etile = rest % geo.ntile_e, tile = rest / geo.ntile_e;
    const int t0 = tile * BM, n0 = etile * N;
    const int nkb = p.H / BK;
    const int kb0 = slice * geo.kb_per;
    const int kb1 = min(nkb, kb0 + geo.kb_per);
    const int nsteps = (kb1 - kb0) * (BK / 16);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            bar_init(&bars->full[s], 1);
            bar_init(&bars->empty[s], 1);
        }
        for (int b = 0; b < G::NBUF; ++b) {
            bar_init(&bars->bfull[b], 1);
            bar_init(&bars->bempty[b], EPI_WARPS);
        }
        bar_init(&bars->drain, 1);
        bars->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&bars->tmem_base)),
                     "r"(G::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = bars->tmem_base;
    pdl_wait();  // the weight split (previous kernel) is complete
    pdl_release();

    if (warp == 0) {
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW)) : "memory");
            bool issued[STAGES] = {false, false, false};
            uint32_t ipar[STAGES] = {0, 0, 0};
            for (int kb = kb0, n = 0; kb < kb1; ++kb, ++n) {
                const int s = n % STAGES;
                const uint32_t ph = (n / STAGES) & 1u;
                if (!wait_or_abort(&bars->empty[s], ph ^ 1u, bars)) break;
                uint8_t* st = smem + s * G::STAGE_BYTES;
                bar_expect_tx(&bars->full[s], G::STAGE_BYTES);
                tma_tile(st, &tmX, &bars->full[s], kb * BK, t0);
#pragma unroll
                for (int part = 0; part < 3; ++part)  // hi, mid, lo planes of Wsplit
                    tma_tile(st + X_BYTES + part * G::W_BYTES, &tmW, &bars->full[s], kb * BK, part * p.E + n0);
                issued[s] = true;
                ipar[s] = ph;
            }
            for (int s = 0; s < STAGES; ++s)
                if (issued[s]) bar_wait(&bars->full[s], ipar[s], kDrainCycles);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(BM, N);
            bool any = false;
            int j = 0;  // k steps so far
            for (int kb = kb0, n = 0; kb < kb1; ++kb, ++n) {
                const int s = n % STAGES;
                if (!wait_or_abort(&bars->full[s], (n / STAGES) & 1u, bars)) break;
                fence_after();
                const uint32_t xa = smem_addr(smem + s * G::STAGE_BYTES);
                const uint32_t wa = xa + X_BYTES;
                bool ok = true;
#pragma unroll 1
                for (int kk = 0; kk < BK / 16; ++kk, ++j) {
                    const int b = j % G::NBUF;
                    if (!wait_or_abort(&bars->bempty[b], ((j / G::NBUF) & 1u) ^ 1u, bars)) {
                        ok = false;
                        break;
                    }
                    fence_after();
                    const uint32_t d = tmem + b * N;
                    const uint64_t xd = desc_sw128(xa + kk * 32);
                    // lo, then mid, then hi into a fresh accumulator
                    mma_ss(d, xd, desc_sw128(wa + 2 * G::W_BYTES + kk * 32), idesc, 0);
                    mma_ss(d, xd, desc_sw128(wa + 1 * G::W_BYTES + kk * 32), idesc, 1);
                    mma_ss(d, xd, desc_sw128(wa + kk * 32), idesc, 1);
                    any = true;
                    commit(&bars->bfull[b]);
                }
                if (!ok) break;
                commit(&bars->empty[s]);
            }
            if (any) {
                commit(&bars->drain);
                bar_wait(&bars->drain, 0, kDrainCycles);
            }
        }
    } else {
        const int q = warp & 3, cq = (warp - 2) >> 2;
        const int m = q * 32 + lane;
        float acc[G::CPW];
#pragma unroll
        for (int i = 0; i < G::CPW; ++i) acc[i] = 0.f;
        bool ok = true;
        const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16) + cq * G::CPW;
        for (int j = 0; j < nsteps; ++j) {
            const int b = j % G::NBUF;
            if (!__all_sync(0xffffffffu, wait_or_abort(&bars->bfull[b], (j / G::NBUF) & 1u, bars))) {
                ok = false;
                break;
            }
            fence_after();
            tmem_add<G::CPW>(lane_base + b * N, acc);
            fence_before();
            __syncwarp();
            if (lane == 0) bar_arrive(&bars->bempty[b]);
        }
        const int t = t0 + m;
        if (ok && t < p.T) {
            float* dst = p.lpart + ((size_t)slice * p.T + t) * p.E + n0 + cq * G::CPW;
#pragma unroll
            for (int i = 0; i < G::CPW; ++i)
                if (n0 + cq * G::CPW + i < p.E) __stcg(dst + i, acc[i]);
        }
    }

    __syncthreads();
    if (threadIdx.x == 0 && bars->abort_flag) atomicOr(&p.ctrl->status, ST_TIMEOUT);
    if (warp == 0) {
        fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(G::TMEM_COLS) : "memory");
    }
}

int tc_router_slices(int E, int H) { return rtc::geometry(E, H).slices; }

namespace {

template <int N>
cudaError_t launch_n(const Params& p, const rtc::Geom& g, const CUtensorMap& mx, const CUtensorMap& mw,
                     cudaStream_t stream) {
    static int attr_set[64];
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64 && !attr_set[dev]) {
        const cudaError_t e = cudaFuncSetAttribute(router_logits_tc_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   rtc::Geo<N>::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set[dev] = 1;
    }
    const int tiles = (p.T + rtc::BM - 1) / rtc::BM;
    return launch_pdl(router_logits_tc_kernel<N>, dim3(tiles * g.ntile_e * g.slices), dim3(rtc::NUM_THREADS),
                      rtc::Geo<N>::SMEM_BYTES, stream, mx, mw, p, g);
}

}  // namespace

cudaError_t launch_router_tc(const Params& p, cudaStream_t stream) {
    const rtc::Geom g = rtc::geometry(p.E, p.H);
    if (g.slices != p.lslices) return cudaErrorInvalidValue;
    CUtensorMap mx, mw;
    if (!encode_tensor_map_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.x, p.H, p.T, rtc::BK, rtc::BM,
                              CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tensor_map_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.wsplit, p.H, 3 * (uint64_t)p.E, rtc::BK,
                              g.N, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const size_t n8 = (size_t)p.E * p.H / 8;
    const int sblocks = (int)((n8 + 255) / 256 < 592 ? (n8 + 255) / 256 : 592);
    cudaError_t err = launch_pdl(router_wsplit_kernel, dim3(sblocks), dim3(256), 0, stream, p);
    if (err != cudaSuccess) return err;
    switch (g.N) {
        case 16: return launch_n<16>(p, g, mx, mw, stream);
        case 32: return launch_n<32>(p, g, mx, mw, stream);
        case 64: return launch_n<64>(p, g, mx, mw, stream);
        case 128: return launch_n<128>(p, g, mx, mw, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
