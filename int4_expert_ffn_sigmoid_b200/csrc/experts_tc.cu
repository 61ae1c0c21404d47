// Large-batch expert kernels: a persistent grouped GEMM on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory) with in-kernel int4
// dequantisation, run twice per layer:
//   GEMM-1: [tokens of a bucket] x [gate rows ; up rows]^T, SwiGLU epilogue -> h (fp16)
//   GEMM-2: [h of a bucket] x [down rows]^T, row-scale epilogue -> y (f32)
// over every non-empty routed bucket and the shared expert.
//
// Method: colibri README (project listing), "What's implemented": packed int4,
// per-row scales, dequant-on-use; batch-union MoE (each expert touched by the
// batch is read once and applied to all of its tokens); nanocolibri-engine
// README, "Converting a checkpoint yourself": per-row symmetric int4, f32 scales.
//
// Tile: 128 tokens (MMA M, one TMEM lane per token) x 256 output columns (MMA
// N) x 64 reduction elements per pipeline stage.  Two rings: TMA stages hold
// the activation and raw int4 tiles of 6 k blocks; 2 slots hold the
// dequantised B operand between the dequantisers and the MMA.  GEMM-1's 256 columns are 128
// gate rows and the 128 up rows of the same features, so one thread of the
// epilogue holds gate and up of one (token, feature) pair.
// Roles (448 threads):
//   warp 0      TMA producer (activation tile, raw int4 weight tile) and TMEM owner
//   warp 1      MMA issuer (one thread, tcgen05.mma kind::f16, M=128 N=256 K=16)
//   warps 2-9   dequantisers, one B row per thread: raw int4 -> exact 16-bit
//               integers in the 128-byte swizzled K-major layout of the B
//               operand (the row scale is applied in the epilogue)
//   warps 10-13 epilogue: tcgen05.ld of the accumulator, scales (staged in
//               shared memory per tile), SwiGLU, stores
// Every mbarrier wait is bounded (clock64); on timeout the CTA records
// ST_TIMEOUT in the status word and stops.  The drains then ignore the abort
// (each with its own bound): the producer waits until every TMA copy it issued
// has landed and the MMA thread until every MMA it issued has completed, and
// only then is tensor memory released and the CTA gone.
#include <cuda.h>

#include "moe_common.cuh"
#include "moe_launch.h"
#include "moe_tc.h"

namespace moe {
namespace tc {

constexpr int BM = 128, BN = 256, BK = 64;
// Two rings: TMA stages (activation tile + raw int4 tile) run TSTAGES k
// blocks ahead to cover load latency; the dequantised B operand needs only
// BSTAGES slots between the dequantisers and the MMA.
constexpr int TSTAGES = 6;
constexpr int BSTAGES = 2;
constexpr int A_BYTES = BM * BK * 2;    // 16 KiB, bf16/fp16 activations
constexpr int B_BYTES = BN * BK * 2;    // 32 KiB, dequantised weights
constexpr int RAW_BYTES = BN * BK / 2;  // 8 KiB, packed int4 weights
constexpr int TSTAGE_BYTES = A_BYTES + RAW_BYTES;
constexpr int RING_BYTES = TSTAGES * TSTAGE_BYTES + BSTAGES * B_BYTES;
constexpr int DEQ_WARPS = 8;
constexpr int NUM_THREADS = 64 + 32 * DEQ_WARPS + 128;
constexpr int TMEM_COLS = 512;          // two 256-column accumulators
constexpr long long kTimeoutCycles = 4000000000LL;
constexpr long long kDrainCycles = 200000000LL;
// MOE_TEST_STALL: the epilogue first waits this long on a barrier nothing
// arrives on (~1 ms), which makes the CTA take its timeout path while its
// copies and MMAs are in flight.
constexpr long long kStallCycles = 1LL << 21;
constexpr int SMEM_BYTES = RING_BYTES + 1024 + 1280;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory of the grouped GEMM");

struct Shared {
    uint64_t full_tma[TSTAGES];  // activation + raw tiles landed (TMA transaction count)
    uint64_t empty_t[TSTAGES];   // MMA done with the activation tile, dequantisers with the raw tile
    uint64_t full_deq[BSTAGES];  // B operand dequantised (one arrival per dequant warp)
    uint64_t empty_b[BSTAGES];   // MMA done with the B operand
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint64_t never;  // nothing arrives on it (MOE_TEST_STALL)
    uint32_t tmem_base;
    int abort_flag;
    float ep_scale[BN];  // the current tile's row scales (epilogue)
    int ep_ok[4];        // per epilogue warp: its accumulator wait succeeded
};
static_assert(sizeof(Shared) <= 1280, "shared control block");

// Barrier among the 4 epilogue warps only.
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait.  Returns false when the CTA aborts (this wait timed out, or
// another role set the abort flag).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, Shared* sh, long long limit = kTimeoutCycles) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*reinterpret_cast<volatile int*>(&sh->abort_flag)) return false;
        if (clock64() - t0 > limit) {
            *reinterpret_cast<volatile int*>(&sh->abort_flag) = 1;
            return false;
        }
    }
}

// Bounded wait that ignores the abort flag: the drains after an abort, which
// must see the CTA's own copies and MMAs complete before its shared memory
// and tensor memory go away.  Returns false only when `limit` runs out.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > limit) return false;
    return true;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
            "r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// Shared-memory matrix descriptor: K-major operand in the 128-byte swizzled
// canonical layout (8-row x 128-byte atoms, atoms 1024 bytes apart).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor, kind::f16, f32 accumulate, both operands K-major.
// fmt: 0 = fp16, 1 = bf16.
__host__ __device__ constexpr uint32_t idesc_f16(int fmt, int M, int N) {
    return (1u << 4) | ((uint32_t)fmt << 7) | ((uint32_t)fmt << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16_ss(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 16 consecutive f32 columns of this thread's TMEM lane.  The load and its
// wait are one asm statement, so no instruction can read the registers early.
__device__ __forceinline__ void tmem_ld16_wait(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        "tcgen05.wait::ld.sync.aligned;\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// Eight int4 codes (a 32-bit word, element j in nibble j) -> four 16-bit pairs
// in natural order: out[j] = (element 2j, element 2j+1), by the exponent-bias
// technique of Kim et al. (2022): (c + 8) in the low mantissa bits of 2^m,
// minus 2^m + 8.  magic = 2^m in both halves, bias = 2^m + 8 in both halves.
template <bool kBf16>
__device__ __forceinline__ void int4x8_natural(uint32_t w, uint32_t (&o)[4]) {
    const uint32_t v = w ^ 0x88888888u;
    const uint32_t v4 = v >> 4;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        // byte j of v (low nibble = element 2j) into half 0, byte j of v>>4
        // (low nibble = element 2j+1) into half 1
        const uint32_t t = __byte_perm(v, v4, j | ((4 + j) << 8)) & 0x000F000Fu;
        if (kBf16) {
            uint32_t u = t | 0x43004300u;
            __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&u),
                                       __halves2bfloat162(__ushort_as_bfloat16(0x4308), __ushort_as_bfloat16(0x4308)));
            o[j] = *reinterpret_cast<uint32_t*>(&r);
        } else {
            uint32_t u = t | 0x64006400u;
            __half2 r = __hsub2(*reinterpret_cast<__half2*>(&u),
                                __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408)));
            o[j] = *reinterpret_cast<uint32_t*>(&r);
        }
    }
}

struct Tile {
    int shared;   // 1: shared expert
    int e;        // expert id (E for shared)
    int n_valid;  // valid tokens in this tile
    int a_row;    // first activation row (TMA y coordinate)
    int slot0;    // first output row of the tile (h row / y slot)
    int col0;     // first output column (GEMM-1: feature j0; GEMM-2: feature n0)
    int nkb;      // k blocks
};

__device__ __forceinline__ Tile decode_tile(const TcArgs& a, int tile) {
    Tile t;
    const int mt_s = a.Is > 0 ? (a.T + BM - 1) / BM : 0;
    const int n_sh = mt_s * a.ntile_s;
    if (tile < n_sh) {
        const int mt = tile % mt_s, nt = tile / mt_s;
        t.shared = 1;
        t.e = a.E;
        t.n_valid = min(BM, a.T - mt * BM);
        t.a_row = mt * BM;
        t.slot0 = mt * BM;
        t.col0 = nt * (a.gemm == 1 ? BN / 2 : BN);
        t.nkb = a.kdim_s / BK;
        return t;
    }
    const int r = tile - n_sh;
    const int nbr = a.ctrl->n_buckets - (a.Is > 0 ? 1 : 0);
    int lo = 0, hi = nbr;  // tstart[lo] <= r < tstart[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(a.tstart + mid) <= r) lo = mid; else hi = mid;
    }
    const int local = r - __ldg(a.tstart + lo);
    const int n = __ldg(a.bucket_n + lo);
    const int off = __ldg(a.bucket_off + lo);
    const int mtiles = (n + BM - 1) / BM;
    const int mt = local % mtiles, nt = local / mtiles;
    t.shared = 0;
    t.e = __ldg(a.bucket_e + lo);
    t.n_valid = min(BM, n - mt * BM);
    t.a_row = off + mt * BM;
    t.slot0 = off + mt * BM;
    t.col0 = nt * (a.gemm == 1 ? BN / 2 : BN);
    t.nkb = a.kdim_r / BK;
    return t;
}

__device__ __forceinline__ int total_tiles(const TcArgs& a) {
    const int mt_s = a.Is > 0 ? (a.T + BM - 1) / BM : 0;
    return mt_s * a.ntile_s + (a.gemm == 1 ? a.ctrl->tc_tiles1 : a.ctrl->tc_tiles2);
}

template <int GEMM>
__global__ void __launch_bounds__(NUM_THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmA_s,
                    const __grid_constant__ CUtensorMap tmB_r, const __grid_constant__ CUtensorMap tmB_s,
                    const TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Shared* sh = reinterpret_cast<Shared*>(smem + RING_BYTES);
    auto a_tile = [&](int s) { return smem + s * TSTAGE_BYTES; };
    auto raw_tile = [&](int s) { return smem + s * TSTAGE_BYTES + A_BYTES; };
    auto b_tile = [&](int s) { return smem + TSTAGES * TSTAGE_BYTES + s * B_BYTES; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < TSTAGES; ++s) {
            mbar_init(&sh->full_tma[s], 1);
            mbar_init(&sh->empty_t[s], 1 + DEQ_WARPS);
        }
        for (int s = 0; s < BSTAGES; ++s) {
            mbar_init(&sh->full_deq[s], DEQ_WARPS);
            mbar_init(&sh->empty_b[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sh->acc_full[b], 1);
            mbar_init(&sh->acc_empty[b], 4);
        }
        mbar_init(&sh->drain, 1);
        mbar_init(&sh->never, 1);
        sh->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sh->tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;
    pdl_wait();  // barriers and TMEM were set up while the previous kernel finished
    pdl_release();
    const int ntiles = total_tiles(a);

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA_r)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA_s)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB_r)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB_s)) : "memory");
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued_par[TSTAGES];
            bool issued[TSTAGES];
            for (int i = 0; i < TSTAGES; ++i) issued[i] = false, issued_par[i] = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
                const Tile t = decode_tile(a, tile);
                const CUtensorMap* mA = t.shared ? &tmA_s : &tmA_r;
                const CUtensorMap* mB = t.shared ? &tmB_s : &tmB_r;
                int brow0, brow1;
                if (GEMM == 1) {
                    const int irow = t.shared ? a.Is : a.I;
                    const int base = t.shared ? 0 : t.e * 2 * a.I;
                    brow0 = base + t.col0;
                    brow1 = base + irow + t.col0;
                } else {
                    const int base = t.shared ? 0 : t.e * a.H;
                    brow0 = base + t.col0;
                    brow1 = base + t.col0 + BN / 2;
                }
                for (int kb = 0; kb < t.nkb; ++kb) {
                    if (!mbar_wait(&sh->empty_t[s], ph ^ 1u, sh)) { ok = false; break; }
                    mbar_expect_tx(&sh->full_tma[s], A_BYTES + RAW_BYTES);
                    tma_load_2d(a_tile(s), mA, &sh->full_tma[s], kb * BK, t.a_row);
                    tma_load_2d(raw_tile(s), mB, &sh->full_tma[s], kb * (BK / 2), brow0);
                    tma_load_2d(raw_tile(s) + RAW_BYTES / 2, mB, &sh->full_tma[s], kb * (BK / 2), brow1);
                    issued[s] = true;
                    issued_par[s] = ph;
                    if (++s == TSTAGES) { s = 0; ph ^= 1u; }
                }
            }
            // make sure no copy is still landing when the CTA leaves
            for (int i = 0; i < TSTAGES; ++i)
                if (issued[i]) mbar_wait_drain(&sh->full_tma[i], issued_par[i], kDrainCycles);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16(GEMM == 1 ? 1 : 0, BM, BN);
            int s = 0, sb = 0;
            uint32_t ph = 0, phb = 0;
            uint32_t acc_ph[2] = {0, 0};
            int buf = 0;
            bool ok = true, any = false;
            for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
                const Tile t = decode_tile(a, tile);
                if (!mbar_wait(&sh->acc_empty[buf], acc_ph[buf] ^ 1u, sh)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem + buf * BN;
                for (int kb = 0; kb < t.nkb; ++kb) {
                    if (!mbar_wait(&sh->full_tma[s], ph, sh) || !mbar_wait(&sh->full_deq[sb], phb, sh)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t aaddr = smem_u32(a_tile(s)), baddr = smem_u32(b_tile(sb));
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        mma_f16_ss(d, smem_desc_sw128(aaddr + kk * 32), smem_desc_sw128(baddr + kk * 32), idesc,
                                   (kb | kk) != 0);
                    }
                    any = true;
                    mma_commit(&sh->empty_t[s]);
                    mma_commit(&sh->empty_b[sb]);
                    if (++s == TSTAGES) { s = 0; ph ^= 1u; }
                    if (++sb == BSTAGES) { sb = 0; phb ^= 1u; }
                }
                if (!ok) break;
                mma_commit(&sh->acc_full[buf]);
                acc_ph[buf] ^= 1u;
                buf ^= 1;
            }
            // Before TMEM is released, every MMA this thread issued must be done:
            // after an abort the epilogue may not wait for the accumulators.
            if (any) {
                mma_commit(&sh->drain);
                mbar_wait_drain(&sh->drain, 0, kDrainCycles);
            }
        }
    } else if (warp < 2 + DEQ_WARPS) {
        // ---------------- dequantisers (one B row per thread) ----------------
        const int r = threadIdx.x - 64;  // B row = output column of the tile
        int s = 0, sb = 0;
        uint32_t ph = 0, phb = 0;
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
            const Tile t = decode_tile(a, tile);
            for (int kb = 0; kb < t.nkb; ++kb) {
                int got = 0;
                if (lane == 0) got = mbar_wait(&sh->full_tma[s], ph, sh) && mbar_wait(&sh->empty_b[sb], phb ^ 1u, sh);
                if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
                const uint8_t* raw = raw_tile(s);
                uint8_t* bt = b_tile(sb);
                {
                    // the two 16-byte halves of this row, the half (r ^ r >> 2) & 1 first:
                    // each quarter-warp's 8 reads then fall on 8 different 16-byte bank
                    // groups (rows are 32 bytes apart)
                    const int h0 = (r ^ (r >> 2)) & 1;
                    const uint4 qa = *reinterpret_cast<const uint4*>(raw + r * 32 + 16 * h0);
                    const uint4 qb = *reinterpret_cast<const uint4*>(raw + r * 32 + 16 * (h0 ^ 1));
                    const uint4 q0 = h0 ? qb : qa, q1 = h0 ? qa : qb;
                    const uint32_t words[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
                    uint8_t* row = bt + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {  // 16-byte chunk c = elements 8c..8c+7
                        uint32_t o[4];
                        int4x8_natural<GEMM == 1>(words[c], o);
                        *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&sh->full_deq[sb]);
                    mbar_arrive(&sh->empty_t[s]);  // this warp is done with the raw tile
                }
                if (++s == TSTAGES) { s = 0; ph ^= 1u; }
                if (++sb == BSTAGES) { sb = 0; phb ^= 1u; }
            }
        }
    } else {
        // ---------------- epilogue (128 threads, one TMEM lane each) ----------------
        const int quarter = warp & 3;
        const int m = quarter * 32 + lane;  // token row of the tile
        uint32_t acc_ph[2] = {0, 0};
        int buf = 0;
        const int et = threadIdx.x - 64 - 32 * DEQ_WARPS;  // 0..127
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
            const Tile t = decode_tile(a, tile);
            const bool valid = m < t.n_valid;
            // this tile's row scales and this thread's token, loaded while the
            // tensor cores still work on the tile
            const int irow = t.shared ? a.Is : a.I;
            epi_bar();  // every epilogue warp is done with the previous tile's scales
            if (GEMM == 1) {
                const float* sc = t.shared ? a.s_s : a.s_r + (size_t)t.e * 2 * a.I;
                sh->ep_scale[et] = __ldg(sc + t.col0 + et);
                sh->ep_scale[BN / 2 + et] = __ldg(sc + irow + t.col0 + et);
            } else {
                const float* sc = t.shared ? a.s_s : a.s_r + (size_t)t.e * a.H;
                sh->ep_scale[et] = __ldg(sc + t.col0 + et);
                sh->ep_scale[BN / 2 + et] = __ldg(sc + t.col0 + BN / 2 + et);
            }
            const int tok = valid ? (t.shared ? t.slot0 + m : __ldg(a.tok_of_slot + t.slot0 + m)) : 0;
            const int hx = __ldg(a.hexp + tok);
            int got = 0;
            if (lane == 0)
                got = (!a.stall || mbar_wait(&sh->never, 0, sh, kStallCycles)) &&
                      mbar_wait(&sh->acc_full[buf], acc_ph[buf], sh);
            if (lane == 0) sh->ep_ok[quarter] = got;
            epi_bar();  // scales visible; every warp's wait outcome known
            if (!(sh->ep_ok[0] && sh->ep_ok[1] && sh->ep_ok[2] && sh->ep_ok[3])) break;
            tc_fence_after();
            const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + buf * BN;
            const float* scs = sh->ep_scale;
            if (GEMM == 1) {
                __half* hrow = (t.shared ? a.h_s : a.h_r) + (size_t)(t.slot0 + m) * irow + t.col0;
                const float hsc = ldexpf(1.0f, -hx);
#pragma unroll 1
                for (int c0 = 0; c0 < BN / 2; c0 += 16) {
                    uint32_t g[16], u[16];
                    tmem_ld16_wait(tbase + c0, g);
                    tmem_ld16_wait(tbase + BN / 2 + c0, u);
                    uint32_t packed[8];
#pragma unroll
                    for (int i = 0; i < 16; i += 2) {
                        const int j = c0 + i;
                        const float g0 = __uint_as_float(g[i]) * scs[j];
                        const float g1 = __uint_as_float(g[i + 1]) * scs[j + 1];
                        const float u0 = __uint_as_float(u[i]) * scs[BN / 2 + j];
                        const float u1 = __uint_as_float(u[i + 1]) * scs[BN / 2 + j + 1];
                        __half2 hv = __floats2half2_rn(silu_mul(g0, u0) * hsc, silu_mul(g1, u1) * hsc);
                        packed[i >> 1] = *reinterpret_cast<uint32_t*>(&hv);
                    }
                    if (valid) {
                        uint4* dst = reinterpret_cast<uint4*>(hrow + c0);
                        dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                        dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
                    }
                }
            } else {
                const size_t slot = t.shared ? (size_t)a.T * a.K + t.slot0 + m : (size_t)(t.slot0 + m);
                float* yrow = a.y + slot * a.H + t.col0;
                const float inv = ldexpf(1.0f, hx);
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 16) {
                    uint32_t v[16];
                    tmem_ld16_wait(tbase + c0, v);
                    if (valid) {
                        float4* dst = reinterpret_cast<float4*>(yrow + c0);
#pragma unroll
                        for (int i = 0; i < 16; i += 4) {
                            const int j = c0 + i;
                            dst[i >> 2] = make_float4(__uint_as_float(v[i]) * (scs[j] * inv),
                                                      __uint_as_float(v[i + 1]) * (scs[j + 1] * inv),
                                                      __uint_as_float(v[i + 2]) * (scs[j + 2] * inv),
                                                      __uint_as_float(v[i + 3]) * (scs[j + 3] * inv));
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh->acc_empty[buf]);
            acc_ph[buf] ^= 1u;
            buf ^= 1;
        }
    }

    __syncthreads();
    if (threadIdx.x == 0 && sh->abort_flag) atomicOr(a.status, ST_TIMEOUT);
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

}  // namespace tc

// ---------------------------------------------------------------------------
// Host side: tensor maps and launches.
// ---------------------------------------------------------------------------

namespace {

PFN_encodeTiled g_encode = nullptr;

bool get_encode() {
    if (g_encode) return true;
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
        return false;
    g_encode = reinterpret_cast<PFN_encodeTiled>(fn);
    return true;
}

// 2-D tensor map over a row-major [rows][inner] matrix.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int esize, const void* base, uint64_t inner, uint64_t rows,
              uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * (uint64_t)esize};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t es[2] = {1, 1};
    const CUresult r = g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, es,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int g_smem_set[64];

}  // namespace

bool encode_tensor_map_2d(CUtensorMap* m, CUtensorMapDataType dt, int esize, const void* base, uint64_t inner,
                          uint64_t rows, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
    return get_encode() && make_map(m, dt, esize, base, inner, rows, box_inner, box_rows, sw);
}

int tc_smem_bytes() { return tc::SMEM_BYTES; }

cudaError_t launch_tc_gemm(const Params& p, int gemm, int grid, cudaStream_t stream) {
    if (!get_encode()) return cudaErrorNotSupported;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !g_smem_set[dev]) {
        cudaError_t e1 = cudaFuncSetAttribute(tc::grouped_gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              tc::SMEM_BYTES);
        cudaError_t e2 = cudaFuncSetAttribute(tc::grouped_gemm_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              tc::SMEM_BYTES);
        if (e1 != cudaSuccess) return e1;
        if (e2 != cudaSuccess) return e2;
        g_smem_set[dev] = 1;
    }
    const int TK = p.T * p.K;
    const int Is = p.Is > 0 ? p.Is : 128;  // any valid map when there is no shared expert
    CUtensorMap mA_r, mA_s, mB_r, mB_s;
    TcArgs a;
    memset(&a, 0, sizeof a);
    a.T = p.T; a.H = p.H; a.E = p.E; a.K = p.K; a.I = p.I; a.Is = p.Is;
    a.gemm = gemm;
    a.ctrl = p.ctrl;
    a.bucket_e = p.bucket_e; a.bucket_n = p.bucket_n; a.bucket_off = p.bucket_off;
    a.status = &p.ctrl->status;
    a.h_r = p.h_r; a.h_s = p.h_s; a.y = p.y;
    a.stall = (p.flags & kFlagTestStall) != 0;
    a.tok_of_slot = p.tok_of_slot; a.hexp = p.hexp;
    bool ok;
    if (gemm == 1) {
        a.kdim_r = p.H; a.kdim_s = p.H;
        a.ntile_r = p.I / 128; a.ntile_s = p.Is / 128;
        a.tstart = p.tcs1;
        a.s_r = p.s13; a.s_s = p.sh_s13;
        ok = make_map(&mA_r, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.x_perm, p.H, TK, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_map(&mA_s, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.x, p.H, p.T, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_map(&mB_r, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.w13, p.H / 2, (uint64_t)p.E * 2 * p.I, 32, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE) &&
             make_map(&mB_s, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.Is > 0 ? (const void*)p.sh_w13 : (const void*)p.w13,
                      p.H / 2, 2 * (uint64_t)Is, 32, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
    } else {
        a.kdim_r = p.I; a.kdim_s = p.Is;
        a.ntile_r = p.H / 256; a.ntile_s = p.H / 256;
        a.tstart = p.tcs2;
        a.s_r = p.s2; a.s_s = p.sh_s2;
        ok = make_map(&mA_r, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, p.h_r, p.I, TK, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_map(&mA_s, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, p.Is > 0 ? (const void*)p.h_s : (const void*)p.h_r,
                      Is, p.T, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_map(&mB_r, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.w2, p.I / 2, (uint64_t)p.E * p.H, 32, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE) &&
             make_map(&mB_s, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.Is > 0 ? (const void*)p.sh_w2 : (const void*)p.w2,
                      Is / 2, p.H, 32, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    if (!ok) return cudaErrorInvalidValue;
    if (gemm == 1)
        return launch_pdl(tc::grouped_gemm_kernel<1>, dim3(grid), dim3(tc::NUM_THREADS), tc::SMEM_BYTES, stream, mA_r,
                          mA_s, mB_r, mB_s, a);
    return launch_pdl(tc::grouped_gemm_kernel<2>, dim3(grid), dim3(tc::NUM_THREADS), tc::SMEM_BYTES, stream, mA_r,
                      mA_s, mB_r, mB_s, a);
}

}  // namespace moe
