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
// The same kernels serve int8 expert weights (the converter's 8-bit expert
// setting): template parameter WB = 4 or 8 sets the raw tile (8 or 16 KiB per
// k block), the ring depths and the code conversion; everything else is shared.
//
// Tile: 128 tokens (MMA M, one TMEM lane per token) x 256 weight rows (MMA N)
// x 64 reduction elements per pipeline stage.  Tokens are the A operand and
// the dequantised weights the B operand, both in shared memory (128-byte
// swizzle).  A tile spans 256 weight rows because the loads from L2 bound the
// kernel: per k block it moves 16 KiB of tokens and 8 KiB of raw int4 for
// 128 x 256 x 64 multiply-adds, twice the weight rows per token byte of a
// 128-row tile.  GEMM-1's 256 rows are 128 gate rows and the 128 up rows of
// the same features, so one epilogue thread holds gate and up of a (token,
// feature) pair.  Two rings: TMA stages hold the token and raw int4 tiles of
// TSTAGES k blocks; BSTAGES slots hold the dequantised B operand.
// Roles (864 threads):
//   warp 0       TMA producer (token tile, raw int4 tile) and TMEM owner
//   warp 1       MMA issuer (one thread, tcgen05.mma kind::f16, M=128 N=256 K=16)
//   warps 2-17   dequantisers, two groups of eight warps: group g takes the k
//                blocks n = g mod 2 of the CTA's sequence (B slot n mod 3),
//                one B row per thread: raw int4 -> exact 16-bit integers in
//                the swizzled K-major layout (the row scale is applied in the
//                epilogue)
//   warp 18      staging: each tile's token rows, h-scale factors and weight
//                row scales into shared memory, a tile or two ahead
//   warps 19-26  epilogue: the warp of lane quarter q and column half c reads
//                tokens 32q..32q+31 and half c of the tile's columns
//                (tcgen05.ld), scales, SwiGLU, stores
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

constexpr int BM = 128;  // tokens per tile (A rows, TMEM lanes)
constexpr int BN = 256;  // weight rows per tile (B rows, accumulator columns)
constexpr int BK = 64;   // reduction elements per stage
static_assert(BM == kTcTokens && BN == 2 * kTcFeat1 && BN == kTcFeat2, "tile geometry");
constexpr int A_BYTES = BM * BK * 2;    // 16 KiB, bf16/fp16 tokens
constexpr int B_BYTES = BN * BK * 2;    // 32 KiB, dequantised weights
// Ring geometry per code width: WB = 4 (packed int4, 32 raw bytes per B row
// and k block) or 8 (int8, 64 bytes).  The int8 raw tile is twice as large,
// so its B ring is one slot shallower (shared memory).  (Deeper TMA rings,
// 5 and 6 stages for int4, measured no faster.)
template <int WB>
struct Geo {
    static_assert(WB == 4 || WB == 8, "int4 or int8 codes");
    static constexpr int TSTAGES = 4;
    static constexpr int BSTAGES = WB == 4 ? 3 : 2;
    static constexpr int RAW_ROW = BK * WB / 8;      // bytes of one raw B row per k block
    static constexpr int RAW_BYTES = BN * RAW_ROW;   // 8 or 16 KiB
    static constexpr int TSTAGE_BYTES = A_BYTES + RAW_BYTES;
    static constexpr int RING_BYTES = TSTAGES * TSTAGE_BYTES + BSTAGES * B_BYTES;
};
constexpr int MAX_TSTAGES = 4, MAX_BSTAGES = 3;
constexpr int EPI_STAGE_BYTES = 2048;  // per epilogue warp: 32 token rows x 64 bytes
constexpr int DEQ_GROUPS = 2;
constexpr int DEQ_WARPS = 8 * DEQ_GROUPS;
constexpr int EPI_WARPS = 8;
constexpr int WARP_STAGE = 2 + DEQ_WARPS;
constexpr int WARP_EPI0 = WARP_STAGE + 1;
constexpr int NUM_THREADS = 32 * (WARP_EPI0 + EPI_WARPS);
constexpr int TMEM_COLS = 512;  // two 256-column accumulators
constexpr long long kTimeoutCycles = 4000000000LL;
constexpr long long kDrainCycles = 200000000LL;
// MOE_TEST_STALL: the epilogue first waits this long on a barrier nothing
// arrives on (~1 ms), which makes the CTA take its timeout path while its
// copies and MMAs are in flight.
constexpr long long kStallCycles = 1LL << 21;

// Per-tile data of the epilogue, written by the staging warp.
struct Stage {
    int slot[BM];   // output row of each token (h row / y slot), -1 past the tile
    float fac[BM];  // per-token factor of the h storage scale (2^-k for GEMM-1, 2^k for GEMM-2)
    float sc[BN];   // scale of each weight row of the tile
};

struct Shared {
    uint64_t full_tma[MAX_TSTAGES];  // token + raw tiles landed (TMA transaction count)
    uint64_t empty_t[MAX_TSTAGES];   // MMA done with the token tile, a dequantiser group with the raw tile
    uint64_t full_b[MAX_BSTAGES];    // B slot written (one arrival per warp of its group)
    uint64_t empty_b[MAX_BSTAGES];   // MMA done with the B slot
    uint64_t acc_full[2];
    uint64_t acc_empty[2];       // one arrival per epilogue warp
    uint64_t stage_full[2];      // one arrival per staging lane
    uint64_t stage_empty[2];     // one arrival per epilogue warp
    uint64_t drain;
    uint64_t never;  // nothing arrives on it (MOE_TEST_STALL)
    uint32_t tmem_base;
    int abort_flag;
    alignas(16) Stage stage[2];
    // epilogue transpose: each warp's 32 rows x 16 columns pass through here so
    // that every global store instruction writes whole row segments
    alignas(128) uint8_t epi[EPI_WARPS][EPI_STAGE_BYTES];
};
template <int WB>
constexpr int smem_bytes() {
    return Geo<WB>::RING_BYTES + 1024 + (int)((sizeof(Shared) + 127) / 128 * 128);
}
static_assert(smem_bytes<4>() <= 227 * 1024 && smem_bytes<8>() <= 227 * 1024, "shared memory of the grouped GEMM");

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory accesses by 32-bit shared address (the tiles sit behind a
// runtime 1024-byte alignment, which generic pointers would not let the
// compiler see as shared).
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ float4 lds128f(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ int lds32(uint32_t a) {
    int v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
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

// Every lane of the warp waits (each then observes the phase and what it
// releases); the warp goes on only if every lane's wait succeeded.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Shared* sh) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, sh)) != 0;
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

// D (tensor memory) += A (shared memory descriptor, 128 x 16) * B (shared
// memory descriptor, N x 16).
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
// The code c + 8 is the nibble with its top bit flipped, so one AND-XOR gives
// the biased code and the exponent together.
template <bool kBf16>
__device__ __forceinline__ void int4x8_natural(uint32_t w, uint32_t* o) {
    const uint32_t w4 = w >> 4;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        // byte j of w (low nibble = element 2j) into half 0, byte j of w>>4
        // (low nibble = element 2j+1) into half 1
        const uint32_t t = __byte_perm(w, w4, j | ((4 + j) << 8));
        if (kBf16) {
            uint32_t u = (t & 0x000F000Fu) ^ 0x43084308u;
            __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&u),
                                       __halves2bfloat162(__ushort_as_bfloat16(0x4308), __ushort_as_bfloat16(0x4308)));
            o[j] = *reinterpret_cast<uint32_t*>(&r);
        } else {
            uint32_t u = (t & 0x000F000Fu) ^ 0x64086408u;
            __half2 r = __hsub2(*reinterpret_cast<__half2*>(&u),
                                __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408)));
            o[j] = *reinterpret_cast<uint32_t*>(&r);
        }
    }
}

// Four int8 codes (a 32-bit word, element j in byte j) -> two 16-bit pairs
// in natural order: o[0] = (element 0, element 1), o[1] = (element 2, 3).
// The same exponent-bias technique: c + 128 (the byte with its top bit
// flipped) in the low mantissa bits of 2^m, minus 2^m + 128.  fp16 has ten
// mantissa bits, so m = 10 works in 16 bits (0x6400 = 1024, 1152 = 0x6480).
// bf16 has seven, too few for eight-bit codes: the value is formed in f32
// (2^23 = 0x4B000000, minus 2^23 + 128), where the integer c is exact, and
// its upper 16 bits, the bf16 encoding of c (the lower 16 are zero), kept.
template <bool kBf16>
__device__ __forceinline__ void int8x4_natural(uint32_t w, uint32_t* o) {
    if (kBf16) {
        const uint32_t u = w ^ 0x80808080u;
        float f[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)  // bytes (u_j, 0, 0, 0x4B): 2^23 + c_j + 128
            f[j] = __uint_as_float(__byte_perm(u, 0x4B000000u, j | 0x7440)) - 8388736.0f;
        o[0] = __byte_perm(__float_as_uint(f[0]), __float_as_uint(f[1]), 0x7632);
        o[1] = __byte_perm(__float_as_uint(f[2]), __float_as_uint(f[3]), 0x7632);
    } else {
        // bytes 0, 1 (then 2, 3) into the low byte of each half, top bit flipped, exponent of 1024
        uint32_t u0 = __byte_perm(w, 0u, 0x4140) ^ 0x64806480u;
        uint32_t u1 = __byte_perm(w, 0u, 0x4342) ^ 0x64806480u;
        const __half2 bias = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
        __half2 r0 = __hsub2(*reinterpret_cast<__half2*>(&u0), bias);
        __half2 r1 = __hsub2(*reinterpret_cast<__half2*>(&u1), bias);
        o[0] = *reinterpret_cast<uint32_t*>(&r0);
        o[1] = *reinterpret_cast<uint32_t*>(&r1);
    }
}

struct Tile {
    int shared;   // 1: shared expert
    int e;        // expert id (E for shared)
    int n_valid;  // valid tokens in this tile
    int slot0;    // first token row of the tile (TMA y coordinate of the token map; h row / y slot)
    int col0;     // GEMM-1: first feature of the unit; GEMM-2: first output feature
    int ncol;     // weight rows (B rows, accumulator columns) of the unit: 256, 128 or 64;
                  // GEMM-1: ncol / 2 features, gate rows then up rows
    int nkb;      // k blocks
};

// Tiles of a launch: the shared expert's first (token tile mt, feature block
// ft: index ft * mt_s + mt), then every routed bucket's (local index
// ft * mtiles + mt, buckets in order, tstart the prefix of their counts).
__device__ __forceinline__ Tile decode_tile(const TcArgs& a, int tile) {
    Tile t;
    const int fw = a.gemm == 1 ? kTcFeat1 : kTcFeat2;
    const int mt_s = a.Is > 0 ? (a.T + BM - 1) / BM : 0;
    const int n_sh = mt_s * a.ntile_s;
    t.ncol = BN;
    if (tile < n_sh) {
        const int mt = tile % mt_s, nt = tile / mt_s;
        t.shared = 1;
        t.e = a.E;
        t.n_valid = min(BM, a.T - mt * BM);
        t.slot0 = mt * BM;
        t.col0 = nt * fw;
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
    t.slot0 = off + mt * BM;
    t.col0 = nt * fw;
    t.nkb = a.kdim_r / BK;
    return t;
}

__device__ __forceinline__ int total_tiles(const TcArgs& a) {
    const int mt_s = a.Is > 0 ? (a.T + BM - 1) / BM : 0;
    return mt_s * a.ntile_s + (a.gemm == 1 ? a.ctrl->tc_tiles1 : a.ctrl->tc_tiles2);
}

// Work units of a launch.  CTA b takes units b, b + grid, ...  The tiles of
// the full waves are units of their own; the tiles of the last, partial wave
// are split by columns into f equal units (f = 1, 2 or 4, as many as the grid
// holds), so that it spreads over more CTAs instead of leaving most of them
// idle while a few finish whole tiles.  A unit covers all of its tile's k
// blocks: every output element is summed exactly as in the unsplit tile.
struct Units {
    int full;   // units that are whole tiles
    int f;      // units per tile of the last wave
    int total;
};
__device__ __forceinline__ Units units_of(int ntiles, int grid) {
    Units u;
    const int rem = ntiles % grid;
    u.full = ntiles - rem;
    u.f = 1;
    while (rem > 0 && u.f < 4 && rem * u.f * 2 <= grid) u.f *= 2;
    u.total = u.full + rem * u.f;
    return u;
}
__device__ __forceinline__ Tile decode_unit(const TcArgs& a, const Units& us, int unit) {
    if (unit < us.full) return decode_tile(a, unit);
    const int i = unit - us.full, part = i % us.f;
    Tile t = decode_tile(a, us.full + i / us.f);
    t.ncol = BN / us.f;
    t.col0 += part * (a.gemm == 1 ? t.ncol / 2 : t.ncol);
    return t;
}

template <int GEMM, int WB>
__global__ void __launch_bounds__(NUM_THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmX_r, const __grid_constant__ CUtensorMap tmX_s,
                    const __grid_constant__ CUtensorMap tmW_r, const __grid_constant__ CUtensorMap tmW_s,
                    const TcArgs a) {
    constexpr int TSTAGES = Geo<WB>::TSTAGES, BSTAGES = Geo<WB>::BSTAGES;
    constexpr int RAW_ROW = Geo<WB>::RAW_ROW, RAW_BYTES = Geo<WB>::RAW_BYTES;
    constexpr int TSTAGE_BYTES = Geo<WB>::TSTAGE_BYTES, RING_BYTES = Geo<WB>::RING_BYTES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Shared* sh = reinterpret_cast<Shared*>(smem + RING_BYTES);
    auto x_tile = [&](int s) { return smem + s * TSTAGE_BYTES; };
    auto raw_tile = [&](int s) { return smem + s * TSTAGE_BYTES + A_BYTES; };
    auto b_tile = [&](int s) { return smem + TSTAGES * TSTAGE_BYTES + s * B_BYTES; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < TSTAGES; ++s) {
            mbar_init(&sh->full_tma[s], 1);
            mbar_init(&sh->empty_t[s], 1 + 8);
        }
        for (int s = 0; s < BSTAGES; ++s) {
            mbar_init(&sh->full_b[s], 8);
            mbar_init(&sh->empty_b[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sh->acc_full[b], 1);
            mbar_init(&sh->acc_empty[b], EPI_WARPS);
            mbar_init(&sh->stage_full[b], 32);
            mbar_init(&sh->stage_empty[b], EPI_WARPS);
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
    const Units us = units_of(ntiles, gridDim.x);

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX_r)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX_s)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW_r)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW_s)) : "memory");
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued_par[TSTAGES];
            bool issued[TSTAGES];
            for (int i = 0; i < TSTAGES; ++i) issued[i] = false, issued_par[i] = 0;
            bool ok = true;
            for (int unit = blockIdx.x; ok && unit < us.total; unit += gridDim.x) {
                const Tile t = decode_unit(a, us, unit);
                const CUtensorMap* mX = t.shared ? &tmX_s : &tmX_r;
                const CUtensorMap* mW = t.shared ? &tmW_s : &tmW_r;
                int wrow0, wrow1;  // raw rows of the two 128-row boxes (a narrower unit uses the first rows of each)
                if (GEMM == 1) {
                    const int irow = t.shared ? a.Is : a.I;
                    const int base = t.shared ? 0 : t.e * 2 * a.I;
                    wrow0 = base + t.col0;         // gate rows
                    wrow1 = base + irow + t.col0;  // up rows of the same features
                } else {
                    wrow0 = (t.shared ? 0 : t.e * a.H) + t.col0;
                    wrow1 = wrow0 + BN / 2;
                }
                for (int kb = 0; kb < t.nkb; ++kb) {
                    if (!mbar_wait(&sh->empty_t[s], ph ^ 1u, sh)) { ok = false; break; }
                    mbar_expect_tx(&sh->full_tma[s], A_BYTES + RAW_BYTES);
                    tma_load_2d(x_tile(s), mX, &sh->full_tma[s], kb * BK, t.slot0);
                    tma_load_2d(raw_tile(s), mW, &sh->full_tma[s], kb * RAW_ROW, wrow0);
                    tma_load_2d(raw_tile(s) + RAW_BYTES / 2, mW, &sh->full_tma[s], kb * RAW_ROW, wrow1);
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
            constexpr int kFmt = GEMM == 1 ? 1 : 0;
            int s = 0, sb = 0;
            uint32_t ph = 0, phb = 0;
            uint32_t acc_ph[2] = {0, 0};
            int buf = 0;
            bool ok = true, any = false;
            for (int unit = blockIdx.x; ok && unit < us.total; unit += gridDim.x) {
                const Tile t = decode_unit(a, us, unit);
                if (!mbar_wait(&sh->acc_empty[buf], acc_ph[buf] ^ 1u, sh)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem + buf * BN;
                const uint32_t idesc = idesc_f16(kFmt, BM, t.ncol);
                for (int kb = 0; kb < t.nkb; ++kb) {
                    if (!mbar_wait(&sh->full_tma[s], ph, sh) || !mbar_wait(&sh->full_b[sb], phb, sh)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t xaddr = smem_u32(x_tile(s)), baddr = smem_u32(b_tile(sb));
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        mma_f16_ss(d, smem_desc_sw128(xaddr + kk * 32), smem_desc_sw128(baddr + kk * 32), idesc,
                                   (kb | kk) != 0);
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
    } else if (warp < WARP_STAGE) {
        // ---------------- dequantisers: one B row per thread ----------------
        // Group g handles the k blocks n = g (mod 2) of the CTA's sequence, which
        // use B slot n mod BSTAGES and TMA stage n mod TSTAGES.
        const int g = (warp - 2) >> 3;
        const int r = ((warp - 2) & 7) * 32 + lane;  // B row = accumulator column
        // int4: the 16-byte half read first; a quarter-warp's eight reads then
        // fall on eight different 16-byte bank groups (raw rows 32 bytes apart).
        // int8: the raw tile lands with the 64-byte swizzle (16-byte chunk q of
        // row r at q ^ ((r >> 1) & 3)), so that every lane reads the same
        // logical quarter at once without bank conflicts and then stores the
        // same B chunks (the B layout's own swizzle keeps those conflict-free).
        const uint32_t brow_off = (r >> 3) * 1024 + (r & 7) * 128;
        const uint32_t ring = smem_u32(smem);
        uint32_t n = 0;  // k blocks of the CTA so far
        bool ok = true;
        for (int unit = blockIdx.x; ok && unit < us.total; unit += gridDim.x) {
            const Tile t = decode_unit(a, us, unit);
            // raw row of this thread's B row: GEMM-1's up rows sit in the second
            // 128-row box, whatever the unit's width; rows past the unit are idle
            const int nf = t.ncol / 2;
            const int rr = (GEMM == 1 && r >= nf) ? BN / 2 + (r - nf) : r;
            const bool active = r < t.ncol;
            const int h0 = (rr ^ (rr >> 2)) & 1;
            const int rot = (rr >> 1) & 3;
            for (int kb = 0; kb < t.nkb; ++kb, ++n) {
                if ((int)(n & (DEQ_GROUPS - 1)) != g) continue;
                const int s = (int)(n % TSTAGES), sb = (int)(n % BSTAGES);
                const uint32_t ph = (n / TSTAGES) & 1u, phb = (n / BSTAGES) & 1u;
                if (!warp_wait(&sh->full_tma[s], ph, sh) || !warp_wait(&sh->empty_b[sb], phb ^ 1u, sh)) {
                    ok = false;
                    break;
                }
                const uint32_t rrow = ring + s * TSTAGE_BYTES + A_BYTES + rr * RAW_ROW;
                const uint32_t brow = ring + TSTAGES * TSTAGE_BYTES + sb * B_BYTES + brow_off;
                if (!active) {
                } else if (WB == 4) {
                    const uint4 qa = lds128(rrow + 16 * h0);
                    const uint4 qb = lds128(rrow + 16 * (h0 ^ 1));
                    const uint4 q0 = h0 ? qb : qa, q1 = h0 ? qa : qb;
                    const uint32_t words[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
                    for (int c = 0; c < 8; ++c) {  // 16-byte chunk c = elements 8c..8c+7
                        uint32_t o[4];
                        int4x8_natural<GEMM == 1>(words[c], o);
                        sts128(brow + ((c ^ (r & 7)) << 4), o[0], o[1], o[2], o[3]);
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {  // raw quarter q = elements 16q..16q+15 = chunks 2q, 2q+1
                        const uint4 v = lds128(rrow + 16 * (q ^ rot));
                        uint32_t o[8];
                        int8x4_natural<GEMM == 1>(v.x, o);
                        int8x4_natural<GEMM == 1>(v.y, o + 2);
                        int8x4_natural<GEMM == 1>(v.z, o + 4);
                        int8x4_natural<GEMM == 1>(v.w, o + 6);
                        sts128(brow + (((2 * q) ^ (r & 7)) << 4), o[0], o[1], o[2], o[3]);
                        sts128(brow + (((2 * q + 1) ^ (r & 7)) << 4), o[4], o[5], o[6], o[7]);
                    }
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the MMA reads through the async proxy
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&sh->full_b[sb]);
                    mbar_arrive(&sh->empty_t[s]);  // this warp is done with the raw tile
                }
            }
        }
    } else if (warp == WARP_STAGE) {
        // ---------------- staging: per-tile token rows, factors and row scales ----------------
        uint32_t st_ph[2] = {0, 0};
        int b = 0;
        for (int unit = blockIdx.x; unit < us.total; unit += gridDim.x) {
            const Tile t = decode_unit(a, us, unit);
            if (!warp_wait(&sh->stage_empty[b], st_ph[b] ^ 1u, sh)) break;
            Stage& st = sh->stage[b];
            const int irow = t.shared ? a.Is : a.I;
            const float* S = GEMM == 1 ? (t.shared ? a.s_s : a.s_r + (size_t)t.e * 2 * a.I)
                                       : (t.shared ? a.s_s : a.s_r + (size_t)t.e * a.H);
#pragma unroll
            for (int j = lane; j < BM; j += 32) {
                if (j < t.n_valid) {
                    const int tok = t.shared ? t.slot0 + j : __ldg(a.tok_of_slot + t.slot0 + j);
                    const int hx = __ldg(a.hexp + tok);
                    st.slot[j] = GEMM == 1 ? t.slot0 + j : (t.shared ? a.T * a.K + t.slot0 + j : t.slot0 + j);
                    st.fac[j] = ldexpf(1.0f, GEMM == 1 ? -hx : hx);
                } else {
                    st.slot[j] = -1;
                    st.fac[j] = 0.f;
                }
            }
            const int nf = t.ncol / 2;  // GEMM-1: features of the unit
#pragma unroll
            for (int j = lane; j < BN; j += 32)
                st.sc[j] = j >= t.ncol ? 0.f
                           : GEMM == 1 ? __ldg(S + (j < nf ? t.col0 + j : irow + t.col0 + (j - nf)))
                                       : __ldg(S + t.col0 + j);
            mbar_arrive(&sh->stage_full[b]);  // every lane: its writes are released with the arrival
            st_ph[b] ^= 1u;
            b ^= 1;
        }
    } else {
        // ---------------- epilogue: tokens of lane quarter q, column half c ----------------
        const int quarter = warp & 3, chalf = (warp - WARP_EPI0) >> 2;
        const int m = quarter * 32 + lane;  // token row of the tile = TMEM lane
        uint32_t acc_ph[2] = {0, 0};
        int buf = 0;
        for (int unit = blockIdx.x; unit < us.total; unit += gridDim.x) {
            const Tile t = decode_unit(a, us, unit);
            const bool got = (!a.stall || mbar_wait(&sh->never, 0, sh, kStallCycles)) &&
                             mbar_wait(&sh->stage_full[buf], acc_ph[buf], sh) &&
                             mbar_wait(&sh->acc_full[buf], acc_ph[buf], sh);
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            const Stage& st = sh->stage[buf];
            const uint32_t st_sc = smem_u32(&st.sc[0]);
            const float fac = __int_as_float(lds32(smem_u32(&st.fac[m])));
            const uint32_t stg = smem_u32(&sh->epi[warp - WARP_EPI0][0]);
            const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + buf * BN;
            if (GEMM == 1) {
                // features of column half c of the unit: gate in column j, up in column nf + j
                const int irow = t.shared ? a.Is : a.I;
                __half* hbase = (t.shared ? a.h_s : a.h_r) + t.col0;
                int rows[2];  // the token rows this lane stores: 16 i + lane / 2
#pragma unroll
                for (int i = 0; i < 2; ++i) rows[i] = lds32(smem_u32(&st.slot[quarter * 32 + 16 * i + (lane >> 1)]));
                const int nf = t.ncol / 2, hw = nf / 2;  // features of the unit, of this warp's half
#pragma unroll 1
                for (int c0 = hw * chalf; c0 < hw * chalf + hw; c0 += 16) {
                    uint32_t gv[16], uv[16];
                    tmem_ld16_wait(tbase + c0, gv);
                    tmem_ld16_wait(tbase + nf + c0, uv);
                    float sg[16], su[16];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 a4 = lds128f(st_sc + 4 * (c0 + 4 * q));
                        const float4 b4 = lds128f(st_sc + 4 * (nf + c0 + 4 * q));
                        sg[4 * q] = a4.x; sg[4 * q + 1] = a4.y; sg[4 * q + 2] = a4.z; sg[4 * q + 3] = a4.w;
                        su[4 * q] = b4.x; su[4 * q + 1] = b4.y; su[4 * q + 2] = b4.z; su[4 * q + 3] = b4.w;
                    }
                    uint32_t packed[8];
#pragma unroll
                    for (int i = 0; i < 16; i += 2) {
                        const float h0v = silu_mul(__uint_as_float(gv[i]) * sg[i], __uint_as_float(uv[i]) * su[i]) * fac;
                        const float h1v =
                            silu_mul(__uint_as_float(gv[i + 1]) * sg[i + 1], __uint_as_float(uv[i + 1]) * su[i + 1]) * fac;
                        __half2 hv = __floats2half2_rn(h0v, h1v);
                        packed[i >> 1] = *reinterpret_cast<uint32_t*>(&hv);
                    }
                    // this lane's 32 bytes (row `lane`) into the warp's stage, 16-byte
                    // chunk c at c ^ ((lane >> 2) & 1); then two lanes per row, 16 rows
                    // per store instruction
                    const int sw = (lane >> 2) & 1;
                    sts128(stg + lane * 32 + 16 * sw, packed[0], packed[1], packed[2], packed[3]);
                    sts128(stg + lane * 32 + 16 * (sw ^ 1), packed[4], packed[5], packed[6], packed[7]);
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const int rr = 16 * i + (lane >> 1), cc = lane & 1;
                        const uint4 val = lds128(stg + rr * 32 + 16 * (cc ^ ((rr >> 2) & 1)));
                        if (rows[i] >= 0)
                            *reinterpret_cast<uint4*>(hbase + (size_t)rows[i] * irow + c0 + 8 * cc) = val;
                    }
                    __syncwarp();  // the stage is read before the next columns overwrite it
                }
            } else {
                // output columns of column half c of the unit
                float* ybase = a.y + t.col0;
                int rows[4];  // the token rows this lane stores: 8 i + lane / 4
#pragma unroll
                for (int i = 0; i < 4; ++i) rows[i] = lds32(smem_u32(&st.slot[quarter * 32 + 8 * i + (lane >> 2)]));
                const int hw = t.ncol / 2;
#pragma unroll 1
                for (int c0 = hw * chalf; c0 < hw * chalf + hw; c0 += 16) {
                    uint32_t v[16];
                    tmem_ld16_wait(tbase + c0, v);
                    float4 o[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 s4 = lds128f(st_sc + 4 * (c0 + 4 * q));
                        o[q] = make_float4(__uint_as_float(v[4 * q]) * (s4.x * fac), __uint_as_float(v[4 * q + 1]) * (s4.y * fac),
                                           __uint_as_float(v[4 * q + 2]) * (s4.z * fac),
                                           __uint_as_float(v[4 * q + 3]) * (s4.w * fac));
                    }
                    // this lane's 64 bytes (row `lane`) into the warp's stage, 16-byte
                    // chunk c at c ^ ((lane >> 1) & 3); then four lanes per row, 8 rows
                    // per store instruction
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        sts128(stg + lane * 64 + 16 * (q ^ ((lane >> 1) & 3)), __float_as_uint(o[q].x),
                               __float_as_uint(o[q].y), __float_as_uint(o[q].z), __float_as_uint(o[q].w));
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int rr = 8 * i + (lane >> 2), cc = lane & 3;
                        const float4 val = lds128f(stg + rr * 64 + 16 * (cc ^ ((rr >> 1) & 3)));
                        if (rows[i] >= 0) *reinterpret_cast<float4*>(ybase + (size_t)rows[i] * a.H + c0 + 4 * cc) = val;
                    }
                    __syncwarp();  // the stage is read before the next columns overwrite it
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sh->acc_empty[buf]);
                mbar_arrive(&sh->stage_empty[buf]);
            }
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

template <int WB>
cudaError_t set_smem_attrs() {
    cudaError_t e = cudaFuncSetAttribute(tc::grouped_gemm_kernel<1, WB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         tc::smem_bytes<WB>());
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(tc::grouped_gemm_kernel<2, WB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tc::smem_bytes<WB>());
    return e;
}

}  // namespace

bool encode_tensor_map_2d(CUtensorMap* m, CUtensorMapDataType dt, int esize, const void* base, uint64_t inner,
                          uint64_t rows, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
    return get_encode() && make_map(m, dt, esize, base, inner, rows, box_inner, box_rows, sw);
}

int tc_smem_bytes() { return tc::smem_bytes<4>(); }

cudaError_t launch_tc_gemm(const Params& p, int gemm, int grid, cudaStream_t stream) {
    if (!get_encode()) return cudaErrorNotSupported;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !g_smem_set[dev]) {
        cudaError_t e = set_smem_attrs<4>();
        if (e == cudaSuccess) e = set_smem_attrs<8>();
        if (e != cudaSuccess) return e;
        g_smem_set[dev] = 1;
    }
    // code width: a row of n elements is n/2 bytes (int4) or n bytes (int8)
    const bool int8w = (p.flags & kFlagWeightsInt8) != 0;
    const int per = int8w ? 1 : 2;
    const uint32_t raw_box = int8w ? tc::Geo<8>::RAW_ROW : tc::Geo<4>::RAW_ROW;
    // int8 raw rows are one 64-byte swizzle span each (the dequantisers undo it)
    const CUtensorMapSwizzle raw_sw = int8w ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE;
    const int TK = p.T * p.K;
    const int Is = p.Is > 0 ? p.Is : 128;  // any valid map when there is no shared expert
    CUtensorMap mX_r, mX_s, mW_r, mW_s;
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
        a.ntile_r = p.I / kTcFeat1; a.ntile_s = p.Is / kTcFeat1;
        a.tstart = p.tcs1;
        a.s_r = p.s13; a.s_s = p.sh_s13;
        ok = make_map(&mX_r, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.x_perm, p.H, TK, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_map(&mX_s, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.x, p.H, p.T, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_map(&mW_r, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.w13, p.H / per, (uint64_t)p.E * 2 * p.I, raw_box,
                      tc::BN / 2, raw_sw) &&
             make_map(&mW_s, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.Is > 0 ? (const void*)p.sh_w13 : (const void*)p.w13,
                      p.H / per, 2 * (uint64_t)Is, raw_box, tc::BN / 2, raw_sw);
    } else {
        a.kdim_r = p.I; a.kdim_s = p.Is;
        a.ntile_r = p.H / kTcFeat2; a.ntile_s = p.H / kTcFeat2;
        a.tstart = p.tcs2;
        a.s_r = p.s2; a.s_s = p.sh_s2;
        ok = make_map(&mX_r, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, p.h_r, p.I, TK, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_map(&mX_s, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, p.Is > 0 ? (const void*)p.h_s : (const void*)p.h_r,
                      Is, p.T, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_map(&mW_r, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.w2, p.I / per, (uint64_t)p.E * p.H, raw_box,
                      tc::BN / 2, raw_sw) &&
             make_map(&mW_s, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.Is > 0 ? (const void*)p.sh_w2 : (const void*)p.w2,
                      Is / per, p.H, raw_box, tc::BN / 2, raw_sw);
    }
    if (!ok) return cudaErrorInvalidValue;
    const dim3 g(grid), b(tc::NUM_THREADS);
    if (int8w)
        return gemm == 1 ? launch_pdl(tc::grouped_gemm_kernel<1, 8>, g, b, tc::smem_bytes<8>(), stream, mX_r, mX_s,
                                      mW_r, mW_s, a)
                         : launch_pdl(tc::grouped_gemm_kernel<2, 8>, g, b, tc::smem_bytes<8>(), stream, mX_r, mX_s,
                                      mW_r, mW_s, a);
    return gemm == 1 ? launch_pdl(tc::grouped_gemm_kernel<1, 4>, g, b, tc::smem_bytes<4>(), stream, mX_r, mX_s, mW_r,
                                  mW_s, a)
                     : launch_pdl(tc::grouped_gemm_kernel<2, 4>, g, b, tc::smem_bytes<4>(), stream, mX_r, mX_s, mW_r,
                                  mW_s, a);
}

}  // namespace moe
