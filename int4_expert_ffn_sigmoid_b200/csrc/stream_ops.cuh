// Device primitives of the weight-streaming kernels (internal): cp.async and
// bulk / tensor copies into shared memory, mbarriers with bounded waits, and
// the int8 mma k-block of the int4 weights against two-part int8
// activations.
#pragma once

#include <cuda.h>

#include "moe_common.cuh"

namespace moe {

// Bytes of padding per staged activation row (16-byte fragment reads of the
// 8 rows of an mma n-tile then fall on different banks).
constexpr int kPadB = 16;
// One TMA stage of the weight rings: a 256-wide k chunk of a row is 128 bytes
// of codes; 64 gate + 64 up rows, or 128 down rows, are 16 KB.
constexpr int kTmaChunk = 256;
constexpr int kTmaRowBytes = kTmaChunk / 2;
constexpr int kTmaWBytes = 2 * kTaskRows13 * kTmaRowBytes;
constexpr int kW2Bytes = kTaskRows2 * kTmaRowBytes;
constexpr int kTmaXStride = kTmaChunk + kPadB;  // staged activation row of a stage
// Limit of every pipeline wait (~2 s at the boost clock).
constexpr long long kBulkWaitCycles = 4000000000LL;
// MOE_TEST_STALL: length of the wait on a flag that nothing sets (~1 ms).
constexpr long long kStallCycles = 1LL << 21;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(smem)), "l"(gmem) : "memory");
}

__device__ __forceinline__ void bar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void bar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
// Arrives on bar once every cp.async this thread issued so far has landed.
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ bool bar_try(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait for phase `parity` of bar.  It does not look at any abort
// flag: the drains before a CTA exits use it, so that every copy the CTA
// issued has landed before its shared memory goes away.
__device__ __forceinline__ bool bar_wait(uint64_t* bar, uint32_t parity, long long limit) {
    if (bar_try(bar, parity)) return true;
    const long long t0 = clock64();
    while (!bar_try(bar, parity))
        if (clock64() - t0 > limit) return false;
    return true;
}
// Bounded pipeline wait that also gives up as soon as *abort is set (by this
// CTA's timeout or another role's); false when it gave up either way.
__device__ __forceinline__ bool bar_wait_or_abort(uint64_t* bar, uint32_t parity, long long limit,
                                                  const volatile int* abort) {
    if (bar_try(bar, parity)) return true;
    const long long t0 = clock64();
    while (!bar_try(bar, parity)) {
        if (*abort) return false;
        if (clock64() - t0 > limit) return false;
    }
    return true;
}
// Waits `limit` cycles for a flag that nothing sets (MOE_TEST_STALL): the
// caller then takes its timeout path.
__device__ __forceinline__ void stall_on_unset_flag(const volatile int* never, long long limit) {
    const long long t0 = clock64();
    while (*never == 0 && clock64() - t0 <= limit) {
    }
}
// bytes (a multiple of 16, both addresses 16-byte aligned) global -> shared,
// completion counted on bar.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(dst)),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}
// A 2-D tensor tile (box of `map`) at (x, y) -> shared, completion counted on bar.
__device__ __forceinline__ void tma_tile(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y)
        : "memory");
}

// One k block of 128 codes: this thread's 16 bytes of weight rows a (mma row
// g) and b (mma row g + 8) against NT n-tiles of staged activations; xrow
// points at staged row g, byte q*32 of the k block, and n-tile i is
// tile_stride bytes further.
template <int NT, int kSets>
__device__ __forceinline__ void kblock8(const uint4& wa, const uint4& wb, const uint8_t* xrow, int tile_stride,
                                        int (&part)[kSets][NT][4]) {
    const uint32_t aw[4] = {wa.x, wa.y, wa.z, wa.w};
    const uint32_t bw[4] = {wb.x, wb.y, wb.z, wb.w};
    uint32_t A[4][4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        A[m][0] = lo8(aw[m]);
        A[m][1] = lo8(bw[m]);
        A[m][2] = hi8(aw[m]);
        A[m][3] = hi8(bw[m]);
    }
#pragma unroll
    for (int i = 0; i < NT; ++i) {
        const uint4 b01 = *reinterpret_cast<const uint4*>(xrow + i * tile_stride);
        const uint4 b23 = *reinterpret_cast<const uint4*>(xrow + i * tile_stride + 16);
        mma_s8(part[0][i], A[0], b01.x, b01.y);
        mma_s8(part[kSets - 1][i], A[1], b01.z, b01.w);
        mma_s8(part[0][i], A[2], b23.x, b23.y);
        mma_s8(part[kSets - 1][i], A[3], b23.z, b23.w);
    }
}

// kblock8 for int8 weight codes (one byte per element): wa0, wa1 hold the 32
// consecutive codes of row g of the block and wb0, wb1 those of row g + 8.
// The MMA k slots take, of every group of eight codes, the even ones and then
// the odd ones (two byte permutes per register), the order in which the
// activations are stored.  The products are c * q (the int4 path's are
// 16 c * q).
template <int NT, int kSets>
__device__ __forceinline__ void kblock8_i8(const uint4& wa0, const uint4& wa1, const uint4& wb0, const uint4& wb1,
                                           const uint8_t* xrow, int tile_stride, int (&part)[kSets][NT][4]) {
    const uint32_t aw[8] = {wa0.x, wa0.y, wa0.z, wa0.w, wa1.x, wa1.y, wa1.z, wa1.w};
    const uint32_t bw[8] = {wb0.x, wb0.y, wb0.z, wb0.w, wb1.x, wb1.y, wb1.z, wb1.w};
    uint32_t A[4][4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        A[m][0] = __byte_perm(aw[2 * m], aw[2 * m + 1], 0x6420);
        A[m][1] = __byte_perm(bw[2 * m], bw[2 * m + 1], 0x6420);
        A[m][2] = __byte_perm(aw[2 * m], aw[2 * m + 1], 0x7531);
        A[m][3] = __byte_perm(bw[2 * m], bw[2 * m + 1], 0x7531);
    }
#pragma unroll
    for (int i = 0; i < NT; ++i) {
        const uint4 b01 = *reinterpret_cast<const uint4*>(xrow + i * tile_stride);
        const uint4 b23 = *reinterpret_cast<const uint4*>(xrow + i * tile_stride + 16);
        mma_s8(part[0][i], A[0], b01.x, b01.y);
        mma_s8(part[kSets - 1][i], A[1], b01.z, b01.w);
        mma_s8(part[0][i], A[2], b23.x, b23.y);
        mma_s8(part[kSets - 1][i], A[3], b23.z, b23.w);
    }
}

// Scale of the int32 sums into activation-scale units: the int4 codes enter
// the MMAs as 16 c, the int8 codes as c.
template <int WB>
constexpr float code_unit() { return WB == 4 ? 0.0625f : 1.0f; }

// Both int8 parts of mma columns 2j, 2j+1 -> the value in units of the
// activation scale times 16.
__device__ __forceinline__ float join(int c0, int c1) { return (float)c0 + (float)c1 * (1.0f / 256.0f); }

}  // namespace moe
