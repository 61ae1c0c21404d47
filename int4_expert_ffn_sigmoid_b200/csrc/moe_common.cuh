// Internal definitions shared by the kernels of the int4 MoE layer library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

// Largest T that takes the weight-streaming (small-batch) path by default.
constexpr int kDecodeMaxTokens = 64;
// Tokens of one bucket handled by one expert-kernel task (2 mma n-tiles of 8).
constexpr int kChunkTokens = 16;
// Large-batch router: tokens per tile and the cap on router CTAs.
constexpr int kRouterTileTokens = 16;
constexpr int kRouterMaxBlocks = 296;
// Small-batch router: tokens and experts per CTA (one warp per expert).
constexpr int kDecodeRouterTok = 8;
constexpr int kDecodeRouterExp = 8;
constexpr int kMaxK = 8;
constexpr int kMaxE = 256;
// The SwiGLU intermediate h of token t is stored in fp16 as h * 2^-k_t, with
// k_t = 8 + floor(log2(mean_h x[t,h]^2)) clamped to [kHExpMin, kHExpMax]:
// h grows like |x|^2, so the stored value stays in fp16's normal range
// whatever the input scale.  The factor is exact and undone in the down
// projection's epilogue.
constexpr int kHExpBase = 8;
constexpr int kHExpMin = -40;
constexpr int kHExpMax = 60;

// Device status bits (set by range checks, read back under MOE_DEBUG_CHECK).
enum : unsigned {
    ST_BAD_EXPERT = 1u,  // a routing index outside [0, E)
    ST_BAD_SLOT = 2u,    // a slot outside [0, T*K)
    ST_BAD_COUNT = 4u,   // bucket counts do not sum to T*K
    ST_BAD_TASK = 8u,    // a task resolved to a bucket outside the list
    ST_TIMEOUT = 16u,    // a bounded pipeline wait of the tensor-core kernel gave up
};

// First 256 bytes of the workspace.  Zeroed at the start of every call.
struct Ctrl {
    unsigned status;
    unsigned done;      // last-CTA-done ticket of the router
    int n_buckets;      // non-empty routed buckets + the shared bucket
    int tasks13;        // gate/up tasks over all buckets
    int tasks2;         // down tasks over all buckets
    int tc_tiles1;      // tensor-core GEMM-1 tiles over the routed buckets
    int tc_tiles2;      // tensor-core GEMM-2 tiles over the routed buckets
    int claim13;        // next gate/up task to claim (weight-streaming kernel)
    int claim2;         // next down task to claim
    unsigned blk_done[kDecodeMaxTokens / 8];  // small-batch router: CTAs done per token block
    unsigned sel_done;  // small-batch router: token blocks whose selection is done
    int pad[46];
};
static_assert(sizeof(Ctrl) == 256, "control block is 256 bytes");

// Everything a kernel needs: shape, inputs, outputs and workspace views.
// Bucket b (0 <= b < n_buckets) is the b-th non-empty routed expert in
// ascending expert order; the shared expert is the last bucket (expert id E),
// whose slots T*K .. T*K+T-1 hold tokens 0..T-1 in order.
struct Params {
    int T, H, E, K, I, Is;
    float scale;
    unsigned flags;
    const __nv_bfloat16* x;
    const float* rw;
    const float* rb;
    const uint8_t* w13;
    const float* s13;
    const uint8_t* w2;
    const float* s2;
    const uint8_t* sh_w13;
    const float* sh_s13;
    const uint8_t* sh_w2;
    const float* sh_s2;
    __nv_bfloat16* out;
    int32_t* topk_idx_out;
    float* topk_w_out;
    // workspace
    Ctrl* ctrl;
    int32_t* idx;         // [T*K] selected experts
    float* wts;           // [T*K] routing weights
    float* logits;        // [T*E] (small-batch router)
    int32_t* counts;      // [E]
    int32_t* offsets;     // [E]   first slot of each expert's bucket
    int32_t* bucket_e;    // [E+1]
    int32_t* bucket_n;    // [E+1]
    int32_t* bucket_off;  // [E+1]
    int32_t* ts13;        // [E+2] exclusive prefix of gate/up tasks per bucket
    int32_t* ts2;         // [E+2] exclusive prefix of down tasks per bucket
    int32_t* tcs1;        // [E+2] exclusive prefix of tensor-core GEMM-1 tiles (routed buckets)
    int32_t* tcs2;        // [E+2] exclusive prefix of tensor-core GEMM-2 tiles (routed buckets)
    __nv_bfloat16* x_perm;  // [T*K][H] tokens gathered in slot order (tensor-core path), or null
    int32_t* tok_of_slot; // [T*K]
    int32_t* slot_of;     // [T*K] slot of (t, k)
    int32_t* hist;        // [router blocks][E]
    __half* h_r;          // [T*K][I]  routed SwiGLU intermediate
    __half* h_s;          // [T][Is]   shared SwiGLU intermediate
    int32_t* hexp;        // [T] per-token exponent k_t of the h storage scale
    float* y;             // [T*K + T][H] expert outputs (already row-scaled)
    int router_blocks;
};

// ---------------------------------------------------------------------------
// int4 -> 16-bit float by the exponent-bias ("magic number") technique of
// Kim et al., "Who Says Elephants Can't Run" (2022): the 4-bit code c, made
// unsigned by flipping its sign bit (c + 8), is OR-ed into the low mantissa
// bits of a 16-bit float equal to 2^m with ulp 1, which gives exactly
// 2^m + 8 + c.  The weight-streaming kernels feed these *biased* values to the
// tensor cores and remove the bias from the f32 result (bias * sum of the
// activations), which saves the subtraction.  bf16: 2^7 = 0x4300 (bias 136);
// fp16: 2^10 = 0x6400 (bias 1032).  Output pair j holds elements (2j, 2j+1)
// of the word, low half first (natural order).
// ---------------------------------------------------------------------------
constexpr uint32_t kMagicBf16 = 0x43004300u;
constexpr uint32_t kMagicF16 = 0x64006400u;
constexpr float kBiasBf16 = 136.0f;
constexpr float kBiasF16 = 1032.0f;
constexpr uint32_t kOnesBf16 = 0x3F803F80u;
constexpr uint32_t kOnesF16 = 0x3C003C00u;

template <uint32_t kMagic>
__device__ __forceinline__ void int4x8_biased(uint32_t w, uint32_t (&o)[4]) {
    const uint32_t v = w ^ 0x88888888u;
    const uint32_t v4 = v >> 4;
    // half 0 <- low nibble of byte j of v (element 2j); half 1 <- low nibble
    // of byte j of v >> 4 (element 2j + 1)
    o[0] = (__byte_perm(v, v4, 0x0400) & 0x000F000Fu) | kMagic;
    o[1] = (__byte_perm(v, v4, 0x0501) & 0x000F000Fu) | kMagic;
    o[2] = (__byte_perm(v, v4, 0x0602) & 0x000F000Fu) | kMagic;
    o[3] = (__byte_perm(v, v4, 0x0703) & 0x000F000Fu) | kMagic;
}

// Streamed weights: read once, keep out of L1.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint4 ld_v4(const void* p) {
    return __ldg(reinterpret_cast<const uint4*>(p));
}

// D(16x8, f32) += A(16x16) * B(16x8), A row-major, B column-major.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ float silu_mul(float g, float u) {
    return g / (1.0f + expf(-g)) * u;
}

// Bucket geometry of the expert kernels.
__device__ __forceinline__ int chunks_of(int n) { return (n + kChunkTokens - 1) / kChunkTokens; }

}  // namespace moe
