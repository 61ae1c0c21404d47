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
// Tensor-core grouped GEMM tiles: 128 tokens x 128 features (GEMM-1: their
// gate and up rows, 256 weight rows) or x 256 output features (GEMM-2).
constexpr int kTcTokens = 128;
constexpr int kTcFeat1 = 128;
constexpr int kTcFeat2 = 256;
// Rows of one weight-streaming task: gate/up (each with its up row); one
// row group of a down task (a down task has Params::rows2 rows, a multiple).
constexpr int kTaskRows13 = 64;
constexpr int kTaskRows2 = 128;
constexpr int kMaxRows2 = 1024;
// Tokens of one bucket handled by one weight-streaming task (Params::chunk):
// each token takes two int8 columns (its two activation parts), so 16 tokens
// fill four mma n-tiles of 8 columns.  Large batches whose expert kernels
// both take the TMA-ring kernels use chunks of kMaxChunk tokens, so that an
// expert's weights are streamed once for up to 32 of its tokens.
constexpr int kChunkTokens = 16;
constexpr int kMaxChunk = 32;
// Reduction slice of the weight-streaming down projection: its activations
// are quantized per (token, slice) and every slice writes its own partial
// output row, summed by the combine.
constexpr int kSliceK = 512;
// Large-batch router: tokens per tile and the cap on router CTAs.
constexpr int kRouterTileTokens = 32;
constexpr int kRouterMaxBlocks = 296;
// Small-batch router: a cluster of kDecodeRouterCtas CTAs per group of
// kDecodeRouterTok tokens; CTA r of the cluster computes the logits of the
// r-th eighth of the experts.
constexpr int kDecodeRouterTok = 8;
constexpr int kDecodeRouterCtas = 8;
constexpr int kDecodeGroups = (64 + kDecodeRouterTok - 1) / kDecodeRouterTok;
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

// Flag bits of Params::flags that the kernels read (the values of the
// MOE_* flags of the C ABI).
constexpr unsigned kFlagResidual = 1u << 0;   // MOE_ADD_RESIDUAL
constexpr unsigned kFlagOutF32 = 1u << 4;     // MOE_OUT_F32
constexpr unsigned kFlagLookahead = 1u << 5;  // MOE_LOOKAHEAD
constexpr unsigned kFlagTestStall = 1u << 6;  // MOE_TEST_STALL
constexpr unsigned kFlagTestBadIndex = 1u << 7;  // MOE_TEST_BAD_INDEX
constexpr unsigned kFlagTrace = 1u << 8;      // MOE_TRACE
constexpr unsigned kFlagWeightsInt8 = 1u << 11;  // MOE_WEIGHTS_INT8

// Adaptive expert top-p over the K picks of one token (one warp; lanes k < K
// hold pick k: expert e_k and sigmoid score s_k; ssum is the K scores' sum).
// A pick is kept when the scores of the picks ordered before it (score
// descending, ties to the lower expert index) sum to less than p * ssum.
// Returns on lane o < K the o-th kept pick (in pick order) with weight
// scale * s / (sum of the kept s, added in pick order), and e = -1, w = 0 past
// the kept ones.  p outside (0, 1): every pick, with weight scale * s / ssum.
__device__ __forceinline__ void topp_picks(int K, float p, float scale, int lane, int my_e, float my_s, float ssum,
                                           int& out_e, float& out_w) {
    if (!(p > 0.f && p < 1.f)) {
        out_e = lane < K ? my_e : -1;
        out_w = lane < K ? scale * my_s / ssum : 0.f;
        return;
    }
    float before = 0.f;
    for (int j = 0; j < K; ++j) {
        const float sj = __shfl_sync(0xffffffffu, my_s, j);
        const int ej = __shfl_sync(0xffffffffu, my_e, j);
        if (j != lane && (sj > my_s || (sj == my_s && ej < my_e))) before += sj;
    }
    const unsigned km = __ballot_sync(0xffffffffu, lane < K && before < p * ssum);
    float kept = 0.f;
    out_e = -1;
    out_w = 0.f;
    int pos = 0;
    for (int j = 0; j < K; ++j) {
        const float sj = __shfl_sync(0xffffffffu, my_s, j);
        if ((km >> j) & 1u) kept += sj;
    }
    for (int j = 0; j < K; ++j) {
        const float sj = __shfl_sync(0xffffffffu, my_s, j);
        const int ej = __shfl_sync(0xffffffffu, my_e, j);
        if ((km >> j) & 1u) {
            if (pos == lane) {
                out_e = ej;
                out_w = scale * sj / kept;
            }
            ++pos;
        }
    }
}

// Device status bits (set by range checks, read back under MOE_DEBUG_CHECK).
enum : unsigned {
    ST_BAD_EXPERT = 1u,  // a routing index outside [0, E)
    ST_BAD_SLOT = 2u,    // a slot outside [0, T*K)
    ST_BAD_COUNT = 4u,   // bucket counts do not sum to T*K
    ST_BAD_TASK = 8u,    // a task resolved to a bucket outside the list
    ST_TIMEOUT = 16u,    // a bounded pipeline wait gave up
};

// First 256 bytes of the workspace.  The first kernel of every call zeroes
// status; every other field is written before it is read within the call,
// so the workspace needs no initialisation.
struct Ctrl {
    unsigned status;
    int n_buckets;      // non-empty routed buckets + the shared bucket
    int tasks13;        // gate/up tasks over all buckets
    int tasks2;         // down tasks over all buckets
    int tc_tiles1;      // tensor-core GEMM-1 tiles over the routed buckets
    int tc_tiles2;      // tensor-core GEMM-2 tiles over the routed buckets
    int pad[58];
};

// Programmatic dependent launch: every kernel of a call is launched so that
// it may start while its predecessor in the stream finishes.  pdl_wait()
// blocks until the predecessor grid has completed and its writes are
// visible; nothing produced by an earlier kernel is touched before it.
// pdl_release() lets the next kernel launch (it still waits for this grid's
// completion before reading anything).  Both are no-ops when the kernel was
// launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Warms L2 with bytes [0, n) of p, spread over the grid (128-byte lines).
__device__ __forceinline__ void prefetch_l2_slice(const void* p, size_t n) {
    const size_t lines = (n + 127) / 128;
    const size_t per = (lines + gridDim.x - 1) / gridDim.x;
    const size_t first = (size_t)blockIdx.x * per;
    for (size_t l = first + threadIdx.x; l < first + per && l < lines; l += blockDim.x)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(static_cast<const char*>(p) + l * 128));
}

// Launches `kernel` with programmatic stream serialization allowed.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}
static_assert(sizeof(Ctrl) == 256, "control block is 256 bytes");

// Everything a kernel needs: shape, inputs, outputs and workspace views.
// Bucket b (0 <= b < n_buckets) is the b-th non-empty routed expert in
// ascending expert order; the shared expert is the last bucket (expert id E),
// whose slots T*K .. T*K+T-1 hold tokens 0..T-1 in order.
struct Params {
    int T, H, E, K, I, Is;
    float scale;
    float topp;  // adaptive expert top-p (0: off); dropped picks are index -1
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
    float* y;             // expert outputs (already row-scaled): [nsl_r][T*K][H] then [nsl_s][T][H]
    int router_blocks;
    // weight-streaming (int8 mma) path
    int8_t* xq;           // [T][2][H] two-part int8 activations (see quant2), or null
    float* xs;            // [T] part-0 scale of xq (part 1: xs / 256); NaN for a non-finite row
    int32_t* rank;        // [T*K] small-batch router: rank of (t, k) among its token group's picks of the expert
    float* h32_r;         // [T*K][I]  routed SwiGLU intermediate (f32)
    float* h32_s;         // [T][Is]   shared SwiGLU intermediate (f32)
    float* hmax_r;        // [T*K][I/64] max |h| of each 64-row block
    float* hmax_s;        // [T][Is/64]
    int nsl_r, nsl_s;     // slices of the down projection's reduction (routed, shared)
    int rows2;            // output rows of one down task (kTaskRows2 times 1..8, dividing H)
    int chunk;            // tokens per weight-streaming task: kChunkTokens or kMaxChunk
    int w13_occ2;         // gate/up on the two-CTAs-per-SM TMA-ring kernel (16-token tasks, int4)
    int decode_groups;    // token groups of the small-batch router (0: tables come from the large router)
    int w2_tables_early;  // small batch: the down kernel builds its tables before its wait
    float* lpart;         // [lslices][T][E] partial router logits (split router or tensor-core router)
    int lslices;          // hidden-dimension slices of lpart (0: the selecting router computes its logits)
    __nv_bfloat16* wsplit;  // [3][E][H] router weights as exact bf16 terms hi, mid, lo (tensor-core router)
    int tc_router;        // 1: the tensor-core router logits run first on the large-batch path
};

// Zeroes the per-call status word (first kernel of a call, one thread,
// after pdl_wait: every kernel of the previous call has completed).
__device__ __forceinline__ void reset_ctrl(const Params& p) {
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) p.ctrl->status = 0;
}

// An f32 weight as three bf16 terms with w = hi + mid + lo exactly (hi =
// bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid): the three 8-bit
// significands cover w's 24 bits), as raw bf16 bits.
__device__ __forceinline__ void split3(float w, uint16_t& hi, uint16_t& mid, uint16_t& lo) {
    const __nv_bfloat16 h = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(h);
    const __nv_bfloat16 m = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(m);
    hi = __bfloat16_as_ushort(h);
    mid = __bfloat16_as_ushort(m);
    lo = __bfloat16_as_ushort(__float2bfloat16_rn(r2));
}


// ---------------------------------------------------------------------------
// int4 -> 16-bit float by the exponent-bias ("magic number") technique of
// Kim et al., "Who Says Elephants Can't Run" (2022): the 4-bit code c, made
// unsigned by flipping its sign bit (c + 8), is OR-ed into the low mantissa
// bits of a 16-bit float equal to 2^m with ulp 1, which gives exactly
// 2^m + 8 + c; subtracting 2^m + 8 leaves c exactly.  bf16: 2^7 = 0x4300;
// fp16: 2^10 = 0x6400.  Output pair j holds elements (2j, 2j+1) of the 32-bit
// word, low half first (natural order).
// ---------------------------------------------------------------------------
template <bool kBf16>
__device__ __forceinline__ void int4x8_to_16(uint32_t w, uint32_t (&o)[4]) {
    const uint32_t v = w ^ 0x88888888u;
    const uint32_t v4 = v >> 4;
    constexpr uint32_t kMagic = kBf16 ? 0x43004300u : 0x64006400u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        // half 0 <- low nibble of byte j of v (element 2j); half 1 <- low
        // nibble of byte j of v >> 4 (element 2j + 1)
        uint32_t t = (__byte_perm(v, v4, j | ((4 + j) << 8)) & 0x000F000Fu) | kMagic;
        if (kBf16) {
            const __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&t),
                                             __halves2bfloat162(__ushort_as_bfloat16(0x4308), __ushort_as_bfloat16(0x4308)));
            o[j] = *reinterpret_cast<const uint32_t*>(&r);
        } else {
            const __half2 r = __hsub2(*reinterpret_cast<__half2*>(&t),
                                      __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408)));
            o[j] = *reinterpret_cast<const uint32_t*>(&r);
        }
    }
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

// silu(g) * u = g * sigmoid(g) * u, with the fast exponential and divide
// intrinsics (a few ulp; for g below about -88 the exponential overflows to
// infinity and the result is a signed zero, the correct limit).
__device__ __forceinline__ float silu_mul(float g, float u) {
    return __fdividef(g, 1.0f + __expf(-g)) * u;
}

// Bucket geometry of the expert kernels.
__device__ __host__ __forceinline__ int chunks_of(int n, int chunk) { return (n + chunk - 1) / chunk; }
__device__ __host__ __forceinline__ int slices_of(int k) { return (k + kSliceK - 1) / kSliceK; }

// ---------------------------------------------------------------------------
// int8 operands of the weight-streaming kernels.
//
// Weights: the int4 code c (two's complement nibble) becomes the int8 value
// 16*c by moving the nibble to the high half of a byte: for a 32-bit word of
// eight codes (element 2j in the low nibble of byte j, 2j+1 in the high one),
//   lo8(w) = (w << 4) & 0xF0F0F0F0  -> byte j = 16 * c[2j]
//   hi8(w) =  w       & 0xF0F0F0F0  -> byte j = 16 * c[2j+1]
// (three logic operations per eight weights; exact).
//
// Activations: a row v (a token's x, or a slice of its SwiGLU intermediate)
// is written as v ~= s * (q0 + q1 / 256) with int8 q0, q1 in [-127, 127] and a
// power of two s chosen from max|v| so that |v| / s <= 127: q0 = rint(v / s),
// then q1 = rint(256 (v - s q0) / s), the residual being exact.  The error is
// at most s / 512 per element (max|v| / 2^15 at worst, usually less), and
// the products with the 16*c weights accumulate exactly in int32.  Within
// every group of eight consecutive elements the bytes are stored in the order
// (0, 2, 4, 6, 1, 3, 5, 7), matching lo8 / hi8 of the weights, so that one
// 8-byte read holds the two mma k-halves of one weight word.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t lo8(uint32_t w) { return (w << 4) & 0xF0F0F0F0u; }
__device__ __forceinline__ uint32_t hi8(uint32_t w) { return w & 0xF0F0F0F0u; }

// max that keeps a NaN once it has seen one
__device__ __forceinline__ float nanmax(float m, float a) { return (a > m || a != a) ? a : m; }

struct QScale {
    float s, inv, inv256;  // s = 2^e; NaN s marks a non-finite row (its q are 0)
};

// Scale of a row whose largest magnitude is amax.  Magnitudes below 2^-113
// (e clamped at -119) quantize to zero.
__device__ __forceinline__ QScale qscale(float amax) {
    QScale r;
    if (!(amax <= 3.402823466e38f)) {  // NaN or infinite
        r.s = __int_as_float(0x7fc00000);
        r.inv = r.inv256 = 0.f;
        return r;
    }
    int e = 0;
    if (amax > 0.f) {
        e = ilogbf(amax) - 6;  // amax / 2^e in [64, 128)
        if (amax > 127.f * __int_as_float((min(max(e, -126), 127) + 127) << 23)) ++e;
        e = min(max(e, -119), 126);
    }
    r.s = __int_as_float((e + 127) << 23);
    r.inv = __int_as_float((127 - e) << 23);
    r.inv256 = __int_as_float((135 - e) << 23);
    return r;
}

// The two int8 parts of v under scale qs.
__device__ __forceinline__ void quant2(float v, const QScale& qs, int& q0, int& q1) {
    const float a = rintf(v * qs.inv);
    const float r = fmaf(-a, qs.s, v);
    const float b = fminf(fmaxf(rintf(r * qs.inv256), -127.f), 127.f);
    q0 = (int)a;
    q1 = (int)b;
}

// Eight consecutive elements -> the two 8-byte groups (part 0, part 1) in the
// (0, 2, 4, 6, 1, 3, 5, 7) byte order.
__device__ __forceinline__ void quant2x8(const float (&v)[8], const QScale& qs, uint2& p0, uint2& p1) {
    int a[8], b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) quant2(v[i], qs, a[i], b[i]);
    auto pack = [](int e0, int e1, int e2, int e3) {
        return (uint32_t)(e0 & 0xff) | ((uint32_t)(e1 & 0xff) << 8) | ((uint32_t)(e2 & 0xff) << 16) |
               ((uint32_t)(e3 & 0xff) << 24);
    };
    p0 = make_uint2(pack(a[0], a[2], a[4], a[6]), pack(a[1], a[3], a[5], a[7]));
    p1 = make_uint2(pack(b[0], b[2], b[4], b[6]), pack(b[1], b[3], b[5], b[7]));
}

// D(16x8, s32) += A(16x32, s8) * B(32x8, s8), A row-major, B column-major.
__device__ __forceinline__ void mma_s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

}  // namespace moe
