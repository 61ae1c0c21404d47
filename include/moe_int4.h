/*
 * moe_int4.h -- C ABI of the B200 (sm_100a) forward pass of one
 * Mixture-of-Experts FFN layer with int4 experts and a sigmoid+bias router.
 *
 * The layer (Colibri-Nano model card, "Architecture"; colibri README in the
 * project listing, "What's implemented"; nanocolibri-engine README,
 * "Converting a checkpoint yourself"):
 *
 *   L[t,e] = sum_h x[t,h] W[e,h]            router logits (f32 weights)
 *   s[t,e] = sigmoid(L[t,e])                 score
 *   S_t    = the K experts with the largest s[t,e] + bias[e]
 *            (the bias only decides the selection; ties go to the lower
 *            expert index; a NaN key counts as -infinity)
 *   w[t,k] = routed_scaling * s[t,e_k] / sum_{j in S_t} s[t,j]
 *   FFN_e(x) = W2_e (silu(Wg_e x) * (Wu_e x)),  silu(z) = z sigmoid(z)
 *   out[t] = sum_k w[t,k] FFN_{e_k}(x_t) + FFN_shared(x_t)  [+ x_t]
 *
 * The shared expert has weight 1 and is not multiplied by routed_scaling.
 * Routed tokens are bucketed by expert ("batch-union": each expert touched by
 * the batch is read once and applied to all its tokens) before the expert
 * FFNs run.
 *
 * Weight format ("per-row symmetric with f32 scales"): every matrix is stored
 * row-major with one row per OUTPUT feature.  A row of n int4 codes takes n/2
 * bytes: byte j holds element 2j in bits 0..3 and element 2j+1 in bits 4..7,
 * each a 4-bit two's-complement code c in [-8, 7].  The dequantised weight is
 * c * scale[row] with one f32 scale per row.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers to caller-owned, contiguous,
 *    row-major memory on the current CUDA device.  Pointers must be 16-byte
 *    aligned.  The library never allocates or frees device memory.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *    stream-ordered and asynchronous: the return value reports argument
 *    errors and launch errors only, unless MOE_DEBUG_CHECK is set.
 *  - Calls are reentrant provided concurrent calls use distinct workspaces
 *    and outputs.  `out` must not alias `x`.
 */
#ifndef MOE_INT4_H
#define MOE_INT4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 2

/* Status codes. */
#define MOE_OK 0
#define MOE_ERR_INVALID_ARG 1  /* NULL pointer, bad struct_size, T < 0, K > E, misaligned pointer */
#define MOE_ERR_UNSUPPORTED 2  /* shape outside the supported set (see moe_cfg_t) */
#define MOE_ERR_WORKSPACE 3    /* workspace NULL or smaller than moe_layer_workspace_bytes() */
#define MOE_ERR_CUDA 4         /* a CUDA runtime call or kernel launch failed */
#define MOE_ERR_DEVICE_CHECK 5 /* MOE_DEBUG_CHECK: a kernel's range check failed */

/* Flags of moe_cfg_t.flags. */
#define MOE_ADD_RESIDUAL (1u << 0)  /* out = x + MoE(x) (one layer of a residual stack) */
#define MOE_DEBUG_CHECK (1u << 1)   /* synchronise the stream and report device range checks */
#define MOE_FORCE_DECODE (1u << 2)  /* use the weight-streaming expert kernels at any T */
#define MOE_FORCE_PREFILL (1u << 3) /* use the grouped-GEMM kernels at any T (H a multiple of 256) */
#define MOE_OUT_F32 (1u << 4)       /* out is f32 [T][H] (the f32 sum, no bf16 rounding): for
                                       checking the arithmetic apart from the output rounding */
#define MOE_LOOKAHEAD (1u << 5)     /* moe_stack_forward, fused kernel: L2 prefetch hints (the
                                       next layer's shared expert, routers and the experts its
                                       router picks on the current input); the output is
                                       bit-identical either way.  Off by default: measured slower
                                       here, the prefetches competing with the demand loads */
#define MOE_TEST_STALL (1u << 6)    /* test only: in the expert kernels that take part (the
                                       tensor-core grouped GEMMs, the TMA-ring weight-streaming
                                       kernels and the fused stack kernel), one role first waits
                                       ~1 ms on a flag that nothing
                                       sets, so that the kernel takes its timeout path while its
                                       copies and MMAs are in flight: it stops, drains what it
                                       issued and records MOE_DEVSTAT_TIMEOUT.  The output is then
                                       undefined; with MOE_DEBUG_CHECK the call returns
                                       MOE_ERR_DEVICE_CHECK.  The next call runs normally. */

#define MOE_TEST_BAD_INDEX (1u << 7) /* test only: the router writes expert index E (out of range)
                                       for token 0's first pick; the kernels' range checks must
                                       catch it (MOE_DEVSTAT_BAD_EXPERT) without an out-of-range
                                       access.  The output is then undefined. */
#define MOE_TRACE (1u << 8)         /* moe_stack_forward, fused kernel: stamp each CTA's phases
                                       with the GPU's nanosecond timer into the workspace (see
                                       moe_stack_trace_offset); the output is unchanged */
#define MOE_DEBUG_POISON (1u << 9)  /* fill the workspace (past the fused kernel's counters) with
                                       0xFF bytes before the kernels run: a kernel that read scratch
                                       it had not written would see NaN / -1; the output must not
                                       change */
#define MOE_STACK_FUSED (1u << 10)  /* moe_stack_forward: take the fused stack kernel wherever it
                                       serves the call (without it the stack runs one
                                       moe_layer_forward per layer, measured faster at every T) */
#define MOE_WEIGHTS_INT8 (1u << 11) /* the expert weights (routed and shared) are int8 codes, one
                                       byte per element: w13 [E][2I][H], w2 [E][H][I], shared
                                       w13 [2Is][H], w2 [H][Is] (byte j of a row = element j, two's
                                       complement; weight = code * row scale).  H must be a
                                       multiple of 256 (else MOE_ERR_UNSUPPORTED).  With H >= 1024
                                       and I, Is multiples of 256 the kernel sequences are int4's
                                       (weight-streaming kernels read the codes as int8 directly;
                                       no fused stack kernel, no tcgen05 streaming gate/up); other
                                       shapes take the tensor-core sequence at every T, and
                                       MOE_FORCE_DECODE on them is MOE_ERR_UNSUPPORTED.  Expert bit
                                       width of the checkpoint converter: nanocolibri-engine
                                       README, "Converting a checkpoint yourself" */

/* Device status word: the first 4 bytes of the workspace hold the OR of these
 * bits after a call completes on the device (0 = no check failed).  Under
 * MOE_DEBUG_CHECK a non-zero word makes the call return MOE_ERR_DEVICE_CHECK. */
#define MOE_DEVSTAT_BAD_EXPERT (1u << 0) /* a routing index outside [0, E) */
#define MOE_DEVSTAT_BAD_SLOT (1u << 1)   /* a bucket slot outside [0, T*K) */
#define MOE_DEVSTAT_BAD_COUNT (1u << 2)  /* bucket counts do not sum to T*K */
#define MOE_DEVSTAT_BAD_TASK (1u << 3)   /* a work item resolved outside the bucket list */
#define MOE_DEVSTAT_TIMEOUT (1u << 4)    /* a bounded wait (about 2 s; MOE_TEST_STALL: ~1 ms) gave up */

/* The always-resident shared expert (intermediate size Is).
 *   w13: uint8 [2*Is][H/2]  rows 0..Is-1 gate, rows Is..2*Is-1 up
 *   s13: f32   [2*Is]       one scale per w13 row
 *   w2 : uint8 [H][Is/2]
 *   s2 : f32   [H]
 * (under MOE_WEIGHTS_INT8: w13 [2*Is][H], w2 [H][Is]) */
typedef struct moe_shared_weights {
    const uint8_t* w13;
    const float* s13;
    const uint8_t* w2;
    const float* s2;
} moe_shared_weights_t;

/* Stages of one forward call, for the optional per-stage event hook. */
#define MOE_STAGE_ROUTE 0   /* router, selection, bucketing */
#define MOE_STAGE_GATE_UP 1 /* expert gate/up projections + SwiGLU (routed and shared) */
#define MOE_STAGE_DOWN 2    /* expert down projections (routed and shared) */
#define MOE_STAGE_COMBINE 3 /* weighted combine (+ shared expert, + residual) */
#define MOE_NUM_STAGES 4

/* Layer configuration.
 *   struct_size    : sizeof(moe_cfg_t) (ABI versioning).
 *   H              : hidden size; multiple of 128, at most 16384.
 *   E              : routed experts, 1..256.
 *   K              : experts per token, 1..8 and K <= E.
 *   I              : routed intermediate size; multiple of 128, at most 8192.
 *   Is             : shared intermediate size; 0 (no shared expert) or a
 *                    multiple of 128, at most 8192.
 *   routed_scaling : factor on the normalised routing weights (finite, > 0).
 *   flags          : MOE_* flags above.
 *   workspace      : device scratch of at least moe_layer_workspace_bytes()
 *                    bytes, 256-byte aligned; its contents need no
 *                    initialisation and are overwritten by every call.
 *   topk_idx_out   : optional device int32 [T][K]: selected experts, in
 *                    decreasing order of s + bias (NULL = not written).
 *   topk_w_out     : optional device f32 [T][K]: their routing weights.
 *   stage_events   : optional array of 2*MOE_NUM_STAGES cudaEvent_t handles
 *                    (created by the caller, e.g. with cudaEventCreate);
 *                    events [2s] and [2s+1] are recorded on `stream` before
 *                    and after stage s.  NULL = no recording.
 *   topp           : adaptive expert top-p (colibri README, "Quick start"
 *                    knobs, "--topp 0.7"): 0 (or >= 1) = plain top-K; for
 *                    0 < topp < 1, of each token's K selected experts the
 *                    fewest highest-scoring ones whose sigmoid scores reach
 *                    topp of the K's total are kept (in selection order, at
 *                    least one), re-weighted as routed_scaling * s /
 *                    (sum of the kept s); the dropped picks are not computed
 *                    and appear in topk_idx_out as -1 (weight 0) after the
 *                    kept ones.  The keep decision is taken in f32. */
typedef struct moe_cfg {
    uint32_t struct_size;
    int32_t H, E, K, I, Is;
    float routed_scaling;
    uint32_t flags;
    void* workspace;
    size_t workspace_bytes;
    int32_t* topk_idx_out;
    float* topk_w_out;
    void* const* stage_events;
    float topp;
} moe_cfg_t;

/* Bytes of workspace moe_layer_forward needs for T tokens under `cfg`
 * (workspace, workspace_bytes and the output pointers are ignored; flags are
 * not: the size depends on the kernel sequence that T and the flags select,
 * and a smaller T can need more; see moe_layer_workspace_bytes_upto).
 * Returns 0 if cfg is NULL or the shape is invalid or unsupported. */
size_t moe_layer_workspace_bytes(const moe_cfg_t* cfg, int32_t T);

/* Bytes of workspace that serve every call of 0..N tokens under `cfg`: the
 * largest moe_layer_workspace_bytes(cfg, T) over T <= N.  Returns 0 if cfg is
 * NULL, the shape is invalid or unsupported, or N is out of range. */
size_t moe_layer_workspace_bytes_upto(const moe_cfg_t* cfg, int32_t N);

/* Forward pass of one MoE layer for T tokens.
 *   x          : bf16 [T][H]
 *   router_w   : f32  [E][H]
 *   router_bias: f32  [E]
 *   packed_w13 : uint8 [E][2I][H/2]  per expert: rows 0..I-1 gate, I..2I-1 up
 *   scales13   : f32  [E][2I]
 *   packed_w2  : uint8 [E][H][I/2]
 *   scales2    : f32  [E][H]
 *                (under MOE_WEIGHTS_INT8: packed_w13 [E][2I][H], packed_w2 [E][H][I])
 *   shared_w   : the shared expert (required when cfg->Is > 0, else ignored)
 *   out        : bf16 [T][H]  (written; one round-to-nearest-even of the f32 sum),
 *                or f32 [T][H] under MOE_OUT_F32
 *   T          : tokens, 0..2^20 (T = 0 returns MOE_OK and launches nothing)
 *   cfg, stream: see above.
 * Arithmetic.  Router logits, scores and routing weights are f32 (on the
 * large-batch sequences the logits are summed on the tensor cores from an
 * exact three-term bf16 split of each f32 router weight, 16 products per
 * step, with f32 adds between steps).  Two kernel sequences compute the
 * experts:
 *  - small batches (T <= moe_decode_max_tokens(), unless MOE_FORCE_PREFILL),
 *    and larger ones when H is not a multiple of 256, when T*K < 32*E (fewer
 *    than 32 picks per routed expert on average; not under
 *    MOE_FORCE_PREFILL), or under MOE_FORCE_DECODE: weight-streaming
 *    kernels (moe_layer_path tells which).  An activation row (x of a
 *    token, or a 512-wide slice of its SwiGLU intermediate h) is written as
 *    s * (q0 + q1/256) with int8 q0, q1 and a power of two s from the row's
 *    largest magnitude, so each element is represented to within 2^-15 of
 *    that magnitude (rows whose largest magnitude is below 2^-113 become
 *    zero; a row holding NaN or infinity gives NaN outputs).  Weight codes
 *    times activation parts accumulate exactly in int32; h is kept in f32.
 *  - otherwise: tensor-core kernels
 *    with bf16 x, f32 accumulation, and h kept in fp16 as h * 2^-k_t with a
 *    per-token power of two 2^-k_t that keeps it in fp16's normal range.
 *    Weight codes (int4 or int8) enter the MMAs exactly as 16-bit values;
 *    the row scales are applied to the f32 accumulators.
 * Expert outputs and their weighted sum are f32 until the output rounding.
 * Returns MOE_OK or an MOE_ERR_* code; on an error nothing is launched
 * (except MOE_ERR_CUDA / MOE_ERR_DEVICE_CHECK, raised after launching). */
int moe_layer_forward(const void* x, const float* router_w, const float* router_bias,
                      const uint8_t* packed_w13, const float* scales13,
                      const uint8_t* packed_w2, const float* scales2,
                      const moe_shared_weights_t* shared_w, void* out, int32_t T,
                      const moe_cfg_t* cfg, void* stream);

/* ---------------------------------------------------------------------------
 * For callers that cannot allocate device memory.
 *
 * moe_layer_forward needs a caller-provided workspace.  Some callers cannot
 * call cudaMalloc or any other allocator: a plug-in running inside a host
 * framework that owns all device memory through its own pool, for example,
 * or code that must not allocate while one of its streams is being captured.
 * moe_layer_forward_static_ws serves them.  The paper has no counterpart of
 * this entry point; it exists for integration only.
 *
 * It takes the same arguments as moe_layer_forward and computes the same
 * result with the same kernels, but ignores cfg->workspace and
 * cfg->workspace_bytes.  Its scratch memory is one array of
 * MOE_STATIC_WORKSPACE_BYTES (32 MiB) that the library itself holds in device
 * memory, on every GPU that loads it, until the process exits.
 *  - A call whose moe_layer_workspace_bytes(cfg, T) exceeds that size returns
 *    MOE_ERR_WORKSPACE and launches nothing.
 *  - It allocates nothing and calls no allocating routine.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current.  Make that first call
 *    before any stream capture begins.  The address belongs to the device's
 *    current driver context: after cudaDeviceReset, or under another
 *    context, the next call looks it up again (so make that call, too,
 *    outside a capture).
 *  - Every call on a device shares the one array, and the array keeps the
 *    last call's contents.  Calls that may run at the same time on the GPU
 *    (on different streams, with nothing ordering them) race on it and must
 *    not be issued; calls ordered on one stream are fine.  No part of the
 *    array has to start at zero: each call sets what it uses.
 * ------------------------------------------------------------------------- */
#define MOE_STATIC_WORKSPACE_BYTES ((size_t)32 << 20)

int moe_layer_forward_static_ws(const void* x, const float* router_w, const float* router_bias,
                                const uint8_t* packed_w13, const float* scales13,
                                const uint8_t* packed_w2, const float* scales2,
                                const moe_shared_weights_t* shared_w, void* out, int32_t T,
                                const moe_cfg_t* cfg, void* stream);

/* ---------------------------------------------------------------------------
 * A stack of L MoE layers: x_{l+1} = MoE_l(x_l) (+ x_l under MOE_ADD_RESIDUAL),
 * each layer as moe_layer_forward defines it, x_0 = x.  (The Colibri-Nano
 * decode runs 23 such MoE layers per token; attention between them is not
 * part of this library.)
 *
 * The weights of all layers are stacked along a leading layer dimension, in
 * the per-layer layouts of moe_layer_forward:
 *   router_w [L][E][H] f32, router_bias [L][E] f32,
 *   w13 [L][E][2I][H/2] uint8, s13 [L][E][2I] f32,
 *   w2 [L][E][H][I/2] uint8, s2 [L][E][H] f32,
 *   shared.w13 [L][2Is][H/2], shared.s13 [L][2Is], shared.w2 [L][H][Is/2],
 *   shared.s2 [L][H]
 * (under MOE_WEIGHTS_INT8 the code rows are H, I and Is bytes long, and every
 * layer takes its own moe_layer_forward call).
 * outs: bf16 [L][T][H]; layer l writes outs[l], which is layer l+1's input.
 * cfg->topk_idx_out / topk_w_out (optional): [L][T][K].
 *
 * Small batches (1 <= T <= 64, H, I and Is multiples of 256, L <= 128, no
 * MOE_FORCE_* flag) can run the whole stack in ONE cooperative kernel with
 * one CTA per SM (MOE_PATH_FUSED_STACK) under MOE_STACK_FUSED.  Without the
 * flag the stack runs one moe_layer_forward per layer, which was measured
 * faster at every T (23-layer Nano stack: 0.51 against 0.56 ms at T = 1,
 * 0.93 against 1.01 ms at T = 64).  The fused
 * kernel: per layer, router units combine the
 * previous layer's expert outputs, compute the router logits on the tensor
 * cores and select; every CTA then builds the layer's buckets and runs its
 * share of the expert tasks, the down projection of an expert starting as
 * soon as that expert's gate/up tasks are done.  Across layers it prefetches
 * into L2 the next layer's shared expert and routers, and the experts that the
 * next layer's router picks when run on the current layer's input (the
 * cross-layer expert prediction of the nanocolibri-engine README, knobs
 * table, PREDICT; colibri README, "How it works") when MOE_LOOKAHEAD is set;
 * the hints change no output bit.  One cudaMemsetAsync of the
 * workspace's counters precedes the kernel.  The arithmetic is the
 * weight-streaming path's (see "Arithmetic" above); the router logits are
 * summed per 128-column block of the hidden dimension, so they can differ
 * from moe_layer_forward's in the last bits.  Other calls run one
 * moe_layer_forward per layer (MOE_PATH_PER_LAYER).
 *
 * MOE_OUT_F32 is rejected (MOE_ERR_INVALID_ARG).  Under MOE_DEBUG_CHECK the
 * call synchronises and reports the device status word (the first 4 bytes of
 * the workspace).  A fused call waits, with bounded waits (~2 s), on counters
 * that other CTAs of the same launch advance; a wait that runs out records
 * MOE_DEVSTAT_TIMEOUT and every CTA stops.
 * ------------------------------------------------------------------------- */
typedef struct moe_stack_weights {
    const float* router_w;
    const float* router_bias;
    const uint8_t* w13;
    const float* s13;
    const uint8_t* w2;
    const float* s2;
    moe_shared_weights_t shared;
} moe_stack_weights_t;

#define MOE_PATH_FUSED_STACK 4 /* moe_stack_forward: one fused kernel for the whole stack */
#define MOE_PATH_PER_LAYER 5   /* moe_stack_forward: one moe_layer_forward per layer */

/* Workspace bytes of moe_stack_forward for T tokens and L layers (0: invalid). */
size_t moe_stack_workspace_bytes(const moe_cfg_t* cfg, int32_t T, int32_t L);

/* MOE_TRACE on the fused path: byte offset in the workspace of the trace,
 * an array [grid][L+1][16] of uint64 %globaltimer stamps (ns) written by each
 * CTA (grid = the number of SMs; a stamp a CTA does not take stays 0) at:
 *  0 entering a layer's router phase, 1 the previous layer's down tasks all
 *  done, 2 its router units done, 3 every token group of the layer selected,
 *  4 the layer's tables built, 5 its gate/up tasks done, 6 its down tasks
 *  done; the CTA's first router unit: 7 combined, 8 partial logits written,
 *  9 counted; the unit that completed a token group: 10 selected, 11 rows
 *  quantized; 12 this layer's prefetches issued; 13 the first gate/up stage
 *  landed; the first down task: 14 its expert ready, 15 its activations
 *  staged.  Row L holds the final combine's stamps 0-2.
 * Returns 0 when the call would not trace (no MOE_TRACE, or not fused). */
size_t moe_stack_trace_offset(const moe_cfg_t* cfg, int32_t T, int32_t L);

/* MOE_PATH_FUSED_STACK or MOE_PATH_PER_LAYER for T tokens and L layers, or 0
 * if T = 0 or the call would be rejected. */
int32_t moe_stack_path(const moe_cfg_t* cfg, int32_t T, int32_t L);

/* Forward of L stacked layers for T tokens (T = 0: MOE_OK, nothing launched).
 * x: bf16 [T][H]; w: the stacked weights; outs: bf16 [L][T][H], not
 * overlapping x.  Returns as moe_layer_forward. */
int moe_stack_forward(const void* x, const moe_stack_weights_t* w, int32_t L, void* outs, int32_t T,
                      const moe_cfg_t* cfg, void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* moe_status_str(int status);

/* MOE_ABI_VERSION of the loaded library. */
int moe_abi_version(void);

/* Largest T for which moe_layer_forward takes the small-batch path when
 * neither MOE_FORCE_* flag is set. */
int32_t moe_decode_max_tokens(void);

/* Number of kernels one moe_layer_forward call launches for T tokens under
 * cfg (the stage events are not kernels).  Returns 0 if T = 0 or the call
 * would be rejected for cfg or T (the pointers in cfg are not looked at). */
int32_t moe_layer_kernel_launches(const moe_cfg_t* cfg, int32_t T);

/* The kernel sequence moe_layer_forward takes for T tokens under cfg (see
 * "Arithmetic" above), or 0 if T = 0 or the call would be rejected. */
#define MOE_PATH_SMALL_BATCH 1     /* cluster router, weight-streaming experts */
#define MOE_PATH_TENSOR_CORE 2     /* large router, tensor-core grouped GEMMs */
#define MOE_PATH_LARGE_STREAMING 3 /* large router, weight-streaming experts */
int32_t moe_layer_path(const moe_cfg_t* cfg, int32_t T);

#ifdef __cplusplus
}
#endif

#endif /* MOE_INT4_H */
