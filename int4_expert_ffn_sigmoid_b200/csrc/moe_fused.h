// Fused small-batch forward of a stack of MoE layers (internal): arguments
// and host entry points of decode_stack_kernel.
#pragma once

#include <cuda_runtime.h>

#include "moe_common.cuh"

namespace moe {

// Layers of one fused call, and the token groups of its router units.
constexpr int kMaxFusedLayers = 128;
constexpr int kMaxGroupsF = kDecodeMaxTokens / 8;
// MOE_TRACE: stamps per (CTA, layer): 0 phase A entered, 1 the previous
// layer's down tasks all done, 2 phase A done, 3 every token group selected,
// 4 tables built, 5 gate/up tasks done, 6 down tasks done; first router unit
// of the CTA: 7 combined, 8 partial logits written, 9 counted; the unit that
// completed a group: 10 selected, 11 rows quantized; 12 prefetches issued;
// 13 the first gate/up stage landed; first down task: 14 its expert ready,
// 15 its activations staged.
constexpr int kTraceSlots = 16;

// Everything the fused kernel reads and writes.  Weights of all L layers are
// stacked along a leading layer dimension (layer l of router_w is at
// rw + l*E*H, and so on); outs is [L][T][H] (layer l's output, which is
// layer l+1's input).
struct FArgs {
    int T, H, E, K, I, Is, L;
    int G, NCB;            // token groups of 8, hidden blocks of 128
    int rows2, nsl_r, nsl_s;
    int r13_r, r13_s;      // gate/up tasks per 16-token chunk of a routed / the shared bucket
    int r2_r, r2_s;        // down tasks per 16-token chunk of a routed / the shared bucket
    float scale;
    float topp;            // adaptive expert top-p (0: off); dropped picks are index -1
    unsigned flags;
    const __nv_bfloat16* x;  // [T][H], layer 0's input
    __nv_bfloat16* outs;     // [L][T][H]
    const float* rw;         // [L][E][H]
    const float* rb;         // [L][E]
    const uint8_t* w13;      // [L][E][2I][H/2]
    const float* s13;        // [L][E][2I]
    const uint8_t* w2;       // [L][E][H][I/2]
    const float* s2;         // [L][E][H]
    const uint8_t* sh_w13;   // [L][2Is][H/2]
    const float* sh_s13;     // [L][2Is]
    const uint8_t* sh_w2;    // [L][H][Is/2]
    const float* sh_s2;      // [L][H]
    int32_t* topk_idx;       // optional [L][T][K]
    float* topk_w;           // optional [L][T][K]
    // workspace: counters (zeroed before every launch)
    unsigned* status;
    int* abort;
    int* grp_cnt;       // [L][kMaxGroupsF]  router units done per token group
    int* groups_done;   // [L]               token groups selected
    int* down_done;     // [L]               CTAs done with the layer's down tasks
    int* ready;         // [L][kMaxE + 1]    gate/up tasks done per expert (E: the shared expert)
    unsigned* pred_bits;  // [L][8]          experts predicted by the lookahead (bit e)
    unsigned long long* trace;  // MOE_TRACE: [grid][L + 1][kTraceSlots] %globaltimer stamps, or null
    // workspace: data
    float* lp;          // [NCB][T][E] partial router logits of the current layer
    float* lpn;         // [NCB][T][E] partial logits of the next layer's router on the current input
    int32_t* idx;       // [T][K]
    float* wts;         // [T][K]
    int8_t* xq;         // [T][2][H]
    float* xs;          // [T]
    float* h32_r;       // [T*K][I]
    float* h32_s;       // [T][Is]
    float* hmax_r;      // [T*K][I/64]
    float* hmax_s;      // [T][Is/64]
    float* y;           // [T*K*nsl_r + T*nsl_s][H]
};

// Whether the fused kernel serves this shape and T (tokens 1..64, H, I and Is
// multiples of 256, up to kMaxFusedLayers layers).
bool fused_supported(int H, int E, int K, int I, int Is, int T, int L);
// Rows of one down task for the fused kernel.
int fused_rows2(int H, int E, int K, int I, int Is, int T, int sms);
// The cooperative grid (one CTA per SM), or -1 if the kernel cannot be resident.
int fused_grid();
size_t fused_smem_bytes();
cudaError_t launch_decode_stack(const FArgs& a, int grid, cudaStream_t stream);

}  // namespace moe
