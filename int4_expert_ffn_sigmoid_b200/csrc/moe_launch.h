// Host-side launch entry points of the kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>

#include "moe_common.cuh"

namespace moe {

// Router + bucketing.  small_path: T <= kDecodeMaxTokens.
cudaError_t launch_router(const Params& p, bool small_path, cudaStream_t stream);
// Hidden-dimension slices of the split small-batch router's partial logits
// (0: the cluster router computes the logits itself).
int router_split_slices(int E, int H);
// Tensor-core router logits of the large-batch path: the weight split and
// the logits kernel (slices of the hidden dimension, partials in lpart).
cudaError_t launch_router_tc(const Params& p, cudaStream_t stream);
// Whether the large-batch path computes the router logits on the tensor cores
// (router_tc.cu; router weights above 512 KB) rather than in router_large_kernel.
bool router_large_uses_tc(int E, int H);
// Hidden slices of the tensor-core router (a function of E and H only).
int tc_router_slices(int E, int H);
// Expert gate/up + SwiGLU (weight-streaming mma.sync kernel).
cudaError_t launch_experts_w13(const Params& p, int grid, cudaStream_t stream);
// Expert down projection (weight-streaming mma.sync kernel).
cudaError_t launch_experts_w2(const Params& p, int grid, cudaStream_t stream);
// CTAs of the weight-streaming kernel `which` (0: gate/up, 1: down) that fit
// on the device at once (the persistent grid size) for hidden size H.  Also
// sets the kernel's shared-memory attribute.
int experts_resident_ctas(int which, int H, bool w2_tma, int chunk, bool int8w, bool occ2 = false);
// Whether the gate/up (down) projection takes the TMA-ring kernel for this shape.
bool experts_w13_tma(int H);
// Whether the large-batch streaming sequence runs gate/up on the tcgen05
// kernel: TMA-ring shapes with at least kTc8MinPicksPerExpert picks per
// routed expert on average (T*K/E), where it outruns the mma.sync kernel.
bool experts_w13_tc8(int H, int I, int Is, int T, int K, int E);
bool experts_w2_tma(int H, int I, int Is);
// Weighted combine + shared expert (+ residual) -> bf16 out.
cudaError_t launch_combine(const Params& p, cudaStream_t stream);

}  // namespace moe
