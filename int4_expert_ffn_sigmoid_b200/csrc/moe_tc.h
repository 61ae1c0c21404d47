// Tensor-core (tcgen05) grouped GEMM of the large-batch expert path (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "moe_common.cuh"

namespace moe {

// Arguments of one grouped-GEMM launch.
struct TcArgs {
    int T, H, E, K, I, Is;
    int gemm;              // 1: gate/up + SwiGLU -> h; 2: down -> y
    int kdim_r, kdim_s;    // reduction length of routed / shared tiles
    int ntile_r, ntile_s;  // output-column tiles per token tile (routed / shared)
    const Ctrl* ctrl;
    const int32_t* bucket_e;
    const int32_t* bucket_n;
    const int32_t* bucket_off;
    const int32_t* tstart;  // exclusive prefix of routed tiles per routed bucket
    const float* s_r;       // routed row scales [E][rows]
    const float* s_s;       // shared row scales [rows]
    __half* h_r;
    __half* h_s;
    float* y;
    const int32_t* tok_of_slot;
    const int32_t* hexp;  // per-token exponent of the h storage scale
    unsigned* status;
    int stall;            // MOE_TEST_STALL: the epilogue's first wait runs out
};

// Signature of cuTensorMapEncodeTiled (fetched from the driver at run time).
typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// A 2-D tensor map over a row-major [rows][inner] matrix of esize-byte
// elements (box box_inner x box_rows); false if the driver entry point is
// missing or rejects the arguments.
bool encode_tensor_map_2d(CUtensorMap* m, CUtensorMapDataType dt, int esize, const void* base, uint64_t inner,
                          uint64_t rows, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw);

// Launch GEMM-1 (gemm = 1) or GEMM-2 (gemm = 2) of the large-batch path.
cudaError_t launch_tc_gemm(const Params& p, int gemm, int grid, cudaStream_t stream);
int tc_smem_bytes();

}  // namespace moe
