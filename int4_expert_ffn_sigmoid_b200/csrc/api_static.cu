// moe_layer_forward_static_ws: the layer forward for callers that cannot
// allocate device memory (see include/moe_int4.h).  The scratch memory the
// kernels need comes from a fixed-size array in this file instead of a
// caller-provided workspace; everything else is moe_layer_forward unchanged.
#include <atomic>

#include "moe_int4.h"

namespace {

// Largest workspace the entry point can serve.  The array below is device
// memory that every GPU which loads this library holds until the process
// exits.
constexpr size_t kStaticWorkspaceBytes = MOE_STATIC_WORKSPACE_BYTES;

__device__ __align__(256) unsigned char g_static_ws[kStaticWorkspaceBytes];

// Device address of g_static_ws per device.  In host code the symbol's name
// is only a host-side stand-in; a kernel given it would fault (or, where the
// GPU can reach host memory, silently use the wrong memory), so the address
// is fetched from the runtime with the device current.
std::atomic<void*> g_static_ws_ptr[64];

}  // namespace

extern "C" {

int moe_layer_forward_static_ws(const void* x, const float* router_w, const float* router_bias,
                                const uint8_t* packed_w13, const float* scales13, const uint8_t* packed_w2,
                                const float* scales2, const moe_shared_weights_t* shared_w, void* out, int32_t T,
                                const moe_cfg_t* cfg, void* stream) {
    if (!cfg || cfg->struct_size != sizeof(moe_cfg_t)) return MOE_ERR_INVALID_ARG;
    const size_t need = moe_layer_workspace_bytes(cfg, T);
    if (need == 0) {
        // an invalid shape or argument: let the regular entry point report it
        moe_cfg_t c = *cfg;
        c.workspace = nullptr;
        c.workspace_bytes = 0;
        const int st = moe_layer_forward(x, router_w, router_bias, packed_w13, scales13, packed_w2, scales2,
                                         shared_w, out, T, &c, stream);
        return st == MOE_OK ? MOE_ERR_INVALID_ARG : st;
    }
    if (need > kStaticWorkspaceBytes) return MOE_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    void* ws = g_static_ws_ptr[dev].load(std::memory_order_acquire);
    if (!ws) {
        if (cudaGetSymbolAddress(&ws, g_static_ws) != cudaSuccess || !ws) return MOE_ERR_CUDA;
        g_static_ws_ptr[dev].store(ws, std::memory_order_release);
    }
    moe_cfg_t c = *cfg;
    c.workspace = ws;
    c.workspace_bytes = kStaticWorkspaceBytes;
    return moe_layer_forward(x, router_w, router_bias, packed_w13, scales13, packed_w2, scales2, shared_w, out, T,
                             &c, stream);
}

}  // extern "C"
