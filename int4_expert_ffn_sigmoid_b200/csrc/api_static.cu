// moe_layer_forward_static_ws: the layer forward for callers that cannot
// allocate device memory (see include/moe_int4.h).  The scratch memory the
// kernels need comes from a fixed-size array in this file instead of a
// caller-provided workspace; everything else is moe_layer_forward unchanged.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "moe_int4.h"

namespace {

// Largest workspace the entry point can serve.  The array below is device
// memory that every GPU which loads this library holds until the process
// exits.
constexpr size_t kStaticWorkspaceBytes = MOE_STATIC_WORKSPACE_BYTES;

__device__ __align__(256) unsigned char g_static_ws[kStaticWorkspaceBytes];

// Device address of g_static_ws per device, with the driver context it
// belongs to.  In host code the symbol's name is only a host-side stand-in; a
// kernel given it would fault (or, where the GPU can reach host memory,
// silently use the wrong memory), so the address is fetched from the runtime
// with the device current.  The module, and so the address, is per context:
// after cudaDeviceReset, or under another context on the same device, the
// address is looked up again.
struct StaticWs {
    void* ctx = nullptr;
    void* ptr = nullptr;
};
StaticWs g_static_ws_of[64];
std::mutex g_static_ws_mu;

typedef CUresult (*PFN_ctxGetCurrent)(CUcontext*);

void* current_context() {
    static PFN_ctxGetCurrent fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<PFN_ctxGetCurrent>(f);
    }();
    CUcontext c = nullptr;
    if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

// The array's device address on device `dev` (current) in the current
// context, or nullptr if the runtime cannot give it.
void* static_ws_address(int dev) {
    std::lock_guard<std::mutex> lock(g_static_ws_mu);
    StaticWs& w = g_static_ws_of[dev];
    void* ctx = current_context();
    if (w.ptr && ctx && ctx == w.ctx) return w.ptr;
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_ws) != cudaSuccess || !ptr) return nullptr;
    w.ptr = ptr;
    w.ctx = current_context();  // the lookup made the runtime's context current if none was
    return ptr;
}

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
    void* ws = static_ws_address(dev);
    if (!ws) return MOE_ERR_CUDA;
    moe_cfg_t c = *cfg;
    c.workspace = ws;
    c.workspace_bytes = kStaticWorkspaceBytes;
    return moe_layer_forward(x, router_w, router_bias, packed_w13, scales13, packed_w2, scales2, shared_w, out, T,
                             &c, stream);
}

}  // extern "C"
