// C ABI of the int4 MoE layer forward: argument validation, workspace
// layout, kernel sequence.  See include/moe_int4.h for the contract.
#include <math.h>
#include <string.h>

#include "moe_common.cuh"
#include "moe_fused.h"
#include "moe_int4.h"
#include "moe_launch.h"
#include "moe_tc.h"

namespace {

using namespace moe;

constexpr unsigned kKnownFlags = MOE_ADD_RESIDUAL | MOE_DEBUG_CHECK | MOE_FORCE_DECODE | MOE_FORCE_PREFILL |
                                 MOE_OUT_F32 | MOE_TEST_STALL | MOE_LOOKAHEAD | MOE_TEST_BAD_INDEX |
                                 MOE_TRACE | MOE_DEBUG_POISON | MOE_STACK_FUSED | MOE_WEIGHTS_INT8;
// Traced CTAs at most (the fused kernel runs one CTA per SM).
constexpr int kMaxGridF = 256;
static_assert(kFlagResidual == MOE_ADD_RESIDUAL && kFlagOutF32 == MOE_OUT_F32 && kFlagTestStall == MOE_TEST_STALL &&
                  kFlagLookahead == MOE_LOOKAHEAD && kFlagTestBadIndex == MOE_TEST_BAD_INDEX &&
                  kFlagTrace == MOE_TRACE && kFlagWeightsInt8 == MOE_WEIGHTS_INT8,
              "kernel flag bits match the C ABI");
static_assert(ST_BAD_EXPERT == MOE_DEVSTAT_BAD_EXPERT && ST_BAD_SLOT == MOE_DEVSTAT_BAD_SLOT &&
                  ST_BAD_COUNT == MOE_DEVSTAT_BAD_COUNT && ST_BAD_TASK == MOE_DEVSTAT_BAD_TASK &&
                  ST_TIMEOUT == MOE_DEVSTAT_TIMEOUT && offsetof(Ctrl, status) == 0,
              "device status bits match the C ABI");
constexpr int32_t kMaxTokens = 1 << 20;

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Kernel sequence of a call: the small-batch router + weight-streaming
// experts; the large router + tensor-core grouped GEMMs; or the large router
// + weight-streaming experts (H not a multiple of 256, or MOE_FORCE_DECODE).
// int8 expert weights stream through the TMA-ring kernels only: shapes those
// do not serve take the tensor-core sequence at every T.
enum class Path { kSmall, kTensorCore, kLargeStreaming };

// Average (token, pick) slots per routed expert below which large batches
// stream the weights instead of running the grouped GEMM: with fewer tokens
// per expert the GEMM's 128-token tiles are mostly padding and the layer is
// bound by reading the touched experts' weights.
constexpr int kTcMinSlotsPerExpert = 32;

// Gate/up tasks per SM from which the 16-token TMA-ring gate/up runs two CTAs
// per SM.
constexpr int kW13TwoPerSmMinTasksPerSm = 4;

bool int8_streams(const moe_cfg_t& c) { return experts_w13_tma(c.H) && experts_w2_tma(c.H, c.I, c.Is); }

Path choose_path(const moe_cfg_t& c, int32_t T) {
    if ((c.flags & MOE_WEIGHTS_INT8) && !int8_streams(c)) return Path::kTensorCore;
    if (T <= kDecodeMaxTokens && !(c.flags & MOE_FORCE_PREFILL)) return Path::kSmall;
    // GEMM-2 of the tensor-core path tiles 256 output columns
    if ((c.flags & MOE_FORCE_DECODE) || c.H % 256 != 0) return Path::kLargeStreaming;
    if (c.flags & MOE_FORCE_PREFILL) return Path::kTensorCore;
    return (long long)T * c.K >= (long long)kTcMinSlotsPerExpert * c.E ? Path::kTensorCore : Path::kLargeStreaming;
}

struct WsLayout {
    size_t ctrl, idx, wts, counts, offsets, bucket_e, bucket_n, bucket_off, ts13, ts2, tcs1, tcs2;
    size_t tok_of_slot, slot_of, hist, rank, hexp, y, lpart, wsplit;
    size_t h_r, h_s, x_perm;                            // tensor-core path
    size_t xq, xs, h32_r, h32_s, hmax_r, hmax_s;        // weight-streaming paths
    size_t total;
};

WsLayout ws_layout(const moe_cfg_t& c, int32_t T) {
    WsLayout L{};
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t r = o;
        o = align256(o + bytes);
        return r;
    };
    const Path path = choose_path(c, T);
    const size_t TK = (size_t)T * c.K, E = (size_t)c.E, H = (size_t)c.H;
    L.ctrl = take(sizeof(Ctrl));
    L.idx = take(TK * 4);
    L.wts = take(TK * 4);
    L.counts = take(E * 4);
    L.offsets = take(E * 4);
    L.bucket_e = take((E + 1) * 4);
    L.bucket_n = take((E + 1) * 4);
    L.bucket_off = take((E + 1) * 4);
    L.ts13 = take((E + 2) * 4);
    L.ts2 = take((E + 2) * 4);
    L.tcs1 = take((E + 2) * 4);
    L.tcs2 = take((E + 2) * 4);
    L.tok_of_slot = take(TK * 4);
    L.slot_of = take(TK * 4);
    L.hist = take((size_t)kRouterMaxBlocks * E * 4);
    L.rank = take(TK * 4);
    L.hexp = take((size_t)T * 4);
    if (path == Path::kSmall) {
        L.lpart = take((size_t)router_split_slices(c.E, c.H) * T * E * 4);
    } else if (router_large_uses_tc(c.E, c.H)) {  // the tensor-core router's partial logits and split weights
        L.lpart = take((size_t)tc_router_slices(c.E, c.H) * T * E * 4);
        L.wsplit = take(3 * E * H * 2);
    }
    const size_t shared_rows = c.Is > 0 ? (size_t)T : 0;
    if (path == Path::kTensorCore) {
        L.h_r = take(TK * (size_t)c.I * 2);
        L.h_s = take((size_t)T * (size_t)c.Is * 2);
        L.x_perm = take(TK * H * 2);
        L.y = take((TK + shared_rows) * H * 4);
    } else {
        L.xq = take((size_t)T * 2 * H);
        L.xs = take((size_t)T * 4);
        L.h32_r = take(TK * (size_t)c.I * 4);
        L.h32_s = take((size_t)T * (size_t)c.Is * 4);
        L.hmax_r = take(TK * (size_t)(c.I / 64) * 4);
        L.hmax_s = take((size_t)T * (size_t)(c.Is / 64) * 4);
        L.y = take((TK * slices_of(c.I) + shared_rows * slices_of(c.Is)) * H * 4);
    }
    L.total = o;
    return L;
}

int validate_cfg(const moe_cfg_t* c) {
    if (!c || c->struct_size != sizeof(moe_cfg_t)) return MOE_ERR_INVALID_ARG;
    if (c->H <= 0 || c->E <= 0 || c->K <= 0 || c->I <= 0 || c->Is < 0 || c->K > c->E) return MOE_ERR_INVALID_ARG;
    if (!(c->routed_scaling > 0.0f) || !isfinite(c->routed_scaling)) return MOE_ERR_INVALID_ARG;
    if (!(c->topp >= 0.0f) || !isfinite(c->topp)) return MOE_ERR_INVALID_ARG;
    if (c->flags & ~kKnownFlags) return MOE_ERR_INVALID_ARG;
    if ((c->flags & MOE_FORCE_DECODE) && (c->flags & MOE_FORCE_PREFILL)) return MOE_ERR_INVALID_ARG;
    if (c->H % 128 || c->H > 16384) return MOE_ERR_UNSUPPORTED;
    // int8 expert weights: the tensor-core sequence (its down projection tiles
    // 256 output columns) or the TMA-ring streaming kernels
    if ((c->flags & MOE_WEIGHTS_INT8) && c->H % 256) return MOE_ERR_UNSUPPORTED;
    if ((c->flags & MOE_WEIGHTS_INT8) && (c->flags & MOE_FORCE_DECODE) && !int8_streams(*c)) return MOE_ERR_UNSUPPORTED;
    if (c->E > kMaxE || c->K > kMaxK) return MOE_ERR_UNSUPPORTED;
    if (c->I % 128 || c->I > 8192) return MOE_ERR_UNSUPPORTED;
    if (c->Is % 128 || c->Is > 8192) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

inline bool aligned(const void* ptr, size_t a) { return ((uintptr_t)ptr % a) == 0; }

int sm_count() {
    static int cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 0 || dev >= 64) dev = 0;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

inline int cdiv(long long a, long long b) { return (int)((a + b - 1) / b); }

// Whether a stack call takes the fused kernel: only under MOE_STACK_FUSED.
// One moe_layer_forward per layer was measured faster at every T (the
// 23-layer Nano stack: 0.507 against 0.561 ms at T = 1, 0.543 against 0.574
// at T = 4, 0.725 against 0.790 at T = 16, 0.926 against 1.008 at T = 64;
// one 6144-hidden layer: 0.084 against 0.123 ms at T = 1).
bool stack_fused(const moe_cfg_t& c, int32_t T, int32_t L) {
    if (c.flags & (MOE_FORCE_DECODE | MOE_FORCE_PREFILL | MOE_WEIGHTS_INT8)) return false;
    if (!(fused_supported(c.H, c.E, c.K, c.I, c.Is, T, L) && fused_grid() > 0)) return false;
    return (c.flags & MOE_STACK_FUSED) != 0;
}

// Workspace of the fused kernel: a zeroed control block and counters, then
// the data regions (see FArgs).
struct FusedLayout {
    size_t ctrl, grp_cnt, groups_done, down_done, ready, pred_bits, counters_end;
    size_t lp, lpn, idx, wts, xq, xs, h32_r, h32_s, hmax_r, hmax_s, y, trace, total;
};

FusedLayout fused_layout(const moe_cfg_t& c, int32_t T, int32_t L) {
    FusedLayout F{};
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t r = o;
        o = align256(o + bytes);
        return r;
    };
    auto take4 = [&](size_t n) {  // counters: packed, 4-byte aligned
        const size_t r = o;
        o += n * 4;
        return r;
    };
    const size_t TK = (size_t)T * c.K, H = c.H, Ls = (size_t)L;
    F.ctrl = take(256);
    F.grp_cnt = take4(Ls * kMaxGroupsF);
    F.groups_done = take4(Ls);
    F.down_done = take4(Ls);
    F.ready = take4(Ls * (kMaxE + 1));
    F.pred_bits = take4(Ls * 8);
    F.counters_end = o;
    o = align256(o);
    const size_t ncb = H / 128;
    F.lp = take(ncb * T * c.E * 4);
    F.lpn = take(ncb * T * c.E * 4);
    F.idx = take(TK * 4);
    F.wts = take(TK * 4);
    F.xq = take((size_t)T * 2 * H);
    F.xs = take((size_t)T * 4);
    F.h32_r = take(TK * c.I * 4);
    F.h32_s = take((size_t)T * c.Is * 4);
    F.hmax_r = take(TK * (c.I / 64) * 4);
    F.hmax_s = take((size_t)T * (c.Is / 64) * 4);
    F.y = take((TK * slices_of(c.I) + (c.Is > 0 ? (size_t)T * slices_of(c.Is) : 0)) * H * 4);
    F.trace = (c.flags & MOE_TRACE) ? take((size_t)kMaxGridF * (Ls + 1) * kTraceSlots * 8) : 0;
    F.total = o;
    return F;
}

int validate_stack(const moe_cfg_t* cfg, int32_t T, int32_t L) {
    const int st = validate_cfg(cfg);
    if (st != MOE_OK) return st;
    if (T < 0 || T > kMaxTokens || L < 1 || L > kMaxFusedLayers) return MOE_ERR_INVALID_ARG;
    if (cfg->flags & MOE_OUT_F32) return MOE_ERR_INVALID_ARG;  // outputs feed the next layer: bf16
    return MOE_OK;
}

}  // namespace

extern "C" {

int moe_abi_version(void) { return MOE_ABI_VERSION; }

int32_t moe_decode_max_tokens(void) { return kDecodeMaxTokens; }

int32_t moe_layer_kernel_launches(const moe_cfg_t* cfg, int32_t T) {
    if (validate_cfg(cfg) != MOE_OK || T <= 0 || T > kMaxTokens) return 0;
    // small batch: [router logits,] cluster router, gate/up, down, combine;
    // otherwise: router (or, with large router weights, the weight split, the
    // tensor-core router logits and the selection), scatter, gate/up, down,
    // combine
    if (choose_path(*cfg, T) != Path::kSmall) return router_large_uses_tc(cfg->E, cfg->H) ? 7 : 5;
    return 4 + (router_split_slices(cfg->E, cfg->H) > 0 ? 1 : 0);
}

int32_t moe_layer_path(const moe_cfg_t* cfg, int32_t T) {
    if (validate_cfg(cfg) != MOE_OK || T <= 0 || T > kMaxTokens) return 0;
    switch (choose_path(*cfg, T)) {
        case Path::kSmall: return MOE_PATH_SMALL_BATCH;
        case Path::kTensorCore: return MOE_PATH_TENSOR_CORE;
        default: return MOE_PATH_LARGE_STREAMING;
    }
}

const char* moe_status_str(int status) {
    switch (status) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK";
        default: return "MOE_ERR_UNKNOWN";
    }
}

size_t moe_layer_workspace_bytes(const moe_cfg_t* cfg, int32_t T) {
    if (validate_cfg(cfg) != MOE_OK || T < 0 || T > kMaxTokens) return 0;
    return ws_layout(*cfg, T).total;
}

size_t moe_layer_workspace_bytes_upto(const moe_cfg_t* cfg, int32_t N) {
    if (validate_cfg(cfg) != MOE_OK || N < 0 || N > kMaxTokens) return 0;
    // The size grows with T within each kernel sequence, so the largest T of
    // each sequence up to N bounds it: N itself, the last small-batch T, and
    // the last T below the tensor-core threshold (T*K < kTcMinSlotsPerExpert*E).
    const long long t_stream = ((long long)kTcMinSlotsPerExpert * cfg->E - 1) / cfg->K;
    const long long cands[3] = {N, kDecodeMaxTokens, t_stream};
    size_t best = 0;
    for (long long t : cands) {
        const int32_t tt = (int32_t)(t < N ? t : N);
        if (tt < 0) continue;
        const size_t b = ws_layout(*cfg, tt).total;
        if (b > best) best = b;
    }
    return best;
}

int moe_layer_forward(const void* x, const float* router_w, const float* router_bias,
                      const uint8_t* packed_w13, const float* scales13, const uint8_t* packed_w2,
                      const float* scales2, const moe_shared_weights_t* shared_w, void* out, int32_t T,
                      const moe_cfg_t* cfg, void* stream) {
    int st = validate_cfg(cfg);
    if (st != MOE_OK) return st;
    if (T < 0 || T > kMaxTokens) return MOE_ERR_INVALID_ARG;
    if (!x || !router_w || !router_bias || !packed_w13 || !scales13 || !packed_w2 || !scales2 || !out)
        return MOE_ERR_INVALID_ARG;
    if (cfg->Is > 0 && (!shared_w || !shared_w->w13 || !shared_w->s13 || !shared_w->w2 || !shared_w->s2))
        return MOE_ERR_INVALID_ARG;
    const void* ptrs[] = {x, router_w, router_bias, packed_w13, scales13, packed_w2, scales2, out,
                          cfg->Is > 0 ? shared_w->w13 : nullptr, cfg->Is > 0 ? shared_w->s13 : nullptr,
                          cfg->Is > 0 ? shared_w->w2 : nullptr, cfg->Is > 0 ? shared_w->s2 : nullptr,
                          cfg->topk_idx_out, cfg->topk_w_out};
    for (const void* ptr : ptrs)
        if (ptr && !aligned(ptr, 16)) return MOE_ERR_INVALID_ARG;
    const size_t xbytes = (size_t)T * cfg->H * 2;
    const size_t obytes = xbytes * ((cfg->flags & MOE_OUT_F32) ? 2 : 1);
    const uintptr_t xa = (uintptr_t)x, oa = (uintptr_t)out;
    if (T > 0 && xa < oa + obytes && oa < xa + xbytes) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(*cfg, T);
    if (!cfg->workspace || cfg->workspace_bytes < L.total) return MOE_ERR_WORKSPACE;
    if (!aligned(cfg->workspace, 256)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;

    char* ws = static_cast<char*>(cfg->workspace);
    const Path path = choose_path(*cfg, T);
    const bool small = path == Path::kSmall, use_tc = path == Path::kTensorCore;
    auto at = [&](size_t off) { return static_cast<void*>(ws + off); };
    Params p;
    memset(&p, 0, sizeof p);
    p.T = T; p.H = cfg->H; p.E = cfg->E; p.K = cfg->K; p.I = cfg->I; p.Is = cfg->Is;
    p.scale = cfg->routed_scaling;
    p.topp = cfg->topp;
    p.flags = cfg->flags;
    p.x = static_cast<const __nv_bfloat16*>(x);
    p.rw = router_w; p.rb = router_bias;
    p.w13 = packed_w13; p.s13 = scales13; p.w2 = packed_w2; p.s2 = scales2;
    if (cfg->Is > 0) {
        p.sh_w13 = shared_w->w13; p.sh_s13 = shared_w->s13; p.sh_w2 = shared_w->w2; p.sh_s2 = shared_w->s2;
    }
    p.out = static_cast<__nv_bfloat16*>(out);
    p.topk_idx_out = cfg->topk_idx_out;
    p.topk_w_out = cfg->topk_w_out;
    p.ctrl = static_cast<Ctrl*>(at(L.ctrl));
    p.idx = static_cast<int32_t*>(at(L.idx));
    p.wts = static_cast<float*>(at(L.wts));
    p.counts = static_cast<int32_t*>(at(L.counts));
    p.offsets = static_cast<int32_t*>(at(L.offsets));
    p.bucket_e = static_cast<int32_t*>(at(L.bucket_e));
    p.bucket_n = static_cast<int32_t*>(at(L.bucket_n));
    p.bucket_off = static_cast<int32_t*>(at(L.bucket_off));
    p.ts13 = static_cast<int32_t*>(at(L.ts13));
    p.ts2 = static_cast<int32_t*>(at(L.ts2));
    p.tcs1 = static_cast<int32_t*>(at(L.tcs1));
    p.tcs2 = static_cast<int32_t*>(at(L.tcs2));
    p.tok_of_slot = static_cast<int32_t*>(at(L.tok_of_slot));
    p.slot_of = static_cast<int32_t*>(at(L.slot_of));
    p.hist = static_cast<int32_t*>(at(L.hist));
    p.rank = static_cast<int32_t*>(at(L.rank));
    p.hexp = static_cast<int32_t*>(at(L.hexp));
    p.y = static_cast<float*>(at(L.y));
    if (use_tc) {
        p.h_r = static_cast<__half*>(at(L.h_r));
        p.h_s = static_cast<__half*>(at(L.h_s));
        p.x_perm = static_cast<__nv_bfloat16*>(at(L.x_perm));
        p.nsl_r = p.nsl_s = 1;
    } else {
        p.xq = static_cast<int8_t*>(at(L.xq));
        p.xs = static_cast<float*>(at(L.xs));
        p.h32_r = static_cast<float*>(at(L.h32_r));
        p.h32_s = static_cast<float*>(at(L.h32_s));
        p.hmax_r = static_cast<float*>(at(L.hmax_r));
        p.hmax_s = static_cast<float*>(at(L.hmax_s));
        p.nsl_r = slices_of(cfg->I);
        p.nsl_s = slices_of(cfg->Is);
    }
    p.decode_groups = small ? cdiv(T, kDecodeRouterTok) : 0;
    if (small) {
        p.lslices = router_split_slices(cfg->E, cfg->H);
    } else if (router_large_uses_tc(cfg->E, cfg->H)) {  // large router weights: logits on the tensor cores
        p.tc_router = 1;
        p.lslices = tc_router_slices(cfg->E, cfg->H);
        p.wsplit = static_cast<__nv_bfloat16*>(at(L.wsplit));
    }
    p.lpart = p.lslices > 0 ? static_cast<float*>(at(L.lpart)) : nullptr;
    const int ntiles = cdiv(T, kRouterTileTokens);
    p.router_blocks = ntiles < kRouterMaxBlocks ? ntiles : kRouterMaxBlocks;
    // large batches whose expert kernels both take the TMA-ring kernels stream
    // an expert's weights once for up to kMaxChunk of its tokens
    const bool w2_tma = experts_w2_tma(cfg->H, cfg->I, cfg->Is);
    p.chunk = path == Path::kLargeStreaming && experts_w13_tma(cfg->H) && w2_tma ? kMaxChunk : kChunkTokens;
    // A down task covers rg 128-row groups (rg up to max(4, H/1024), dividing
    // H/128): the task's h slice is quantized once for all of them and it
    // streams enough weight bytes to outweigh its per-task costs.  rg stays
    // small enough that the down tasks (counted from the upper bound of the
    // routed buckets) still give every SM one.
    {
        const long long TKl = (long long)T * cfg->K;
        const long long bucket_slices = (cfg->E < TKl ? cfg->E : TKl) * slices_of(cfg->I) +
                                        (cfg->Is > 0 ? (long long)cdiv(T, p.chunk) * slices_of(cfg->Is) : 0);
        const int groups = cfg->H / kTaskRows2, want = cfg->H / 1024 > 4 ? cfg->H / 1024 : 4;
        int rg = 1;
        for (int c : {8, 6, 4, 3, 2})
            if (c <= want && groups % c == 0 && (long long)(groups / c) * bucket_slices >= sm_count()) {
                rg = c;
                break;
            }
        p.rows2 = kTaskRows2 * rg;
    }

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const long long TK = (long long)T * cfg->K;
    const long long routed_buckets = (cfg->E < TK ? cfg->E : TK) + cdiv(TK, p.chunk);
    const long long shared_chunks = cfg->Is > 0 ? cdiv(T, p.chunk) : 0;
    // upper bounds of the weight-streaming kernels' CTA tasks
    const long long tasks13 = (long long)(cfg->I / 64) * routed_buckets + (long long)(cfg->Is / 64) * shared_chunks;
    const long long tasks2 = (long long)(cfg->H / p.rows2) *
                             (routed_buckets * slices_of(cfg->I) + shared_chunks * slices_of(cfg->Is));
    int grid13 = 0, grid2 = 0;
    if (!use_tc) {
        const bool int8w = (cfg->flags & MOE_WEIGHTS_INT8) != 0;
        // 16-token gate/up tasks: two CTAs per SM (shallower rings) once there
        // are enough tasks for both to have several (measured: Nano stack at
        // T = 64 0.996 -> 0.940 ms, large layer T = 32 0.475 -> 0.443 ms; at
        // T = 16, 304 tasks, 1% slower)
        p.w13_occ2 = !int8w && p.chunk == kChunkTokens && experts_w13_tma(cfg->H) &&
                     tasks13 >= (long long)kW13TwoPerSmMinTasksPerSm * sm_count();
        const long long cap13 = experts_resident_ctas(0, cfg->H, w2_tma, p.chunk, int8w, p.w13_occ2 != 0);
        const long long cap2 = experts_resident_ctas(1, cfg->H, w2_tma, p.chunk, int8w);
        grid13 = (int)(tasks13 < cap13 ? tasks13 : cap13);
        grid2 = (int)(tasks2 < cap2 ? tasks2 : cap2);
        // The TMA down kernel builds its tables before its wait where its CTAs
        // can start while the gate/up kernel still runs: SMs the gate/up grid
        // leaves free, or the two-CTAs-per-SM gate/up's uneven finish
        // (measured on the Nano stack: T = 1 0.481 -> 0.444 ms, T = 64 0.905
        // -> 0.871 ms; with one gate/up CTA on every SM, T = 16, 1.8% slower)
        p.w2_tables_early = small && w2_tma && (grid13 < sm_count() || p.w13_occ2);
    }

    void* const* ev = cfg->stage_events;
    auto mark = [&](int idx) -> cudaError_t {
        return ev ? cudaEventRecord(static_cast<cudaEvent_t>(ev[idx]), s) : cudaSuccess;
    };
    cudaError_t err = cudaSuccess;
    if (cfg->flags & MOE_DEBUG_POISON)  // every byte a kernel reads must have been written first
        err = cudaMemsetAsync(ws, 0xFF, L.total, s);
    if (err == cudaSuccess) err = mark(2 * MOE_STAGE_ROUTE);
    if (err == cudaSuccess) err = launch_router(p, small, s);
    if (err == cudaSuccess) err = mark(2 * MOE_STAGE_ROUTE + 1);
    int tc_grid1 = 0, tc_grid2 = 0;
    if (use_tc) {
        const long long mt_routed = (cfg->E < TK ? cfg->E : TK) + cdiv(TK, kTcTokens);
        const long long mt_shared = cfg->Is > 0 ? cdiv(T, kTcTokens) : 0;
        const long long t1 = mt_routed * (cfg->I / kTcFeat1) + mt_shared * (cfg->Is / kTcFeat1);
        const long long t2 = (mt_routed + mt_shared) * (cfg->H / kTcFeat2);
        const int sms = sm_count();
        tc_grid1 = (int)(t1 < sms ? t1 : sms);
        tc_grid2 = (int)(t2 < sms ? t2 : sms);
    }
    if (err == cudaSuccess) err = mark(2 * MOE_STAGE_GATE_UP);
    if (err == cudaSuccess) err = use_tc ? launch_tc_gemm(p, 1, tc_grid1, s) : launch_experts_w13(p, grid13, s);
    if (err == cudaSuccess) err = mark(2 * MOE_STAGE_GATE_UP + 1);
    if (err == cudaSuccess) err = mark(2 * MOE_STAGE_DOWN);
    if (err == cudaSuccess) err = use_tc ? launch_tc_gemm(p, 2, tc_grid2, s) : launch_experts_w2(p, grid2, s);
    if (err == cudaSuccess) err = mark(2 * MOE_STAGE_DOWN + 1);
    if (err == cudaSuccess) err = mark(2 * MOE_STAGE_COMBINE);
    if (err == cudaSuccess) err = launch_combine(p, s);
    if (err == cudaSuccess) err = mark(2 * MOE_STAGE_COMBINE + 1);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
    if (cfg->flags & MOE_DEBUG_CHECK) {
        unsigned status = 0;
        err = cudaMemcpyAsync(&status, &p.ctrl->status, sizeof status, cudaMemcpyDeviceToHost, s);
        if (err == cudaSuccess) err = cudaStreamSynchronize(s);
        if (err != cudaSuccess) return MOE_ERR_CUDA;
        if (status != 0) return MOE_ERR_DEVICE_CHECK;
    }
    return MOE_OK;
}

size_t moe_stack_workspace_bytes(const moe_cfg_t* cfg, int32_t T, int32_t L) {
    if (validate_stack(cfg, T, L) != MOE_OK) return 0;
    if (T > 0 && stack_fused(*cfg, T, L)) return fused_layout(*cfg, T, L).total;
    return ws_layout(*cfg, T).total;
}

size_t moe_stack_trace_offset(const moe_cfg_t* cfg, int32_t T, int32_t L) {
    if (validate_stack(cfg, T, L) != MOE_OK || T <= 0 || !(cfg->flags & MOE_TRACE) || !stack_fused(*cfg, T, L))
        return 0;
    return fused_layout(*cfg, T, L).trace;
}

int32_t moe_stack_path(const moe_cfg_t* cfg, int32_t T, int32_t L) {
    if (validate_stack(cfg, T, L) != MOE_OK || T <= 0) return 0;
    return stack_fused(*cfg, T, L) ? MOE_PATH_FUSED_STACK : MOE_PATH_PER_LAYER;
}

int moe_stack_forward(const void* x, const moe_stack_weights_t* w, int32_t L, void* outs, int32_t T,
                      const moe_cfg_t* cfg, void* stream) {
    int st = validate_stack(cfg, T, L);
    if (st != MOE_OK) return st;
    if (!x || !w || !outs || !w->router_w || !w->router_bias || !w->w13 || !w->s13 || !w->w2 || !w->s2)
        return MOE_ERR_INVALID_ARG;
    const moe_shared_weights_t& shw = w->shared;
    if (cfg->Is > 0 && (!shw.w13 || !shw.s13 || !shw.w2 || !shw.s2)) return MOE_ERR_INVALID_ARG;
    const void* ptrs[] = {x, outs, w->router_w, w->router_bias, w->w13, w->s13, w->w2, w->s2,
                          cfg->Is > 0 ? shw.w13 : nullptr, cfg->Is > 0 ? shw.s13 : nullptr,
                          cfg->Is > 0 ? shw.w2 : nullptr, cfg->Is > 0 ? shw.s2 : nullptr,
                          cfg->topk_idx_out, cfg->topk_w_out};
    for (const void* ptr : ptrs)
        if (ptr && !aligned(ptr, 16)) return MOE_ERR_INVALID_ARG;
    const size_t H = cfg->H, E = cfg->E, I = cfg->I, Is = cfg->Is;
    const size_t xbytes = (size_t)T * H * 2, obytes = xbytes * L;
    const uintptr_t xa = (uintptr_t)x, oa = (uintptr_t)outs;
    if (T > 0 && xa < oa + obytes && oa < xa + xbytes) return MOE_ERR_INVALID_ARG;
    const size_t need = moe_stack_workspace_bytes(cfg, T, L);
    if (!cfg->workspace || cfg->workspace_bytes < need) return MOE_ERR_WORKSPACE;
    if (!aligned(cfg->workspace, 256)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t TK = (size_t)T * cfg->K;
    if (!stack_fused(*cfg, T, L)) {
        // one moe_layer_forward call per layer, each layer's output the next one's input;
        // a code row of n elements is n/2 bytes (int4) or n bytes (int8)
        const size_t per = (cfg->flags & MOE_WEIGHTS_INT8) ? 1 : 2;
        for (int32_t l = 0; l < L; ++l) {
            moe_cfg_t c = *cfg;
            c.flags &= ~(unsigned)MOE_LOOKAHEAD;
            c.topk_idx_out = cfg->topk_idx_out ? cfg->topk_idx_out + l * TK : nullptr;
            c.topk_w_out = cfg->topk_w_out ? cfg->topk_w_out + l * TK : nullptr;
            c.stage_events = nullptr;
            moe_shared_weights_t sl{};
            if (Is > 0) {
                sl.w13 = shw.w13 + l * 2 * Is * (H / per);
                sl.s13 = shw.s13 + l * 2 * Is;
                sl.w2 = shw.w2 + l * H * (Is / per);
                sl.s2 = shw.s2 + l * H;
            }
            const void* in = l == 0 ? x : static_cast<const char*>(outs) + (size_t)(l - 1) * xbytes;
            void* out = static_cast<char*>(outs) + (size_t)l * xbytes;
            st = moe_layer_forward(in, w->router_w + l * E * H, w->router_bias + l * E, w->w13 + l * E * 2 * I * (H / per),
                                   w->s13 + l * E * 2 * I, w->w2 + l * E * H * (I / per), w->s2 + l * E * H, &sl, out, T,
                                   &c, stream);
            if (st != MOE_OK) return st;
        }
        return MOE_OK;
    }
    const FusedLayout F = fused_layout(*cfg, T, L);
    char* ws = static_cast<char*>(cfg->workspace);
    FArgs a;
    memset(&a, 0, sizeof a);
    a.T = T; a.H = cfg->H; a.E = cfg->E; a.K = cfg->K; a.I = cfg->I; a.Is = cfg->Is; a.L = L;
    a.G = cdiv(T, 8);
    a.NCB = cfg->H / 128;
    a.rows2 = fused_rows2(cfg->H, cfg->E, cfg->K, cfg->I, cfg->Is, T, fused_grid());
    a.nsl_r = slices_of(cfg->I);
    a.nsl_s = cfg->Is > 0 ? slices_of(cfg->Is) : 0;
    a.r13_r = cfg->I / kTaskRows13;
    a.r13_s = cfg->Is / kTaskRows13;
    a.r2_r = (cfg->H / a.rows2) * a.nsl_r;
    a.r2_s = (cfg->H / a.rows2) * a.nsl_s;
    a.scale = cfg->routed_scaling;
    a.topp = cfg->topp;
    a.flags = cfg->flags;
    a.x = static_cast<const __nv_bfloat16*>(x);
    a.outs = static_cast<__nv_bfloat16*>(outs);
    a.rw = w->router_w; a.rb = w->router_bias;
    a.w13 = w->w13; a.s13 = w->s13; a.w2 = w->w2; a.s2 = w->s2;
    if (cfg->Is > 0) {
        a.sh_w13 = shw.w13; a.sh_s13 = shw.s13; a.sh_w2 = shw.w2; a.sh_s2 = shw.s2;
    }
    a.topk_idx = cfg->topk_idx_out;
    a.topk_w = cfg->topk_w_out;
    a.status = reinterpret_cast<unsigned*>(ws + F.ctrl);
    a.abort = reinterpret_cast<int*>(ws + F.ctrl + 4);
    a.grp_cnt = reinterpret_cast<int*>(ws + F.grp_cnt);
    a.groups_done = reinterpret_cast<int*>(ws + F.groups_done);
    a.down_done = reinterpret_cast<int*>(ws + F.down_done);
    a.ready = reinterpret_cast<int*>(ws + F.ready);
    a.pred_bits = reinterpret_cast<unsigned*>(ws + F.pred_bits);
    a.trace = (cfg->flags & MOE_TRACE) ? reinterpret_cast<unsigned long long*>(ws + F.trace) : nullptr;
    a.lp = reinterpret_cast<float*>(ws + F.lp);
    a.lpn = reinterpret_cast<float*>(ws + F.lpn);
    a.idx = reinterpret_cast<int32_t*>(ws + F.idx);
    a.wts = reinterpret_cast<float*>(ws + F.wts);
    a.xq = reinterpret_cast<int8_t*>(ws + F.xq);
    a.xs = reinterpret_cast<float*>(ws + F.xs);
    a.h32_r = reinterpret_cast<float*>(ws + F.h32_r);
    a.h32_s = reinterpret_cast<float*>(ws + F.h32_s);
    a.hmax_r = reinterpret_cast<float*>(ws + F.hmax_r);
    a.hmax_s = reinterpret_cast<float*>(ws + F.hmax_s);
    a.y = reinterpret_cast<float*>(ws + F.y);
    if (fused_grid() > kMaxGridF && (cfg->flags & MOE_TRACE)) return MOE_ERR_UNSUPPORTED;
    cudaError_t err = cudaSuccess;
    if (cfg->flags & MOE_DEBUG_POISON)  // every byte a kernel reads must have been written first
        err = cudaMemsetAsync(ws + F.counters_end, 0xFF, F.total - F.counters_end, s);
    if (err == cudaSuccess) err = cudaMemsetAsync(ws, 0, F.counters_end, s);
    if (err == cudaSuccess && (cfg->flags & MOE_TRACE))  // stamps a CTA does not take stay 0
        err = cudaMemsetAsync(ws + F.trace, 0, F.total - F.trace, s);
    if (err == cudaSuccess) err = launch_decode_stack(a, fused_grid(), s);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
    if (cfg->flags & MOE_DEBUG_CHECK) {
        unsigned status = 0;
        err = cudaMemcpyAsync(&status, a.status, sizeof status, cudaMemcpyDeviceToHost, s);
        if (err == cudaSuccess) err = cudaStreamSynchronize(s);
        if (err != cudaSuccess) return MOE_ERR_CUDA;
        if (status != 0) return MOE_ERR_DEVICE_CHECK;
    }
    return MOE_OK;
}

}  // extern "C"
