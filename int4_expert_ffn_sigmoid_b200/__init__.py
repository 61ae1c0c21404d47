"""B200 (sm_100a) forward pass of one int4 expert-FFN MoE layer with a
sigmoid+bias router: the Python binding of ``libmoe_int4.so``.

This module only marshals arguments: every step of the layer (router,
selection, bucketing, expert FFNs, shared expert, combine) runs in the
library's CUDA kernels.  torch provides device memory and streams.  There is
no fallback: if the library is missing, importing the binding raises.

The C ABI is declared in ``include/moe_int4.h``; the names here mirror it.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "MoeError", "moe_cfg_t", "moe_shared_weights_t", "lib", "EXPORTED_SYMBOLS",
    "MOE_ADD_RESIDUAL", "MOE_DEBUG_CHECK", "MOE_FORCE_DECODE", "MOE_FORCE_PREFILL", "MOE_OUT_F32",
    "MOE_TEST_STALL", "MOE_LOOKAHEAD", "MOE_TEST_BAD_INDEX", "MOE_TRACE", "MOE_DEBUG_POISON", "MOE_STACK_FUSED",
    "MOE_WEIGHTS_INT8", "weight_flags",
    "MOE_DEVSTAT_TIMEOUT", "MOE_DEVSTAT_BAD_EXPERT", "device_status", "stack_trace",
    "moe_stack_weights_t", "stack_workspace_bytes", "stack_path", "stack_forward", "stack_layers",
    "MOE_PATH_FUSED_STACK", "MOE_PATH_PER_LAYER",
    "workspace_bytes", "workspace_bytes_upto", "layer_forward", "MoELayer", "decode_max_tokens", "kernel_launches", "layer_path",
    "MOE_PATH_SMALL_BATCH", "MOE_PATH_TENSOR_CORE", "MOE_PATH_LARGE_STREAMING", "LIB_PATH",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_int4.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE_CHECK = 5

MOE_ADD_RESIDUAL = 1 << 0
MOE_DEBUG_CHECK = 1 << 1
MOE_FORCE_DECODE = 1 << 2
MOE_FORCE_PREFILL = 1 << 3
MOE_OUT_F32 = 1 << 4
MOE_LOOKAHEAD = 1 << 5
MOE_TEST_STALL = 1 << 6
MOE_TEST_BAD_INDEX = 1 << 7
MOE_TRACE = 1 << 8
MOE_DEBUG_POISON = 1 << 9
MOE_STACK_FUSED = 1 << 10
MOE_WEIGHTS_INT8 = 1 << 11
TRACE_SLOTS = 16  # MOE_TRACE stamps per (CTA, layer)
# device status word (the first 4 bytes of the workspace)
MOE_DEVSTAT_BAD_EXPERT = 1 << 0
MOE_DEVSTAT_BAD_SLOT = 1 << 1
MOE_DEVSTAT_BAD_COUNT = 1 << 2
MOE_DEVSTAT_BAD_TASK = 1 << 3
MOE_DEVSTAT_TIMEOUT = 1 << 4
# kernel sequences (moe_layer_path)
MOE_PATH_SMALL_BATCH = 1
MOE_PATH_TENSOR_CORE = 2
MOE_PATH_LARGE_STREAMING = 3
MOE_PATH_FUSED_STACK = 4
MOE_PATH_PER_LAYER = 5

MOE_STAGE_ROUTE, MOE_STAGE_GATE_UP, MOE_STAGE_DOWN, MOE_STAGE_COMBINE = range(4)
MOE_NUM_STAGES = 4
STAGE_NAMES = ("route", "gate_up", "down", "combine")

# Every function declared in include/moe_int4.h.
EXPORTED_SYMBOLS = ("moe_layer_workspace_bytes", "moe_layer_forward", "moe_status_str",
                    "moe_abi_version", "moe_decode_max_tokens", "moe_layer_forward_static_ws",
                    "moe_layer_kernel_launches", "moe_layer_path", "moe_layer_workspace_bytes_upto",
                    "moe_stack_workspace_bytes", "moe_stack_path", "moe_stack_forward", "moe_stack_trace_offset")

# Scratch capacity of moe_layer_forward_static_ws (the entry point for callers
# that cannot allocate device memory).
MOE_STATIC_WORKSPACE_BYTES = 32 << 20


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str = "moe_layer_forward"):
        self.status = status
        super().__init__(f"{what} failed: {status_str(status)} ({status})")


class moe_cfg_t(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("H", ctypes.c_int32), ("E", ctypes.c_int32),
                ("K", ctypes.c_int32), ("I", ctypes.c_int32), ("Is", ctypes.c_int32),
                ("routed_scaling", ctypes.c_float), ("flags", ctypes.c_uint32),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("topk_idx_out", ctypes.c_void_p), ("topk_w_out", ctypes.c_void_p),
                ("stage_events", ctypes.c_void_p), ("topp", ctypes.c_float)]


class moe_shared_weights_t(ctypes.Structure):
    _fields_ = [("w13", ctypes.c_void_p), ("s13", ctypes.c_void_p),
                ("w2", ctypes.c_void_p), ("s2", ctypes.c_void_p)]


class moe_stack_weights_t(ctypes.Structure):
    _fields_ = [("router_w", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
                ("w13", ctypes.c_void_p), ("s13", ctypes.c_void_p),
                ("w2", ctypes.c_void_p), ("s2", ctypes.c_void_p),
                ("shared", moe_shared_weights_t)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python int4_expert_ffn_sigmoid_b200/_build.py`")
    L = ctypes.CDLL(LIB_PATH)
    vp = ctypes.c_void_p
    L.moe_layer_workspace_bytes.argtypes = [ctypes.POINTER(moe_cfg_t), ctypes.c_int32]
    L.moe_layer_workspace_bytes.restype = ctypes.c_size_t
    L.moe_layer_workspace_bytes_upto.argtypes = [ctypes.POINTER(moe_cfg_t), ctypes.c_int32]
    L.moe_layer_workspace_bytes_upto.restype = ctypes.c_size_t
    L.moe_layer_forward.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.POINTER(moe_shared_weights_t),
                                    vp, ctypes.c_int32, ctypes.POINTER(moe_cfg_t), vp]
    L.moe_layer_forward.restype = ctypes.c_int
    L.moe_layer_forward_static_ws.argtypes = L.moe_layer_forward.argtypes
    L.moe_layer_forward_static_ws.restype = ctypes.c_int
    L.moe_status_str.argtypes = [ctypes.c_int]
    L.moe_status_str.restype = ctypes.c_char_p
    L.moe_abi_version.argtypes = []
    L.moe_abi_version.restype = ctypes.c_int
    L.moe_decode_max_tokens.argtypes = []
    L.moe_decode_max_tokens.restype = ctypes.c_int32
    L.moe_layer_kernel_launches.argtypes = [ctypes.POINTER(moe_cfg_t), ctypes.c_int32]
    L.moe_layer_kernel_launches.restype = ctypes.c_int32
    L.moe_layer_path.argtypes = [ctypes.POINTER(moe_cfg_t), ctypes.c_int32]
    L.moe_layer_path.restype = ctypes.c_int32
    L.moe_stack_workspace_bytes.argtypes = [ctypes.POINTER(moe_cfg_t), ctypes.c_int32, ctypes.c_int32]
    L.moe_stack_workspace_bytes.restype = ctypes.c_size_t
    L.moe_stack_path.argtypes = [ctypes.POINTER(moe_cfg_t), ctypes.c_int32, ctypes.c_int32]
    L.moe_stack_path.restype = ctypes.c_int32
    L.moe_stack_forward.argtypes = [vp, ctypes.POINTER(moe_stack_weights_t), ctypes.c_int32, vp, ctypes.c_int32,
                                    ctypes.POINTER(moe_cfg_t), vp]
    L.moe_stack_forward.restype = ctypes.c_int
    L.moe_stack_trace_offset.argtypes = [ctypes.POINTER(moe_cfg_t), ctypes.c_int32, ctypes.c_int32]
    L.moe_stack_trace_offset.restype = ctypes.c_size_t
    if L.moe_abi_version() != 2:
        raise ImportError("libmoe_int4.so ABI version mismatch")
    return L


lib = _load()


def status_str(status: int) -> str:
    return lib.moe_status_str(int(status)).decode()


def decode_max_tokens() -> int:
    return int(lib.moe_decode_max_tokens())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def make_cfg(shape, flags: int = 0, workspace: Optional[torch.Tensor] = None,
             topk_idx: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None,
             stage_events=None, topp: float = 0.0) -> moe_cfg_t:
    c = moe_cfg_t()
    c.topp = float(topp)
    c.struct_size = ctypes.sizeof(moe_cfg_t)
    c.H, c.E, c.K, c.I, c.Is = shape.H, shape.E, shape.K, shape.I, shape.Is
    c.routed_scaling = float(shape.routed_scaling)
    c.flags = int(flags)
    if workspace is not None:
        c.workspace = workspace.data_ptr()
        c.workspace_bytes = workspace.numel() * workspace.element_size()
    c.topk_idx_out = None if topk_idx is None else topk_idx.data_ptr()
    c.topk_w_out = None if topk_w is None else topk_w.data_ptr()
    if stage_events is not None:
        if len(stage_events) != 2 * MOE_NUM_STAGES:
            raise ValueError(f"stage_events needs {2 * MOE_NUM_STAGES} events")
        arr = (ctypes.c_void_p * len(stage_events))(*[int(e.cuda_event) for e in stage_events])
        c._events_keepalive = arr
        c.stage_events = ctypes.cast(arr, ctypes.c_void_p).value
    return c


def kernel_launches(shape, T: int, flags: int = 0) -> int:
    """Kernels one layer_forward call launches for T tokens (0: invalid)."""
    c = make_cfg(shape, flags)
    return int(lib.moe_layer_kernel_launches(ctypes.byref(c), int(T)))


def layer_path(shape, T: int, flags: int = 0) -> int:
    """MOE_PATH_* of a layer_forward call for T tokens (0: invalid)."""
    c = make_cfg(shape, flags)
    return int(lib.moe_layer_path(ctypes.byref(c), int(T)))


def workspace_bytes(shape, T: int, flags: int = 0) -> int:
    c = make_cfg(shape, flags)
    return int(lib.moe_layer_workspace_bytes(ctypes.byref(c), int(T)))


def workspace_bytes_upto(shape, T: int, flags: int = 0) -> int:
    c = make_cfg(shape, flags)
    return int(lib.moe_layer_workspace_bytes_upto(ctypes.byref(c), int(T)))


def new_workspace(shape, T: int, device, flags: int = 0) -> torch.Tensor:
    """A workspace for any call of up to T tokens under `flags`."""
    n = workspace_bytes_upto(shape, T, flags)
    if n == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED, "moe_layer_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def _check_dev(name, t, dtype, shape=None):
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor, got {t.dtype} on {t.device}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


def weight_flags(layer: dict, shape) -> int:
    """MOE_WEIGHTS_INT8 when ``layer``'s expert codes are one byte per element
    (w13 rows of H bytes), 0 for packed int4 (H/2 bytes)."""
    n = layer["w13"].shape[-1]
    if n == shape.H:
        return MOE_WEIGHTS_INT8
    if 2 * n == shape.H:
        return 0
    raise ValueError(f"w13 rows of {n} bytes fit neither int4 nor int8 codes of H={shape.H}")


def layer_forward(x: torch.Tensor, layer: dict, shape, out: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, flags: int = 0,
                  topk_idx: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None, stage_events=None, topp: float = 0.0) -> torch.Tensor:
    """Call ``moe_layer_forward`` on torch tensors (see include/moe_int4.h).

    ``layer`` holds router_w, router_bias, w13, s13, w2, s2 and, when
    shape.Is > 0, sh_w13, sh_s13, sh_w2, sh_s2 (the layout of
    ``workloads.make_layer``).  With int8 expert weights (one byte per element)
    ``flags`` must hold MOE_WEIGHTS_INT8.  Returns ``out`` (bf16 [T, H]).  ``stage_events``:
    optional sequence of 2*MOE_NUM_STAGES ``torch.cuda.Event`` already recorded
    once (so that they exist); the library records them around each stage."""
    T = x.shape[0]
    H, E, I, Is = shape.H, shape.E, shape.I, shape.Is
    per = 1 if flags & MOE_WEIGHTS_INT8 else 2  # code elements per byte
    _check_dev("x", x, torch.bfloat16, (T, H))
    _check_dev("router_w", layer["router_w"], torch.float32, (E, H))
    _check_dev("router_bias", layer["router_bias"], torch.float32, (E,))
    _check_dev("w13", layer["w13"], torch.uint8, (E, 2 * I, H // per))
    _check_dev("s13", layer["s13"], torch.float32, (E, 2 * I))
    _check_dev("w2", layer["w2"], torch.uint8, (E, H, I // per))
    _check_dev("s2", layer["s2"], torch.float32, (E, H))
    sh = moe_shared_weights_t()
    if Is > 0:
        _check_dev("sh_w13", layer["sh_w13"], torch.uint8, (2 * Is, H // per))
        _check_dev("sh_s13", layer["sh_s13"], torch.float32, (2 * Is,))
        _check_dev("sh_w2", layer["sh_w2"], torch.uint8, (H, Is // per))
        _check_dev("sh_s2", layer["sh_s2"], torch.float32, (H,))
        sh.w13, sh.s13 = layer["sh_w13"].data_ptr(), layer["sh_s13"].data_ptr()
        sh.w2, sh.s2 = layer["sh_w2"].data_ptr(), layer["sh_s2"].data_ptr()
    odt = torch.float32 if flags & MOE_OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty((T, H), dtype=odt, device=x.device)
    _check_dev("out", out, odt, (T, H))
    if workspace is None:
        workspace = new_workspace(shape, T, x.device, flags)
    if topk_idx is not None:
        _check_dev("topk_idx", topk_idx, torch.int32, (T, shape.K))
    if topk_w is not None:
        _check_dev("topk_w", topk_w, torch.float32, (T, shape.K))
    cfg = make_cfg(shape, flags, workspace, topk_idx, topk_w, stage_events, topp)
    s = stream if stream is not None else torch.cuda.current_stream(x.device)
    st = lib.moe_layer_forward(_ptr(x), _ptr(layer["router_w"]), _ptr(layer["router_bias"]),
                               _ptr(layer["w13"]), _ptr(layer["s13"]), _ptr(layer["w2"]),
                               _ptr(layer["s2"]), ctypes.byref(sh), _ptr(out), int(T),
                               ctypes.byref(cfg), ctypes.c_void_p(s.cuda_stream))
    if st != MOE_OK:
        raise MoeError(st)
    return out


STACK_KEYS = ("router_w", "router_bias", "w13", "s13", "w2", "s2", "sh_w13", "sh_s13", "sh_w2", "sh_s2")


def stack_layers(layers) -> dict:
    """Stacks per-layer weight dicts (``workloads.make_layer``'s layout) along a
    new leading layer dimension: the layout moe_stack_forward reads."""
    keys = [k for k in STACK_KEYS if k in layers[0]]
    return {k: torch.stack([l[k] for l in layers]).contiguous() for k in keys}


def stack_workspace_bytes(shape, T: int, L: int, flags: int = 0) -> int:
    c = make_cfg(shape, flags)
    return int(lib.moe_stack_workspace_bytes(ctypes.byref(c), int(T), int(L)))


def stack_path(shape, T: int, L: int, flags: int = 0) -> int:
    """MOE_PATH_FUSED_STACK or MOE_PATH_PER_LAYER of a stack_forward call (0: invalid)."""
    c = make_cfg(shape, flags)
    return int(lib.moe_stack_path(ctypes.byref(c), int(T), int(L)))


def stack_forward(x: torch.Tensor, stacked: dict, shape, outs: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, flags: int = 0,
                  topk_idx: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None, topp: float = 0.0) -> torch.Tensor:
    """Call ``moe_stack_forward`` on torch tensors: ``stacked`` holds the
    weights of L layers stacked along dimension 0 (see ``stack_layers``).
    Returns ``outs`` (bf16 [L, T, H]; outs[l] is layer l's output).
    ``topk_idx`` / ``topk_w``: optional [L, T, K]."""
    T = x.shape[0]
    H, E, K, I, Is = shape.H, shape.E, shape.K, shape.I, shape.Is
    L = stacked["router_w"].shape[0]
    per = 1 if flags & MOE_WEIGHTS_INT8 else 2  # code elements per byte
    _check_dev("x", x, torch.bfloat16, (T, H))
    _check_dev("router_w", stacked["router_w"], torch.float32, (L, E, H))
    _check_dev("router_bias", stacked["router_bias"], torch.float32, (L, E))
    _check_dev("w13", stacked["w13"], torch.uint8, (L, E, 2 * I, H // per))
    _check_dev("s13", stacked["s13"], torch.float32, (L, E, 2 * I))
    _check_dev("w2", stacked["w2"], torch.uint8, (L, E, H, I // per))
    _check_dev("s2", stacked["s2"], torch.float32, (L, E, H))
    w = moe_stack_weights_t()
    w.router_w, w.router_bias = stacked["router_w"].data_ptr(), stacked["router_bias"].data_ptr()
    w.w13, w.s13 = stacked["w13"].data_ptr(), stacked["s13"].data_ptr()
    w.w2, w.s2 = stacked["w2"].data_ptr(), stacked["s2"].data_ptr()
    if Is > 0:
        _check_dev("sh_w13", stacked["sh_w13"], torch.uint8, (L, 2 * Is, H // per))
        _check_dev("sh_s13", stacked["sh_s13"], torch.float32, (L, 2 * Is))
        _check_dev("sh_w2", stacked["sh_w2"], torch.uint8, (L, H, Is // per))
        _check_dev("sh_s2", stacked["sh_s2"], torch.float32, (L, H))
        w.shared.w13, w.shared.s13 = stacked["sh_w13"].data_ptr(), stacked["sh_s13"].data_ptr()
        w.shared.w2, w.shared.s2 = stacked["sh_w2"].data_ptr(), stacked["sh_s2"].data_ptr()
    if outs is None:
        outs = torch.empty((L, T, H), dtype=torch.bfloat16, device=x.device)
    _check_dev("outs", outs, torch.bfloat16, (L, T, H))
    if workspace is None:
        n = stack_workspace_bytes(shape, T, L, flags)
        if n == 0:
            raise MoeError(MOE_ERR_UNSUPPORTED, "moe_stack_workspace_bytes")
        workspace = torch.empty(n, dtype=torch.uint8, device=x.device)
    if topk_idx is not None:
        _check_dev("topk_idx", topk_idx, torch.int32, (L, T, K))
    if topk_w is not None:
        _check_dev("topk_w", topk_w, torch.float32, (L, T, K))
    cfg = make_cfg(shape, flags, workspace, topk_idx, topk_w, topp=topp)
    s = stream if stream is not None else torch.cuda.current_stream(x.device)
    st = lib.moe_stack_forward(_ptr(x), ctypes.byref(w), int(L), _ptr(outs), int(T), ctypes.byref(cfg),
                               ctypes.c_void_p(s.cuda_stream))
    if st != MOE_OK:
        raise MoeError(st, "moe_stack_forward")
    return outs


def stack_trace(workspace: torch.Tensor, shape, T: int, L: int, flags: int, grid: int) -> torch.Tensor:
    """The MOE_TRACE stamps of the last fused call on ``workspace``: int64
    [grid, L + 1, 16] nanosecond timer values, 0 where a CTA took no stamp
    (see moe_stack_trace_offset).  Synchronises the stream."""
    c = make_cfg(shape, flags | MOE_TRACE)
    off = int(lib.moe_stack_trace_offset(ctypes.byref(c), int(T), int(L)))
    if off == 0:
        raise ValueError("this call does not trace (not the fused kernel, or no MOE_TRACE)")
    n = grid * (L + 1) * TRACE_SLOTS
    return workspace[off:off + 8 * n].view(torch.int64).view(grid, L + 1, TRACE_SLOTS).cpu()


def device_status(workspace: torch.Tensor) -> int:
    """The device status word (MOE_DEVSTAT_* bits) that the last call on
    ``workspace`` left in its first 4 bytes (synchronises the stream)."""
    return int(workspace[:4].view(torch.int32).item()) & 0xFFFFFFFF


class MoELayer:
    """One layer's device weights plus a workspace sized for every call of up
    to ``max_tokens`` tokens under any per-call flags (the kernel sequence,
    and so the workspace, depends on MOE_FORCE_DECODE / MOE_FORCE_PREFILL).
    The code width of the expert weights (int4 or int8) is read from their
    shapes and its flag added to every call."""

    def __init__(self, layer: dict, shape, max_tokens: int, device=None):
        self.layer = layer
        self.shape = shape
        self.device = torch.device(device) if device is not None else layer["w13"].device
        self.max_tokens = int(max_tokens)
        self.weight_flags = weight_flags(layer, shape)
        n = max(workspace_bytes_upto(shape, self.max_tokens, f | self.weight_flags)
                for f in (0, MOE_FORCE_DECODE, MOE_FORCE_PREFILL))
        if n == 0:
            raise MoeError(MOE_ERR_UNSUPPORTED, "moe_layer_workspace_bytes")
        self.workspace = torch.empty(n, dtype=torch.uint8, device=self.device)

    def __call__(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, residual: bool = False,
                 flags: int = 0, topk_idx=None, topk_w=None, stage_events=None) -> torch.Tensor:
        if x.shape[0] > self.max_tokens:
            raise ValueError(f"T={x.shape[0]} exceeds max_tokens={self.max_tokens}")
        f = flags | self.weight_flags | (MOE_ADD_RESIDUAL if residual else 0)
        return layer_forward(x, self.layer, self.shape, out=out, workspace=self.workspace, flags=f,
                             topk_idx=topk_idx, topk_w=topk_w, stage_events=stage_events)
