"""CPU oracle for the int4 expert-FFN MoE layer forward.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(the CUDA library and its binding) never imports it, and this package never
imports the product.

Two independent formulations live here:
  * ``moe_oracle.c`` (loaded through ctypes): the plain per-token definition
    in double precision, dequantising each int4 row as it is used;
  * ``dense_masked.py``: a dense NumPy formulation for tiny shapes (every
    expert applied to every token, times a 0/1 routing mask), used to pin the
    C oracle.

Which page passage each step follows is stated in the header of
``moe_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_i32p = ctypes.POINTER(ctypes.c_int32)
_f64p = ctypes.POINTER(ctypes.c_double)
_f32p = ctypes.POINTER(ctypes.c_float)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, -O2, no FMA contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_unpack_int4.argtypes = [_u8p, ctypes.c_int64, _i32p]
            lib.oracle_route.argtypes = [_u16p, _f32p, _f32p, ctypes.c_int32, ctypes.c_int32,
                                         ctypes.c_int32, ctypes.c_int32, ctypes.c_double, ctypes.c_double,
                                         _f64p, _f64p, _i32p, _f64p, _f64p, _f64p]
            lib.oracle_select_topk.argtypes = [_f64p, _f32p, ctypes.c_int32, ctypes.c_int32,
                                               ctypes.c_int32, _i32p, _f64p]
            lib.oracle_expert_ffn.argtypes = [_f64p, ctypes.c_int32, ctypes.c_int32, _u8p, _f32p,
                                              _u8p, _f32p, ctypes.c_int32, _f64p, _f64p]
            lib.oracle_moe_tokens.argtypes = (
                [_u16p] + [ctypes.c_int32] * 6 + [ctypes.c_double, ctypes.c_double, ctypes.c_int32]
                + [_f32p, _f32p, _u8p, _f32p, _u8p, _f32p, _u8p, _f32p, _u8p, _f32p, ctypes.c_int32]
                + [_i32p, ctypes.c_int32, _i32p, _f64p, _i32p, _f64p, _f64p])
            for fn in ("oracle_unpack_int4", "oracle_route", "oracle_select_topk",
                       "oracle_expert_ffn", "oracle_moe_tokens"):
                getattr(lib, fn).restype = ctypes.c_int
            _lib = lib
    return _lib


def _np(a, dtype):
    """torch tensor or array-like -> C-contiguous numpy array of ``dtype``."""
    if a is None:
        return None
    if hasattr(a, "detach"):
        import torch
        t = a.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            a = t.view(torch.int16).numpy().view(np.uint16)
        else:
            a = t.numpy()
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a, ctype):
    return None if a is None else a.ctypes.data_as(ctype)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"{what}: oracle returned {rc}")


def unpack_int4(row, n: int) -> np.ndarray:
    r = _np(row, np.uint8)
    out = np.empty(n, np.int32)
    _check(_load().oracle_unpack_int4(_ptr(r, _u8p), n, _ptr(out, _i32p)), "unpack_int4")
    return out


def route(x, router_w, router_bias, K: int, scale: float, topp: float = 0.0) -> dict:
    """Router of every token.  x: bf16 [T,H] (torch) or uint16 bf16 bits.
    topp: 0 = plain top-K, 0 < topp < 1 = adaptive expert top-p (dropped picks
    are -1, after the kept ones; ``topp_margin`` tells how close each token's
    top-p decision came to going the other way, relative to its score sum)."""
    xb = _np(x, np.uint16)
    W = _np(router_w, np.float32)
    b = _np(router_bias, np.float32)
    T, H = xb.shape
    E = W.shape[0]
    logits = np.empty((T, E)); scores = np.empty((T, E))
    idx = np.empty((T, K), np.int32); w = np.empty((T, K)); margin = np.empty(T); pm = np.empty(T)
    _check(_load().oracle_route(_ptr(xb, _u16p), _ptr(W, _f32p), _ptr(b, _f32p), T, H, E, K,
                                float(scale), float(topp), _ptr(logits, _f64p), _ptr(scores, _f64p),
                                _ptr(idx, _i32p), _ptr(w, _f64p), _ptr(margin, _f64p), _ptr(pm, _f64p)),
           "route")
    return dict(logits=logits, scores=scores, idx=idx, weights=w, margin=margin, topp_margin=pm)


def select_topk(scores, bias, K: int):
    """Top-K of scores + bias per token.  Returns (idx [T,K], margin [T])."""
    sc = _np(scores, np.float64)
    b = _np(bias, np.float32)
    T, E = sc.shape
    idx = np.empty((T, K), np.int32); margin = np.empty(T)
    _check(_load().oracle_select_topk(_ptr(sc, _f64p), _ptr(b, _f32p), T, E, K, _ptr(idx, _i32p),
                                      _ptr(margin, _f64p)), "select_topk")
    return idx, margin


def weight_bits(w13, H: int) -> int:
    """Code width of expert weights from their row bytes: H/2 (packed int4) or H (int8)."""
    n = _np(w13, np.uint8).shape[-1]
    if n * 2 == H:
        return 4
    if n == H:
        return 8
    raise ValueError(f"expert rows of {n} bytes fit neither int4 nor int8 codes of {H} elements")


def expert_ffn(xvec, w13, s13, w2, s2):
    """One expert on one token (x given as float64 [H]).  Returns (h, y).
    The code width (int4 or int8) follows from the rows' byte counts."""
    xv = _np(xvec, np.float64)
    a13 = _np(w13, np.uint8); a2 = _np(w2, np.uint8)
    f13 = _np(s13, np.float32); f2 = _np(s2, np.float32)
    H = xv.shape[0]
    I = f13.shape[0] // 2
    wb = weight_bits(a13, H)
    h = np.empty(I); y = np.empty(H)
    _check(_load().oracle_expert_ffn(_ptr(xv, _f64p), H, I, _ptr(a13, _u8p), _ptr(f13, _f32p),
                                     _ptr(a2, _u8p), _ptr(f2, _f32p), wb, _ptr(h, _f64p),
                                     _ptr(y, _f64p)), "expert_ffn")
    return h, y


def moe_tokens(x, layer: dict, shape, residual: bool = False, tokens=None,
               idx_override=None, topp: float = 0.0) -> dict:
    """Layer output (float64) for ``tokens`` (default: all tokens).

    ``layer`` is the dict produced by ``workloads.make_layer``; ``shape`` a
    ``workloads.LayerShape``.  ``idx_override`` [n,K] evaluates the given
    experts instead of the router's choice (with ``topp``, -1 entries are
    dropped picks).  ``topp``: 0 = plain top-K, else the adaptive top-p.
    """
    xb = _np(x, np.uint16)
    T, H = xb.shape
    E, K, I, Is = shape.E, shape.K, shape.I, shape.Is
    tok = None if tokens is None else _np(tokens, np.int32).reshape(-1)
    n = T if tok is None else tok.shape[0]
    ov = None if idx_override is None else _np(idx_override, np.int32).reshape(n, K)
    arrs = dict(
        rw=_np(layer["router_w"], np.float32), rb=_np(layer["router_bias"], np.float32),
        w13=_np(layer["w13"], np.uint8), s13=_np(layer["s13"], np.float32),
        w2=_np(layer["w2"], np.uint8), s2=_np(layer["s2"], np.float32))
    if Is > 0:
        arrs.update(sw13=_np(layer["sh_w13"], np.uint8), ss13=_np(layer["sh_s13"], np.float32),
                    sw2=_np(layer["sh_w2"], np.uint8), ss2=_np(layer["sh_s2"], np.float32))
    wb = weight_bits(arrs["w13"], H)
    out = np.empty((n, H)); idx = np.empty((n, K), np.int32); w = np.empty((n, K)); m = np.empty(n)
    _check(_load().oracle_moe_tokens(
        _ptr(xb, _u16p), T, H, E, K, I, Is, float(shape.routed_scaling), float(topp), int(bool(residual)),
        _ptr(arrs["rw"], _f32p), _ptr(arrs["rb"], _f32p), _ptr(arrs["w13"], _u8p),
        _ptr(arrs["s13"], _f32p), _ptr(arrs["w2"], _u8p), _ptr(arrs["s2"], _f32p),
        _ptr(arrs.get("sw13"), _u8p), _ptr(arrs.get("ss13"), _f32p),
        _ptr(arrs.get("sw2"), _u8p), _ptr(arrs.get("ss2"), _f32p), wb,
        _ptr(tok, _i32p), n, _ptr(ov, _i32p), _ptr(out, _f64p), _ptr(idx, _i32p),
        _ptr(w, _f64p), _ptr(m, _f64p)), "moe_tokens")
    return dict(out=out, idx=idx, weights=w, margin=m)


def bf16_bits_to_f64(x) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly."""
    b = _np(x, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
