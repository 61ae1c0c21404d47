"""Dense-masked formulation of the MoE layer, in NumPy float64, for tiny shapes.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

A second, structurally different algorithm used to pin the C oracle: the
weights are dequantised in full, *every* expert is applied to *every* token
with batched ``einsum`` contractions, and the routing enters only as a dense
[T, E] weight matrix that is zero outside each token's selected experts.  The
C oracle instead routes first and evaluates only the selected experts, one
token at a time.  Both follow the formulas stated in ``moe_oracle.c``'s header
(sigmoid+bias router of the Colibri-Nano model card "Architecture" and the
colibri README "What's implemented"; per-row int4 with f32 scales of the
nanocolibri-engine README "Converting a checkpoint yourself").
"""
from __future__ import annotations

import numpy as np

from . import _np, bf16_bits_to_f64


def decode_int4(packed: np.ndarray) -> np.ndarray:
    """Packed bytes [..., n/2] -> int codes [..., n] (low nibble = even element)."""
    p = packed.astype(np.int16)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    codes = np.empty(packed.shape[:-1] + (2 * packed.shape[-1],), np.int16)
    codes[..., 0::2] = np.where(lo >= 8, lo - 16, lo)
    codes[..., 1::2] = np.where(hi >= 8, hi - 16, hi)
    return codes


def decode_codes(raw: np.ndarray, n: int) -> np.ndarray:
    """Expert weight bytes [..., n/2] (packed int4) or [..., n] (int8, byte j
    = element j, two's complement) -> int codes [..., n]."""
    if raw.shape[-1] * 2 == n:
        return decode_int4(raw)
    if raw.shape[-1] == n:
        return raw.view(np.int8).astype(np.int16)
    raise ValueError(f"rows of {raw.shape[-1]} bytes fit neither int4 nor int8 codes of {n} elements")


def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def topp_keep(s_sel: np.ndarray, e_sel: np.ndarray, p: float) -> np.ndarray:
    """Adaptive expert top-p over one token's K picks (scores s_sel, experts
    e_sel): a boolean mask of the picks kept -- the fewest of the
    highest-scoring ones (ties: lower expert index) whose scores reach p of the
    K picks' total.  Written as a search over prefix lengths: the smallest n
    such that the n best picks carry at least p of the total (a pick is needed
    while the mass before it is still below p)."""
    order = sorted(range(len(s_sel)), key=lambda k: (-s_sel[k], e_sel[k]))
    total = float(np.sum(s_sel))
    keep = np.zeros(len(s_sel), bool)
    for n in range(1, len(order) + 1):
        if sum(s_sel[order[j]] for j in range(n - 1)) >= p * total:
            break
        keep[order[n - 1]] = True
    return keep


def routing_matrix(x: np.ndarray, W: np.ndarray, bias: np.ndarray, K: int, scale: float, forced=None,
                   topp: float = 0.0):
    """Dense routing weights R [T,E]: R[t,e] = w[t,k] if e = e_k, else 0.

    ``forced`` [T,K] (optional) replaces the selection by the given experts
    (-1 entries: none); their weights still come from the unbiased scores,
    normalised over the forced set.  ``topp`` (0 < p < 1): the adaptive expert
    top-p drops picks (``topp_keep``) and the kept ones are normalised over the
    kept set."""
    s = _sigmoid(x @ W.T.astype(np.float64))
    key = s + bias.astype(np.float64)[None, :]
    key = np.where(np.isnan(key), -np.inf, key)
    T, E = s.shape
    R = np.zeros((T, E))
    for t in range(T):
        if forced is None:
            order = np.argsort(-key[t], kind="stable")  # equal keys keep index order
            sel = order[:K]
            if 0.0 < topp < 1.0:
                sel = sel[topp_keep(s[t, sel], sel, topp)]
        else:
            sel = np.asarray([e for e in forced[t] if e >= 0], np.int64)
        R[t, sel] = scale * s[t, sel] / s[t, sel].sum()
    return R


def moe_dense(x, layer: dict, shape, residual: bool = False, forced=None, topp: float = 0.0):
    """Layer output [T,H] in float64.  x: bf16 [T,H] (torch) or bf16 bits.
    ``forced`` [T,K]: evaluate these experts instead of the router's choice.
    ``topp``: the adaptive expert top-p (0 = off)."""
    xf = bf16_bits_to_f64(x)
    E, K, I, Is = shape.E, shape.K, shape.I, shape.Is
    R = routing_matrix(xf, _np(layer["router_w"], np.float64), _np(layer["router_bias"], np.float64),
                       K, shape.routed_scaling, forced, topp)
    H = xf.shape[1]
    W13 = decode_codes(_np(layer["w13"], np.uint8), H) * _np(layer["s13"], np.float64)[..., None]
    W2 = decode_codes(_np(layer["w2"], np.uint8), I) * _np(layer["s2"], np.float64)[..., None]
    G = np.einsum("th,eih->tei", xf, W13[:, :I])
    U = np.einsum("th,eih->tei", xf, W13[:, I:])
    Hh = G * _sigmoid(G) * U
    Y = np.einsum("tei,eji->tej", Hh, W2)
    out = np.einsum("te,tej->tj", R, Y)
    if Is > 0:
        S13 = decode_codes(_np(layer["sh_w13"], np.uint8), H) * _np(layer["sh_s13"], np.float64)[:, None]
        S2 = decode_codes(_np(layer["sh_w2"], np.uint8), Is) * _np(layer["sh_s2"], np.float64)[:, None]
        g = xf @ S13[:Is].T
        u = xf @ S13[Is:].T
        out = out + (g * _sigmoid(g) * u) @ S2.T
    if residual:
        out = out + xf
    return out, R
