"""Comparison of the CUDA path with the CPU oracle (helpers for GPU tests).

Bars (the layer's stated acceptance criteria):
  * the set of selected experts identical to the oracle's, except for
    "ties": tokens whose oracle margin (K-th minus (K+1)-th selection key) is
    below 1e-6.  For a tie the GPU's choice must lie in the tie set: every
    selected expert's oracle key >= the oracle's K-th key - 1e-6, no repeats.
    (The order inside the set follows the keys, which two selected experts
    may share to within rounding; the set and each expert's weight are what
    the layer uses);
  * routing weights within 1e-5 relative of the oracle's, expert by expert.
    The router weights stay f32 (nanocolibri-engine README, "Converting a
    checkpoint yourself"), so the logits carry f32 rounding of order
    2^-24 * sum_h |x_h W_eh|, which reaches ~1.5e-6 relative in the weights
    when that sum is ~20 (raw-code cases with 5x router weights); 1e-5 bounds
    it, while a real error (the bias inside the weights, a dropped scaling
    factor) is >= 1e-2;
  * layer output: per-token relative L2 error ||out - ref|| / ||ref|| <= 2e-3,
    with out the GPU's bf16 output widened exactly and ref the oracle's f64
    result evaluated with the GPU's selection (identical to the oracle's own
    selection except at ties).

Two further bars, derived from the arithmetic, for shapes whose rows are too
short for the 2e-3 bar to leave room above the bf16 output rounding (that
rounding alone averages ~1.7e-3 and varies more when a token has few elements):
  * OUT_F32_TOL: the f32 output mode (no output rounding) against the exact
    result.  The kernels' own error is dominated by the fp16 intermediate h
    (unit roundoff 2^-11 = 4.9e-4, i.e. ~2.8e-4 RMS relative), so 1e-3 is met
    with margin and any wrong term (relative error O(1)) fails it;
  * and, bit for bit, the bf16 output equals round-to-nearest-even of the f32
    output of the same call (the output rounding is the only difference).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TIE_MARGIN = 1e-6
W_RTOL = 1e-5
OUT_TOL = 2e-3
OUT_F32_TOL = 1e-3


def to_cpu_layer(layer: dict) -> dict:
    return {k: v.detach().cpu() for k, v in layer.items()}


def check_routing(idx_gpu: np.ndarray, w_gpu: np.ndarray, ref: dict, bias: np.ndarray, K: int,
                  topp: float = 0.0):
    """Returns (tie token indices, max weight rel error over non-tie tokens).

    With the adaptive top-p (0 < topp < 1) each row holds the kept picks and
    then -1 entries (weight 0).  A token is also a tie when its top-p decision
    came within 1e-6 of the score sum of going the other way (the kernels take
    it in f32); for such tokens the kept picks must be the oracle's kept ones,
    possibly plus or minus the one at the boundary."""
    T = idx_gpu.shape[0]
    margin = ref["margin"]
    keys = ref["scores"] + bias.astype(np.float64)[None, :]
    use_topp = 0.0 < topp < 1.0
    tie = margin < TIE_MARGIN
    if use_topp:
        tie |= ref["topp_margin"] < TIE_MARGIN
    ties = np.nonzero(tie)[0]
    non = ~tie
    # dropped picks (-1) come after the kept ones
    kept = idx_gpu >= 0
    assert np.all(kept[:, 0]), "a token with no expert"
    assert np.all(kept[:, :-1] | ~kept[:, 1:]), "a dropped pick before a kept one"
    if not use_topp:
        assert np.all(kept), "-1 entries without the top-p"
    assert np.all(w_gpu[~kept] == 0.0)
    big = np.iinfo(np.int32).max
    sg = np.sort(np.where(kept, idx_gpu, big), axis=1)
    so = np.sort(np.where(ref["idx"] >= 0, ref["idx"], big), axis=1)
    bad = np.nonzero(non & np.any(sg != so, axis=1))[0]
    assert bad.size == 0, (f"{bad.size} non-tie tokens select different experts; first {bad[:5]}: "
                           f"gpu {idx_gpu[bad[:3]]} oracle {ref['idx'][bad[:3]]} margin {margin[bad[:3]]}")
    for t in ties:
        sel = idx_gpu[t][kept[t]]
        assert len(set(sel.tolist())) == len(sel), (t, sel)
        kth = np.sort(keys[t])[::-1][K - 1]
        assert np.all(keys[t, sel] >= kth - TIE_MARGIN), (t, sel, keys[t, sel], kth)
    # the documented order of topk_idx_out: decreasing s + bias over the kept
    # picks (two selected experts whose keys agree to within rounding may come
    # in either order)
    sel_keys = np.where(kept, np.take_along_axis(keys, np.maximum(idx_gpu, 0).astype(np.int64), axis=1), -1e300)
    drop = sel_keys[:, :-1] - sel_keys[:, 1:]
    bad = np.nonzero(np.any((drop < -TIE_MARGIN) & kept[:, 1:], axis=1))[0]
    assert bad.size == 0, f"selection not in decreasing key order at tokens {bad[:5]}: {sel_keys[bad[:3]]}"
    werr = 0.0
    if non.any():
        og = np.argsort(np.where(kept, idx_gpu, big), axis=1)
        oo = np.argsort(np.where(ref["idx"] >= 0, ref["idx"], big), axis=1)
        wg = np.take_along_axis(w_gpu, og, axis=1)[non]
        wo = np.take_along_axis(ref["weights"], oo, axis=1)[non]
        m = wo > 0
        werr = float(np.max(np.abs(wg[m] - wo[m]) / np.abs(wo[m])))
        assert werr <= W_RTOL, f"routing weight relative error {werr:.3e} > {W_RTOL}"
    return ties, werr


def rel_l2(out_gpu: torch.Tensor, ref: np.ndarray, against=None) -> np.ndarray:
    """||out - against|| / ||ref|| per token (against defaults to ref)."""
    o = out_gpu.detach().float().cpu().numpy().astype(np.float64)
    a = ref if against is None else against
    num = np.linalg.norm(o - a, axis=1)
    den = np.linalg.norm(ref, axis=1)
    return num / np.maximum(den, 1e-300)


def bf16_round(ref: np.ndarray) -> np.ndarray:
    return torch.from_numpy(ref).to(torch.bfloat16).double().numpy()


def oracle_tokens(x, layer_cpu: dict, shape, residual: bool, tokens: np.ndarray, idx_override: np.ndarray,
                  threads: int = 0, topp: float = 0.0) -> np.ndarray:
    """The oracle's output for `tokens` (with the given selections), the
    tokens split over host threads (the oracle is plain C called through
    ctypes, which releases the interpreter lock; it keeps no state between
    calls)."""
    import concurrent.futures
    import os
    n = len(tokens)
    threads = threads or max(1, min(16, os.cpu_count() or 1))
    if n <= 8 or threads == 1:
        return oracle.moe_tokens(x, layer_cpu, shape, residual=residual, tokens=tokens.astype(np.int32),
                                 idx_override=idx_override, topp=topp)["out"]
    parts = np.array_split(np.arange(n), min(threads, n))

    def run(sel):
        return oracle.moe_tokens(x, layer_cpu, shape, residual=residual, tokens=tokens[sel].astype(np.int32),
                                 idx_override=idx_override[sel], topp=topp)["out"]

    with concurrent.futures.ThreadPoolExecutor(len(parts)) as ex:
        outs = list(ex.map(run, parts))
    return np.concatenate(outs, axis=0)


def compare_layer(x: torch.Tensor, out: torch.Tensor, idx: torch.Tensor, w: torch.Tensor, layer_cpu: dict,
                  shape, residual: bool, sample=None, tol: float = OUT_TOL, rounded: bool = False,
                  topp: float = 0.0) -> dict:
    """Full comparison.  Routing is checked on every token; outputs on
    ``sample`` (token indices; default all).  ``rounded``: compare with the
    correctly rounded bf16 result instead of the exact one."""
    xc = x.detach().cpu()
    ref_r = oracle.route(xc, layer_cpu["router_w"], layer_cpu["router_bias"], shape.K, shape.routed_scaling, topp)
    idx_g = idx.detach().cpu().numpy()
    w_g = w.detach().cpu().numpy().astype(np.float64)
    ties, werr = check_routing(idx_g, w_g, ref_r, layer_cpu["router_bias"].numpy(), shape.K, topp)
    T = x.shape[0]
    tok = np.arange(T) if sample is None else np.unique(np.asarray(sample, np.int64))
    ref = oracle_tokens(xc, layer_cpu, shape, residual, tok, np.ascontiguousarray(idx_g[tok]), topp=topp)
    o = out[torch.from_numpy(tok).to(out.device)]
    err = rel_l2(o, ref, bf16_round(ref) if rounded else None)
    assert np.all(np.isfinite(err)), "non-finite output"
    worst = int(tok[int(np.argmax(err))])
    assert err.max() <= tol, f"per-token rel L2 {err.max():.3e} > {tol} at token {worst}"
    return dict(ties=len(ties), max_rel_l2=float(err.max()), mean_rel_l2=float(err.mean()),
                max_w_rel=werr, tokens_checked=len(tok))


def tile_cover(idx: np.ndarray, E: int, tile: int, shared: bool) -> np.ndarray:
    """Tokens that put at least one checked token into every work unit of the
    expert kernels: every `tile`-slot piece of every routed bucket (buckets in
    ascending expert order, each listing its tokens in (t, k) order, as the
    kernels lay out their slots) and, with a shared expert, every `tile`-token
    piece of the shared bucket (tokens in order).  Greedy: a unit not yet
    covered adds its first token, which also covers the units of that token's
    other picks and its shared piece.  The last token of every bucket (its
    ragged tail) is added as well when the bucket spans several units."""
    T, K = idx.shape
    flat = idx.reshape(-1).astype(np.int64)
    tok = np.repeat(np.arange(T), K)
    order = np.argsort(flat, kind="stable")  # (t, k) order within each expert
    se, st = flat[order], tok[order]
    start = np.searchsorted(se, np.arange(E))
    unit_of = np.full(T * K, -1, np.int64)  # unit id of each (t, k) pick (-1: a pick the top-p dropped)
    units_first = []
    uid = 0
    for e in range(E):
        lo, hi = start[e], (start[e + 1] if e + 1 < E else se.size)
        for m0 in range(lo, hi, tile):
            m1 = min(hi, m0 + tile)
            unit_of[order[m0:m1]] = uid
            units_first.append(int(st[m0]))
            uid += 1
    n_routed = uid
    covered = np.zeros(n_routed + (-(-T // tile) if shared else 0), bool)
    picks_of = unit_of.reshape(T, K)
    chosen = []

    def take(t):
        chosen.append(t)
        u = picks_of[t]
        covered[u[u >= 0]] = True
        if shared:
            covered[n_routed + t // tile] = True

    for u in range(n_routed):
        if not covered[u]:
            take(units_first[u])
    if shared:
        for m in range(-(-T // tile)):
            if not covered[n_routed + m]:
                take(m * tile)
    assert covered.all()
    ends = np.append(start[1:], se.size)
    tails = [int(st[ends[e] - 1]) for e in range(E) if ends[e] - start[e] > tile]
    return np.unique(np.asarray(chosen + tails + [T - 1], np.int64))


def sample_tokens(T: int, n: int = 32, seed: int = 0, extra=()) -> np.ndarray:
    """First and last few tokens (ragged tail) plus a seeded random draw."""
    rng = np.random.default_rng(seed)
    head = np.arange(min(T, 4))
    tail = np.arange(max(0, T - 4), T)
    mid = rng.choice(T, size=min(T, n), replace=False)
    return np.unique(np.concatenate([head, tail, mid, np.asarray(extra, np.int64)]))
