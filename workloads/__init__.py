"""Seeded synthetic inputs for the int4 expert-FFN MoE layer.

This module is shared by the CPU oracle tests and the CUDA path's tests and
benchmark.  It only *produces inputs*: random activations, random router
weights and biases, and the offline per-row symmetric int4 quantisation of
random expert weights (the container format the hot path consumes).  It holds
none of the layer's forward arithmetic (no router scores, no selection, no
expert FFN, no combine).

Shapes and distributions follow the workloads of the Colibri-Nano model card
("Architecture": 64 experts, top-2, 2048-wide shared expert, hidden 1024) and
the colibri GLM-5.2 README ("How it works": 256 routed experts of ~19 MB at
int4, top-8), with the quantisation rule of the nanocolibri-engine README
("Converting a checkpoint yourself": per-row symmetric, f32 scales in a
sibling tensor, router weight and bias kept f32).

Quantisation rule (per output row r of a [rows, cols] matrix, computed in f32):
    scale_r = max_c |w[r, c]| / 7
    q[r, c] = clamp(round_half_even(w[r, c] / scale_r), -8, 7)     (0 if scale_r == 0)
Packing: byte j of a row holds element 2j in bits 0..3 and element 2j+1 in
bits 4..7, each a 4-bit two's-complement code.

The int8 expert weights (the engine's ``--ebits 8`` conversion, nanocolibri-engine
README "Converting a checkpoint yourself") use the same per-row rule with 127:
    scale_r = max_c |w[r, c]| / 127
    q[r, c] = clamp(round_half_even(w[r, c] / scale_r), -128, 127)
one byte per element, two's complement, in column order.

Randomness: every tensor is drawn from its own ``torch.Generator`` seeded with
a fixed integer derived from (workload id, layer, tensor id, chunk), on the
device the caller asks for.  The CPU and CUDA generators are different
streams, so a comparison always feeds both sides the same materialised arrays.
"""
from __future__ import annotations

import dataclasses
import os
from typing import Dict, Iterable, List, Optional

import torch

__all__ = [
    "LayerShape", "NANO", "LARGE", "LARGE_E32", "Workload", "WORKLOADS",
    "quantize_rows_int4", "quantize_rows_int8", "pack_int4", "random_int4_codes",
    "make_layer", "make_x", "zipf_bias_path", "load_zipf_bias",
    "layer_weight_bytes", "expert_bytes",
]


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """Static shape of one MoE layer.

    H: hidden size; E: routed experts; K: experts selected per token;
    I: routed SwiGLU intermediate; Is: shared-expert intermediate (0 = none);
    routed_scaling: factor applied to the normalised routing weights.
    """
    H: int
    E: int
    K: int
    I: int
    Is: int
    routed_scaling: float


# Colibri-Nano: hidden 1024, 64 experts top-2, routed intermediate 512,
# a 2048-wide shared expert, scaling factor 1.0.
NANO = LayerShape(H=1024, E=64, K=2, I=512, Is=2048, routed_scaling=1.0)
# Layer shaped like the 744B streaming engine's: hidden 6144, 256 experts,
# top-8, intermediate 2048 (routed and shared), scaling factor 2.5.
LARGE = LayerShape(H=6144, E=256, K=8, I=2048, Is=2048, routed_scaling=2.5)
# The same expert shapes with 32 experts (profiling stand-in).
LARGE_E32 = LayerShape(H=6144, E=32, K=8, I=2048, Is=2048, routed_scaling=2.5)


@dataclasses.dataclass(frozen=True)
class Workload:
    """A named synthetic workload.

    wid: integer id used in the seeds; layers: stacked layers (each with its
    own weights); tokens: the token counts the workload is run at;
    bias_mode: "uniform" (U(-0.1, 0.1)), "zero", or "zipf" (calibrated
    popularity bias read from a data file); residual: whether each layer adds
    its input (x_{l+1} = x_l + MoE_l(x_l)); wbits: expert code width (4 or 8).
    """
    name: str
    wid: int
    shape: LayerShape
    layers: int
    tokens: tuple
    bias_mode: str
    residual: bool
    description: str
    wbits: int = 4


WORKLOADS: Dict[str, Workload] = {
    w.name: w for w in [
        Workload("nano_layer_t16", 0, NANO, 1, (16,), "uniform", False,
                 "one Nano MoE layer, T=16"),
        Workload("nano_decode_stack", 1, NANO, 23, (1, 2, 3, 4, 16, 64), "uniform", True,
                 "23 stacked Nano MoE layers with residual, decode T in {1,4,16,64} and "
                 "speculative-verify T in {2,3,4}"),
        Workload("nano_prefill_t4096", 2, NANO, 1, (4096,), "zero", False,
                 "one Nano MoE layer, T=4096, zero router bias (balanced loads)"),
        Workload("nano_zipf_t16384", 3, NANO, 1, (16384,), "zipf", False,
                 "one Nano MoE layer, T=16384, Zipf(1.2) expert popularity via router bias"),
        Workload("nano_prefill_t4096_int8", 6, NANO, 1, (4096,), "zero", False,
                 "one Nano MoE layer with int8 expert weights (the converter's 8-bit expert setting), "
                 "T=4096, zero router bias", wbits=8),
        Workload("large_layer", 4, LARGE, 1, (1, 32, 512), "uniform", False,
                 "one 6144-hidden 256-expert top-8 layer, T in {1,32,512}"),
        Workload("large_layer_e32", 5, LARGE_E32, 1, (4,), "uniform", False,
                 "the large layer's expert shapes with 32 experts (about 0.6 GB of weights), T=4: "
                 "about one token per touched expert, as in the large layer at T=32; sized for "
                 "profiler captures of its kernels"),
    ]
}

# tensor ids used in the seeds
_TID_X, _TID_RW, _TID_RB, _TID_W13, _TID_W2, _TID_SW13, _TID_SW2 = range(7)
# experts are drawn in chunks of this many experts per generator call
_EXPERT_CHUNK = 8
_WEIGHT_STD = 0.02


def _seed(wid: int, layer: int, tid: int, chunk: int = 0) -> int:
    return ((((wid * 1009) + layer) * 101 + tid) * 100003 + chunk) & 0x7FFF_FFFF_FFFF


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def pack_int4(q: torch.Tensor) -> torch.Tensor:
    """Pack int4 codes (int8 tensor with values in [-8, 7], last dim even)
    into bytes, element 2j in the low nibble of byte j."""
    if q.shape[-1] % 2:
        raise ValueError("last dimension must be even")
    u = q.to(torch.int16) & 0xF
    return (u[..., 0::2] | (u[..., 1::2] << 4)).to(torch.uint8)


def quantize_rows_int4(w: torch.Tensor):
    """Per-row symmetric int4 quantisation of an f32 tensor [..., cols].

    Returns (packed uint8 [..., cols/2], scales f32 [...]).  Computed in f32;
    torch.round rounds half to even.  An all-zero row gets scale 0 and codes 0.
    """
    w = w.to(torch.float32)
    scale = w.abs().amax(dim=-1) / 7.0
    safe = torch.where(scale > 0, scale, torch.ones_like(scale))
    q = torch.round(w / safe.unsqueeze(-1)).clamp_(-8, 7)
    q = torch.where(scale.unsqueeze(-1) > 0, q, torch.zeros_like(q)).to(torch.int8)
    return pack_int4(q), scale.contiguous()


def quantize_rows_int8(w: torch.Tensor):
    """Per-row symmetric int8 quantisation of an f32 tensor [..., cols].

    Returns (codes uint8 [..., cols], the int8 two's-complement bytes, and
    scales f32 [...]).  Same rounding and zero-row rule as the int4 quantiser.
    """
    w = w.to(torch.float32)
    scale = w.abs().amax(dim=-1) / 127.0
    safe = torch.where(scale > 0, scale, torch.ones_like(scale))
    q = torch.round(w / safe.unsqueeze(-1)).clamp_(-128, 127)
    q = torch.where(scale.unsqueeze(-1) > 0, q, torch.zeros_like(q)).to(torch.int8)
    return q.view(torch.uint8).contiguous(), scale.contiguous()


def random_int4_codes(shape, generator: torch.Generator, device) -> torch.Tensor:
    """Uniformly random packed bytes: every one of the 16 codes (including -8,
    which the quantiser never emits) appears in both nibbles."""
    return torch.randint(0, 256, shape, generator=generator, device=device, dtype=torch.int32).to(torch.uint8)


def zipf_bias_path(E: int = 64, s: float = 1.2) -> str:
    return os.path.join(os.path.dirname(__file__), "data", f"zipf_bias_e{E}_s{s:g}.txt")


def load_zipf_bias(E: int = 64, s: float = 1.2) -> torch.Tensor:
    """Router bias calibrated so expert popularity follows Zipf(s).

    The values are written by ``oracle/calibrate_zipf_bias.py``.  They are an
    input of the Zipf workload, not an expected result."""
    path = zipf_bias_path(E, s)
    vals: List[float] = []
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                vals.append(float(line))
    if len(vals) != E:
        raise ValueError(f"{path}: expected {E} values, found {len(vals)}")
    return torch.tensor(vals, dtype=torch.float32)


def _normal(shape, g, device, std=_WEIGHT_STD):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).mul_(std)


def make_layer(shape: LayerShape, wid: int, layer: int = 0, device="cpu",
               bias_mode: str = "uniform", raw_codes: bool = False,
               experts: Optional[Iterable[int]] = None, wbits: int = 4) -> Dict[str, torch.Tensor]:
    """Materialise one layer's weights on ``device``.

    Returns a dict with router_w f32 [E,H], router_bias f32 [E],
    w13 u8 [E,2I,H/2] (rows 0..I-1 gate, I..2I-1 up), s13 f32 [E,2I],
    w2 u8 [E,H,I/2], s2 f32 [E,H], and, when Is > 0, sh_w13 u8 [2Is,H/2],
    sh_s13 f32 [2Is], sh_w2 u8 [H,Is/2], sh_s2 f32 [H].

    raw_codes=True replaces the quantised expert weights by uniformly random
    packed codes with random positive scales (exercises code -8).
    ``experts`` restricts the routed experts that are generated (the others
    stay zero): only used to keep CPU tests small.
    wbits=8 gives int8 expert and shared weights instead (one byte per
    element: w13 u8 [E,2I,H], w2 u8 [E,H,I], sh_w13 [2Is,H], sh_w2 [H,Is]);
    raw_codes then draws every byte value, -128 included.
    """
    if wbits not in (4, 8):
        raise ValueError("wbits must be 4 or 8")
    H, E, I, Is = shape.H, shape.E, shape.I, shape.Is
    per = 2 if wbits == 4 else 1          # elements per byte
    quant = quantize_rows_int4 if wbits == 4 else quantize_rows_int8
    dev = torch.device(device)
    out: Dict[str, torch.Tensor] = {}
    out["router_w"] = _normal((E, H), _gen(dev, _seed(wid, layer, _TID_RW)), dev)
    if bias_mode == "uniform":
        g = _gen(dev, _seed(wid, layer, _TID_RB))
        out["router_bias"] = torch.rand((E,), generator=g, device=dev).mul_(0.2).sub_(0.1)
    elif bias_mode == "zero":
        out["router_bias"] = torch.zeros((E,), device=dev)
    elif bias_mode == "zipf":
        out["router_bias"] = load_zipf_bias(E).to(dev)
    else:
        raise ValueError(bias_mode)

    w13 = torch.zeros((E, 2 * I, H // per), dtype=torch.uint8, device=dev)
    s13 = torch.zeros((E, 2 * I), dtype=torch.float32, device=dev)
    w2 = torch.zeros((E, H, I // per), dtype=torch.uint8, device=dev)
    s2 = torch.zeros((E, H), dtype=torch.float32, device=dev)
    wanted = set(range(E)) if experts is None else set(int(e) for e in experts)
    for c0 in range(0, E, _EXPERT_CHUNK):
        c1 = min(E, c0 + _EXPERT_CHUNK)
        if not wanted.intersection(range(c0, c1)):
            continue
        chunk = c0 // _EXPERT_CHUNK
        g13 = _gen(dev, _seed(wid, layer, _TID_W13, chunk))
        g2 = _gen(dev, _seed(wid, layer, _TID_W2, chunk))
        n = c1 - c0
        if raw_codes:
            w13[c0:c1] = random_int4_codes((n, 2 * I, H // per), g13, dev)
            s13[c0:c1] = torch.rand((n, 2 * I), generator=g13, device=dev).mul_(0.01).add_(0.001)
            w2[c0:c1] = random_int4_codes((n, H, I // per), g2, dev)
            s2[c0:c1] = torch.rand((n, H), generator=g2, device=dev).mul_(0.01).add_(0.001)
        else:
            p, s = quant(_normal((n, 2 * I, H), g13, dev))
            w13[c0:c1], s13[c0:c1] = p, s
            p, s = quant(_normal((n, H, I), g2, dev))
            w2[c0:c1], s2[c0:c1] = p, s
    if experts is not None:
        keep = torch.zeros(E, dtype=torch.bool, device=dev)
        keep[list(wanted)] = True
        w13[~keep] = 0
        s13[~keep] = 0
        w2[~keep] = 0
        s2[~keep] = 0
    out.update(w13=w13, s13=s13, w2=w2, s2=s2)
    if Is > 0:
        g13 = _gen(dev, _seed(wid, layer, _TID_SW13))
        g2 = _gen(dev, _seed(wid, layer, _TID_SW2))
        if raw_codes:
            out["sh_w13"] = random_int4_codes((2 * Is, H // per), g13, dev)
            out["sh_s13"] = torch.rand((2 * Is,), generator=g13, device=dev).mul_(0.01).add_(0.001)
            out["sh_w2"] = random_int4_codes((H, Is // per), g2, dev)
            out["sh_s2"] = torch.rand((H,), generator=g2, device=dev).mul_(0.01).add_(0.001)
        else:
            out["sh_w13"], out["sh_s13"] = quant(_normal((2 * Is, H), g13, dev))
            out["sh_w2"], out["sh_s2"] = quant(_normal((H, Is), g2, dev))
    return out


def make_x(shape: LayerShape, T: int, wid: int, batch: int = 0, device="cpu",
           std: float = 1.0) -> torch.Tensor:
    """Activations x: bf16 [T, H], drawn as f32 N(0, std^2) and rounded to
    bf16 (round to nearest even).  ``batch`` selects an independent draw."""
    g = _gen(torch.device(device), _seed(wid, 10_000 + batch, _TID_X, T))
    return torch.randn((T, shape.H), generator=g, device=device, dtype=torch.float32).mul_(std).to(torch.bfloat16)


def expert_bytes(shape: LayerShape, wbits: int = 4) -> int:
    """Bytes of one routed expert at int4 (or int8) plus its f32 row scales."""
    H, I = shape.H, shape.I
    return 3 * H * I * wbits // 8 + (2 * I + H) * 4


def layer_weight_bytes(shape: LayerShape, wbits: int = 4) -> Dict[str, int]:
    H, E, I, Is = shape.H, shape.E, shape.I, shape.Is
    shared = (3 * H * Is * wbits // 8 + (2 * Is + H) * 4) if Is else 0
    return {
        "router": E * H * 4 + E * 4,
        "expert": expert_bytes(shape, wbits),
        "experts_total": E * expert_bytes(shape, wbits),
        "shared": shared,
    }
