"""int8 expert weights (MOE_WEIGHTS_INT8) against the CPU oracle, through the
C ABI.

The engine's checkpoint converter sets the experts' bit width
(nanocolibri-engine README, "Converting a checkpoint yourself"); with 8 bits
every routed and shared weight is one two's-complement byte times its row
scale.  Shapes the TMA-ring streaming kernels serve take int4's kernel
sequences (small batch, large-batch streaming, tensor cores); others take the
tensor-core grouped GEMMs at every T.  Cases: quantised and uniformly random
codes (-128 included), one token, ragged token tiles, several tiles per
bucket, no shared expert, the f32 output mode, the stack entry point, and an
int4 layer re-encoded one code per byte, which must give the int4 call's
output bit for bit on every sequence (the same codes reach the same MMAs:
16 c on the int4 streaming path against c here, the factor 16 taken out of the
exact activation scale).
"""
import numpy as np
import pytest
import torch

import workloads
from tests._parity import OUT_F32_TOL, compare_layer, sample_tokens, tile_cover, to_cpu_layer

pytestmark = pytest.mark.gpu

NANO = workloads.NANO
CASES = [
    # (shape, T values, raw codes): Nano streams at T <= 1023; H = 512 and I = 384 have no int8
    # streaming kernels (tensor cores at every T)
    (NANO, (1, 16, 64, 300, 1100), False),
    (NANO, (3, 130), True),
    (workloads.LayerShape(H=512, E=16, K=8, I=256, Is=0, routed_scaling=2.5), (1, 77, 400), True),
    (workloads.LayerShape(H=2048, E=32, K=4, I=384, Is=640, routed_scaling=2.5), (200,), False),
    (workloads.LayerShape(H=1536, E=24, K=3, I=256, Is=0, routed_scaling=2.5), (5, 40, 150), True),
]


@pytest.fixture(scope="module")
def moe(cuda_device):
    import int4_expert_ffn_sigmoid_b200 as m
    return m


def run(moe, x, layer, shape, flags):
    T = x.shape[0]
    idx = torch.empty((T, shape.K), dtype=torch.int32, device=x.device)
    w = torch.empty((T, shape.K), dtype=torch.float32, device=x.device)
    out = moe.layer_forward(x, layer, shape, flags=flags | moe.MOE_WEIGHTS_INT8 | moe.MOE_DEBUG_CHECK,
                            topk_idx=idx, topk_w=w)
    torch.cuda.synchronize()
    return out, idx, w


@pytest.mark.parametrize("case", range(len(CASES)))
def test_int8_layer_matches_oracle(moe, cuda_device, case):
    shape, Ts, raw = CASES[case]
    layer = workloads.make_layer(shape, 700 + case, 0, cuda_device, raw_codes=raw, wbits=8)
    assert layer["w13"].shape[-1] == shape.H
    cpu = to_cpu_layer(layer)
    for T in Ts:
        path = moe.layer_path(shape, T, moe.MOE_WEIGHTS_INT8)
        assert path != 0
        x = workloads.make_x(shape, T, 700 + case, device=cuda_device)
        out, idx, w = run(moe, x, layer, shape, 0)
        cover = tile_cover(idx.cpu().numpy(), shape.E, 128 if path == moe.MOE_PATH_TENSOR_CORE else 16, shape.Is > 0)
        sample = np.union1d(cover, sample_tokens(T, 24, 7 + case))
        r = compare_layer(x, out, idx, w, cpu, shape, residual=False, sample=sample)
        print(f"case {case} T={T} path={path} raw={raw} {r}")
        # the f32 output against the exact result, and the bf16 output its rounding
        o32, idx32, w32 = run(moe, x, layer, shape, moe.MOE_OUT_F32)
        assert torch.equal(idx32, idx) and torch.equal(w32, w)
        r32 = compare_layer(x, o32, idx, w, cpu, shape, residual=False, sample=sample, tol=OUT_F32_TOL)
        assert torch.equal(o32.to(torch.bfloat16), out)
        print(f"  f32 output {r32['max_rel_l2']:.2e}")


def test_int8_equals_int4_recoded(moe, cuda_device):
    """The int4 call and the same codes one per byte (MOE_WEIGHTS_INT8) give
    identical bits, on each kernel sequence."""
    shape = NANO
    layer4 = workloads.make_layer(shape, 710, 0, cuda_device, raw_codes=True)
    table = torch.tensor([0, 1, 2, 3, 4, 5, 6, 7, -8, -7, -6, -5, -4, -3, -2, -1], dtype=torch.int16,
                         device=cuda_device)

    def recode(p):
        lo, hi = table[(p & 0xF).long()], table[(p >> 4).long()]
        return torch.stack([lo, hi], dim=-1).reshape(*p.shape[:-1], 2 * p.shape[-1]).to(torch.int8).view(torch.uint8)
    layer8 = dict(layer4)
    for k in ("w13", "w2", "sh_w13", "sh_w2"):
        layer8[k] = recode(layer4[k]).contiguous()
    for T, f in ((1, moe.MOE_FORCE_PREFILL), (200, moe.MOE_FORCE_PREFILL), (2048, 0), (1, 0), (16, 0), (64, 0),
                 (200, moe.MOE_FORCE_DECODE), (300, 0)):
        x = workloads.make_x(shape, T, 710, device=cuda_device)
        a = moe.layer_forward(x, layer4, shape, flags=f | moe.MOE_DEBUG_CHECK)
        b = moe.layer_forward(x, layer8, shape, flags=f | moe.MOE_WEIGHTS_INT8 | moe.MOE_DEBUG_CHECK)
        torch.cuda.synchronize()
        assert moe.layer_path(shape, T, f) == moe.layer_path(shape, T, f | moe.MOE_WEIGHTS_INT8)
        if moe.layer_path(shape, T, f) == moe.MOE_PATH_LARGE_STREAMING and T * shape.K >= 12 * shape.E:
            continue  # int4 gate/up on tcgen05 there, int8 on mma.sync: equal to rounding, not bit for bit
        assert torch.equal(a, b), (T, f)


def test_int8_stack_and_layer_object(moe, cuda_device):
    """moe_stack_forward with int8 weights: one layer call per layer (residual),
    bit-identical to chaining layer_forward; MoELayer adds the flag itself."""
    shape = NANO
    L, T = 3, 12
    layers = [workloads.make_layer(shape, 720, l, cuda_device, wbits=8) for l in range(L)]
    stacked = moe.stack_layers(layers)
    x = workloads.make_x(shape, T, 720, device=cuda_device)
    f = moe.MOE_WEIGHTS_INT8 | moe.MOE_ADD_RESIDUAL | moe.MOE_DEBUG_CHECK
    assert moe.stack_path(shape, T, L, f) == moe.MOE_PATH_PER_LAYER
    outs = moe.stack_forward(x, stacked, shape, flags=f)
    h = x
    for l in range(L):
        obj = moe.MoELayer(layers[l], shape, max_tokens=64)
        assert obj.weight_flags == moe.MOE_WEIGHTS_INT8
        h = obj(h, residual=True, flags=moe.MOE_DEBUG_CHECK)
        torch.cuda.synchronize()
        assert torch.equal(outs[l], h), l
    cpu = to_cpu_layer(layers[0])
    idx = torch.empty((T, shape.K), dtype=torch.int32, device=cuda_device)
    w = torch.empty((T, shape.K), dtype=torch.float32, device=cuda_device)
    o0 = moe.layer_forward(x, layers[0], shape, flags=f, topk_idx=idx, topk_w=w)
    torch.cuda.synchronize()
    compare_layer(x, o0, idx, w, cpu, shape, residual=True)
