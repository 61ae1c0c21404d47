"""Seeded random configurations of the layer against the CPU oracle, through
the C ABI.

Shapes, token counts, kernel sequences and options are drawn together, so
that combinations no hand-written case names are checked too: a split last
wave of the grouped GEMM, int8 weights with ragged buckets, top-p on either
expert sequence, a residual on the large-batch paths, expert counts that are
not multiples of any tile.  Each case compares the f32 output (no output
rounding) with the exact result at the f32 bar, and checks that the bf16
output of the same call is that f32 output rounded to nearest-even, bit for
bit.
"""
import numpy as np
import pytest
import torch

import workloads
from tests._parity import OUT_F32_TOL, compare_layer, sample_tokens, tile_cover, to_cpu_layer

pytestmark = pytest.mark.gpu

N_CASES = 40


def draw(i):
    rng = np.random.default_rng(1000 + i)
    H = int(rng.choice([256, 512, 768, 1024, 1536, 2048]))
    E = int(rng.integers(4, 161))
    K = int(rng.integers(1, min(8, E) + 1))
    I = int(rng.choice([128, 256, 384, 512]))
    Is = int(rng.choice([0, 128, 256, 640]))
    T = int(rng.choice([1, 7, 33, 64, 65, 129, 300, 777]))
    mode = str(rng.choice(["auto", "prefill", "decode", "int8"]))
    if H % 256 and mode in ("prefill", "int8"):
        mode = "decode"
    opts = dict(residual=bool(rng.random() < 0.3), topp=float(rng.choice([0.0, 0.0, 0.0, 0.7])),
                raw=bool(rng.random() < 0.3), scale=float(rng.choice([1.0, 2.5])))
    return H, E, K, I, Is, T, mode, opts


@pytest.fixture(scope="module")
def moe(cuda_device):
    import int4_expert_ffn_sigmoid_b200 as m
    return m


@pytest.mark.parametrize("case", range(N_CASES))
def test_random_configuration(moe, cuda_device, case):
    H, E, K, I, Is, T, mode, opts = draw(case)
    shape = workloads.LayerShape(H=H, E=E, K=K, I=I, Is=Is, routed_scaling=opts["scale"])
    flags = {"auto": 0, "prefill": moe.MOE_FORCE_PREFILL, "decode": moe.MOE_FORCE_DECODE,
             "int8": moe.MOE_WEIGHTS_INT8}[mode]
    if opts["residual"]:
        flags |= moe.MOE_ADD_RESIDUAL
    wbits = 8 if mode == "int8" else 4
    layer = workloads.make_layer(shape, 1000 + case, 0, cuda_device, raw_codes=opts["raw"], wbits=wbits)
    x = workloads.make_x(shape, T, 1000 + case, device=cuda_device)
    path = moe.layer_path(shape, T, flags)
    assert path != 0, (shape, T, flags)
    idx = torch.empty((T, K), dtype=torch.int32, device=cuda_device)
    w = torch.empty((T, K), dtype=torch.float32, device=cuda_device)
    f = flags | moe.MOE_DEBUG_CHECK
    o32 = moe.layer_forward(x, layer, shape, flags=f | moe.MOE_OUT_F32, topk_idx=idx, topk_w=w, topp=opts["topp"])
    o16 = moe.layer_forward(x, layer, shape, flags=f, topp=opts["topp"])
    torch.cuda.synchronize()
    assert torch.equal(o32.to(torch.bfloat16), o16), "bf16 output is not the f32 output rounded"
    unit = 128 if path == moe.MOE_PATH_TENSOR_CORE else 16
    sample = np.union1d(tile_cover(idx.cpu().numpy(), E, unit, Is > 0), sample_tokens(T, 16, case))
    r = compare_layer(x, o32, idx, w, to_cpu_layer(layer), shape, residual=opts["residual"], sample=sample,
                      tol=OUT_F32_TOL, topp=opts["topp"])
    print(f"case {case}: H={H} E={E} K={K} I={I} Is={Is} T={T} mode={mode} path={path} {opts} {r}")
