"""The adaptive expert top-p (cfg.topp, opt-in) on every kernel sequence,
against the CPU oracle with the same top-p.

Of each token's K selected experts the kernels keep the fewest
highest-scoring ones whose scores reach p of the K's total (the keep decision
taken in f32), re-weighted over the kept set; the dropped picks are not
computed and appear as -1 after the kept ones.  Compared: the kept sets and
their order and weights on every token (tokens whose top-p decision lies
within 1e-6 of the boundary may keep one pick more or fewer), outputs against
the oracle evaluated with the GPU's kept picks.  Without top-p nothing
changes, bit for bit.
"""
import numpy as np
import pytest
import torch

import workloads
from tests._parity import OUT_F32_TOL, compare_layer, to_cpu_layer

pytestmark = pytest.mark.gpu

TOPP = 0.7


@pytest.fixture(scope="module")
def moe(cuda_device):
    import int4_expert_ffn_sigmoid_b200 as m
    return m


def run(moe, x, layer, shape, flags=0, topp=TOPP):
    T = x.shape[0]
    idx = torch.empty((T, shape.K), dtype=torch.int32, device=x.device)
    w = torch.empty((T, shape.K), dtype=torch.float32, device=x.device)
    out = moe.layer_forward(x, layer, shape, flags=flags | moe.MOE_DEBUG_CHECK, topk_idx=idx, topk_w=w, topp=topp)
    torch.cuda.synchronize()
    return out, idx, w


CASES = [
    # (what, shape, T, flags)
    ("small-batch kernels, large layer shape", "large", 32, 0),
    ("small-batch kernels", workloads.LayerShape(1024, 64, 8, 512, 2048, 2.5), 40, 0),
    ("tensor-core kernels", workloads.LayerShape(512, 16, 8, 256, 384, 2.5), 130, "prefill"),
    ("large-batch streaming kernels", workloads.LayerShape(1024, 64, 8, 512, 2048, 2.5), 150, "decode"),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_topp_per_layer_paths(moe, cuda_device, case):
    what, shape, T, f = CASES[case]
    if shape == "large":
        wl = workloads.WORKLOADS["large_layer"]
        shape, layer = wl.shape, workloads.make_layer(wl.shape, wl.wid, 0, cuda_device, wl.bias_mode)
        x = workloads.make_x(shape, T, wl.wid, device=cuda_device)
    else:
        layer = workloads.make_layer(shape, 360 + case, 0, cuda_device)
        layer["router_w"].mul_(8)  # a spread of scores, so the top-p drops picks
        x = workloads.make_x(shape, T, 360 + case, device=cuda_device)
    flags = {0: 0, "prefill": moe.MOE_FORCE_PREFILL, "decode": moe.MOE_FORCE_DECODE}[f]
    out, idx, w = run(moe, x, layer, shape, flags)
    dropped = int((idx < 0).sum())
    assert dropped > 0, what
    cpu = to_cpu_layer(layer)
    r = compare_layer(x, out, idx, w, cpu, shape, False, topp=TOPP,
                      sample=np.arange(T) if T <= 64 else np.unique(np.r_[np.arange(8), np.arange(T - 8, T),
                                                                           np.arange(0, T, 7)]))
    print(what, f"dropped {dropped} of {T * shape.K} picks", r)
    # the f32 output mode: the kernels' own error without the output rounding
    of32, _, _ = run(moe, x, layer, shape, flags | moe.MOE_OUT_F32)
    compare_layer(x, of32, idx, w, cpu, shape, False, topp=TOPP, tol=OUT_F32_TOL,
                  sample=np.arange(min(T, 24)))
    # topp 0 and 1 are plain top-K, bit for bit
    a, ia, _ = run(moe, x, layer, shape, flags, topp=0.0)
    b, ib, _ = run(moe, x, layer, shape, flags, topp=1.0)
    assert torch.equal(a, b) and torch.equal(ia, ib) and bool((ia >= 0).all())


def test_topp_fused_stack(moe, cuda_device):
    shape = workloads.LayerShape(1024, 64, 8, 512, 2048, 2.5)
    layers = [workloads.make_layer(shape, 370, l, cuda_device) for l in range(3)]
    for layer in layers:
        layer["router_w"].mul_(8)
    stacked = moe.stack_layers(layers)
    T = 24
    x = workloads.make_x(shape, T, 370, device=cuda_device)
    f = moe.MOE_ADD_RESIDUAL | moe.MOE_DEBUG_CHECK | moe.MOE_STACK_FUSED
    assert moe.stack_path(shape, T, 3, f) == moe.MOE_PATH_FUSED_STACK
    idx = torch.empty((3, T, shape.K), dtype=torch.int32, device=cuda_device)
    w = torch.empty((3, T, shape.K), dtype=torch.float32, device=cuda_device)
    outs = moe.stack_forward(x, stacked, shape, flags=f, topk_idx=idx, topk_w=w, topp=TOPP)
    torch.cuda.synchronize()
    assert int((idx < 0).sum()) > 0
    for l in range(3):
        inp = x if l == 0 else outs[l - 1]
        compare_layer(inp, outs[l], idx[l], w[l], to_cpu_layer(layers[l]), shape, True, topp=TOPP)
