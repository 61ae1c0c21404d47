"""The tcgen05 (kind::i8) gate/up kernel of the large-batch weight-streaming
sequence against the CPU oracle, through the C ABI.

It runs under MOE_FORCE_DECODE (or below the grouped GEMM's threshold) when
the shape takes the TMA-ring kernels and the batch averages at least 12 picks
per routed expert.  Cases: 12.5 and 31 picks per expert (tasks of 13 and of
the full 32 tokens), K = 1 and K = 6, a skewed router that gives one expert
many 32-token chunks, the shared expert's 32-token chunks, and a token's
result independent of the rest of the batch (bit-exact, same sequence).
"""
import numpy as np
import pytest
import torch

import workloads
from tests._parity import compare_layer, sample_tokens, tile_cover, to_cpu_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(cuda_device):
    import int4_expert_ffn_sigmoid_b200 as m
    return m


def run(moe, x, layer, shape, flags):
    T = x.shape[0]
    idx = torch.empty((T, shape.K), dtype=torch.int32, device=x.device)
    w = torch.empty((T, shape.K), dtype=torch.float32, device=x.device)
    out = moe.layer_forward(x, layer, shape, flags=flags | moe.MOE_DEBUG_CHECK, topk_idx=idx, topk_w=w)
    torch.cuda.synchronize()
    return out, idx, w


CASES = [
    # (H, E, K, I, Is, T): T*K/E picks per expert
    (1024, 64, 2, 512, 2048, 400),    # 12.5
    (1024, 64, 2, 512, 2048, 1000),   # 31
    (2048, 32, 1, 512, 512, 500),     # K = 1, 15.6
    (1536, 48, 6, 256, 768, 200),     # K = 6, 25, a 768-wide shared expert
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_tc8_gate_up(moe, cuda_device, case):
    H, E, K, I, Is, T = CASES[case]
    shape = workloads.LayerShape(H=H, E=E, K=K, I=I, Is=Is, routed_scaling=2.5)
    f = moe.MOE_FORCE_DECODE
    assert moe.layer_path(shape, T, f) == moe.MOE_PATH_LARGE_STREAMING
    assert T * K >= 12 * E
    layer = workloads.make_layer(shape, 700 + case, 0, cuda_device)
    cpu = to_cpu_layer(layer)
    x = workloads.make_x(shape, T, 700 + case, device=cuda_device)
    out, idx, w = run(moe, x, layer, shape, f)
    sample = np.union1d(tile_cover(idx.cpu().numpy(), E, 16, Is > 0), sample_tokens(T, 24, case))
    r = compare_layer(x, out, idx, w, cpu, shape, residual=False, sample=sample)
    print(f"case {case}: {r}")
    # batch independence within the sequence: a sub-batch that still averages
    # >= 12 picks per expert gives the same bits
    sub = (12 * E + K - 1) // K + 7
    o1, i1, _ = run(moe, x[3:3 + sub].contiguous(), layer, shape, f)
    assert torch.equal(i1, idx[3:3 + sub]) and torch.equal(o1, out[3:3 + sub])


def test_tc8_hot_expert(moe, cuda_device):
    """A router bias that sends most tokens to expert 5: its bucket spans many
    32-token chunks (the tasks walk them in order), the other experts few."""
    shape = workloads.LayerShape(H=1024, E=64, K=2, I=512, Is=2048, routed_scaling=1.0)
    layer = workloads.make_layer(shape, 720, 0, cuda_device)
    layer["router_bias"][5] += 4.0
    x = workloads.make_x(shape, 600, 720, device=cuda_device)
    out, idx, w = run(moe, x, layer, shape, moe.MOE_FORCE_DECODE)
    assert (idx == 5).sum().item() > 300
    sample = np.union1d(tile_cover(idx.cpu().numpy(), shape.E, 16, True), sample_tokens(600, 24, 1))
    r = compare_layer(x, out, idx, w, to_cpu_layer(layer), shape, residual=False, sample=sample)
    print(r)
