"""The large-batch router for small router weights (at most 512 KB,
router_large_kernel), through the C ABI against the CPU oracle: both
large-batch expert sequences, expert counts below and above 64 and one that
is not a multiple of the 8-expert MMA tile, ragged token tiles, and a token's
result independent of the rest of the batch (bit-exact).
"""
import pytest
import torch

import workloads
from tests._parity import compare_layer, sample_tokens, to_cpu_layer

pytestmark = pytest.mark.gpu

# (E, H, K, I, Is, launches at T = 300)
CASES = [(60, 768, 3, 128, 256, 5), (64, 1024, 2, 256, 512, 5), (128, 512, 4, 256, 256, 5)]


@pytest.fixture(scope="module")
def moe(cuda_device):
    import int4_expert_ffn_sigmoid_b200 as m
    return m


def run(moe, x, layer, shape, flags=0):
    T = x.shape[0]
    idx = torch.empty((T, shape.K), dtype=torch.int32, device=x.device)
    w = torch.empty((T, shape.K), dtype=torch.float32, device=x.device)
    out = moe.layer_forward(x, layer, shape, flags=flags | moe.MOE_DEBUG_CHECK, topk_idx=idx, topk_w=w)
    torch.cuda.synchronize()
    return out, idx, w


@pytest.mark.parametrize("case", range(len(CASES)))
def test_large_router_small_weights(moe, cuda_device, case):
    E, H, K, I, Is, launches = CASES[case]
    assert E * H * 4 <= 512 * 1024
    shape = workloads.LayerShape(H=H, E=E, K=K, I=I, Is=Is, routed_scaling=2.5)
    assert moe.kernel_launches(shape, 300, moe.MOE_FORCE_DECODE) == launches
    layer = workloads.make_layer(shape, 800 + case, 0, cuda_device)
    cpu = to_cpu_layer(layer)
    modes = [(300, moe.MOE_FORCE_DECODE), (77, moe.MOE_FORCE_DECODE)]
    if H % 256 == 0:
        modes += [(300, moe.MOE_FORCE_PREFILL), (1, moe.MOE_FORCE_PREFILL)]
    for T, flags in modes:
        x = workloads.make_x(shape, T, 800 + case, device=cuda_device)
        out, idx, w = run(moe, x, layer, shape, flags)
        r = compare_layer(x, out, idx, w, cpu, shape, residual=False, sample=sample_tokens(T, 40, 11 + case))
        print(f"E={E} H={H} K={K} T={T} flags={flags} {r}")
    # batch independence within a sequence: sub-batches in other token tiles give the same bits
    x = workloads.make_x(shape, 300, 900 + case, device=cuda_device)
    full, idx_full, _ = run(moe, x, layer, shape, moe.MOE_FORCE_DECODE)
    for t0, sub in ((0, 65), (37, 150), (235, 65)):
        o1, i1, _ = run(moe, x[t0:t0 + sub].contiguous(), layer, shape, moe.MOE_FORCE_DECODE)
        assert torch.equal(i1, idx_full[t0:t0 + sub])
        assert torch.equal(o1, full[t0:t0 + sub])
