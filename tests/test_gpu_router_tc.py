"""The tensor-core router logits of the large-batch path (router weights above
512 KB) against the CPU oracle, through the C ABI.

The four expert-tile widths of the logits kernel (16, 32, 64 and 128 experts,
the last with a second tile holding 2 experts), ragged token tiles, one token
under MOE_FORCE_PREFILL, both large-batch expert sequences, and a token's
result independent of the rest of the batch (bit-exact: the hidden slices
depend on H alone).
"""
import pytest
import torch

import workloads
from tests._parity import compare_layer, sample_tokens, to_cpu_layer

pytestmark = pytest.mark.gpu

# (E, H, K): E*H*4 bytes of router weights above 512 KB in every case
CASES = [(16, 16384, 2), (24, 8192, 4), (40, 4096, 8), (130, 1024, 6)]


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
def test_tensor_core_router(moe, cuda_device, case):
    E, H, K = CASES[case]
    assert E * H * 4 > 512 * 1024
    shape = workloads.LayerShape(H=H, E=E, K=K, I=128, Is=128, routed_scaling=2.5)
    assert moe.kernel_launches(shape, 300) == 7  # weight split, logits, selection, scatter, experts, combine
    layer = workloads.make_layer(shape, 500 + case, 0, cuda_device)
    cpu = to_cpu_layer(layer)
    for T, flags in ((1, moe.MOE_FORCE_PREFILL), (65, 0), (300, moe.MOE_FORCE_DECODE), (300, moe.MOE_FORCE_PREFILL)):
        x = workloads.make_x(shape, T, 500 + case, device=cuda_device)
        out, idx, w = run(moe, x, layer, shape, flags)
        r = compare_layer(x, out, idx, w, cpu, shape, residual=False, sample=sample_tokens(T, 40, 3 + case))
        print(f"E={E} H={H} K={K} T={T} flags={flags} {r}")
    # batch independence: sub-batches (other token tiles, other tile counts) give the same bits
    x = workloads.make_x(shape, 300, 600 + case, device=cuda_device)
    full, idx_full, _ = run(moe, x, layer, shape)
    for t0, sub in ((0, 65), (37, 150), (299, 1)):
        flags = moe.MOE_FORCE_PREFILL if sub <= 64 else 0
        o1, i1, _ = run(moe, x[t0:t0 + sub].contiguous(), layer, shape, flags)
        assert torch.equal(i1, idx_full[t0:t0 + sub])
        if moe.layer_path(shape, sub, flags) == moe.layer_path(shape, 300):  # the same expert sequence
            assert torch.equal(o1, full[t0:t0 + sub])
