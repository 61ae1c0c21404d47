"""The fused stack kernel (moe_stack_forward, one launch for all layers) against
the CPU oracle, through the C ABI.

Every layer is compared with the oracle fed the GPU's bf16 input of that
layer (its previous layer's output): routing on every token, outputs on every
token.  Also: the lookahead prefetch changes no bit, a token's result does not
depend on the rest of the batch (bit for bit), shapes with E not a multiple of
8 or 32, K = 1 and K = E, no shared expert, raw int4 codes, the 23-layer Nano
stack over the decode and verify sizes T in {1, 2, 3, 4, 16, 64}, the large
layer at T = 1 and 32, the per-layer path beyond 64 tokens, and the timeout
path.
"""
import numpy as np
import pytest
import torch

import workloads
from tests._parity import OUT_TOL, compare_layer, to_cpu_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(cuda_device):
    import int4_expert_ffn_sigmoid_b200 as m
    return m


def run_stack(moe, x, stacked, shape, flags=0):
    L = stacked["router_w"].shape[0]
    T = x.shape[0]
    idx = torch.empty((L, T, shape.K), dtype=torch.int32, device=x.device)
    w = torch.empty((L, T, shape.K), dtype=torch.float32, device=x.device)
    # the fused kernel wherever it serves the call (opt-in: the default runs one layer call per layer)
    outs = moe.stack_forward(x, stacked, shape, flags=flags | moe.MOE_DEBUG_CHECK | moe.MOE_STACK_FUSED, topk_idx=idx,
                             topk_w=w)
    torch.cuda.synchronize()
    return outs, idx, w


def layer_of(stacked, l):
    return {k: v[l] for k, v in stacked.items()}


def check_stack(moe, x, stacked, shape, residual, flags=0, rounded=False, layers_cpu=None, sample=None):
    f = flags | (moe.MOE_ADD_RESIDUAL if residual else 0)
    L = stacked["router_w"].shape[0]
    assert moe.stack_path(shape, x.shape[0], L, f | moe.MOE_STACK_FUSED) == moe.MOE_PATH_FUSED_STACK
    outs, idx, w = run_stack(moe, x, stacked, shape, f)
    worst = 0.0
    for l in range(L):
        inp = x if l == 0 else outs[l - 1]
        cpu = layers_cpu[l] if layers_cpu is not None else to_cpu_layer(layer_of(stacked, l))
        r = compare_layer(inp, outs[l], idx[l], w[l], cpu, shape, residual, sample=sample, rounded=rounded)
        worst = max(worst, r["max_rel_l2"])
    print(f"T={x.shape[0]} L={L} worst per-token rel L2 {worst:.3e}")
    return outs, idx, w


@pytest.fixture(scope="module")
def nano_stack(moe, cuda_device):
    wl = workloads.WORKLOADS["nano_decode_stack"]
    layers = [workloads.make_layer(wl.shape, wl.wid, l, cuda_device, wl.bias_mode) for l in range(wl.layers)]
    stacked = moe.stack_layers(layers)
    del layers
    cpu = [to_cpu_layer(layer_of(stacked, l)) for l in range(wl.layers)]
    return wl, stacked, cpu


@pytest.mark.parametrize("T", [1, 2, 3, 4, 16, 64])
def test_nano_decode_stack_fused(moe, cuda_device, nano_stack, T):
    wl, stacked, cpu = nano_stack
    x = workloads.make_x(wl.shape, T, wl.wid, device=cuda_device)
    outs, _, _ = check_stack(moe, x, stacked, wl.shape, residual=True, layers_cpu=cpu)
    assert torch.isfinite(outs.float()).all()


def test_lookahead_changes_no_bit(moe, cuda_device, nano_stack):
    wl, stacked, _ = nano_stack
    f = moe.MOE_ADD_RESIDUAL
    for T in (1, 64):
        x = workloads.make_x(wl.shape, T, wl.wid, batch=3, device=cuda_device)
        a, ia, wa = run_stack(moe, x, stacked, wl.shape, f)
        b, ib, wb = run_stack(moe, x, stacked, wl.shape, f | moe.MOE_LOOKAHEAD)
        assert torch.equal(a, b) and torch.equal(ia, ib) and torch.equal(wa, wb)


def test_stack_batch_independence_and_permutation(moe, cuda_device, nano_stack):
    wl, stacked, _ = nano_stack
    f = moe.MOE_ADD_RESIDUAL
    T = 40
    x = workloads.make_x(wl.shape, T, wl.wid, batch=4, device=cuda_device)
    out, _, _ = run_stack(moe, x, stacked, wl.shape, f)
    perm = torch.randperm(T, generator=torch.Generator().manual_seed(7)).to(cuda_device)
    outp, _, _ = run_stack(moe, x[perm].contiguous(), stacked, wl.shape, f)
    assert torch.equal(outp, out[:, perm])
    for t0, sub in ((0, 1), (9, 17), (39, 1)):
        o1, _, _ = run_stack(moe, x[t0:t0 + sub].contiguous(), stacked, wl.shape, f)
        assert torch.equal(o1, out[:, t0:t0 + sub])


SHAPES = [
    dict(H=256, E=8, K=8, I=256, Is=0, scale=1.0, L=3),      # K = E, no shared expert
    dict(H=512, E=40, K=3, I=256, Is=256, scale=1.3, L=4),   # E not a multiple of 8
    dict(H=1024, E=33, K=1, I=512, Is=768, scale=2.5, L=2),  # K = 1, a 768-wide shared expert (slices 512 + 256)
    dict(H=768, E=256, K=8, I=256, Is=512, scale=2.5, L=2),  # 256 experts, top-8
]


@pytest.mark.parametrize("case", range(len(SHAPES)))
@pytest.mark.parametrize("T", [1, 7, 17, 64])
@pytest.mark.parametrize("raw", [False, True])
def test_stack_shapes(moe, cuda_device, case, T, raw):
    c = SHAPES[case]
    shape = workloads.LayerShape(c["H"], c["E"], c["K"], c["I"], c["Is"], c["scale"])
    layers = [workloads.make_layer(shape, 400 + case, l, cuda_device, "uniform", raw_codes=raw) for l in range(c["L"])]
    if raw:  # larger router weights so raw-code experts still see a spread of scores
        for layer in layers:
            layer["router_w"].mul_(5)
    stacked = moe.stack_layers(layers)
    x = workloads.make_x(shape, T, 400 + case, device=cuda_device)
    residual = (T + case) % 2 == 0
    check_stack(moe, x, stacked, shape, residual, rounded=True)


@pytest.mark.parametrize("T", [1, 32])
def test_large_layer_fused(moe, cuda_device, T):
    wl = workloads.WORKLOADS["large_layer"]
    layer = workloads.make_layer(wl.shape, wl.wid, 0, cuda_device, wl.bias_mode)
    stacked = moe.stack_layers([layer])
    del layer
    x = workloads.make_x(wl.shape, T, wl.wid, device=cuda_device)
    check_stack(moe, x, stacked, wl.shape, residual=False)


def test_per_layer_path_beyond_64_tokens(moe, cuda_device, nano_stack):
    wl, stacked, _ = nano_stack
    sub = {k: v[:3].contiguous() for k, v in stacked.items()}
    T = 100
    assert moe.stack_path(wl.shape, T, 3) == moe.MOE_PATH_PER_LAYER
    x = workloads.make_x(wl.shape, T, wl.wid, batch=6, device=cuda_device)
    outs, _, _ = run_stack(moe, x, sub, wl.shape, moe.MOE_ADD_RESIDUAL)
    inp = x
    for l in range(3):
        ref = moe.layer_forward(inp, layer_of(sub, l), wl.shape, flags=moe.MOE_ADD_RESIDUAL)
        assert torch.equal(outs[l], ref)
        inp = ref


def test_fused_stall_reports_timeout_then_recovers(moe, cuda_device, nano_stack):
    wl, stacked, _ = nano_stack
    sub = {k: v[:4].contiguous() for k, v in stacked.items()}
    x = workloads.make_x(wl.shape, 16, wl.wid, batch=8, device=cuda_device)
    f = moe.MOE_ADD_RESIDUAL | moe.MOE_DEBUG_CHECK | moe.MOE_STACK_FUSED
    ws = torch.empty(moe.stack_workspace_bytes(wl.shape, 16, 4, f), dtype=torch.uint8, device=cuda_device)
    good = moe.stack_forward(x, sub, wl.shape, workspace=ws, flags=f).clone()
    assert moe.device_status(ws) == 0
    with pytest.raises(moe.MoeError) as err:
        moe.stack_forward(x, sub, wl.shape, workspace=ws, flags=f | moe.MOE_TEST_STALL)
    assert err.value.status == moe.MOE_ERR_DEVICE_CHECK
    assert moe.device_status(ws) & moe.MOE_DEVSTAT_TIMEOUT
    again = moe.stack_forward(x, sub, wl.shape, workspace=ws, flags=f)
    torch.cuda.synchronize()
    assert moe.device_status(ws) == 0
    assert torch.equal(again, good)
