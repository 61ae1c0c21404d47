"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Every workload of the layer is covered: the Nano layer at T=16, the 23-layer
Nano decode stack at T in {1,4,16,64} (compared layer by layer, the oracle fed
the GPU's bf16 input of that layer), Nano prefill at T=4096, Zipf-skewed
routing at T=16384, and the 256-expert top-8 layer at T in {1,32,512}.  Large
cases check routing on every token and outputs on sampled tokens.  Edge cases:
ragged T, raw int4 codes (code -8), no shared expert, K=1, K=E, E not a
multiple of 32, exact ties, NaN bias, maximum H, batch independence and token
permutation (bit-exact).
"""
import numpy as np
import pytest
import torch

import workloads
from tests._parity import OUT_F32_TOL, compare_layer, sample_tokens, tile_cover, to_cpu_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(cuda_device):
    import int4_expert_ffn_sigmoid_b200 as m
    return m


def run(moe, x, layer, shape, residual=False, flags=0):
    T = x.shape[0]
    idx = torch.empty((T, shape.K), dtype=torch.int32, device=x.device)
    w = torch.empty((T, shape.K), dtype=torch.float32, device=x.device)
    f = flags | (moe.MOE_ADD_RESIDUAL if residual else 0) | moe.MOE_DEBUG_CHECK
    out = moe.layer_forward(x, layer, shape, flags=f, topk_idx=idx, topk_w=w)
    torch.cuda.synchronize()
    return out, idx, w


def check(moe, x, layer, shape, residual=False, sample=None, flags=0, layer_cpu=None, **kw):
    out, idx, w = run(moe, x, layer, shape, residual, flags)
    r = compare_layer(x, out, idx, w, layer_cpu or to_cpu_layer(layer), shape, residual, sample, **kw)
    print(f"T={x.shape[0]} flags={flags} {r}")
    return out, idx, w, r


def test_nano_layer_t16(moe, cuda_device):
    wl = workloads.WORKLOADS["nano_layer_t16"]
    layer = workloads.make_layer(wl.shape, wl.wid, 0, cuda_device, wl.bias_mode)
    x = workloads.make_x(wl.shape, 16, wl.wid, device=cuda_device)
    cpu = to_cpu_layer(layer)
    check(moe, x, layer, wl.shape, layer_cpu=cpu)
    _, _, _, r = check(moe, x, layer, wl.shape, flags=moe.MOE_OUT_F32, layer_cpu=cpu, tol=OUT_F32_TOL)
    assert r["max_rel_l2"] < 5e-4


@pytest.mark.parametrize("T", [1, 4, 16, 64])
def test_nano_decode_stack(moe, cuda_device, T):
    wl = workloads.WORKLOADS["nano_decode_stack"]
    x = workloads.make_x(wl.shape, T, wl.wid, device=cuda_device)
    x0 = x.clone()
    for l in range(wl.layers):
        layer = workloads.make_layer(wl.shape, wl.wid, l, cuda_device, wl.bias_mode)
        x, _, _, r = check(moe, x, layer, wl.shape, residual=True)
        del layer
    assert torch.isfinite(x.float()).all()
    assert not torch.equal(x, x0)


def work_unit_sample(moe, shape, T, idx, n, seed, extra=()):
    """Checked tokens of a full-size case: at least one token of every work
    unit of the expert kernels that ran (every 128-token tile of every bucket
    on the tensor-core path; every 16-token piece of every bucket, which
    covers the 32-token tasks too, on the weight-streaming paths), every
    multi-unit bucket's last token, head and tail tokens and a seeded draw."""
    path = moe.layer_path(shape, T)
    tile = 128 if path == moe.MOE_PATH_TENSOR_CORE else 16
    cover = tile_cover(idx.cpu().numpy(), shape.E, tile, shape.Is > 0)
    return np.union1d(cover, sample_tokens(T, n, seed, extra))


def test_nano_prefill_t4096(moe, cuda_device):
    wl = workloads.WORKLOADS["nano_prefill_t4096"]
    layer = workloads.make_layer(wl.shape, wl.wid, 0, cuda_device, wl.bias_mode)
    x = workloads.make_x(wl.shape, 4096, wl.wid, device=cuda_device)
    out, idx, w = run(moe, x, layer, wl.shape)
    sample = work_unit_sample(moe, wl.shape, 4096, idx, 40, 1)
    r = compare_layer(x, out, idx, w, to_cpu_layer(layer), wl.shape, False, sample)
    print("prefill", r)
    loads = torch.bincount(idx.flatten().long(), minlength=64)
    assert int(loads.min()) > 0            # zero bias: every expert receives tokens


def test_nano_zipf_t16384(moe, cuda_device):
    wl = workloads.WORKLOADS["nano_zipf_t16384"]
    layer = workloads.make_layer(wl.shape, wl.wid, 0, cuda_device, wl.bias_mode)
    x = workloads.make_x(wl.shape, 16384, wl.wid, device=cuda_device)
    out, idx, w = run(moe, x, layer, wl.shape)
    idx_np = idx.cpu().numpy()
    loads = np.bincount(idx_np.reshape(-1), minlength=64)
    hot = np.nonzero(idx_np == np.argmax(loads))[0][:3]
    cold = np.nonzero(idx_np == np.argmin(loads))[0][:3]
    sample = work_unit_sample(moe, wl.shape, 16384, idx, 32, 2, extra=np.concatenate([hot, cold]))
    r = compare_layer(x, out, idx, w, to_cpu_layer(layer), wl.shape, False, sample)
    print("zipf loads", sorted(loads.tolist(), reverse=True)[:5], "...", sorted(loads.tolist())[:3], r)
    assert loads.max() > 2000 and loads.min() < 200


@pytest.mark.parametrize("T,n", [(1, 1), (32, 8), (512, 10)])
def test_large_layer(moe, cuda_device, T, n):
    wl = workloads.WORKLOADS["large_layer"]
    layer = workloads.make_layer(wl.shape, wl.wid, 0, cuda_device, wl.bias_mode)
    x = workloads.make_x(wl.shape, T, wl.wid, device=cuda_device)
    out, idx, w = run(moe, x, layer, wl.shape)
    r = compare_layer(x, out, idx, w, to_cpu_layer(layer), wl.shape, False, work_unit_sample(moe, wl.shape, T, idx, n, 3))
    print(f"large T={T}", r)


# --- edge cases on small shapes -------------------------------------------------

SMALL = [
    dict(H=128, E=40, K=3, I=128, Is=128, scale=1.3),
    dict(H=256, E=8, K=8, I=256, Is=0, scale=1.0),     # K = E, no shared expert
    dict(H=384, E=33, K=1, I=128, Is=256, scale=2.5),  # K = 1, E not a multiple of 32
    dict(H=128, E=256, K=8, I=128, Is=128, scale=2.5),
]


@pytest.mark.parametrize("case", range(len(SMALL)))
@pytest.mark.parametrize("T", [1, 3, 17, 64, 65, 300])
@pytest.mark.parametrize("raw", [False, True])
def test_small_shapes(moe, cuda_device, case, T, raw):
    c = SMALL[case]
    shape = workloads.LayerShape(c["H"], c["E"], c["K"], c["I"], c["Is"], c["scale"])
    layer = workloads.make_layer(shape, 200 + case, 0, cuda_device, "uniform", raw_codes=raw)
    if raw:  # larger router weights so raw-code experts still see a spread of scores
        layer["router_w"].mul_(5)
    x = workloads.make_x(shape, T, 200 + case, device=cuda_device)
    cpu = to_cpu_layer(layer)
    res = T % 2 == 1
    of32, _, _, _ = check(moe, x, layer, shape, residual=res, flags=moe.MOE_OUT_F32, layer_cpu=cpu,
                          tol=OUT_F32_TOL)
    # the bf16 output is the round-to-nearest-even of that same f32 sum, bit for bit
    ob16, _, _ = run(moe, x, layer, shape, residual=res)
    assert torch.equal(ob16, of32.to(torch.bfloat16))


def test_force_flags_same_result(moe, cuda_device):
    c = SMALL[0]
    shape = workloads.LayerShape(c["H"], c["E"], c["K"], c["I"], c["Is"], c["scale"])
    layer = workloads.make_layer(shape, 210, 0, cuda_device)
    x = workloads.make_x(shape, 40, 210, device=cuda_device)
    a, _, _ = run(moe, x, layer, shape)
    b, _, _ = run(moe, x, layer, shape, flags=moe.MOE_FORCE_DECODE)
    assert torch.equal(a, b)  # T <= 64 takes the small-batch path anyway
    for f in (moe.MOE_FORCE_PREFILL, moe.MOE_FORCE_DECODE):
        check(moe, x, layer, shape, flags=f | moe.MOE_OUT_F32, tol=OUT_F32_TOL)


def test_tensor_core_path_small_batch(moe, cuda_device):
    """MOE_FORCE_PREFILL runs the tensor-core grouped GEMMs at small T: ragged
    token tiles (1..130 tokens), several experts per tile list, K = 8."""
    shape = workloads.LayerShape(H=512, E=16, K=8, I=256, Is=384, routed_scaling=2.5)
    layer = workloads.make_layer(shape, 215, 0, cuda_device)
    cpu = to_cpu_layer(layer)
    for T in (1, 5, 130):
        x = workloads.make_x(shape, T, 215, device=cuda_device)
        check(moe, x, layer, shape, flags=moe.MOE_FORCE_PREFILL | moe.MOE_OUT_F32, layer_cpu=cpu,
              tol=OUT_F32_TOL, residual=True)


def test_max_hidden(moe, cuda_device):
    shape = workloads.LayerShape(H=16384, E=8, K=2, I=128, Is=128, routed_scaling=1.0)
    layer = workloads.make_layer(shape, 220, 0, cuda_device)
    cpu = to_cpu_layer(layer)
    for T in (5, 70):
        x = workloads.make_x(shape, T, 220, device=cuda_device)
        check(moe, x, layer, shape, layer_cpu=cpu)


def test_split_router(moe, cuda_device):
    """Router weights of 2 MB or more take the split small-batch router (a
    logits kernel over slices of the hidden dimension, then the cluster
    selection): a ragged last slice (22 blocks of 128 in slices of 3), E not a
    multiple of 32, and a token's result independent of the rest of the batch."""
    shape = workloads.LayerShape(H=2816, E=200, K=6, I=128, Is=128, routed_scaling=2.5)
    assert moe.kernel_launches(shape, 9) == 5
    layer = workloads.make_layer(shape, 250, 0, cuda_device)
    cpu = to_cpu_layer(layer)
    x = workloads.make_x(shape, 64, 250, device=cuda_device)
    out, _, _, _ = check(moe, x, layer, shape, layer_cpu=cpu)
    for t0, sub in ((0, 1), (5, 9), (40, 24)):
        o1, _, _ = run(moe, x[t0:t0 + sub].contiguous(), layer, shape)
        assert torch.equal(o1, out[t0:t0 + sub])
    # large batches: the tensor-core router logits (a 128-token tile and a
    # ragged one of 22; expert tiles of 128 and 72) feeding the large router's
    # selection
    assert moe.kernel_launches(shape, 150) == 7
    x = workloads.make_x(shape, 150, 250, batch=1, device=cuda_device)
    out, _, _, _ = check(moe, x, layer, shape, layer_cpu=cpu, sample=sample_tokens(150, 40, 5))
    o1, _, _ = run(moe, x[10:110].contiguous(), layer, shape)
    assert torch.equal(o1, out[10:110])


@pytest.mark.parametrize("H", [1152, 2176, 2304])
def test_streaming_kernel_variants(moe, cuda_device, H):
    """Hidden sizes above 1024: gate/up takes the register-ring kernels when H
    is not a multiple of 256 (whole-row activations up to 2048, slices beyond)
    and the TMA-ring kernel otherwise; the down projection takes its TMA-ring
    kernel (I and Is multiples of 256; a 768-wide I gives slices of 512 and
    256).  T = 100 runs the large-batch router with the weight-streaming
    kernels (H not a multiple of 256, or MOE_FORCE_DECODE)."""
    shape = workloads.LayerShape(H=H, E=16, K=3, I=768, Is=256, routed_scaling=1.5)
    layer = workloads.make_layer(shape, 260, 0, cuda_device)
    cpu = to_cpu_layer(layer)
    for T in (5, 40, 100):
        x = workloads.make_x(shape, T, 260, device=cuda_device)
        flags = moe.MOE_FORCE_DECODE if T > 64 else 0
        check(moe, x, layer, shape, layer_cpu=cpu, residual=True, flags=flags)


def test_hot_expert_many_chunks(moe, cuda_device):
    """Large-batch weight streaming with 32-token tasks: one expert picked by
    every token (a bucket of 150 = 4 x 32 + 22 tokens), next to the shared
    expert's chunks and the light buckets of the other experts."""
    wl = workloads.WORKLOADS["nano_layer_t16"]
    layer = workloads.make_layer(wl.shape, wl.wid, 0, cuda_device, wl.bias_mode)
    layer["router_bias"][7] = 5.0
    x = workloads.make_x(wl.shape, 150, wl.wid, batch=9, device=cuda_device)
    assert moe.layer_path(wl.shape, 150, moe.MOE_FORCE_DECODE) == moe.MOE_PATH_LARGE_STREAMING
    out, idx, w = run(moe, x, layer, wl.shape, flags=moe.MOE_FORCE_DECODE)
    sample = np.union1d(tile_cover(idx.cpu().numpy(), wl.shape.E, 16, True), sample_tokens(150, 40, 7))
    compare_layer(x, out, idx, w, to_cpu_layer(layer), wl.shape, False, sample)
    assert idx[:, 0].eq(7).all()


def test_large_intermediate_values(moe, cuda_device):
    """Inputs around +-300 drive the SwiGLU intermediate to ~1e5 (beyond fp16's
    65504 unless it is stored scaled); outputs stay finite and match."""
    wl = workloads.WORKLOADS["nano_layer_t16"]
    layer = workloads.make_layer(wl.shape, wl.wid, 0, cuda_device, wl.bias_mode)
    cpu = to_cpu_layer(layer)
    for T in (3, 100):
        x = workloads.make_x(wl.shape, T, wl.wid, batch=7, device=cuda_device, std=300.0)
        check(moe, x, layer, wl.shape, layer_cpu=cpu, residual=True)


def test_exact_ties_lower_index(moe, cuda_device):
    shape = workloads.LayerShape(H=128, E=8, K=2, I=128, Is=0, routed_scaling=1.0)
    layer = workloads.make_layer(shape, 230, 0, cuda_device)
    layer["router_w"][5] = layer["router_w"][1]
    layer["router_w"][6] = layer["router_w"][1]
    layer["router_bias"][:] = -1.0
    layer["router_bias"][[1, 5, 6]] = 0.5
    x = workloads.make_x(shape, 20, 230, device=cuda_device)
    out, idx, w = run(moe, x, layer, shape)
    assert idx[:, 0].eq(1).all() and idx[:, 1].eq(5).all()
    torch.testing.assert_close(w, torch.full_like(w, 0.5), rtol=1e-6, atol=0)


def test_nan_bias_never_selected(moe, cuda_device):
    shape = workloads.LayerShape(H=128, E=8, K=3, I=128, Is=128, routed_scaling=1.0)
    layer = workloads.make_layer(shape, 240, 0, cuda_device)
    layer["router_bias"][2] = float("nan")
    layer["router_bias"][4] = 10.0
    x = workloads.make_x(shape, 9, 240, device=cuda_device)
    out, idx, _, _ = check(moe, x, layer, shape)
    assert not idx.eq(2).any() and idx[:, 0].eq(4).all()


def test_batch_independence_and_permutation(moe, cuda_device):
    """A token's output does not depend on the rest of the batch, bit for bit,
    within each path: the small-batch path (T <= 64), the large-batch
    weight-streaming path (T = 200 gives ~6 picks per expert) and the
    tensor-core path (forced)."""
    wl = workloads.WORKLOADS["nano_layer_t16"]
    layer = workloads.make_layer(wl.shape, wl.wid, 0, cuda_device, wl.bias_mode)
    cases = ((16, 1, 0, moe.MOE_PATH_SMALL_BATCH), (200, 70, 0, moe.MOE_PATH_LARGE_STREAMING),
             (200, 70, moe.MOE_FORCE_PREFILL, moe.MOE_PATH_TENSOR_CORE))
    for T, sub, flags, path in cases:
        assert moe.layer_path(wl.shape, T, flags) == path
        assert moe.layer_path(wl.shape, sub, flags) == path
        x = workloads.make_x(wl.shape, T, wl.wid, batch=5, device=cuda_device)
        out, _, _ = run(moe, x, layer, wl.shape, flags=flags)
        perm = torch.randperm(T, generator=torch.Generator().manual_seed(T)).to(cuda_device)
        outp, _, _ = run(moe, x[perm].contiguous(), layer, wl.shape, flags=flags)
        assert torch.equal(outp, out[perm])
        for t0 in (0, T // 2, T - sub):
            o1, _, _ = run(moe, x[t0:t0 + sub].contiguous(), layer, wl.shape, flags=flags)
            assert torch.equal(o1, out[t0:t0 + sub])


def test_workspace_reuse_and_stream(moe, cuda_device):
    """Two calls on one workspace, the second on a side stream, are independent."""
    wl = workloads.WORKLOADS["nano_layer_t16"]
    layer = workloads.make_layer(wl.shape, wl.wid, 0, cuda_device, wl.bias_mode)
    m = moe.MoELayer(layer, wl.shape, 300)
    xa = workloads.make_x(wl.shape, 300, wl.wid, batch=1, device=cuda_device)
    xb = workloads.make_x(wl.shape, 7, wl.wid, batch=2, device=cuda_device)
    ra = m(xa).clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        rb = m(xb)
    s.synchronize()
    assert torch.equal(m(xa), ra)
    assert torch.equal(rb, moe.layer_forward(xb, layer, wl.shape))
