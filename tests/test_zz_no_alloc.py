"""The entry point for callers that cannot allocate device memory.

moe_layer_forward_static_ws serves callers that cannot call cudaMalloc (a
plug-in whose host framework owns all device memory, code that must not
allocate while a stream is being captured): its scratch memory is a fixed
array inside the library instead of a caller-provided workspace.  These tests
call it through the C ABI and check it against moe_layer_forward, twice in a
row on the shared array, and check that oversized calls are refused.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from tests._parity import OUT_TOL, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(cuda_device):
    import int4_expert_ffn_sigmoid_b200 as m
    return m


def _static_call(moe, x, layer, shape, out, flags=0):
    cfg = moe.make_cfg(shape, flags)  # no workspace
    sh = moe.moe_shared_weights_t()
    if shape.Is > 0:
        sh.w13, sh.s13 = layer["sh_w13"].data_ptr(), layer["sh_s13"].data_ptr()
        sh.w2, sh.s2 = layer["sh_w2"].data_ptr(), layer["sh_s2"].data_ptr()
    vp = ctypes.c_void_p
    stream = torch.cuda.current_stream().cuda_stream
    return moe.lib.moe_layer_forward_static_ws(
        vp(x.data_ptr()), vp(layer["router_w"].data_ptr()), vp(layer["router_bias"].data_ptr()),
        vp(layer["w13"].data_ptr()), vp(layer["s13"].data_ptr()), vp(layer["w2"].data_ptr()),
        vp(layer["s2"].data_ptr()), ctypes.byref(sh), vp(out.data_ptr()), int(x.shape[0]),
        ctypes.byref(cfg), vp(stream))


@pytest.mark.parametrize("T", [16, 64, 300])
def test_static_workspace_matches_regular_entry_point(moe, cuda_device, T):
    wl = workloads.WORKLOADS["nano_layer_t16"]
    layer = workloads.make_layer(wl.shape, wl.wid, 0, cuda_device, wl.bias_mode)
    xs = [workloads.make_x(wl.shape, T, wl.wid, batch=b, device=cuda_device) for b in (11, 12)]
    assert moe.workspace_bytes(wl.shape, T) <= moe.MOE_STATIC_WORKSPACE_BYTES
    for x in xs:  # two calls in a row on the one shared array
        ref = moe.layer_forward(x, layer, wl.shape)
        out = torch.empty_like(ref)
        assert _static_call(moe, x, layer, wl.shape, out) == moe.MOE_OK
        torch.cuda.synchronize()
        err = rel_l2(out, ref.double().cpu().numpy())
        assert np.all(np.isfinite(err)) and err.max() <= OUT_TOL
        # the same kernels on the same inputs: the same result, bit for bit
        assert torch.equal(out, ref)


def test_static_workspace_rejects_oversized_calls(moe, cuda_device):
    wl = workloads.WORKLOADS["nano_layer_t16"]
    T = 16384
    assert moe.workspace_bytes(wl.shape, T) > moe.MOE_STATIC_WORKSPACE_BYTES
    layer = workloads.make_layer(wl.shape, wl.wid, 0, cuda_device, wl.bias_mode)
    x = workloads.make_x(wl.shape, T, wl.wid, device=cuda_device)
    out = torch.full((T, wl.shape.H), 7.0, dtype=torch.bfloat16, device=cuda_device)
    assert _static_call(moe, x, layer, wl.shape, out) == moe.MOE_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)  # nothing was launched
