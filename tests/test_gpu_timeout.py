"""Failure detection on the device: a bounded wait that runs out, a
corrupted routing index, and a poisoned workspace.

MOE_TEST_STALL makes one role of each expert kernel that takes part wait ~1 ms
on a flag that nothing sets.  The kernel then takes its timeout path while its
copies and MMAs are in flight: it stops, drains what it issued (bounded waits
that ignore the abort), releases tensor memory and exits, and the status word
records MOE_DEVSTAT_TIMEOUT.  Under MOE_DEBUG_CHECK the call reports
MOE_ERR_DEVICE_CHECK.  No fault and no hang: the context stays usable, and the
next normal call must give the same result, bit for bit, as before the
stalled one.
"""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(cuda_device):
    import int4_expert_ffn_sigmoid_b200 as m
    return m


CASES = [
    # (description, shape, T, flags): the kernels that take part
    ("tensor-core grouped GEMMs", workloads.LayerShape(H=512, E=16, K=8, I=256, Is=384, routed_scaling=2.5), 130,
     "prefill"),
    ("TMA-ring weight-streaming kernels", workloads.LayerShape(H=1024, E=64, K=2, I=512, Is=2048, routed_scaling=1.0),
     16, "decode"),
    ("tcgen05 streaming gate/up kernel", workloads.LayerShape(H=1024, E=64, K=2, I=512, Is=2048, routed_scaling=1.0),
     400, "decode"),
    ("tensor-core grouped GEMMs, int8 weights", workloads.LayerShape(H=512, E=16, K=8, I=256, Is=384, routed_scaling=2.5),
     130, "int8"),
    ("TMA-ring weight-streaming kernels, int8 weights",
     workloads.LayerShape(H=1024, E=64, K=2, I=512, Is=2048, routed_scaling=1.0), 16, "int8"),
]


def _wbits(mode):
    return 8 if mode == "int8" else 4


@pytest.mark.parametrize("case", range(len(CASES)))
def test_stalled_wait_reports_timeout_then_recovers(moe, cuda_device, case):
    what, shape, T, mode = CASES[case]
    if mode == "int8":
        base = moe.MOE_WEIGHTS_INT8
        path = moe.MOE_PATH_TENSOR_CORE if shape.H < 1024 else moe.MOE_PATH_SMALL_BATCH
    else:
        base = moe.MOE_FORCE_PREFILL if mode == "prefill" else (moe.MOE_FORCE_DECODE if T > 64 else 0)
        path = moe.MOE_PATH_TENSOR_CORE if mode == "prefill" else (moe.MOE_PATH_LARGE_STREAMING if T > 64 else
                                                                      moe.MOE_PATH_SMALL_BATCH)
    assert moe.layer_path(shape, T, base) == path, what
    layer = workloads.make_layer(shape, 300 + case, 0, cuda_device, wbits=_wbits(mode))
    x = workloads.make_x(shape, T, 300 + case, device=cuda_device)
    ws = moe.new_workspace(shape, T, cuda_device, base)
    good = moe.layer_forward(x, layer, shape, workspace=ws, flags=base | moe.MOE_DEBUG_CHECK).clone()
    assert moe.device_status(ws) == 0
    with pytest.raises(moe.MoeError) as err:
        moe.layer_forward(x, layer, shape, workspace=ws, flags=base | moe.MOE_TEST_STALL | moe.MOE_DEBUG_CHECK)
    assert err.value.status == moe.MOE_ERR_DEVICE_CHECK, what
    assert moe.device_status(ws) & moe.MOE_DEVSTAT_TIMEOUT, what
    # the context is intact and the next call runs normally
    again = moe.layer_forward(x, layer, shape, workspace=ws, flags=base | moe.MOE_DEBUG_CHECK)
    torch.cuda.synchronize()
    assert moe.device_status(ws) == 0
    assert torch.equal(again, good), what


# --- a corrupted routing index and a poisoned workspace --------------------------

PATHS = [
    # (description, shape, T, flags)
    ("small-batch kernels", workloads.LayerShape(1024, 64, 2, 512, 2048, 1.0), 16, 0),
    ("tensor-core kernels", workloads.LayerShape(512, 16, 8, 256, 384, 2.5), 130, "prefill"),
    ("large-batch streaming kernels", workloads.LayerShape(1024, 64, 2, 512, 2048, 1.0), 150, "decode"),
    ("large-batch streaming, tcgen05 gate/up", workloads.LayerShape(1024, 64, 2, 512, 2048, 1.0), 400, "decode"),
    ("tensor-core kernels, int8 weights", workloads.LayerShape(512, 16, 8, 256, 384, 2.5), 130, "int8"),
    ("large-batch streaming kernels, int8 weights", workloads.LayerShape(1024, 64, 2, 512, 2048, 1.0), 150, "int8"),
]


def _flags(moe, f):
    return {0: 0, "prefill": moe.MOE_FORCE_PREFILL, "decode": moe.MOE_FORCE_DECODE, "int8": moe.MOE_WEIGHTS_INT8}[f]


@pytest.mark.parametrize("case", range(len(PATHS)))
def test_bad_routing_index_is_caught(moe, cuda_device, case):
    """The router hands an out-of-range expert index to the kernels that
    follow (MOE_TEST_BAD_INDEX); their range checks report it and nothing
    reads or writes out of bounds: the next normal call is bit-identical."""
    what, shape, T, f = PATHS[case]
    base = _flags(moe, f)
    layer = workloads.make_layer(shape, 320 + case, 0, cuda_device, wbits=_wbits(f))
    x = workloads.make_x(shape, T, 320 + case, device=cuda_device)
    ws = moe.new_workspace(shape, T, cuda_device, base)
    good = moe.layer_forward(x, layer, shape, workspace=ws, flags=base | moe.MOE_DEBUG_CHECK).clone()
    with pytest.raises(moe.MoeError) as err:
        moe.layer_forward(x, layer, shape, workspace=ws, flags=base | moe.MOE_TEST_BAD_INDEX | moe.MOE_DEBUG_CHECK)
    assert err.value.status == moe.MOE_ERR_DEVICE_CHECK, what
    assert moe.device_status(ws) & moe.MOE_DEVSTAT_BAD_EXPERT, what
    again = moe.layer_forward(x, layer, shape, workspace=ws, flags=base | moe.MOE_DEBUG_CHECK)
    torch.cuda.synchronize()
    assert torch.equal(again, good), what


@pytest.mark.parametrize("case", range(len(PATHS)))
def test_poisoned_workspace_changes_nothing(moe, cuda_device, case):
    """Every scratch byte the kernels read was written first in the same call:
    filling the workspace with 0xFF (NaN / -1) beforehand changes no output bit."""
    what, shape, T, f = PATHS[case]
    base = _flags(moe, f)
    layer = workloads.make_layer(shape, 330 + case, 0, cuda_device, wbits=_wbits(f))
    x = workloads.make_x(shape, T, 330 + case, device=cuda_device)
    a = moe.layer_forward(x, layer, shape, flags=base | moe.MOE_DEBUG_CHECK)
    b = moe.layer_forward(x, layer, shape, flags=base | moe.MOE_DEBUG_POISON | moe.MOE_DEBUG_CHECK)
    torch.cuda.synchronize()
    assert torch.equal(a, b), what


def test_fused_stack_bad_index_and_poison(moe, cuda_device):
    shape = workloads.LayerShape(1024, 64, 2, 512, 2048, 1.0)
    layers = [workloads.make_layer(shape, 340, l, cuda_device) for l in range(3)]
    stacked = moe.stack_layers(layers)
    x = workloads.make_x(shape, 24, 340, device=cuda_device)
    f = moe.MOE_ADD_RESIDUAL | moe.MOE_DEBUG_CHECK | moe.MOE_STACK_FUSED
    assert moe.stack_path(shape, 24, 3, f) == moe.MOE_PATH_FUSED_STACK
    ws = torch.empty(moe.stack_workspace_bytes(shape, 24, 3, f), dtype=torch.uint8, device=cuda_device)
    good = moe.stack_forward(x, stacked, shape, workspace=ws, flags=f).clone()
    with pytest.raises(moe.MoeError) as err:
        moe.stack_forward(x, stacked, shape, workspace=ws, flags=f | moe.MOE_TEST_BAD_INDEX)
    assert err.value.status == moe.MOE_ERR_DEVICE_CHECK
    assert moe.device_status(ws) & moe.MOE_DEVSTAT_BAD_EXPERT
    poisoned = moe.stack_forward(x, stacked, shape, workspace=ws, flags=f | moe.MOE_DEBUG_POISON)
    torch.cuda.synchronize()
    assert torch.equal(poisoned, good)
