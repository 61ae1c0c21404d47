"""Failure detection on the device: a bounded wait that runs out.

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
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_stalled_wait_reports_timeout_then_recovers(moe, cuda_device, case):
    what, shape, T, mode = CASES[case]
    base = moe.MOE_FORCE_PREFILL if mode == "prefill" else 0
    path = moe.MOE_PATH_TENSOR_CORE if mode == "prefill" else moe.MOE_PATH_SMALL_BATCH
    assert moe.layer_path(shape, T, base) == path, what
    layer = workloads.make_layer(shape, 300 + case, 0, cuda_device)
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
