"""The algorithmic bytes and flops that bench.py divides by its measured
times (the roofline numerators), counted again from the tensors themselves.

Bytes: the stored size of every tensor a layer pass reads (router weights and
bias, the touched routed experts' code rows and row scales, the shared
expert) plus the bf16 activations in and out.  Flops: two per multiply-add of
every matrix-vector product the layer definition performs for one token,
taken from the weight matrices' shapes (a code row of n elements is n/2 bytes
at int4, n bytes at int8).
"""
import pytest

import bench
import workloads

SHAPES = [
    workloads.LayerShape(H=256, E=8, K=2, I=128, Is=256, routed_scaling=1.0),
    workloads.LayerShape(H=512, E=16, K=4, I=256, Is=0, routed_scaling=2.5),
]


def tensor_bytes(layer, e=None, part=None):
    if part == "router":
        return layer["router_w"].nbytes + layer["router_bias"].nbytes
    if part == "shared":
        return sum(layer[k].nbytes for k in ("sh_w13", "sh_s13", "sh_w2", "sh_s2")) if "sh_w13" in layer else 0
    if part == "gate_up":
        return layer["w13"][e].nbytes + layer["s13"][e].nbytes
    if part == "down":
        return layer["w2"][e].nbytes + layer["s2"][e].nbytes
    raise ValueError(part)


def matvec_macs(layer, wbits):
    """Multiply-adds per token of each matrix, from the stored shapes."""
    per = 8 // wbits  # code elements per byte
    rw = layer["router_w"]
    w13, w2 = layer["w13"][0], layer["w2"][0]
    macs = {"router": rw.shape[0] * rw.shape[1],
            "gate_up": w13.shape[0] * w13.shape[1] * per,
            "down": w2.shape[0] * w2.shape[1] * per}
    if "sh_w13" in layer:
        macs["sh_gate_up"] = layer["sh_w13"].shape[0] * layer["sh_w13"].shape[1] * per
        macs["sh_down"] = layer["sh_w2"].shape[0] * layer["sh_w2"].shape[1] * per
    else:
        macs["sh_gate_up"] = macs["sh_down"] = 0
    return macs


@pytest.mark.parametrize("wbits", [4, 8])
@pytest.mark.parametrize("si", range(len(SHAPES)))
def test_layer_weight_bytes_are_the_stored_sizes(si, wbits):
    shape = SHAPES[si]
    layer = workloads.make_layer(shape, 40 + si, 0, "cpu", wbits=wbits)
    lb = workloads.layer_weight_bytes(shape, wbits)
    assert lb["router"] == tensor_bytes(layer, part="router")
    assert lb["shared"] == tensor_bytes(layer, part="shared")
    for e in (0, shape.E - 1):
        assert lb["expert"] == tensor_bytes(layer, e, "gate_up") + tensor_bytes(layer, e, "down")
    assert lb["experts_total"] == sum(tensor_bytes(layer, e, "gate_up") + tensor_bytes(layer, e, "down")
                                      for e in range(shape.E))


@pytest.mark.parametrize("wbits", [4, 8])
@pytest.mark.parametrize("si", range(len(SHAPES)))
def test_step_bytes_and_flops(si, wbits):
    shape = SHAPES[si]
    layer = workloads.make_layer(shape, 50 + si, 0, "cpu", wbits=wbits)
    T, uniq = 5, [3, shape.E, 1]  # touched routed experts in each of three layers
    nbytes, flops = bench.step_bytes_flops(shape, T, uniq, wbits)
    per_layer = [tensor_bytes(layer, part="router") + tensor_bytes(layer, part="shared")
                 + sum(tensor_bytes(layer, e, "gate_up") + tensor_bytes(layer, e, "down") for e in range(u))
                 + 2 * T * shape.H * 2 for u in uniq]
    assert nbytes == sum(per_layer)
    m = matvec_macs(layer, wbits)
    per_token = m["router"] + shape.K * (m["gate_up"] + m["down"]) + m["sh_gate_up"] + m["sh_down"]
    assert flops == len(uniq) * 2 * T * per_token


@pytest.mark.parametrize("wbits", [4, 8])
@pytest.mark.parametrize("si", range(len(SHAPES)))
def test_stage_work_splits_the_expert_weights(si, wbits):
    """Each stage counts its own weight matrices (and scales) once per
    touched expert, and the flops of its products; activations and expert
    outputs on top."""
    shape = SHAPES[si]
    layer = workloads.make_layer(shape, 60 + si, 0, "cpu", wbits=wbits)
    H, K, I, Is = shape.H, shape.K, shape.I, shape.Is
    T, u = 7, 4
    m = matvec_macs(layer, wbits)
    sh = "sh_w13" in layer
    gb, gf = bench.stage_work("gate_up", shape, T, u, wbits)
    sh13 = (layer["sh_w13"].nbytes + layer["sh_s13"].nbytes) if sh else 0
    acts13 = T * H * 2 + T * K * I * 2 + T * Is * 2  # x read once, h written (16-bit)
    assert gb == u * tensor_bytes(layer, 0, "gate_up") + sh13 + acts13
    assert gf == 2 * T * (K * m["gate_up"] + m["sh_gate_up"])
    db, df = bench.stage_work("down", shape, T, u, wbits)
    sh2 = (layer["sh_w2"].nbytes + layer["sh_s2"].nbytes) if sh else 0
    acts2 = T * K * I * 2 + T * Is * 2 + (T * K + (T if sh else 0)) * H * 4  # h read, y written (f32)
    assert db == u * tensor_bytes(layer, 0, "down") + sh2 + acts2
    assert df == 2 * T * (K * m["down"] + m["sh_down"])
    # the two stages' weights are one layer's touched experts and shared expert
    lb = workloads.layer_weight_bytes(shape, wbits)
    assert (gb - acts13) + (db - acts2) == u * lb["expert"] + lb["shared"]
