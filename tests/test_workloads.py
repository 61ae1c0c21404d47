"""The synthetic workloads: shapes, sizes against the pages, determinism."""
import os

import numpy as np
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _sizes():
    vals = {}
    with open(os.path.join(GOLDEN, "page_sizes.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, v, tol, *_ = line.split()
            vals[k] = (float(v), float(tol))
    return vals


def test_sizes_match_pages():
    s = _sizes()
    L = workloads.LARGE
    eb = workloads.expert_bytes(L)
    assert eb == 3 * 6144 * 2048 // 2 + (2 * 2048 + 6144) * 4
    v, tol = s["large_expert_mb"]
    assert abs(eb / 1e6 - v) <= tol
    v, tol = s["large_token_cold_gb"]
    assert abs(75 * 8 * eb / 1e9 - v) <= tol
    v, tol = s["nano_routed_experts_gb"]
    n_layers = int(s["nano_moe_layers"][0])
    assert n_layers == workloads.WORKLOADS["nano_decode_stack"].layers
    assert abs(n_layers * 64 * workloads.expert_bytes(workloads.NANO) / 1e9 - v) <= tol


def test_generator_shapes_and_determinism():
    shape = workloads.LayerShape(H=64, E=10, K=2, I=32, Is=48, routed_scaling=1.0)
    a = workloads.make_layer(shape, 5, 1)
    b = workloads.make_layer(shape, 5, 1)
    c = workloads.make_layer(shape, 5, 2)
    assert a["w13"].shape == (10, 64, 32) and a["s13"].shape == (10, 64)
    assert a["w2"].shape == (10, 64, 16) and a["s2"].shape == (10, 64)
    assert a["sh_w13"].shape == (96, 32) and a["sh_w2"].shape == (64, 24)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    assert not torch.equal(a["w13"], c["w13"])
    assert float(a["router_bias"].abs().max()) <= 0.1
    x = workloads.make_x(shape, 5, 5)
    assert x.dtype == torch.bfloat16 and x.shape == (5, 64)
    assert torch.equal(x, workloads.make_x(shape, 5, 5))
    assert not torch.equal(x, workloads.make_x(shape, 5, 5, batch=1))


def test_raw_codes_cover_minus_eight():
    shape = workloads.LayerShape(H=64, E=2, K=1, I=32, Is=0, routed_scaling=1.0)
    a = workloads.make_layer(shape, 6, raw_codes=True)
    codes = oracle.unpack_int4(a["w13"].reshape(-1).numpy(), a["w13"].numel() * 2)
    assert set(np.unique(codes).tolist()) == set(range(-8, 8))


def test_zipf_bias_file():
    b = workloads.load_zipf_bias(64)
    assert b.shape == (64,)
    # popularity decreases with the expert index over the hot head
    assert float(b[0]) > float(b[1]) > float(b[2]) > float(b[3])
