"""Pins of the CPU oracle against facts fixed outside it.

Each test targets a mistake the oracle could plausibly contain: the nibble
order or sign of the int4 codes, the orientation of a weight matrix, gate and
up swapped, the bias leaking into the routing weights, a dropped scaling
factor, the shared expert being scaled, the tie-break, NaN handling.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads
from oracle import dense_masked

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --- int4 code layout -------------------------------------------------------

# 4-bit two's complement, written out code by code.
CODE_OF_NIBBLE = {0x0: 0, 0x1: 1, 0x2: 2, 0x3: 3, 0x4: 4, 0x5: 5, 0x6: 6, 0x7: 7,
                  0x8: -8, 0x9: -7, 0xA: -6, 0xB: -5, 0xC: -4, 0xD: -3, 0xE: -2, 0xF: -1}


def test_unpack_every_byte():
    """Byte j holds element 2j in its low nibble and 2j+1 in its high nibble."""
    row = np.arange(256, dtype=np.uint8)
    codes = oracle.unpack_int4(row, 512)
    for b in range(256):
        assert codes[2 * b] == CODE_OF_NIBBLE[b & 0xF], b
        assert codes[2 * b + 1] == CODE_OF_NIBBLE[b >> 4], b


def test_unpack_literal_examples():
    assert list(oracle.unpack_int4(np.array([0x21], np.uint8), 2)) == [1, 2]
    assert list(oracle.unpack_int4(np.array([0x8F], np.uint8), 2)) == [-1, -8]
    assert list(oracle.unpack_int4(np.array([0x7A, 0x09], np.uint8), 4)) == [-6, 7, -7, 0]


def test_dense_decoder_matches_table():
    codes = dense_masked.decode_int4(np.arange(256, dtype=np.uint8)[None, :])[0]
    for b in range(256):
        assert codes[2 * b] == CODE_OF_NIBBLE[b & 0xF]
        assert codes[2 * b + 1] == CODE_OF_NIBBLE[b >> 4]


# --- quantiser (input generator) -------------------------------------------

def test_quantiser_bounds_and_roundtrip():
    g = torch.Generator().manual_seed(5)
    w = torch.randn(37, 96, generator=g) * 0.02
    w[3] = 0.0                       # all-zero row
    packed, scale = workloads.quantize_rows_int4(w)
    assert packed.shape == (37, 48) and packed.dtype == torch.uint8
    codes = np.stack([oracle.unpack_int4(packed[r].numpy(), 96) for r in range(37)])
    assert codes.min() >= -8 and codes.max() <= 7
    s = scale.numpy().astype(np.float64)
    deq = codes * s[:, None]
    err = np.abs(w.numpy().astype(np.float64) - deq)
    assert np.all(err <= s[:, None] / 2 * (1 + 1e-6) + 1e-12)
    # the largest-magnitude element of every nonzero row maps to +-7
    for r in range(37):
        if r == 3:
            assert s[r] == 0 and np.all(codes[r] == 0)
            continue
        j = int(np.argmax(np.abs(w[r].numpy())))
        assert abs(codes[r, j]) == 7
        assert np.isclose(s[r], np.abs(w[r].numpy()).max() / 7, rtol=1e-6)


def test_quantiser_int8_bounds_and_roundtrip():
    g = torch.Generator().manual_seed(6)
    w = torch.randn(29, 80, generator=g) * 0.02
    w[5] = 0.0
    codes8, scale = workloads.quantize_rows_int8(w)
    assert codes8.shape == (29, 80) and codes8.dtype == torch.uint8
    codes = codes8.numpy().view(np.int8).astype(np.int64)
    assert codes.min() >= -127 and codes.max() <= 127
    s = scale.numpy().astype(np.float64)
    err = np.abs(w.numpy().astype(np.float64) - codes * s[:, None])
    assert np.all(err <= s[:, None] / 2 * (1 + 1e-6) + 1e-12)
    for r in range(29):
        if r == 5:
            assert s[r] == 0 and np.all(codes[r] == 0)
            continue
        j = int(np.argmax(np.abs(w[r].numpy())))
        assert abs(codes[r, j]) == 127
        assert np.isclose(s[r], np.abs(w[r].numpy()).max() / 127, rtol=1e-6)


# --- int8 code layout ---------------------------------------------------------

def test_int8_decode_literal():
    """Byte j of an int8 row is element j in two's complement."""
    raw = np.array([[0x00, 0x7F, 0x80, 0xFF, 0x01, 0xFE]], np.uint8)
    assert dense_masked.decode_codes(raw, 6)[0].tolist() == [0, 127, -128, -1, 1, -2]
    assert dense_masked.decode_codes(np.array([[0x8F]], np.uint8), 2)[0].tolist() == [-1, -8]


def test_int8_expert_hand_example():
    """One int8 expert at x = (1, -2), power-of-two scales, extreme codes:
    gate (127/128, 2), up (-1, -254/128), h = (-silu(127/128), silu(2) * -254/128),
    y = (127 h0 - 128 h1, (h0 - h1) / 2)."""
    silu = lambda z: z / (1 + math.exp(-z))
    b = lambda v: v & 0xFF
    w13 = np.array([[b(127), 0], [0, b(-128)], [b(-128), 0], [0, b(127)]], np.uint8)
    s13 = np.array([2.0 ** -7, 2.0 ** -7, 2.0 ** -7, 2.0 ** -7], np.float32)
    w2 = np.array([[b(127), b(-128)], [1, b(-1)]], np.uint8)
    s2 = np.array([1.0, 0.5], np.float32)
    h, y = oracle.expert_ffn(np.array([1.0, -2.0]), w13, s13, w2, s2)
    h_exp = [silu(127 / 128) * -1.0, silu(2.0) * (-254 / 128)]
    np.testing.assert_allclose(h, h_exp, rtol=1e-15)
    np.testing.assert_allclose(y, [127 * h_exp[0] - 128 * h_exp[1], 0.5 * (h_exp[0] - h_exp[1])], rtol=1e-14)


def test_int8_layer_equals_int4_recoded():
    """An int4 layer re-encoded one code per byte gives the same outputs, bit
    for bit: the int8 path only changes how codes are read."""
    shape = workloads.LayerShape(H=32, E=6, K=3, I=16, Is=8, routed_scaling=2.5)
    layer4 = workloads.make_layer(shape, 91, device="cpu", raw_codes=True)
    table = np.array([CODE_OF_NIBBLE[v] for v in range(16)], np.int16)

    def recode(packed):
        p = packed.numpy()
        codes = np.stack([table[p & 0xF], table[p >> 4]], axis=-1).reshape(*p.shape[:-1], 2 * p.shape[-1])
        return torch.from_numpy((codes & 0xFF).astype(np.uint8))
    layer8 = dict(layer4)
    for k in ("w13", "w2", "sh_w13", "sh_w2"):
        layer8[k] = recode(layer4[k])
    assert oracle.weight_bits(layer8["w13"], shape.H) == 8
    x = workloads.make_x(shape, 6, 91)
    r4 = oracle.moe_tokens(x, layer4, shape)
    r8 = oracle.moe_tokens(x, layer8, shape)
    np.testing.assert_array_equal(r8["out"], r4["out"])
    np.testing.assert_array_equal(r8["idx"], r4["idx"])
    d8, _ = dense_masked.moe_dense(x, layer8, shape)
    np.testing.assert_allclose(d8, r4["out"], rtol=1e-12, atol=1e-13)


# --- selection --------------------------------------------------------------

@pytest.mark.parametrize("K", [1, 2, 3])
def test_selection_bruteforce_subsets(K):
    """Top-K = the unique K-subset with the largest sum of keys (distinct keys)."""
    rng = np.random.default_rng(K)
    E = 8
    for trial in range(50):
        scores = rng.uniform(0.01, 0.99, size=(1, E))
        bias = rng.uniform(-0.2, 0.2, size=E).astype(np.float32)
        idx, margin = oracle.select_topk(scores, bias, K)
        key = scores[0] + bias.astype(np.float64)
        best = max(itertools.combinations(range(E), K), key=lambda S: sum(key[list(S)]))
        assert sorted(idx[0].tolist()) == sorted(best)
        # listed in decreasing key order
        assert all(key[idx[0][i]] >= key[idx[0][i + 1]] for i in range(K - 1))
        rest = sorted(set(range(E)) - set(best), key=lambda e: -key[e])
        assert math.isclose(margin[0], key[idx[0][-1]] - key[rest[0]], rel_tol=0, abs_tol=1e-15)


def test_selection_ties_prefer_lower_index():
    # identical router rows and equal biases give exactly equal keys
    shape = workloads.LayerShape(H=8, E=6, K=2, I=2, Is=0, routed_scaling=1.0)
    W = torch.zeros(6, 8)
    W[1] = W[4] = torch.tensor([0.3, -0.1, 0.2, 0.0, 0.5, 0.1, -0.2, 0.4])
    W[2] = W[5] = torch.tensor([0.1, 0.1, 0.1, 0.1, 0.1, 0.1, 0.1, 0.1])
    x = torch.ones(1, 8).to(torch.bfloat16)
    bias = torch.zeros(6)
    r = oracle.route(x, W, bias, shape.K, 1.0)
    assert r["idx"][0].tolist() == [1, 4]
    assert r["margin"][0] > 0
    r3 = oracle.route(x, W, bias, 3, 1.0)
    assert r3["idx"][0].tolist() == [1, 4, 2]
    assert r3["margin"][0] == 0.0        # expert 5 ties expert 2


def test_selection_nan_is_minus_infinity():
    scores = np.array([[0.9, np.nan, 0.1, 0.5]])
    idx, _ = oracle.select_topk(scores, np.zeros(4, np.float32), 2)
    assert idx[0].tolist() == [0, 3]
    idx, _ = oracle.select_topk(scores, np.zeros(4, np.float32), 4)
    assert idx[0].tolist() == [0, 3, 2, 1]


def test_weights_sum_to_scaling_factor():
    shape = workloads.LayerShape(H=64, E=16, K=4, I=8, Is=0, routed_scaling=2.5)
    layer = workloads.make_layer(shape, 77, device="cpu", experts=[])
    x = workloads.make_x(shape, 33, 77)
    r = oracle.route(x, layer["router_w"], layer["router_bias"], shape.K, shape.routed_scaling)
    np.testing.assert_allclose(r["weights"].sum(1), 2.5, rtol=0, atol=1e-12)
    # weights are proportional to the unbiased sigmoid scores of the selection
    for t in range(33):
        s = r["scores"][t, r["idx"][t]]
        np.testing.assert_allclose(r["weights"][t] / s, r["weights"][t, 0] / s[0], rtol=1e-12)
    # scores are the logistic function of the logits
    np.testing.assert_allclose(r["scores"] * (1 + np.exp(-r["logits"])), 1.0, rtol=1e-14)


# --- hand-worked example ----------------------------------------------------

def _hand_example():
    ln3 = np.float32(math.log(3.0))
    shape = workloads.LayerShape(H=2, E=4, K=2, I=2, Is=2, routed_scaling=2.0)
    W = np.array([[ln3, 0], [0, 0], [0, np.float32(ln3 / 2)], [2, 1]], np.float32)
    bias = np.array([0, 0.1, 0.3, 0], np.float32)

    def pk(rows):
        return workloads.pack_int4(torch.tensor(rows, dtype=torch.int8)).numpy()
    w13 = np.zeros((4, 4, 1), np.uint8); s13 = np.ones((4, 4), np.float32)
    w2 = np.zeros((4, 2, 1), np.uint8); s2 = np.ones((4, 2), np.float32)
    w13[0] = pk([[1, 0], [0, 1], [2, 0], [0, -1]]); s13[0] = [1, 1, 0.5, 1]
    w2[0] = pk([[1, 0], [0, -3]]); s2[0] = [1, 0.5]
    w13[1] = pk([[0, 1], [1, 1], [1, 1], [-8, 0]]); s13[1] = [1, 1, 1, 0.25]
    w2[1] = pk([[2, 0], [1, 1]]); s2[1] = [1, 1]
    for e in (2, 3):
        w13[e] = pk([[7, 7]] * 4)
        w2[e] = pk([[7, 7]] * 2)
    layer = dict(router_w=W, router_bias=bias, w13=w13, s13=s13, w2=w2, s2=s2,
                 sh_w13=pk([[1, 0], [0, 0], [0, -1], [1, 0]]), sh_s13=np.ones(4, np.float32),
                 sh_w2=pk([[1, 1], [-1, 0]]), sh_s2=np.array([0.5, 1], np.float32))
    x = torch.tensor([[1.0, -2.0]]).to(torch.bfloat16)
    return shape, layer, x


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, *v = line.split()
            vals[k] = [float(t) for t in v]
    return vals


@pytest.mark.parametrize("residual", [False, True])
def test_hand_example(residual):
    """4 experts, top-2, hand-derived closed form (tests/golden/hand_example_e4_k2.txt).

    Expected values assume sigmoid(ln 3) = 3/4 exactly; the router holds the
    f32 value nearest ln 3, which moves results by ~1e-8 relative, hence 1e-7."""
    g = _read_golden("hand_example_e4_k2.txt")
    shape, layer, x = _hand_example()
    r = oracle.moe_tokens(x, layer, shape, residual=residual)
    assert r["idx"][0].tolist() == [int(v) for v in g["idx"]]
    np.testing.assert_allclose(r["weights"][0], g["weights"], rtol=1e-7)
    np.testing.assert_allclose(r["margin"][0], g["margin"][0], rtol=1e-6)
    expect = np.array([g["out0"][0], g["out1"][0]]) + (np.array([1.0, -2.0]) if residual else 0)
    np.testing.assert_allclose(r["out"][0], expect, rtol=1e-7, atol=1e-9)
    # the dense-masked formulation agrees
    dense, _ = dense_masked.moe_dense(x, layer, shape, residual)
    np.testing.assert_allclose(dense[0], expect, rtol=1e-7, atol=1e-9)


def test_hand_example_expert_h():
    """Intermediate of expert 0 at x=(1,-2): h = (silu(1), 2*silu(-2))."""
    shape, layer, x = _hand_example()
    silu = lambda z: z / (1 + math.exp(-z))
    h, y = oracle.expert_ffn(np.array([1.0, -2.0]), layer["w13"][0], layer["s13"][0],
                             layer["w2"][0], layer["s2"][0])
    np.testing.assert_allclose(h, [silu(1), 2 * silu(-2)], rtol=1e-15)
    np.testing.assert_allclose(y, [silu(1), -3 * silu(-2)], rtol=1e-15)


# --- dense-masked formulation vs per-token oracle ---------------------------

@pytest.mark.parametrize("case", [
    dict(H=32, E=8, K=2, I=16, Is=24, scale=1.0, T=7, residual=False, raw=False),
    dict(H=64, E=16, K=4, I=32, Is=0, scale=2.5, T=5, residual=True, raw=False),
    dict(H=32, E=6, K=6, I=8, Is=8, scale=1.5, T=3, residual=False, raw=True),
    dict(H=16, E=5, K=1, I=4, Is=6, scale=1.0, T=9, residual=True, raw=True),
    dict(H=32, E=8, K=2, I=16, Is=24, scale=1.0, T=7, residual=False, raw=False, wbits=8),
    dict(H=16, E=5, K=3, I=6, Is=10, scale=2.5, T=6, residual=True, raw=True, wbits=8),
])
def test_dense_masked_equals_per_token(case):
    shape = workloads.LayerShape(case["H"], case["E"], case["K"], case["I"], case["Is"], case["scale"])
    layer = workloads.make_layer(shape, 90, device="cpu", raw_codes=case["raw"], wbits=case.get("wbits", 4))
    x = workloads.make_x(shape, case["T"], 90)
    r = oracle.moe_tokens(x, layer, shape, residual=case["residual"])
    dense, R = dense_masked.moe_dense(x, layer, shape, case["residual"])
    np.testing.assert_allclose(r["out"], dense, rtol=1e-12, atol=1e-13)
    for t in range(case["T"]):
        assert sorted(np.nonzero(R[t])[0].tolist()) == sorted(r["idx"][t].tolist())
    # token subsets give the same rows
    sub = oracle.moe_tokens(x, layer, shape, residual=case["residual"], tokens=[case["T"] - 1, 0])
    np.testing.assert_allclose(sub["out"], r["out"][[case["T"] - 1, 0]], rtol=0, atol=0)


# --- identity-like expert -----------------------------------------------------

def test_identity_like_expert_reproduces_input():
    """silu(z) - silu(-z) = z, so gate rows +-c*e_i, up rows selecting a
    constant-1 channel and down rows (e_i - e_{I/2+i}) * d give
    y_i = c*d*u*x_i.  Every expert is this identity, so whatever the routing,
    out_i = routed_scaling * c*d*u * x_i for i < I/2 and 0 elsewhere."""
    H, E, K, I = 16, 4, 2, 8
    shape = workloads.LayerShape(H, E, K, I, 0, 2.5)
    c0 = H - 1
    q13 = np.zeros((2 * I, H), np.int8)
    q2 = np.zeros((H, I), np.int8)
    for i in range(I // 2):
        q13[i, i] = 7
        q13[I // 2 + i, i] = -7
        q2[i, i] = 7
        q2[i, I // 2 + i] = -7
    q13[I:, c0] = 7
    s_g, s_u, s_d = np.float32(0.125), np.float32(1 / 7), np.float32(0.3)
    s13 = np.concatenate([np.full(I, s_g), np.full(I, s_u)]).astype(np.float32)
    s2 = np.full(H, s_d, np.float32)
    p13 = workloads.pack_int4(torch.tensor(q13)).numpy()
    p2 = workloads.pack_int4(torch.tensor(q2)).numpy()
    g = torch.Generator().manual_seed(3)
    layer = dict(router_w=torch.randn(E, H, generator=g).numpy() * 0.5,
                 router_bias=np.zeros(E, np.float32),
                 w13=np.stack([p13] * E), s13=np.stack([s13] * E),
                 w2=np.stack([p2] * E), s2=np.stack([s2] * E))
    x = torch.randn(6, H, generator=g)
    x[:, c0] = 1.0
    x = x.to(torch.bfloat16)
    r = oracle.moe_tokens(x, layer, shape)
    xf = oracle.bf16_bits_to_f64(x)
    factor = 2.5 * (7 * float(s_g)) * (7 * float(s_d)) * (7 * float(s_u))
    np.testing.assert_allclose(r["out"][:, :I // 2], factor * xf[:, :I // 2], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(r["out"][:, I // 2:], 0.0, atol=1e-15)


# --- relabelling --------------------------------------------------------------

def test_expert_relabelling_invariance():
    shape = workloads.LayerShape(H=32, E=8, K=3, I=16, Is=8, routed_scaling=1.7)
    layer = workloads.make_layer(shape, 91, device="cpu")
    x = workloads.make_x(shape, 6, 91)
    r = oracle.moe_tokens(x, layer, shape)
    perm = np.array([5, 2, 7, 0, 1, 6, 3, 4])
    layer_p = dict(layer)
    for k in ("router_w", "router_bias", "w13", "s13", "w2", "s2"):
        layer_p[k] = layer[k][torch.from_numpy(perm)]
    rp = oracle.moe_tokens(x, layer_p, shape)
    np.testing.assert_allclose(rp["out"], r["out"], rtol=1e-13, atol=1e-15)
    for t in range(6):
        assert sorted(perm[rp["idx"][t]].tolist()) == sorted(r["idx"][t].tolist())


def test_override_with_own_choice_is_identity():
    shape = workloads.LayerShape(H=32, E=8, K=2, I=16, Is=8, routed_scaling=1.0)
    layer = workloads.make_layer(shape, 92, device="cpu")
    x = workloads.make_x(shape, 4, 92)
    r = oracle.moe_tokens(x, layer, shape)
    r2 = oracle.moe_tokens(x, layer, shape, idx_override=r["idx"])
    np.testing.assert_array_equal(r2["out"], r["out"])


def test_override_evaluates_the_forced_experts():
    """idx_override replaces the selection: the oracle then evaluates exactly
    the forced experts, weighted by their unbiased sigmoid scores normalised
    over the forced set (the bias only ever decides a selection), which the
    dense-masked formulation computes independently.  The forced experts are
    each token's K lowest keys, so an override that were ignored, or that only
    reordered the router's own choice, would fail."""
    shape = workloads.LayerShape(H=32, E=8, K=3, I=16, Is=8, routed_scaling=2.5)
    layer = workloads.make_layer(shape, 93, device="cpu")
    x = workloads.make_x(shape, 6, 93)
    own = oracle.moe_tokens(x, layer, shape)
    rt = oracle.route(x, layer["router_w"], layer["router_bias"], shape.K, shape.routed_scaling)
    keys = rt["scores"] + layer["router_bias"].double().numpy()[None, :]
    forced = np.argsort(keys, axis=1, kind="stable")[:, :shape.K][:, ::-1].astype(np.int32).copy()
    assert not np.any(np.isin(forced, own["idx"]).all(axis=1))
    r = oracle.moe_tokens(x, layer, shape, residual=True, idx_override=forced)
    np.testing.assert_array_equal(r["idx"], forced)
    s = rt["scores"][np.arange(6)[:, None], forced]
    np.testing.assert_allclose(r["weights"], 2.5 * s / s.sum(axis=1, keepdims=True), rtol=1e-14)
    ref, R = dense_masked.moe_dense(x, layer, shape, residual=True, forced=forced)
    np.testing.assert_allclose(r["out"], ref, rtol=0, atol=1e-12 * np.abs(ref).max())
    assert np.abs(r["out"] - oracle.moe_tokens(x, layer, shape, residual=True)["out"]).max() > 1e-3
    # a subset of tokens with their own overrides
    tok = np.array([4, 1], np.int32)
    r2 = oracle.moe_tokens(x, layer, shape, residual=True, tokens=tok, idx_override=forced[tok])
    np.testing.assert_array_equal(r2["out"], r["out"][tok])


def test_sigmoid_saturation_finite():
    shape = workloads.LayerShape(H=8, E=4, K=2, I=2, Is=0, routed_scaling=1.0)
    W = np.full((4, 8), 500.0, np.float32)
    W[1] *= -1
    x = torch.ones(1, 8).to(torch.bfloat16)
    r = oracle.route(x, W, np.zeros(4, np.float32), 2, 1.0)
    assert np.all(np.isfinite(r["weights"]))
    assert r["idx"][0].tolist() == [0, 2]


# --- adaptive expert top-p (opt-in) ---------------------------------------------

def _route_with_scores(scores, K, scale=1.0, topp=0.0):
    """oracle.route on one token whose sigmoid scores are (close to) `scores`:
    x = [1, 0], router row e = [logit(s_e), 0], bias 0."""
    s = np.asarray(scores, np.float64)
    W = np.zeros((len(s), 2), np.float32)
    W[:, 0] = np.log(s / (1.0 - s))
    x = torch.tensor([[1.0, 0.0]]).to(torch.bfloat16)
    return oracle.route(x, W, np.zeros(len(s), np.float32), K, scale, topp)


def test_topp_hand_worked():
    """Scores 0.5, 0.3, 0.2 (all three picked, K = 3): with p = 0.7 the two
    best carry 0.8 >= 0.7 of the mass, so the third is dropped and the weights
    become scale * (0.5, 0.3) / 0.8; with p = 0.45 the best alone reaches it;
    with p = 0.81 all three are needed; p = 1 (or 0) is plain top-K."""
    for p, kept, w in ((0.7, [0, 1], [0.625, 0.375]), (0.45, [0], [1.0]), (0.81, [0, 1, 2], [0.5, 0.3, 0.2]),
                       (1.0, [0, 1, 2], [0.5, 0.3, 0.2]), (0.0, [0, 1, 2], [0.5, 0.3, 0.2])):
        r = _route_with_scores([0.5, 0.3, 0.2], 3, scale=2.5, topp=p)
        n = len(kept)
        assert r["idx"][0, :n].tolist() == kept, (p, r["idx"])
        assert np.all(r["idx"][0, n:] == -1) and np.all(r["weights"][0, n:] == 0.0)
        np.testing.assert_allclose(r["weights"][0, :n], 2.5 * np.array(w), rtol=2e-6)


def test_topp_brute_force_over_subsets():
    """The kept picks are the smallest subset of the K picks whose scores reach
    p of their total, the highest-mass one among subsets of that size (checked
    against every subset), kept in selection order; their weights are
    normalised over the kept set."""
    rng = np.random.default_rng(11)
    for trial in range(200):
        E, K = 7, int(rng.integers(1, 6))
        s = rng.uniform(0.05, 0.95, E)
        p = float(rng.uniform(0.05, 0.99))
        r = _route_with_scores(s, K, scale=1.3, topp=p)
        sc = r["scores"][0]
        picks = np.argsort(-sc, kind="stable")[:K]  # zero bias: the K best scores
        total = sc[picks].sum()
        best = None
        for size in range(1, K + 1):
            cands = [c for c in itertools.combinations(picks.tolist(), size) if sc[list(c)].sum() >= p * total]
            if cands:
                best = max(cands, key=lambda c: sc[list(c)].sum())
                break
        got = [e for e in r["idx"][0] if e >= 0]
        assert set(got) == set(best), (trial, got, best)
        assert got == [e for e in picks if e in set(best)]  # selection order kept
        np.testing.assert_allclose(r["weights"][0, :len(got)], 1.3 * sc[got] / sc[got].sum(), rtol=1e-12)


def test_topp_layer_matches_dense_formulation():
    shape = workloads.LayerShape(H=32, E=8, K=4, I=16, Is=8, routed_scaling=2.5)
    layer = workloads.make_layer(shape, 94, device="cpu")
    layer["router_w"].mul_(20)  # a wide spread of scores, so the top-p drops picks
    x = workloads.make_x(shape, 9, 94)
    for p in (0.3, 0.6, 0.9):
        r = oracle.moe_tokens(x, layer, shape, residual=True, topp=p)
        assert np.any(r["idx"] == -1)
        ref, R = dense_masked.moe_dense(x, layer, shape, residual=True, topp=p)
        np.testing.assert_allclose(r["out"], ref, rtol=0, atol=1e-12 * np.abs(ref).max())
        # the override path evaluates the same kept picks (-1 = dropped)
        r2 = oracle.moe_tokens(x, layer, shape, residual=True, topp=p, idx_override=r["idx"])
        np.testing.assert_array_equal(r2["out"], r["out"])
    plain = oracle.moe_tokens(x, layer, shape, residual=True)
    np.testing.assert_array_equal(oracle.moe_tokens(x, layer, shape, residual=True, topp=1.0)["out"], plain["out"])
