"""The C-ABI library without a GPU: it loads, exports every function that
include/moe_int4.h declares, and its host-side validation returns the
documented status codes before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_int4.h")


@pytest.fixture(scope="module")
def moe():
    import __graft_entry__
    __graft_entry__._load_build_module().build()
    import int4_expert_ffn_sigmoid_b200 as m
    return m


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(moe_\w+)\s*\(", text, flags=re.M)))


def test_exports_every_declared_function(moe):
    names = _declared_functions()
    assert set(names) == set(moe.EXPORTED_SYMBOLS), names
    for n in names:
        assert hasattr(moe.lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True, text=True).stdout
    for n in names:
        assert re.search(rf"\bT {n}$", out, flags=re.M), n


def test_struct_layout_matches_c(moe, tmp_path):
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "moe_int4.h"\n'
        "int main(void){printf(\"%zu %zu %zu %zu %zu %zu %zu\\n\", sizeof(moe_cfg_t),"
        " offsetof(moe_cfg_t, routed_scaling), offsetof(moe_cfg_t, flags),"
        " offsetof(moe_cfg_t, workspace), offsetof(moe_cfg_t, workspace_bytes),"
        " offsetof(moe_cfg_t, topk_w_out), sizeof(moe_shared_weights_t));"
        " printf(\"%zu \", offsetof(moe_cfg_t, topp));"
        " printf(\"%zu %zu %zu\\n\", sizeof(moe_stack_weights_t), offsetof(moe_stack_weights_t, s2),"
        " offsetof(moe_stack_weights_t, shared)); return 0;}\n")
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)])
    c_vals = [int(v) for v in subprocess.check_output([str(exe)]).split()]
    cfg = moe.moe_cfg_t
    py_vals = [ctypes.sizeof(cfg), cfg.routed_scaling.offset, cfg.flags.offset, cfg.workspace.offset,
               cfg.workspace_bytes.offset, cfg.topk_w_out.offset, ctypes.sizeof(moe.moe_shared_weights_t),
               cfg.topp.offset,
               ctypes.sizeof(moe.moe_stack_weights_t), moe.moe_stack_weights_t.s2.offset,
               moe.moe_stack_weights_t.shared.offset]
    assert c_vals == py_vals


def test_header_constants_match_binding(moe):
    text = open(HEADER).read()
    for name in ("MOE_STATIC_WORKSPACE_BYTES", "MOE_OUT_F32", "MOE_FORCE_DECODE",
                 "MOE_FORCE_PREFILL", "MOE_ADD_RESIDUAL", "MOE_DEBUG_CHECK",
                 "MOE_PATH_SMALL_BATCH", "MOE_PATH_TENSOR_CORE", "MOE_PATH_LARGE_STREAMING",
                 "MOE_LOOKAHEAD", "MOE_TEST_STALL", "MOE_TEST_BAD_INDEX", "MOE_TRACE", "MOE_DEBUG_POISON",
                 "MOE_DEVSTAT_TIMEOUT", "MOE_DEVSTAT_BAD_EXPERT", "MOE_PATH_FUSED_STACK", "MOE_PATH_PER_LAYER",
                 "MOE_STACK_FUSED", "MOE_WEIGHTS_INT8"):
        m = re.search(rf"#define {name} (.+)", text)
        assert m, name
        expr = m.group(1).split("/*")[0].replace("(size_t)", "").replace("u", "")
        assert eval(expr) == getattr(moe, name), name


def test_version_and_strings(moe):
    assert moe.lib.moe_abi_version() == 2
    assert moe.status_str(0) == "MOE_OK"
    assert moe.status_str(3) == "MOE_ERR_WORKSPACE"
    assert moe.status_str(99) == "MOE_ERR_UNKNOWN"
    assert moe.decode_max_tokens() == 64


def _shape(**kw):
    import workloads
    base = dict(H=1024, E=64, K=2, I=512, Is=2048, routed_scaling=1.0)
    base.update(kw)
    return workloads.LayerShape(**base)


def test_workspace_query(moe):
    a = moe.workspace_bytes(_shape(), 16)
    b = moe.workspace_bytes(_shape(), 4096)
    assert 0 < a < b
    assert a % 256 == 0
    assert moe.workspace_bytes(_shape(H=1000), 16) == 0      # H not a multiple of 128
    assert moe.workspace_bytes(_shape(K=65, E=64), 16) == 0  # K > E
    assert moe.workspace_bytes(_shape(E=300), 16) == 0       # E > 256
    assert moe.workspace_bytes(_shape(), -1) == 0
    assert moe.workspace_bytes(_shape(Is=0), 16) < a         # no shared-expert scratch


def test_kernel_launch_count(moe):
    nano = _shape()
    large = _shape(H=6144, E=256, K=8, I=2048, Is=2048, routed_scaling=2.5)
    assert moe.kernel_launches(nano, 0) == 0
    assert moe.kernel_launches(nano, 16) == 4       # cluster router, gate/up, down, combine
    assert moe.kernel_launches(nano, 4096) == 5     # router, scatter, 2 GEMMs, combine
    assert moe.kernel_launches(nano, 16, moe.MOE_FORCE_PREFILL) == 5
    assert moe.kernel_launches(nano, 4096, moe.MOE_FORCE_DECODE) == 5
    assert moe.kernel_launches(large, 1) == 5       # + the split router's logits kernel
    # weight split, tensor-core router logits, selection, scatter, 2 expert kernels, combine
    assert moe.kernel_launches(large, 512) == 7
    assert moe.kernel_launches(_shape(H=1000), 16) == 0
    assert moe.kernel_launches(nano, (1 << 20) + 1) == 0


def test_workspace_upto_covers_every_smaller_call(moe):
    """A smaller T can need more workspace (the weight-streaming sequence keeps
    f32 h and per-slice partial rows); the _upto query is the maximum over
    every T up to N, checked here against all T."""
    for shape in (_shape(), _shape(H=6144, E=256, K=8, I=2048, Is=2048, routed_scaling=2.5),
                  _shape(H=1152, E=16, K=3, I=768, Is=256)):
        for flags in (0, moe.MOE_FORCE_DECODE, moe.MOE_FORCE_PREFILL):
            for N in (1, 64, 65, 700, 1100, 3000):
                sizes = [moe.workspace_bytes(shape, t, flags) for t in range(N + 1)]
                assert moe.workspace_bytes_upto(shape, N, flags) == max(sizes), (shape, flags, N)
    nano = _shape()
    # the example that needs it: a workspace for 1100 tokens sized at T = 1100 alone is too small
    assert moe.workspace_bytes(nano, 1100) < moe.workspace_bytes(nano, 1000)
    assert moe.workspace_bytes_upto(_shape(H=1000), 16) == 0


def test_path_choice(moe):
    nano = _shape()
    large = _shape(H=6144, E=256, K=8, I=2048, Is=2048, routed_scaling=2.5)
    S, TC, LS = moe.MOE_PATH_SMALL_BATCH, moe.MOE_PATH_TENSOR_CORE, moe.MOE_PATH_LARGE_STREAMING
    assert moe.layer_path(nano, 0) == 0
    assert moe.layer_path(nano, 64) == S
    assert moe.layer_path(nano, 65) == LS             # 130 picks over 64 experts: streaming
    assert moe.layer_path(nano, 1023) == LS           # T*K = 2046 < 32*E = 2048
    assert moe.layer_path(nano, 1024) == TC
    assert moe.layer_path(nano, 4096) == TC
    assert moe.layer_path(nano, 4096, moe.MOE_FORCE_DECODE) == LS
    assert moe.layer_path(nano, 16, moe.MOE_FORCE_PREFILL) == TC
    assert moe.layer_path(nano, 100, moe.MOE_FORCE_PREFILL) == TC
    assert moe.layer_path(_shape(H=1152), 4096) == LS  # H not a multiple of 256
    assert moe.layer_path(large, 512) == LS            # 16 picks per expert
    assert moe.layer_path(large, 1024) == TC


def test_int8_weights_flag(moe):
    """int8 expert weights take int4's kernel sequences where the TMA-ring
    streaming kernels serve the shape (H >= 1024, H, I, Is multiples of 256),
    else the tensor-core sequence at every T; never the fused stack kernel."""
    nano = _shape()
    I8 = moe.MOE_WEIGHTS_INT8
    S, TC, LS = moe.MOE_PATH_SMALL_BATCH, moe.MOE_PATH_TENSOR_CORE, moe.MOE_PATH_LARGE_STREAMING
    for T, path in ((1, S), (16, S), (64, S), (65, LS), (1023, LS), (4096, TC)):
        assert moe.layer_path(nano, T, I8) == path == moe.layer_path(nano, T), T
        assert moe.kernel_launches(nano, T, I8) == moe.kernel_launches(nano, T), T
        assert moe.workspace_bytes(nano, T, I8) == moe.workspace_bytes(nano, T), T
    assert moe.layer_path(nano, 16, I8 | moe.MOE_FORCE_PREFILL) == TC
    assert moe.layer_path(nano, 4096, I8 | moe.MOE_FORCE_DECODE) == LS
    # shapes without int8 streaming kernels: the tensor-core sequence at every T
    small = _shape(H=512, I=256, Is=256)
    for T in (1, 16, 300):
        assert moe.layer_path(small, T, I8) == TC, T
    assert moe.layer_path(small, 16, I8 | moe.MOE_FORCE_DECODE) == 0
    assert _call(moe, small, T=4, flags=I8 | moe.MOE_FORCE_DECODE) == moe.MOE_ERR_UNSUPPORTED
    assert moe.layer_path(_shape(H=1152), 4096, I8) == 0
    assert _call(moe, _shape(H=1152), T=4, flags=I8) == moe.MOE_ERR_UNSUPPORTED
    assert moe.workspace_bytes_upto(small, 300, I8) == moe.workspace_bytes(small, 300, I8)
    for T in (1, 4, 16):
        assert moe.stack_path(nano, T, 23, I8) == moe.MOE_PATH_PER_LAYER
        assert moe.stack_path(nano, T, 23, I8 | moe.MOE_STACK_FUSED) == moe.MOE_PATH_PER_LAYER
    # the binding reads the code width from the weight shapes
    assert moe.weight_flags({"w13": torch.empty(2, 4, 1024, dtype=torch.uint8)}, nano) == I8
    assert moe.weight_flags({"w13": torch.empty(2, 4, 512, dtype=torch.uint8)}, nano) == 0
    with pytest.raises(ValueError):
        moe.weight_flags({"w13": torch.empty(2, 4, 100, dtype=torch.uint8)}, nano)


# Fake device pointers: validation runs before any dereference or CUDA call.
FAKE = 1 << 20


def _call(moe, shape, T=0, ws_bytes=1 << 30, flags=0, x=FAKE, out=FAKE * 64, shared=True,
          cfg_patch=None, ws=FAKE * 256):
    cfg = moe.make_cfg(shape, flags)
    cfg.workspace = ws
    cfg.workspace_bytes = ws_bytes
    if cfg_patch:
        cfg_patch(cfg)
    sh = moe.moe_shared_weights_t(FAKE, FAKE, FAKE, FAKE) if shared else None
    vp = ctypes.c_void_p
    return moe.lib.moe_layer_forward(vp(x), vp(FAKE), vp(FAKE), vp(FAKE), vp(FAKE), vp(FAKE), vp(FAKE),
                                     ctypes.byref(sh) if sh is not None else None, vp(out), T,
                                     ctypes.byref(cfg), None)


def test_forward_validation_codes(moe):
    s = _shape()
    assert _call(moe, s) == 0                                           # T = 0: no-op
    assert _call(moe, s, T=-1) == moe.MOE_ERR_INVALID_ARG
    assert _call(moe, s, x=0) == moe.MOE_ERR_INVALID_ARG                # NULL x
    assert _call(moe, s, x=FAKE + 4) == moe.MOE_ERR_INVALID_ARG         # misaligned
    assert _call(moe, s, shared=False) == moe.MOE_ERR_INVALID_ARG       # Is > 0 needs shared
    assert _call(moe, _shape(Is=0), shared=False) == 0
    assert _call(moe, s, T=4, out=FAKE) == moe.MOE_ERR_INVALID_ARG      # out aliases x
    assert _call(moe, s, T=4, ws_bytes=100) == moe.MOE_ERR_WORKSPACE
    assert _call(moe, s, T=4, ws=0) == moe.MOE_ERR_WORKSPACE
    assert _call(moe, s, ws=FAKE * 256 + 16) == moe.MOE_ERR_INVALID_ARG  # workspace alignment
    assert _call(moe, _shape(H=1000)) == moe.MOE_ERR_UNSUPPORTED
    assert _call(moe, _shape(I=200)) == moe.MOE_ERR_UNSUPPORTED
    assert _call(moe, _shape(K=9, E=64)) == moe.MOE_ERR_UNSUPPORTED
    assert _call(moe, _shape(K=5, E=4)) == moe.MOE_ERR_INVALID_ARG
    assert _call(moe, _shape(routed_scaling=0.0)) == moe.MOE_ERR_INVALID_ARG
    assert _call(moe, s, flags=1 << 12) == moe.MOE_ERR_INVALID_ARG  # an unknown flag

    def topp(v):
        def patch(c):
            c.topp = v
        return patch
    assert _call(moe, s, cfg_patch=topp(float("nan"))) == moe.MOE_ERR_INVALID_ARG
    assert _call(moe, s, cfg_patch=topp(-0.5)) == moe.MOE_ERR_INVALID_ARG
    assert _call(moe, s, cfg_patch=topp(0.7)) == 0
    assert _call(moe, s, flags=moe.MOE_FORCE_DECODE | moe.MOE_FORCE_PREFILL) == moe.MOE_ERR_INVALID_ARG

    def bad_size(c):
        c.struct_size = 12
    assert _call(moe, s, cfg_patch=bad_size) == moe.MOE_ERR_INVALID_ARG
    assert moe.lib.moe_layer_forward(None, None, None, None, None, None, None, None, None, 0, None,
                                     None) == moe.MOE_ERR_INVALID_ARG


def _stack_call(moe, shape, T=0, L=2, x=None, outs=None, ws=None, ws_bytes=1 << 30, flags=0, null_field=None):
    w = moe.moe_stack_weights_t()
    for f in ("router_w", "router_bias", "w13", "s13", "w2", "s2"):
        setattr(w, f, FAKE)
    w.shared.w13 = w.shared.s13 = w.shared.w2 = w.shared.s2 = FAKE
    if null_field:
        setattr(w, null_field, None)
    cfg = moe.make_cfg(shape, flags)
    cfg.workspace = FAKE * 256 if ws is None else ws
    cfg.workspace_bytes = ws_bytes
    vp = ctypes.c_void_p
    return moe.lib.moe_stack_forward(vp(FAKE * 2 if x is None else x), ctypes.byref(w), L,
                                     vp(FAKE * 64 if outs is None else outs), T, ctypes.byref(cfg), None)


def test_stack_validation_codes(moe):
    """moe_stack_forward checks its arguments before launching anything."""
    s = _shape()
    assert _stack_call(moe, s) == 0                                               # T = 0: no-op
    assert _stack_call(moe, s, L=0) == moe.MOE_ERR_INVALID_ARG
    assert _stack_call(moe, s, L=129) == moe.MOE_ERR_INVALID_ARG                  # more layers than supported
    assert _stack_call(moe, s, T=-1) == moe.MOE_ERR_INVALID_ARG
    assert _stack_call(moe, s, flags=moe.MOE_OUT_F32) == moe.MOE_ERR_INVALID_ARG  # outputs feed the next layer
    assert _stack_call(moe, s, null_field="w2") == moe.MOE_ERR_INVALID_ARG
    assert _stack_call(moe, s, x=FAKE * 2 + 8) == moe.MOE_ERR_INVALID_ARG         # misaligned
    assert _stack_call(moe, s, T=4, outs=FAKE * 2) == moe.MOE_ERR_INVALID_ARG     # outs overlaps x
    assert _stack_call(moe, s, T=4, ws_bytes=100) == moe.MOE_ERR_WORKSPACE
    assert _stack_call(moe, s, flags=1 << 12) == moe.MOE_ERR_INVALID_ARG
    assert moe.stack_workspace_bytes(s, 64, 23) > 0
    assert moe.stack_workspace_bytes(s, 64, 0) == 0
    # without a GPU the fused kernel cannot be resident: every call takes the per-layer path
    assert moe.stack_path(s, 0, 23) == 0
    assert moe.stack_path(s, 16, 23, moe.MOE_STACK_FUSED) in (moe.MOE_PATH_FUSED_STACK, moe.MOE_PATH_PER_LAYER)
    # without MOE_STACK_FUSED every stack runs one layer call per layer (measured faster at every T)
    for T in (1, 4, 16, 64):
        assert moe.stack_path(s, T, 23) == moe.MOE_PATH_PER_LAYER
    assert moe.stack_path(s, 4, 1) == moe.MOE_PATH_PER_LAYER
    assert moe.stack_path(s, 100, 23, moe.MOE_STACK_FUSED) == moe.MOE_PATH_PER_LAYER  # beyond 64 tokens
    assert moe.stack_path(s, 16, 23, moe.MOE_FORCE_DECODE) == moe.MOE_PATH_PER_LAYER
