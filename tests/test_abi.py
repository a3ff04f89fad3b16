"""CPU-side checks of the C ABI: the library loads, exports every function
include/vggt_attn.h declares, and rejects bad arguments on the host before
touching any device (so these run without a GPU)."""
import ctypes
import os
import re

import pytest

import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def V():
    import __graft_entry__
    __graft_entry__._build_module().build()
    import vit_attention_b200
    return vit_attention_b200


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(vggt_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_debug_build_exports_every_declared_function(V):
    import __graft_entry__
    lib_path = __graft_entry__._build_module().build(debug=True)
    assert lib_path.endswith("libvggt_attn_debug.so")
    lib = ctypes.CDLL(lib_path)
    for n in declared_functions():
        assert hasattr(lib, n), n
    lib.vggt_attn_error_string.restype = ctypes.c_char_p
    assert b"bounds check" in lib.vggt_attn_error_string(V.ERR_BOUNDS)


def test_library_exports_every_declared_function(V):
    names = declared_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(V.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert V.vggt_attn_abi_version() == 4


def test_error_strings(V):
    for code in range(0, -8, -1):
        assert V.error_string(code) and "unknown" not in V.error_string(code)
    assert "unknown" in V.error_string(-99)


def test_workspace_size_formula(V):
    s = W.workload(3).shape
    n = s.S * s.T
    qk = (n * 16 * 64 * 2 + 255) // 256 * 256
    assert V.vggt_attn_workspace_size(s, "global") == 256 + 2 * qk
    assert V.vggt_attn_workspace_size(s, "frame") == 256 + 2 * qk
    nr = s.S * s.n_special * 16 * 64 * 2
    r = (nr + 255) // 256 * 256
    assert V.vggt_attn_workspace_size(s, "register") == 256 + 3 * r
    bad = V.make_shape(s)
    bad.head_dim = 32
    assert V.vggt_attn_workspace_size(bad, "global") == 0
    assert V.vggt_attn_workspace_size(s, 7) == 0


def _call(V, fn, shape, qkv=4096, g=8192, out=1 << 30, ws=1 << 32, wsb=None, mode="global"):
    s = V.make_shape(shape)
    wsb = V.vggt_attn_workspace_size(s, mode) if wsb is None else wsb
    return fn(ctypes.byref(s), qkv, g, g + 256, g + 512, g + 768, out, ws, wsb, 0)


def test_host_validation_without_device(V):
    lib = V.library()
    s = W.workload(0).shape
    f = lib.vggt_attn_global
    bad = V.make_shape(s)
    bad.head_dim = 128
    assert _call(V, f, bad) == V.ERR_UNSUPPORTED_SHAPE
    bad = V.make_shape(s)
    bad.T = s.T + 1
    assert _call(V, f, bad) == V.ERR_UNSUPPORTED_SHAPE
    bad = V.make_shape(s)
    bad.ln_eps = float("nan")
    assert _call(V, f, bad) == V.ERR_INVALID_ARG
    assert _call(V, f, s, qkv=0) == V.ERR_INVALID_ARG
    assert _call(V, f, s, qkv=4098) == V.ERR_MISALIGNED
    assert _call(V, f, s, ws=(1 << 32) + 16) == V.ERR_MISALIGNED
    assert _call(V, f, s, wsb=100) == V.ERR_WORKSPACE_TOO_SMALL
    assert _call(V, f, s, out=4096) == V.ERR_INVALID_ARG          # out aliases qkv
    nospecial = W.Shape(S=2, T=16, H=2, n_special=0, grid_h=4, grid_w=4)
    assert _call(V, lib.vggt_attn_register, nospecial, mode="register") == V.ERR_UNSUPPORTED_SHAPE
    assert lib.vggt_attn_selftest_timeout(None, 10, None) == V.ERR_INVALID_ARG
    assert lib.vggt_attn_selftest_timeout(256, 0, None) == V.ERR_INVALID_ARG


def test_valid_call_without_gpu_fails_loudly(V):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc = _call(V, V.library().vggt_attn_global, W.workload(0).shape)
    assert rc in (V.ERR_CUDA, V.ERR_UNSUPPORTED_DEVICE)
    with pytest.raises(V.VggtAttnError):
        V.vggt_attn_global(W.workload(0).shape, 4096, 8192, 8448, 8704, 8960, 1 << 30, 1 << 32,
                           V.vggt_attn_workspace_size(W.workload(0).shape, "global"), stream=0)


def test_block_and_pipeline_validation_without_device(V):
    """Argument errors of the newer entry points are caught on the host, before any device work."""
    s = W.Shape(S=2, T=68, H=4, n_special=5, grid_h=7, grid_w=9)
    good = {f: (1 << 20) + 256 * i for i, f in enumerate(V.BLOCK_WEIGHT_FIELDS)}
    wsb = V.vggt_block_workspace_size(s, "frame")
    assert wsb > 0 and V.vggt_block_workspace_size(W.Shape(S=2, T=68, H=2, n_special=5, grid_h=7, grid_w=9),
                                                    "frame") == 0          # C = 128: not a multiple of 256
    lib = V.library()
    shape = V.make_shape(s)
    x = 1 << 34
    ws = 1 << 36

    def block(weights, eps=1e-6, nbytes=wsb, xx=x):
        w = V.make_block_weights(weights)
        return lib.vggt_block_forward(0, ctypes.byref(shape), xx, ctypes.byref(w), eps, ws, nbytes, None)

    assert block(dict(good, ls1=None)) == V.ERR_INVALID_ARG
    assert block(dict(good, w_fc1=(1 << 20) + 8)) == V.ERR_MISALIGNED
    assert block(good, eps=0.0) == V.ERR_INVALID_ARG
    assert block(good, nbytes=wsb - 1) == V.ERR_WORKSPACE_TOO_SMALL
    assert block(good, xx=ws + 256) == V.ERR_INVALID_ARG                   # x inside the workspace
    assert block(dict(good, w_qkv=x)) == V.ERR_INVALID_ARG                 # a weight overlapping x
    # the schedule: a register layer index out of range
    w = V.make_block_weights(good)
    arr = (V.vggt_block_weights * 1)(w)
    regs = (ctypes.c_int * 1)(3)
    assert lib.vggt_aggregator_forward(ctypes.byref(shape), x, arr, arr, 1, regs, 1, 1e-6, ws,
                                       V.vggt_aggregator_workspace_size(s), None) == V.ERR_INVALID_ARG
    # host pipeline: missing host pointers; sharded core: too many ranks for the fused form
    qs = (ctypes.c_void_p * 1)(None)
    assert lib.vggt_attn_host_pipeline(1, ctypes.byref(shape), 1, qs, 256, 512, 768, 1024, qs, ws,
                                       V.vggt_attn_host_pipeline_workspace_size(s, "global"), None, None,
                                       None) == V.ERR_INVALID_ARG
    ks = (ctypes.c_void_p * 9)(*([1 << 24] * 9))
    assert lib.vggt_attn_global_shard_core_peers(ctypes.byref(shape), 9, ks, ks, x, ws, 1 << 30,
                                                 None) == V.ERR_UNSUPPORTED_SHAPE
    # descriptor attention: window sizes must be >= 1
    assert lib.vggt_attn_global_desc(ctypes.byref(shape), 0, 2, 4096, 256, 512, 768, 1024, x, ws, 1 << 30,
                                     None) == V.ERR_INVALID_ARG


def test_empty_and_oversized_shapes_are_rejected_on_the_host(V):
    lib = V.library()
    f = lib.vggt_attn_global
    for S, T, ns, gh, gw in ((0, 69, 5, 8, 8), (2, 0, 0, 0, 0)):
        s = W.Shape(S=S, T=T, H=4, n_special=ns, grid_h=gh, grid_w=gw)
        assert V.vggt_attn_workspace_size(s, "global") == 0
        assert _call(V, f, s, wsb=1 << 30) == V.ERR_UNSUPPORTED_SHAPE
    # more tokens than the kernels' 32-bit token indices allow
    huge = W.Shape(S=2_100_000, T=1031, H=16, n_special=17, grid_h=26, grid_w=39)
    assert V.vggt_attn_workspace_size(huge, "global") == 0
    assert _call(V, f, huge, wsb=1 << 40) == V.ERR_UNSUPPORTED_SHAPE
    # zero heads
    assert _call(V, f, W.Shape(S=2, T=69, H=0, n_special=5, grid_h=8, grid_w=8), wsb=1 << 30) == V.ERR_UNSUPPORTED_SHAPE


def test_overlapped_shard_core_validation_without_device(V):
    """The overlapped sharded core's argument errors come back from the host before any device work, and
    its workspace holds the partial softmax state (fp32 sums, row sum and max per row and head) on top of
    the gathered buffers."""
    import dataclasses
    s = W.Shape(S=2, T=68, H=4, n_special=5, grid_h=7, grid_w=9)
    lib = V.library()
    shape = V.make_shape(s)
    world = 2
    L = s.S * s.T
    wsb = V.vggt_attn_shard_workspace_size(s, world)
    fused = V.vggt_attn_shard_fused_workspace_size(s)
    assert wsb >= fused + 2 * world * L * s.H * 128 + s.H * L * (64 + 2) * 4
    ws, out = 1 << 36, 1 << 34
    local = lib.vggt_attn_global_shard_core_local
    remote = lib.vggt_attn_global_shard_core_remote
    assert local(ctypes.byref(shape), world, None, wsb, None) == V.ERR_INVALID_ARG
    assert local(ctypes.byref(shape), world, ws + 16, wsb, None) == V.ERR_MISALIGNED
    assert local(ctypes.byref(shape), world, ws, wsb - 1, None) == V.ERR_WORKSPACE_TOO_SMALL
    assert local(ctypes.byref(shape), world, ws, fused, None) == V.ERR_WORKSPACE_TOO_SMALL   # the fused form's prefix only
    one = V.make_shape(dataclasses.replace(s, S=4))
    assert remote(ctypes.byref(one), 1, 0, out, ws, 1 << 32, None) == V.ERR_UNSUPPORTED_SHAPE   # nothing remote
    assert remote(ctypes.byref(shape), 10, 0, out, ws, 1 << 32, None) == V.ERR_UNSUPPORTED_SHAPE  # > 8 remote maps
    assert remote(ctypes.byref(shape), world, world, out, ws, wsb, None) == V.ERR_INVALID_ARG
    assert remote(ctypes.byref(shape), world, -1, out, ws, wsb, None) == V.ERR_INVALID_ARG
    assert remote(ctypes.byref(shape), world, 0, out, ws, wsb - 1, None) == V.ERR_WORKSPACE_TOO_SMALL
    assert remote(ctypes.byref(shape), world, 0, None, ws, wsb, None) == V.ERR_INVALID_ARG
    assert remote(ctypes.byref(shape), world, 0, out + 8, ws, wsb, None) == V.ERR_MISALIGNED
    assert remote(ctypes.byref(shape), world, 0, ws + 256, ws, wsb, None) == V.ERR_INVALID_ARG   # out inside the workspace
