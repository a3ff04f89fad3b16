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


def test_library_exports_every_declared_function(V):
    names = declared_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(V.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert V.vggt_attn_abi_version() == 3


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
