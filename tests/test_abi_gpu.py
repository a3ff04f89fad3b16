"""Behaviour of the C ABI on a GPU: untouched patch rows in register mode,
determinism, non-default streams, stage split, device status word and the
bounded-wait error path (no GPU fault is provoked)."""
import ctypes

import numpy as np
import pytest

import workloads as W
from parity import assert_close, rows, run_gpu, to_device, query_sample
import oracle as O

pytestmark = pytest.mark.gpu


def shp(S, H, ns, gh, gw):
    return W.Shape(S=S, T=ns + gh * gw, H=H, n_special=ns, grid_h=gh, grid_w=gw)


def test_register_mode_leaves_patch_rows_untouched():
    import torch
    shape = shp(9, 2, 17, 5, 6)
    x = W.make_random_inputs(shape, 31)
    sentinel = torch.full((shape.S, shape.T, shape.H, 64), -7.25, dtype=torch.bfloat16, device="cuda")
    out = run_gpu("register", shape, x, out=sentinel)
    patch = out[:, shape.n_special:]
    assert torch.equal(patch, torch.full_like(patch, -7.25))
    q = query_sample("register", shape, 1 << 62, 0)
    assert_close(rows(out, shape, q), O.attn_register(shape, x, q), "register rows")


@pytest.mark.parametrize("mode", ["frame", "global", "register"])
def test_two_runs_are_bitwise_identical(mode):
    import torch
    shape = shp(4, 3, 17, 9, 11)
    dev = to_device(W.make_random_inputs(shape, 32))
    a = run_gpu(mode, shape, dev_inputs=dev).clone()
    b = run_gpu(mode, shape, dev_inputs=dev)
    if mode == "register":
        a, b = a[:, :shape.n_special], b[:, :shape.n_special]
    assert torch.equal(a, b)


def test_nondefault_stream_and_stage_split():
    import torch
    import vit_attention_b200 as V
    shape = shp(3, 2, 17, 8, 9)
    x = W.make_random_inputs(shape, 33)
    qkv, p = to_device(x)
    ref = run_gpu("global", shape, dev_inputs=(qkv, p))
    s = torch.cuda.Stream()
    out = torch.empty_like(ref)
    ws = torch.empty(V.vggt_attn_workspace_size(shape, "global"), dtype=torch.uint8, device="cuda")
    with torch.cuda.stream(s):
        V.vggt_attn_prologue("global", shape, qkv, p["q_gamma"], p["q_beta"], p["k_gamma"], p["k_beta"], ws,
                             stream=s)
        V.vggt_attn_core("global", shape, qkv, out, ws, stream=s)
    s.synchronize()
    assert V.vggt_attn_read_status(ws, s) == 0
    assert torch.equal(out, ref)


def test_argument_errors_are_reported_before_launch():
    import torch
    import vit_attention_b200 as V
    shape = shp(2, 2, 5, 3, 3)
    x = W.make_random_inputs(shape, 34)
    qkv, p = to_device(x)
    out = torch.full((2, shape.T, 2, 64), 3.0, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(V.vggt_attn_workspace_size(shape, "frame"), dtype=torch.uint8, device="cuda")
    lib = V.library()
    s = V.make_shape(shape)
    args = lambda **kw: [ctypes.byref(kw.get("shape", s)), kw.get("qkv", qkv.data_ptr()), p["q_gamma"].data_ptr(),
                         p["q_beta"].data_ptr(), p["k_gamma"].data_ptr(), p["k_beta"].data_ptr(),
                         kw.get("out", out.data_ptr()), kw.get("ws", ws.data_ptr()), kw.get("wsb", ws.numel()),
                         torch.cuda.current_stream().cuda_stream]
    assert lib.vggt_attn_frame(*args(wsb=ws.numel() - 1)) == V.ERR_WORKSPACE_TOO_SMALL
    assert lib.vggt_attn_frame(*args(qkv=qkv.data_ptr() + 2)) == V.ERR_MISALIGNED
    assert lib.vggt_attn_frame(*args(out=qkv.data_ptr())) == V.ERR_INVALID_ARG     # aliasing
    assert lib.vggt_attn_frame(*args(out=0)) == V.ERR_INVALID_ARG
    bad = V.make_shape(shape)
    bad.head_dim = 128
    assert lib.vggt_attn_frame(*args(shape=bad)) == V.ERR_UNSUPPORTED_SHAPE
    torch.cuda.synchronize()
    assert torch.equal(out, torch.full_like(out, 3.0))                             # nothing ran


def test_bounded_wait_reports_timeout_and_context_survives():
    import torch
    import vit_attention_b200 as V
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    V.vggt_attn_selftest_timeout(ws, 2000)          # 2 ms wait on a barrier nothing arrives at
    assert V.vggt_attn_read_status(ws) == V.ERR_TIMEOUT
    assert V.vggt_attn_read_status(ws) == 0         # read clears it
    shape = shp(2, 2, 5, 4, 4)                      # the context is still usable
    x = W.make_random_inputs(shape, 35)
    out = run_gpu("global", shape, x)
    assert_close(rows(out, shape, np.arange(shape.S * shape.T)), O.attn_global(shape, x), "after timeout")
