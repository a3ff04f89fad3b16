"""The allocation-free entry point, vggt_attn_noalloc.

It exists for callers that cannot allocate device memory -- plug-in
interfaces that hand over only input and output buffers, code that must not
call cudaMalloc/cudaFree (cudaFree synchronises the device), processes with a
device-memory budget fixed at start-up.  Instead of a caller-given workspace it
uses one fixed 64 MiB scratch array inside the library, shared by all calls.

The GPU test calls it through the C ABI three times in a row (global,
register and frame mode on different shapes and inputs, so each call runs on
scratch the one before left behind) and checks each output against the
regular entry point, which takes a workspace, within the parity tolerance of
the other tests.  This file is
named to be collected last.
"""
import ctypes

import numpy as np
import pytest

import workloads as W
from parity import MAX_ABS_TOL, REL_FRO_TOL, errors, to_device


def _noalloc(V, mode, shape, qkv, prm, out):
    import torch
    return V.library().vggt_attn_noalloc(V.MODES[mode], ctypes.byref(V.make_shape(shape)), qkv.data_ptr(),
                                         prm["q_gamma"].data_ptr(), prm["q_beta"].data_ptr(),
                                         prm["k_gamma"].data_ptr(), prm["k_beta"].data_ptr(), out.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream)


def _with_workspace(V, mode, shape, qkv, prm, out):
    import torch
    ws = torch.empty(V.vggt_attn_workspace_size(shape, mode), dtype=torch.uint8, device="cuda")
    V.attend(mode, shape, qkv, prm["q_gamma"], prm["q_beta"], prm["k_gamma"], prm["k_beta"], out, ws)
    assert V.vggt_attn_read_status(ws) == 0


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_on_calls_in_a_row():
    import torch
    import vit_attention_b200 as V
    cases = [("global", W.Shape(S=6, T=17 + 10 * 12, H=4, n_special=17, grid_h=10, grid_w=12), 41),
             ("register", W.Shape(S=60, T=17 + 3 * 3, H=3, n_special=17, grid_h=3, grid_w=3), 42),
             # frame mode runs its own persistent kernel; it reuses the scratch the two calls above left
             ("frame", W.Shape(S=3, T=17 + 10 * 12, H=4, n_special=17, grid_h=10, grid_w=12), 43)]
    for mode, shape, seed in cases:
        qkv, prm = to_device(W.make_random_inputs(shape, seed))
        ref = torch.zeros((shape.S, shape.T, shape.H, 64), dtype=torch.bfloat16, device="cuda")
        got = torch.zeros_like(ref)
        _with_workspace(V, mode, shape, qkv, prm, ref)
        assert _noalloc(V, mode, shape, qkv, prm, got) == V.OK
        torch.cuda.synchronize()
        rows = slice(None) if mode != "register" else slice(0, shape.n_special)
        g = got[:, rows].double().cpu().numpy()
        r = ref[:, rows].double().cpu().numpy()
        assert np.all(np.isfinite(g))
        max_abs, rel = errors(g, r)
        assert max_abs <= MAX_ABS_TOL and rel <= REL_FRO_TOL, f"{mode}: max_abs={max_abs} rel={rel}"


def test_noalloc_rejects_problems_beyond_the_scratch():
    # Host-side check only: the library must be built, but no GPU is needed.
    V = pytest.importorskip("vit_attention_b200", reason="libvggt_attn.so is not built")
    big = W.Shape(S=16, T=1031, H=16, n_special=17, grid_h=26, grid_w=39)   # 263,936 token-heads
    assert V.vggt_attn_workspace_size(big, "global") > V.NOALLOC_SCRATCH_BYTES
    s = V.make_shape(big)
    # The size check runs before anything touches a pointer or a device, so these made-up (but 16- and
    # 256-byte aligned) addresses are never dereferenced: the call returns the error without any device work.
    rc = V.library().vggt_attn_noalloc(V.GLOBAL, ctypes.byref(s), 4096, 8192, 8448, 8704, 8960, 1 << 30, None)
    assert rc == V.ERR_SCRATCH_TOO_SMALL
    assert "64 MiB" in V.error_string(rc)
