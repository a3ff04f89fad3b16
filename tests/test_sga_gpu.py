"""GPU parity of subsampled global attention (vggt_attn_global_sga) against the
fp64 oracle (oracle/sga.py), through the C ABI binding."""
import numpy as np
import pytest

import oracle as O
import workloads as W
from parity import assert_close, rows, to_device

pytestmark = pytest.mark.gpu


def _run(shape, inputs, s_h, s_w):
    import torch
    import vit_attention_b200 as V
    qkv, prm = to_device(inputs)
    out = torch.empty((shape.S, shape.T, shape.H, 64), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(V.vggt_attn_sga_workspace_size(shape, s_h, s_w), dtype=torch.uint8, device="cuda")
    V.vggt_attn_global_sga(shape, s_h, s_w, qkv, prm["q_gamma"], prm["q_beta"], prm["k_gamma"], prm["k_beta"], out, ws)
    assert V.vggt_attn_read_status(ws) == 0
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("s_h,s_w", [(1, 1), (2, 2), (3, 2), (8, 8)])
def test_sga_small_matches_oracle(s_h, s_w):
    shape = W.workload(0).shape
    inputs = W.make_random_inputs(shape, 61)
    out = _run(shape, inputs, s_h, s_w)
    q = np.arange(shape.S * shape.T)
    assert_close(rows(out, shape, q), O.attn_global_sga(shape, inputs, s_h, s_w, q), f"sga {s_h}x{s_w}")


def test_sga_no_subsampling_is_global_mode():
    import torch
    shape = W.workload(0).shape
    inputs = W.make_random_inputs(shape, 62)
    from parity import run_gpu
    a = _run(shape, inputs, 1, 1)
    b = run_gpu("global", shape, inputs)
    assert torch.equal(a, b)


def test_sga_frames_of_1031_tokens_sampled():
    shape = W.Shape(S=4, T=1031, H=16, n_special=17, grid_h=26, grid_w=39)
    inputs = W.make_random_inputs(shape, 63)
    out = _run(shape, inputs, 3, 3)
    q = W.query_subset(shape.S * shape.T, 192, 64)
    assert_close(rows(out, shape, q), O.attn_global_sga(shape, inputs, 3, 3, q), "sga 3x3 S=4")


def test_sga_rejects_bad_strides():
    import torch
    import vit_attention_b200 as V
    shape = W.workload(0).shape
    assert V.vggt_attn_sga_workspace_size(shape, 0, 2) == 0
    inputs = W.make_random_inputs(shape, 65)
    qkv, prm = to_device(inputs)
    out = torch.empty((shape.S, shape.T, shape.H, 64), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(V.vggt_attn_sga_workspace_size(shape, 2, 2), dtype=torch.uint8, device="cuda")
    with pytest.raises(V.VggtAttnError) as e:
        V.vggt_attn_global_sga(shape, 0, 2, qkv, prm["q_gamma"], prm["q_beta"], prm["k_gamma"], prm["k_beta"], out, ws)
    assert e.value.code == V.ERR_INVALID_ARG
