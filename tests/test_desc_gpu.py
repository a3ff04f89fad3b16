"""GPU parity of descriptor attention (vggt_attn_global_desc) against its fp64
oracle (oracle/descriptor.py); 1x1 windows must reproduce global mode bit for bit."""
import numpy as np
import pytest

import oracle as O
import workloads as W
from parity import assert_close, query_sample, rows, to_device

pytestmark = pytest.mark.gpu


def shp(S, H, ns, gh, gw):
    return W.Shape(S=S, T=ns + gh * gw, H=H, n_special=ns, grid_h=gh, grid_w=gw)


def _run(shape, dev, s_h, s_w):
    import torch
    import vit_attention_b200 as V
    qkv, prm = dev
    out = torch.zeros((shape.S, shape.T, shape.H, 64), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(V.vggt_attn_sga_workspace_size(shape, s_h, s_w), dtype=torch.uint8, device="cuda")
    V.vggt_attn_global_desc(shape, s_h, s_w, qkv, prm["q_gamma"], prm["q_beta"], prm["k_gamma"], prm["k_beta"],
                            out, ws)
    assert V.vggt_attn_read_status(ws) == 0
    return out


CASES = [(shp(3, 4, 5, 7, 9), 2, 2), (shp(3, 4, 5, 7, 9), 3, 2), (shp(2, 2, 17, 26, 39), 4, 4),
         (shp(4, 2, 3, 5, 5), 5, 5), (shp(2, 2, 4, 0, 1), 2, 2)]


@pytest.mark.parametrize("shape,s_h,s_w", CASES, ids=[f"S{s.S}T{s.T}-{a}x{b}" for s, a, b in CASES])
def test_desc_matches_oracle(shape, s_h, s_w):
    x = W.make_random_inputs(shape, 300 + shape.T + s_h)
    got = _run(shape, to_device(x), s_h, s_w)
    q = query_sample("global", shape, 1 << 62, 0)
    assert_close(rows(got, shape, q), O.attn_global_desc(shape, x, s_h, s_w, q), f"desc {s_h}x{s_w}")


def test_desc_unit_windows_equal_global_bitwise():
    import torch
    from parity import run_gpu
    shape = shp(3, 4, 17, 10, 12)
    x = W.make_random_inputs(shape, 310)
    dev = to_device(x)
    want = run_gpu("global", shape, dev_inputs=dev)
    assert torch.equal(_run(shape, dev, 1, 1).view(torch.int16), want.view(torch.int16))


def test_desc_workload2_sampled():
    w = W.workload(2)
    x = W.make_inputs(w)
    got = _run(w.shape, to_device(x), 2, 2)
    q = query_sample("global", w.shape, 512, w.seed)
    assert_close(rows(got, w.shape, q), O.attn_global_desc(w.shape, x, 2, 2, q), "desc 2x2, 24 frames")


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=20, deadline=None)
@given(S=st.integers(1, 4), H=st.integers(1, 2), ns=st.integers(1, 6), gh=st.integers(0, 9), gw=st.integers(1, 9),
       s_h=st.integers(1, 4), s_w=st.integers(1, 4), seed=st.integers(0, 10_000))
def test_random_shapes_and_windows(S, H, ns, gh, gw, s_h, s_w, seed):
    """Descriptor and subsampled global attention on random shapes and window sizes (ragged edge windows)."""
    import vit_attention_b200 as V
    import torch
    shape = shp(S, H, ns, gh, gw)
    x = W.make_random_inputs(shape, seed)
    dev = to_device(x)
    q = query_sample("global", shape, 1 << 62, 0)
    assert_close(rows(_run(shape, dev, s_h, s_w), shape, q), O.attn_global_desc(shape, x, s_h, s_w, q), "desc")
    qkv, prm = dev
    out = torch.zeros((shape.S, shape.T, shape.H, 64), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(V.vggt_attn_sga_workspace_size(shape, s_h, s_w), dtype=torch.uint8, device="cuda")
    V.vggt_attn_global_sga(shape, s_h, s_w, qkv, prm["q_gamma"], prm["q_beta"], prm["k_gamma"], prm["k_beta"], out, ws)
    assert V.vggt_attn_read_status(ws) == 0
    assert_close(rows(out, shape, q), O.attn_global_sga(shape, x, s_h, s_w, q), "sga")
