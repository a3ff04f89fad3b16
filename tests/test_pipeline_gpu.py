"""Host-memory pipeline (vggt_attn_host_pipeline): several scenes from pinned
host buffers, copies on their own streams overlapping the kernels; every
scene's output must equal the single device call's bit for bit, and register
mode must leave the patch rows of the host outputs untouched."""
import numpy as np
import pytest

import workloads as W
from parity import run_gpu, to_device

pytestmark = pytest.mark.gpu


def shp(S, H, ns, gh, gw):
    return W.Shape(S=S, T=ns + gh * gw, H=H, n_special=ns, grid_h=gh, grid_w=gw)


@pytest.mark.parametrize("mode", ["global", "frame", "register"])
@pytest.mark.parametrize("separate_streams", [True, False])
def test_pipeline_matches_single_calls(mode, separate_streams):
    import torch
    import vit_attention_b200 as V
    shape = shp(4, 4, 5, 7, 9)
    n = 5
    xs = [W.make_random_inputs(shape, 400 + i) for i in range(n)]
    for x in xs[1:]:                       # one set of gamma/beta for all scenes
        for k in ("q_gamma", "q_beta", "k_gamma", "k_beta"):
            x[k] = xs[0][k]
    _, prm = to_device(xs[0])
    h_qkv = [torch.from_numpy(x["qkv"].view(np.int16)).view(torch.bfloat16).pin_memory() for x in xs]
    sentinel = torch.tensor(-3.0, dtype=torch.bfloat16)
    h_out = [torch.full((shape.S, shape.T, shape.H, 64), -3.0, dtype=torch.bfloat16).pin_memory() for _ in xs]
    ws = torch.empty(V.vggt_attn_host_pipeline_workspace_size(shape, mode), dtype=torch.uint8, device="cuda")
    streams = [torch.cuda.Stream() for _ in range(3)] if separate_streams else [torch.cuda.current_stream()] * 3
    V.vggt_attn_host_pipeline(mode, shape, h_qkv, prm["q_gamma"], prm["q_beta"], prm["k_gamma"], prm["k_beta"],
                              h_out, ws, compute_stream=streams[0], h2d_stream=streams[1], d2h_stream=streams[2])
    torch.cuda.synchronize()
    assert V.vggt_attn_read_status(ws) == 0
    for i, x in enumerate(xs):
        want = run_gpu(mode, shape, x).cpu()
        if mode == "register":
            sp = want.view(shape.S, shape.T, -1)[:, :shape.n_special]
            got = h_out[i].view(shape.S, shape.T, -1)
            assert torch.equal(got[:, :shape.n_special].view(torch.int16), sp.view(torch.int16))
            assert bool((got[:, shape.n_special:] == sentinel).all())
        else:
            assert torch.equal(h_out[i].view(torch.int16), want.view(torch.int16))


def test_pipeline_rejects_pageable_host_memory():
    import torch
    import vit_attention_b200 as V
    shape = shp(2, 4, 5, 7, 9)
    x = W.make_random_inputs(shape, 9)
    _, prm = to_device(x)
    h_qkv = [torch.from_numpy(x["qkv"].view(np.int16)).view(torch.bfloat16)]          # not pinned
    h_out = [torch.empty((shape.S, shape.T, shape.H, 64), dtype=torch.bfloat16).pin_memory()]
    ws = torch.empty(V.vggt_attn_host_pipeline_workspace_size(shape, "global"), dtype=torch.uint8, device="cuda")
    with pytest.raises(V.VggtAttnError) as e:
        V.vggt_attn_host_pipeline("global", shape, h_qkv, prm["q_gamma"], prm["q_beta"], prm["k_gamma"],
                                  prm["k_beta"], h_out, ws)
    assert e.value.code == V.ERR_INVALID_ARG
