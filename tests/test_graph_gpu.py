"""The entry points enqueue kernels only (no allocation, no host synchronisation),
so they can be captured into a CUDA graph: a captured transformer-block layer
and a captured attention call replay to the eager results bit for bit."""
import numpy as np
import pytest

import workloads as W
from parity import run_gpu, to_device

pytestmark = pytest.mark.gpu


def shp(S, H, ns, gh, gw):
    return W.Shape(S=S, T=ns + gh * gw, H=H, n_special=ns, grid_h=gh, grid_w=gw)


def _dev_weights(w):
    import torch
    return {k: (torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).cuda().view(torch.bfloat16)
                if v.dtype == np.uint16 else torch.from_numpy(v).cuda()) for k, v in w.items()}


def test_captured_layer_replays_eager_result():
    import torch
    import vit_attention_b200 as V
    shape = shp(4, 4, 5, 7, 9)
    fw = _dev_weights(W.make_transformer_block_weights(shape.H, 130))
    iw = _dev_weights(W.make_transformer_block_weights(shape.H, 131))
    x0 = torch.from_numpy(W.make_tokens(shape, 132).view(np.int16)).cuda().view(torch.bfloat16)
    ws = torch.empty(V.vggt_aggregator_workspace_size(shape), dtype=torch.uint8, device="cuda")

    def layer(x, stream):
        V.vggt_block_forward("frame", shape, x, fw, 1e-6, ws, stream=stream)
        V.vggt_block_forward("register", shape, x, iw, 1e-6, ws, stream=stream)
        V.vggt_block_forward("global", shape, x, iw, 1e-6, ws, stream=stream)

    eager = x0.clone()
    layer(eager, None)
    torch.cuda.synchronize()
    x = x0.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            layer(x, s)
    torch.cuda.synchronize()
    for _ in range(2):                      # the graph updates x in place: reset before each replay
        x.copy_(x0)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(x.view(torch.int16), eager.view(torch.int16))
    assert V.vggt_attn_read_status(ws) == 0


def test_captured_attention_call_replays_eager_result():
    import torch
    import vit_attention_b200 as V
    shape = shp(3, 4, 17, 10, 12)
    x = W.make_random_inputs(shape, 133)
    qkv, prm = to_device(x)
    want = run_gpu("global", shape, dev_inputs=(qkv, prm))
    out = torch.zeros_like(want)
    ws = torch.empty(V.vggt_attn_workspace_size(shape, "global"), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            V.vggt_attn_global(shape, qkv, prm["q_gamma"], prm["q_beta"], prm["k_gamma"], prm["k_beta"], out, ws,
                               stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), want.view(torch.int16))
