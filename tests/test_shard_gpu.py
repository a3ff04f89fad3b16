"""Query-sharded global attention (vggt_attn_global_shard_prologue / _core)
on one GPU: the ranks run one after another (no rank waits on another), the
all-gather is done with device copies, and the concatenated outputs must equal
vggt_attn_global on the whole scene bit for bit (every query row sees the
same keys in the same 64-key steps); one case is also checked against the
fp64 oracle."""
import numpy as np
import pytest

import oracle as O
import workloads as W
from parity import assert_close, query_sample, rows, to_device

pytestmark = pytest.mark.gpu


def shp(S, H, ns, gh, gw):
    return W.Shape(S=S, T=ns + gh * gw, H=H, n_special=ns, grid_h=gh, grid_w=gw)


def _dev(x):
    qkv, prm = to_device(x)
    return dict(qkv=qkv, **prm)


def _run_global(shape, dev):
    import torch
    import vit_attention_b200 as V
    out = torch.zeros((shape.S, shape.T, shape.H, 64), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(V.vggt_attn_workspace_size(shape, "global"), dtype=torch.uint8, device="cuda")
    V.vggt_attn_global(shape, dev["qkv"], dev["q_gamma"], dev["q_beta"], dev["k_gamma"], dev["k_beta"], out, ws)
    assert V.vggt_attn_read_status(ws) == 0
    return out


def _run_sharded(shape, dev, world):
    import dataclasses
    import torch
    import vit_attention_b200 as V
    local = dataclasses.replace(shape, S=shape.S // world)
    wss, sends = [], []
    for r in range(world):
        ws = torch.empty(V.vggt_attn_shard_workspace_size(local, world), dtype=torch.uint8, device="cuda")
        qkv_r = dev["qkv"][r * local.S:(r + 1) * local.S]
        V.vggt_attn_global_shard_prologue(local, world, qkv_r, dev["q_gamma"], dev["q_beta"], dev["k_gamma"],
                                          dev["k_beta"], ws)
        wss.append(ws)
        sends.append(V.vggt_attn_shard_buffers(local, world, ws)[:2])
    k_cat = torch.cat([k for k, _ in sends])
    v_cat = torch.cat([v for _, v in sends])
    outs = []
    for r in range(world):
        _, _, k_all, v_all = V.vggt_attn_shard_buffers(local, world, wss[r])
        k_all.copy_(k_cat)
        v_all.copy_(v_cat)
        out = torch.zeros((local.S, local.T, local.H, 64), dtype=torch.bfloat16, device="cuda")
        V.vggt_attn_global_shard_core(local, world, out, wss[r])
        assert V.vggt_attn_read_status(wss[r]) == 0
        outs.append(out)
    return torch.cat(outs)


CASES = [(shp(6, 4, 5, 7, 9), 3), (shp(6, 4, 5, 7, 9), 1), (shp(4, 2, 17, 10, 30), 2)]


@pytest.mark.parametrize("shape,world", CASES, ids=[f"S{s.S}T{s.T}H{s.H}-w{w}" for s, w in CASES])
def test_sharded_equals_global_bitwise(shape, world):
    import torch
    x = W.make_random_inputs(shape, 200 + shape.T)
    dev = _dev(x)
    want = _run_global(shape, dev)
    got = _run_sharded(shape, dev, world)
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))


def test_sharded_workload2_four_ranks_against_oracle():
    import torch
    w = W.workload(2)                                  # 24 frames x 1031 tokens, 16 heads
    x = W.make_inputs(w)
    dev = _dev(x)
    got = _run_sharded(w.shape, dev, 4)
    assert torch.equal(got.view(torch.int16), _run_global(w.shape, dev).view(torch.int16))
    q = query_sample("global", w.shape, 512, w.seed)
    assert_close(rows(got, w.shape, q), O.attn_global(w.shape, x, q), "sharded global, 4 ranks")


def test_single_rank_helper_without_process_group():
    import torch
    import vit_attention_b200 as V
    from vit_attention_b200.sharded import global_attention_sharded
    shape = shp(3, 4, 5, 7, 9)
    x = W.make_random_inputs(shape, 17)
    dev = _dev(x)
    out = torch.zeros((shape.S, shape.T, shape.H, 64), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(V.vggt_attn_shard_workspace_size(shape, 1), dtype=torch.uint8, device="cuda")
    global_attention_sharded(shape, dev["qkv"], dev["q_gamma"], dev["q_beta"], dev["k_gamma"], dev["k_beta"], out, ws)
    assert torch.equal(out.view(torch.int16), _run_global(shape, dev).view(torch.int16))
