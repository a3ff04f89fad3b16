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


# ------------------------------------------------------------------ overlapped form (own keys, then the others')
def _run_overlapped(shape, dev, world):
    """Every rank's prologue and own-keys core (the launch that runs beside the all-gather), the gather
    emulated with device copies, then each rank's core over the other ranks' keys with the merge."""
    import dataclasses
    import torch
    import vit_attention_b200 as V
    local = dataclasses.replace(shape, S=shape.S // world)
    wss, sends = [], []
    for r in range(world):
        ws = torch.empty(V.vggt_attn_shard_workspace_size(local, world), dtype=torch.uint8, device="cuda")
        V.vggt_attn_global_shard_prologue(local, world, dev["qkv"][r * local.S:(r + 1) * local.S], dev["q_gamma"],
                                          dev["q_beta"], dev["k_gamma"], dev["k_beta"], ws)
        V.vggt_attn_global_shard_core_local(local, world, ws)
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
        V.vggt_attn_global_shard_core_remote(local, world, r, out, wss[r])
        assert V.vggt_attn_read_status(wss[r]) == 0
        outs.append(out)
    return torch.cat(outs)


# ragged local token counts (136, 634, 14) and the largest world (8 remote rank maps)
OVERLAP = [(shp(6, 4, 5, 7, 9), 3), (shp(4, 2, 17, 10, 30), 2), (shp(8, 2, 5, 3, 4), 8), (shp(9, 2, 5, 3, 4), 9)]


@pytest.mark.parametrize("shape,world", OVERLAP, ids=[f"S{s.S}T{s.T}H{s.H}-w{w}" for s, w in OVERLAP])
def test_overlapped_ranks_match_oracle(shape, world):
    """Every query row against the fp64 oracle; and against the one-pass gathered core to bf16 rounding
    (the key order and the 64-key step boundaries differ, so not bit for bit)."""
    import torch
    x = W.make_random_inputs(shape, 240 + shape.T + world)
    dev = _dev(x)
    got = _run_overlapped(shape, dev, world)
    q = query_sample("global", shape, 1 << 62, 0)
    assert_close(rows(got, shape, q), O.attn_global(shape, x, q), f"overlapped sharded global, {world} ranks")
    one_pass = _run_sharded(shape, dev, world).float()
    diff = (got.float() - one_pass).abs().max().item()
    assert diff <= 2.0 ** -5, f"overlapped vs one-pass core: max |diff| = {diff}"


def test_overlapped_workload2_four_ranks_against_oracle():
    w = W.workload(2)                                  # 24 frames x 1031 tokens, 16 heads
    x = W.make_inputs(w)
    got = _run_overlapped(w.shape, _dev(x), 4)
    q = query_sample("global", w.shape, 512, w.seed + 1)
    assert_close(rows(got, w.shape, q), O.attn_global(w.shape, x, q), "overlapped sharded global, 4 ranks")


def test_overlapped_merge_with_distant_maxima():
    """Rank 0's keys point along -u, rank 1's along +u, and the queries alternate between +u and -u, so for
    every rank some rows find their maxima among their own keys and others among the other rank's, 15-20
    units (base 2) above the rest: the merge scales one side by about 2^-18.  The bf16 storage points alone
    err by 1.8e-3 (max-abs) / 3.5e-3 (rel.) on these inputs (CPU emulation, as in test_parity_gpu); a merge
    that scaled the wrong side would be off by O(1)."""
    shape = W.Shape(S=4, T=40, H=2, n_special=40, grid_h=0, grid_w=1)
    x = W.make_random_inputs(shape, 250)
    qkv = O.bf16_to_f64(x["qkv"])
    u = np.random.default_rng(251).standard_normal(64)
    u -= u.mean()
    u /= np.linalg.norm(u)
    for s in range(shape.S):
        qkv[s, :, 1] += (16.0 if s >= shape.S // 2 else -16.0) * u
        qkv[s, :, 0] += np.where(np.arange(shape.T) % 2 == 0, 16.0, -16.0)[:, None, None] * u
    x["qkv"] = W.f32_to_bf16_bits(qkv.astype(np.float32))
    got = _run_overlapped(shape, _dev(x), 2)
    q = np.arange(shape.S * shape.T)
    assert_close(rows(got, shape, q), O.attn_global(shape, x, q), "overlapped sharded global, distant maxima")


def test_overlapped_remote_rejects_bad_world_and_rank():
    import dataclasses
    import torch
    import vit_attention_b200 as V
    shape = shp(10, 2, 5, 3, 4)
    for world, rank in ((1, 0), (10, 0), (2, 2), (2, -1)):
        local = dataclasses.replace(shape, S=shape.S // world)
        ws = torch.empty(V.vggt_attn_shard_workspace_size(local, world), dtype=torch.uint8, device="cuda")
        out = torch.zeros((local.S, local.T, local.H, 64), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(RuntimeError):
            V.vggt_attn_global_shard_core_remote(local, world, rank, out, ws)


# ------------------------------------------------------------------ fused form (keys read in place)
def _fused_emulated(shape, dev, world):
    """All ranks in this process: W prologues into W workspaces, then each rank's core reads the W send
    buffers in place (on one GPU they are simply this GPU's memory)."""
    import dataclasses
    import torch
    import vit_attention_b200 as V
    local = dataclasses.replace(shape, S=shape.S // world)
    wss, ks, vs = [], [], []
    for r in range(world):
        ws = torch.empty(V.vggt_attn_shard_fused_workspace_size(local), dtype=torch.uint8, device="cuda")
        V.vggt_attn_global_shard_prologue(local, world, dev["qkv"][r * local.S:(r + 1) * local.S], dev["q_gamma"],
                                          dev["q_beta"], dev["k_gamma"], dev["k_beta"], ws)
        k_send, v_send, _, _ = V.vggt_attn_shard_buffers(local, world, ws)
        wss.append(ws)
        ks.append(k_send)
        vs.append(v_send)
    outs = []
    for r in range(world):
        out = torch.zeros((local.S, local.T, local.H, 64), dtype=torch.bfloat16, device="cuda")
        V.vggt_attn_global_shard_core_peers(local, world, ks, vs, out, wss[r])
        assert V.vggt_attn_read_status(wss[r]) == 0
        outs.append(out)
    return torch.cat(outs)


FUSED = [(shp(6, 4, 5, 7, 9), 3), (shp(4, 2, 17, 10, 30), 2), (shp(8, 2, 5, 3, 4), 8)]


@pytest.mark.parametrize("shape,world", FUSED, ids=[f"S{s.S}T{s.T}H{s.H}-w{w}" for s, w in FUSED])
def test_fused_ranks_match_oracle(shape, world):
    x = W.make_random_inputs(shape, 210 + shape.T)
    dev = _dev(x)
    got = _fused_emulated(shape, dev, world)
    q = query_sample("global", shape, 1 << 62, 0)
    assert_close(rows(got, shape, q), O.attn_global(shape, x, q), f"fused sharded global, {world} ranks")


def test_fused_single_rank_equals_global_bitwise():
    import torch
    shape = shp(3, 4, 17, 10, 12)
    x = W.make_random_inputs(shape, 220)
    dev = _dev(x)
    assert torch.equal(_fused_emulated(shape, dev, 1).view(torch.int16), _run_global(shape, dev).view(torch.int16))


def _ipc_worker(rank, world, port, seed, results):
    """One rank of a 2-process run on one GPU: the other rank's keys/values are read through a CUDA IPC
    mapping of its workspace (no kernel waits on the other process; the ranks meet at host barriers)."""
    import dataclasses
    import datetime
    import os
    import sys
    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(0)
    import vit_attention_b200 as V
    import workloads as W
    from parity import to_device
    from vit_attention_b200.sharded import PeerShards
    shape = W.Shape(S=4, T=68, H=4, n_special=5, grid_h=7, grid_w=9)
    local = dataclasses.replace(shape, S=shape.S // world)
    x = W.make_random_inputs(shape, seed)
    qkv, prm = to_device(x)
    ws = torch.empty(V.vggt_attn_shard_fused_workspace_size(local), dtype=torch.uint8, device="cuda")
    peers = PeerShards(local, ws)
    out = torch.zeros((local.S, local.T, local.H, 64), dtype=torch.bfloat16, device="cuda")
    peers.attend(qkv[rank * local.S:(rank + 1) * local.S], prm["q_gamma"], prm["q_beta"], prm["k_gamma"],
                 prm["k_beta"], out)
    torch.cuda.synchronize()
    results[rank] = (V.vggt_attn_read_status(ws), out.float().cpu().numpy())
    dist.barrier()
    del peers
    dist.destroy_process_group()


def test_fused_two_processes_share_one_gpu_through_ipc():
    import socket
    import numpy as np
    import torch.multiprocessing as mp
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    seed = 230
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.spawn(_ipc_worker, args=(2, port, seed, results), nprocs=2, join=True)
        res = dict(results)
    assert res[0][0] == 0 and res[1][0] == 0
    shape = W.Shape(S=4, T=68, H=4, n_special=5, grid_h=7, grid_w=9)
    x = W.make_random_inputs(shape, seed)
    got = np.concatenate([res[0][1], res[1][1]]).reshape(-1, shape.H, 64).astype(np.float64)
    assert_close(got, O.attn_global(shape, x), "fused sharded global over IPC, 2 processes")


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=12, deadline=None)
@given(world=st.integers(1, 8), frames_per_rank=st.integers(1, 3), H=st.integers(1, 2), ns=st.integers(1, 6),
       gh=st.integers(0, 7), gw=st.integers(1, 7), seed=st.integers(0, 10_000))
def test_random_sharded_shapes(world, frames_per_rank, H, ns, gh, gw, seed):
    """Gathered and fused sharded forms over random rank counts and shapes (rank blocks of any length)."""
    import torch
    shape = shp(world * frames_per_rank, H, ns, gh, gw)
    x = W.make_random_inputs(shape, seed)
    dev = _dev(x)
    want = _run_global(shape, dev)
    assert torch.equal(_run_sharded(shape, dev, world).view(torch.int16), want.view(torch.int16))
    got = _fused_emulated(shape, dev, world)
    q = query_sample("global", shape, 1 << 62, 0)
    assert_close(rows(got, shape, q), O.attn_global(shape, x, q), "fused sharded global")
