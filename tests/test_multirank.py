"""Host-side logic of the multi-GPU bench path, run as 2 gloo ranks on CPU:
each rank gets its own independent workload copy (weak scaling, no data
exchange) and the timed region is the max over ranks; the exchange step of
query-sharded global attention (the all-gather in rank order) and the order of
the overlapped form's host steps (streams and library calls recorded by fakes)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import datetime
    import sys
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    r, w, lr = bench.dist_env()
    plan = bench.shard_plan(w, r, 1003)
    local_ms = 10.0 + 5.0 * rank                     # rank 1 is the slow one
    bench.barrier()
    mx = bench.reduce_max(local_ms)
    results[rank] = (r, w, lr, plan["seed"], plan["problems"], mx)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    assert sorted(res) == [0, 1]
    seeds = {res[r][3] for r in res}
    assert len(seeds) == 2                            # independent inputs per rank
    for r in res:
        assert res[r][0] == r and res[r][1] == world and res[r][4] == 1
        assert res[r][5] == 15.0                      # max over ranks, seen by every rank


def test_single_process_defaults():
    import bench
    os.environ.pop("RANK", None)
    os.environ.pop("WORLD_SIZE", None)
    assert bench.dist_env()[:2] == (0, 1)
    assert bench.reduce_max(3.5) == 3.5
    assert bench.shard_plan(1, 0, 1003)["seed"] == 1003


def _gather_worker(rank, world, port, results):
    import datetime
    import sys
    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from vit_attention_b200.sharded import gather_kv
    L, H = 5, 2
    k_send = torch.full((L, H, 64), float(rank + 1))
    v_send = -k_send - 0.5
    k_all = torch.empty((world * L, H, 64))
    v_all = torch.empty((world * L, H, 64))
    gather_kv(k_send, v_send, k_all, v_all)
    results[rank] = (k_all[:, 1, 63].tolist(), v_all[:, 0, 0].tolist())
    dist.barrier()
    dist.destroy_process_group()


def test_sharded_global_gathers_kv_in_rank_order():
    """The exchange step of query-sharded global attention: every rank ends with
    all ranks' key/value rows, rank r's block at token offset r * L."""
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.spawn(_gather_worker, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    for r in range(world):
        k, v = res[r]
        assert k == [1.0] * 5 + [2.0] * 5
        assert v == [-1.5] * 5 + [-2.5] * 5


# ---------------------------------------------------------------- bench --sharded: one scene split by frames
def test_scene_frames_partition_covers_the_scene_in_rank_order():
    import bench
    for world in (1, 2, 4, 5):
        parts = [bench.scene_frames(100, world, r) for r in range(world)]
        assert [f for p in parts for f in p] == list(range(100))
        assert len({len(p) for p in parts}) == 1
    with pytest.raises(ValueError):
        bench.scene_frames(100, 8, 0)


def test_frame_range_draw_equals_the_whole_scene_draw():
    import numpy as np
    import workloads as W
    shape = W.Shape(S=6, T=9, H=2, n_special=1, grid_h=2, grid_w=4)
    full = W.make_qkv(shape, 1234, 0.5)
    np.testing.assert_array_equal(W.make_qkv(shape, 1234, 0.5, range(2, 5)), full[2:5])
    np.testing.assert_array_equal(W.make_qkv(shape, 1234, 0.0, range(0, 6)), W.make_qkv(shape, 1234, 0.0))


def _scene_worker(rank, world, port, results):
    import datetime
    import sys
    import numpy as np
    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    import workloads as W
    from vit_attention_b200.sharded import gather_kv
    shape = W.Shape(S=4, T=5, H=2, n_special=1, grid_h=2, grid_w=2)
    frames = bench.scene_frames(shape.S, world, rank)
    mine = W.make_qkv(shape, 77, 0.5, frames)                       # [S/world, T, 3, H, 64] bits
    # this rank's keys and values token-major, as the shard prologue's send buffers hold them
    k_send = torch.from_numpy(mine[:, :, 1].reshape(-1, shape.H, 64).astype(np.float32))
    v_send = torch.from_numpy(mine[:, :, 2].reshape(-1, shape.H, 64).astype(np.float32))
    k_all = torch.empty((world * k_send.shape[0], shape.H, 64))
    v_all = torch.empty_like(k_all)
    gather_kv(k_send, v_send, k_all, v_all)
    full = W.make_qkv(shape, 77, 0.5)
    ok_k = np.array_equal(k_all.numpy(), full[:, :, 1].reshape(-1, shape.H, 64).astype(np.float32))
    ok_v = np.array_equal(v_all.numpy(), full[:, :, 2].reshape(-1, shape.H, 64).astype(np.float32))
    results[rank] = (list(frames), ok_k, ok_v, bench.reduce_max(float(rank)))
    dist.barrier()
    dist.destroy_process_group()


def test_sharded_scene_gathers_the_whole_scene_on_every_rank():
    """bench --sharded's host side on 2 gloo ranks: each rank draws only its frames, and the all-gather in rank
    order rebuilds the whole scene's keys and values exactly (the layout the shard core reads)."""
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.spawn(_scene_worker, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    assert res[0][0] == [0, 1] and res[1][0] == [2, 3]
    for r in range(world):
        assert res[r][1] and res[r][2]
        assert res[r][3] == 1.0


# ---------------------------------------------------------------- overlapped form: the order of the host's steps
class _Stream:
    def __init__(self, name, log):
        self.name, self.log, self.device = name, log, "cuda:0"

    def wait_stream(self, other):
        self.log.append(("wait", self.name, other.name))


class _Buf:
    def __init__(self, name, log):
        self.name, self.log = name, log

    def copy_(self, src):
        self.log.append(("copy", self.name, src.name))


def _fake_sharded(monkeypatch, world, rank):
    """sharded.global_attention_sharded with the library calls, the streams and the process group replaced
    by recorders: returns (the call, the log).  Each log entry names the stream it was enqueued on."""
    V = pytest.importorskip("vit_attention_b200", reason="libvggt_attn.so is not built")
    import contextlib
    import torch
    import torch.distributed as dist
    from vit_attention_b200 import sharded
    log = []
    main, comm = _Stream("main", log), _Stream("comm", log)
    current = [main]

    @contextlib.contextmanager
    def on(stream):
        prev = current[0]
        current[0] = stream
        try:
            yield
        finally:
            current[0] = prev

    bufs = [_Buf(n, log) for n in ("k_send", "v_send", "k_all", "v_all")]
    monkeypatch.setattr(torch.cuda, "stream", on)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a: current[0])
    monkeypatch.setattr(sharded, "_side_stream", lambda device: comm)
    monkeypatch.setattr(dist, "is_initialized", lambda: True)
    monkeypatch.setattr(dist, "get_world_size", lambda group=None: world)
    monkeypatch.setattr(dist, "get_rank", lambda group=None: rank)
    monkeypatch.setattr(sharded, "gather_kv", lambda *a, **k: log.append(("gather", current[0].name)))
    monkeypatch.setattr(V, "vggt_attn_shard_buffers", lambda *a, **k: bufs)
    monkeypatch.setattr(V, "vggt_attn_global_shard_prologue", lambda *a, stream=None, **k: log.append(("prologue", stream.name)))
    monkeypatch.setattr(V, "vggt_attn_global_shard_core", lambda *a, stream=None, **k: log.append(("core", stream.name)))
    monkeypatch.setattr(V, "vggt_attn_global_shard_core_local",
                        lambda *a, stream=None, **k: log.append(("core_local", stream.name)))
    monkeypatch.setattr(V, "vggt_attn_global_shard_core_remote",
                        lambda shape, w, r, *a, stream=None, **k: log.append(("core_remote", stream.name, r)))

    def call(**kw):
        sharded.global_attention_sharded("shape", None, None, None, None, None, "out", "ws", stream=main, **kw)
        return log
    return call


@pytest.mark.parametrize("world,rank", [(2, 1), (8, 3), (9, 8)])
def test_overlapped_steps_gather_beside_the_own_keys_core(monkeypatch, world, rank):
    log = _fake_sharded(monkeypatch, world, rank)(overlap=True)
    assert log == [("prologue", "main"),
                   ("wait", "comm", "main"),          # the side stream waits for the send buffers
                   ("gather", "comm"),                # the all-gather on the side stream ...
                   ("core_local", "main"),            # ... beside the own keys' core, which does not wait for it
                   ("wait", "main", "comm"),          # the remote keys' core waits for the gather
                   ("core_remote", "main", rank)]


@pytest.mark.parametrize("world,overlap", [(2, None), (2, False), (10, True)])
def test_gather_then_one_core_without_overlap(monkeypatch, world, overlap):
    kw = {} if overlap is None else {"overlap": overlap}      # the default is the one-pass core
    log = _fake_sharded(monkeypatch, world, 0)(**kw)
    assert log == [("prologue", "main"), ("gather", "main"), ("core", "main")]


def test_one_rank_copies_instead_of_gathering(monkeypatch):
    log = _fake_sharded(monkeypatch, 1, 0)()
    assert log == [("prologue", "main"), ("copy", "k_all", "k_send"), ("copy", "v_all", "v_send"), ("core", "main")]
