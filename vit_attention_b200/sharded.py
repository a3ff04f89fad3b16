"""Query-sharded global attention over the ranks of a torch.distributed group
(one GPU per rank, NCCL over NVLink): each rank holds the same number of
consecutive frames of one scene; its queries attend to the keys of every
frame.  The exchange step is one all-gather of the normalised, rotated keys and
one of the values (token-major, rank-major); the prologue before it and the
attention core after it are the library's kernels (vggt_attn_global_shard_*).

Overlapped (optional, 2 to 9 ranks): the all-gather runs on a side stream
while the compute stream runs the core over the rank's own keys
(vggt_attn_global_shard_core_local, which leaves each row's softmax state);
after the gather the core runs over the other ranks' keys and merges that
state (vggt_attn_global_shard_core_remote).  Only the gather time beyond the
local keys' attention stays exposed, but the two launches cost 4-7 % more
than the one-pass core (100-frame scene, 2-5 ranks, measured on a B200 with
the ranks run one after another), more than an all-gather at NVLink 5
speeds takes (1-4 % of the core), so it is off by default; it pays where the
link is much slower than the core.

The collective is the only data-path communication: head-sharded global
attention (each rank a subset of heads over all tokens) needs none and is plain
vggt_attn_global on a head slice of qkv.

Fused form (`PeerShards`): no gathered copy at all.  Every rank maps the
others' workspaces once (CUDA IPC handles exchanged over the process group);
after the prologues, one attention kernel per rank reads each rank's keys and
values straight from that rank's send buffers -- peer loads over NVLink,
tile by tile, overlapping the products (vggt_attn_global_shard_core_peers).
The ranks meet at a host barrier after their prologues (the buffers are
written) and after the core (they have been read) -- no kernel waits on
another rank.
"""
from __future__ import annotations


def gather_kv(k_send, v_send, k_all, v_all, group=None) -> None:
    """k_all <- [k_send of rank 0; rank 1; ...] and v_all likewise (rank order = frame order)."""
    import torch.distributed as dist
    dist.all_gather_into_tensor(k_all, k_send, group=group)
    dist.all_gather_into_tensor(v_all, v_send, group=group)


# The overlapped core's second launch reads one tensor map per remote rank.
MAX_OVERLAP_WORLD = 9

_side_streams = {}


def _side_stream(device):
    import torch
    key = torch.device(device).index
    if key not in _side_streams:
        _side_streams[key] = torch.cuda.Stream(device=device)
    return _side_streams[key]


def overlapped(world: int, overlap: bool) -> bool:
    """Whether global_attention_sharded runs the all-gather beside the local keys' attention."""
    return overlap and 2 <= world <= MAX_OVERLAP_WORLD


def global_attention_sharded(shape, qkv, q_gamma, q_beta, k_gamma, k_beta, out, workspace, group=None,
                             stream=None, overlap=False) -> None:
    """This rank's rows of global attention over the whole scene.

    shape: the LOCAL shape (S = frames on this rank, equal on every rank);
    qkv: this rank's frames, bf16 [S][T][3][H][64]; out: bf16 [S][T][H][64];
    workspace: uint8 tensor of vggt_attn_shard_workspace_size(shape, world) bytes.
    overlap: run the all-gather on a side stream beside the attention over the
    rank's own keys (2 to 9 ranks; equal to the one-pass result to rounding);
    otherwise gather first, then one core over all keys (bit for bit
    vggt_attn_global's rows).
    """
    import torch
    import torch.distributed as dist
    import vit_attention_b200 as V
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    V.vggt_attn_global_shard_prologue(shape, world, qkv, q_gamma, q_beta, k_gamma, k_beta, workspace,
                                      stream=stream)
    k_send, v_send, k_all, v_all = V.vggt_attn_shard_buffers(shape, world, workspace)
    s = stream if stream is not None else torch.cuda.current_stream()
    if world == 1:
        with torch.cuda.stream(s):
            k_all.copy_(k_send)
            v_all.copy_(v_send)
    elif overlapped(world, overlap):
        comm = _side_stream(s.device)
        comm.wait_stream(s)                       # the prologue has written the send buffers
        with torch.cuda.stream(comm):
            gather_kv(k_send, v_send, k_all, v_all, group)
        V.vggt_attn_global_shard_core_local(shape, world, workspace, stream=s)
        s.wait_stream(comm)                       # every rank's keys and values are gathered
        V.vggt_attn_global_shard_core_remote(shape, world, rank, out, workspace, stream=s)
        return
    else:
        with torch.cuda.stream(s):
            gather_kv(k_send, v_send, k_all, v_all, group)
    V.vggt_attn_global_shard_core(shape, world, out, workspace, stream=stream)


class PeerShards:
    """This rank's view of every rank's send buffers for the fused form.

    Built once per (workspace, shape): the workspace tensors of all ranks are
    shared through CUDA IPC (torch's tensor reduction), so every rank holds a
    mapping of every other rank's workspace.  ``group`` must be a CPU-capable
    process group (gloo) or any group supporting ``all_gather_object``.
    """

    def __init__(self, shape, workspace, group=None):
        import torch.distributed as dist
        from torch.multiprocessing.reductions import reduce_tensor
        import vit_attention_b200 as V
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.group = group
        self.shape = shape
        self.workspace = workspace
        k_send, v_send, _, _ = V.vggt_attn_shard_buffers(shape, self.world, workspace)
        k_off = k_send.data_ptr() - workspace.data_ptr()
        v_off = v_send.data_ptr() - workspace.data_ptr()
        if self.world == 1:
            self.peers = [workspace]
        else:
            handles = [None] * self.world
            dist.all_gather_object(handles, reduce_tensor(workspace), group=group)
            self.peers = [workspace if r == self.rank else fn(*args) for r, (fn, args) in enumerate(handles)]
        self.k_ptrs = [t.data_ptr() + k_off for t in self.peers]
        self.v_ptrs = [t.data_ptr() + v_off for t in self.peers]

    def attend(self, qkv, q_gamma, q_beta, k_gamma, k_beta, out, stream=None) -> None:
        """This rank's rows of global attention over the whole scene (see global_attention_sharded)."""
        import torch
        import torch.distributed as dist
        import vit_attention_b200 as V
        V.vggt_attn_global_shard_prologue(self.shape, self.world, qkv, q_gamma, q_beta, k_gamma, k_beta,
                                          self.workspace, stream=stream)
        if self.world > 1:
            (stream or torch.cuda.current_stream()).synchronize()
            dist.barrier(group=self.group)            # every rank's keys and values are written
        V.vggt_attn_global_shard_core_peers(self.shape, self.world, self.k_ptrs, self.v_ptrs, out, self.workspace,
                                            stream=stream)
        if self.world > 1:
            (stream or torch.cuda.current_stream()).synchronize()
            dist.barrier(group=self.group)            # and read: the next prologue may overwrite them
