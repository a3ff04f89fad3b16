"""Query-sharded global attention over the ranks of a torch.distributed group
(one GPU per rank, NCCL over NVLink): each rank holds the same number of
consecutive frames of one scene; its queries attend to the keys of every
frame.  The exchange step is one all-gather of the normalised, rotated keys and
one of the values (token-major, rank-major); the prologue before it and the
attention core after it are the library's kernels (vggt_attn_global_shard_*).

The collective is the only data-path communication: head-sharded global
attention (each rank a subset of heads over all tokens) needs none and is plain
vggt_attn_global on a head slice of qkv.
"""
from __future__ import annotations


def gather_kv(k_send, v_send, k_all, v_all, group=None) -> None:
    """k_all <- [k_send of rank 0; rank 1; ...] and v_all likewise (rank order = frame order)."""
    import torch.distributed as dist
    dist.all_gather_into_tensor(k_all, k_send, group=group)
    dist.all_gather_into_tensor(v_all, v_send, group=group)


def global_attention_sharded(shape, qkv, q_gamma, q_beta, k_gamma, k_beta, out, workspace, group=None,
                             stream=None) -> None:
    """This rank's rows of global attention over the whole scene.

    shape: the LOCAL shape (S = frames on this rank, equal on every rank);
    qkv: this rank's frames, bf16 [S][T][3][H][64]; out: bf16 [S][T][H][64];
    workspace: uint8 tensor of vggt_attn_shard_workspace_size(shape, world) bytes.
    """
    import torch
    import torch.distributed as dist
    import vit_attention_b200 as V
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    V.vggt_attn_global_shard_prologue(shape, world, qkv, q_gamma, q_beta, k_gamma, k_beta, workspace,
                                      stream=stream)
    k_send, v_send, k_all, v_all = V.vggt_attn_shard_buffers(shape, world, workspace)
    if world == 1:
        k_all.copy_(k_send)
        v_all.copy_(v_send)
    else:
        s = stream if stream is not None else torch.cuda.current_stream()
        with torch.cuda.stream(s):
            gather_kv(k_send, v_send, k_all, v_all, group)
    V.vggt_attn_global_shard_core(shape, world, out, workspace, stream=stream)
