"""fp64 oracle of the projections around the attention core (test infrastructure).

Source, cited by page title and section:
  [P1] VGGT-Omega Aggregator explainer -- section 3: every attention block of
       the alternating-attention layer maps its C = 16 x 64 = 1024 channels to
       q, k and v (one linear projection, then the per-head QK-norm and RoPE of
       the attention core) and maps the attention output back to C channels.

Readings where the page is silent: the projections are
nn.Linear maps y = x W^T + b with W stored [out_features][in_features]; the
3C outputs of the QKV projection are ordered [q | k | v], each [H][64].
"""
from __future__ import annotations

import numpy as np

from .attention import HEAD_DIM, attn_mode, bf16_to_f64


def linear(x, w, b=None) -> np.ndarray:
    """y = x W^T + b in fp64; x, w are bf16 bit patterns ([M, K], [N, K]), b fp32 [N] or None."""
    y = bf16_to_f64(x) @ bf16_to_f64(w).T
    if b is not None:
        y = y + np.asarray(b, dtype=np.float64)
    return y


def projected_qkv(shape, block) -> np.ndarray:
    """fp64 qkv [S, T, 3, H, 64] of a block's QKV projection of x ([P1] section 3)."""
    y = linear(block["x"], block["w_qkv"], block.get("b_qkv"))
    return y.reshape(shape.S, shape.T, 3, shape.H, HEAD_DIM)


def attention_block(mode: str, shape, block, queries=None) -> np.ndarray:
    """One attention block on token features x: QKV projection, the attention
    core (QK-norm, RoPE, softmax attention in ``mode``), output projection.

    ``queries``: flat token indices (default all).  Returns fp64 ``[n_q, C]``.
    """
    inputs = {"qkv_f64": projected_qkv(shape, block)}
    for name in ("q_gamma", "q_beta", "k_gamma", "k_beta"):
        inputs[name] = block[name]
    attn = attn_mode(mode, shape, inputs, queries)               # [n_q, H, 64]
    a = attn.reshape(attn.shape[0], shape.H * HEAD_DIM)
    y = a @ bf16_to_f64(block["w_out"]).T
    if block.get("b_out") is not None:
        y = y + np.asarray(block["b_out"], dtype=np.float64)
    return y
