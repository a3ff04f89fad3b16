"""fp64 oracle of descriptor attention (test infrastructure).

Source, cited by page title and section:
  [P2] FlashVGGT article, abstract: instead of dense global attention over all
       tokens, the spatial information of each frame is compressed into a
       compact set of descriptor tokens, and global attention becomes
       cross-attention between the full set of image tokens (queries) and the
       descriptors (keys and values).

Readings where the page is silent:
  * a frame's descriptors are its camera/register tokens, unchanged, plus one
    descriptor per s_h x s_w window of the patch grid (windows tile the grid
    from (0, 0); the last row/column of windows may be smaller) whose key is
    the mean of the window's QK-normalised, rotated keys and whose value is the
    mean of the window's values;
  * every query (all S*T tokens, normalised and rotated as in global mode)
    attends to the descriptors of all frames with ordinary softmax attention;
  * the chunk-recursive online mode (cached descriptors of earlier chunks) is
    not part of the operation.
With s_h = s_w = 1 every descriptor is one token and this is global attention.
"""
from __future__ import annotations

import numpy as np

from .attention import normalized_tokens, resolved_scale, softmax_attention


def descriptor_windows(shape, s_h: int, s_w: int):
    """List, per descriptor of all frames in order, of the flat token indices it averages."""
    nh = -(-shape.grid_h // s_h) if shape.grid_h > 0 else 0
    nw = -(-shape.grid_w // s_w) if shape.grid_w > 0 else 0
    out = []
    for s in range(shape.S):
        base = s * shape.T
        for t in range(shape.n_special):
            out.append(np.array([base + t]))
        for wr in range(nh):
            for wc in range(nw):
                rows = np.arange(wr * s_h, min((wr + 1) * s_h, shape.grid_h))
                cols = np.arange(wc * s_w, min((wc + 1) * s_w, shape.grid_w))
                t = shape.n_special + (rows[:, None] * shape.grid_w + cols[None, :]).reshape(-1)
                out.append(base + t)
    return out


def attn_global_desc(shape, inputs, s_h: int, s_w: int, queries=None) -> np.ndarray:
    """Descriptor attention output ``[n_q, H, 64]`` for flat query indices (default all)."""
    N = shape.S * shape.T
    qi = np.arange(N, dtype=np.int64) if queries is None else np.asarray(queries, dtype=np.int64)
    kv = normalized_tokens(shape, inputs, np.arange(N), ("k", "v"))          # [H, N, 64]
    qn = normalized_tokens(shape, inputs, qi, ("q",))["q"]                   # [H, n_q, 64]
    windows = descriptor_windows(shape, s_h, s_w)
    kd = np.stack([kv["k"][:, w].mean(axis=1) for w in windows], axis=1)    # [H, Nd, 64]
    vd = np.stack([kv["v"][:, w].mean(axis=1) for w in windows], axis=1)
    scale = resolved_scale(shape)
    out = np.empty((len(qi), shape.H, shape.head_dim))
    for h in range(shape.H):
        out[:, h] = softmax_attention(qn[h], kd[h], vd[h], scale)
    return out
