"""fp64 oracle of subsampled global attention (test infrastructure).

Source, cited by page title and section:
  [P4] AVGGT article, section B ("De Versnellingsstrategie"), point 2,
       "Subsampling van Globale Attention (SGA)": in the global layers the
       keys/values are subsampled on a 2D grid (one token per s_h x s_w window)
       while every query is kept; each token keeps its diagonal self-attention;
       all discarded columns are stood in for by one mean key-value pair.

Readings where the page is silent:
  * kept keys K = every camera/register token of every frame, plus the patch
    tokens at (row, col) with row % s_h == 0 and col % s_w == 0 (the first
    token of each window), in every frame;
  * discarded set D = all S*T tokens not in K; the mean pair is the mean over D
    of the QK-normalised, rotated keys and of the raw values;
  * query i attends to K, to itself when i is in D (the diagonal), and to the
    mean pair counted n_i = |D| - [i in D] times (the discarded columns it does
    not already see);
  * q, k normalisation, RoPE and the softmax scale are those of global mode.
With s_h = s_w = 1, D is empty and this is exact global attention.
"""
from __future__ import annotations

import numpy as np

from .attention import normalized_tokens, patch_row_col, resolved_scale


def sga_kept_tokens(shape, s_h: int, s_w: int) -> np.ndarray:
    """Sorted flat indices (s*T + t) of the kept keys K."""
    t = np.arange(shape.T)
    is_patch, row, col = patch_row_col(t, shape.n_special, shape.grid_w)
    keep_t = np.nonzero(~is_patch | ((row % s_h == 0) & (col % s_w == 0)))[0]
    return (np.arange(shape.S)[:, None] * shape.T + keep_t[None, :]).reshape(-1)


def attn_global_sga(shape, inputs, s_h: int, s_w: int, queries=None) -> np.ndarray:
    """SGA output ``[n_q, H, 64]`` for the given flat query indices (default all)."""
    N = shape.S * shape.T
    qi = np.arange(N, dtype=np.int64) if queries is None else np.asarray(queries, dtype=np.int64)
    kept = sga_kept_tokens(shape, s_h, s_w)
    in_kept = np.zeros(N, dtype=bool)
    in_kept[kept] = True
    disc = np.nonzero(~in_kept)[0]
    kv_all = normalized_tokens(shape, inputs, np.arange(N), ("k", "v"))      # [H, N, 64]
    qn = normalized_tokens(shape, inputs, qi, ("q",))["q"]                   # [H, n_q, 64]
    scale = resolved_scale(shape)
    out = np.empty((len(qi), shape.H, shape.head_dim))
    for h in range(shape.H):
        k, v = kv_all["k"][h], kv_all["v"][h]
        kK, vK = k[kept], v[kept]
        has_d = len(disc) > 0
        k_mean = k[disc].mean(axis=0) if has_d else np.zeros(shape.head_dim)
        v_mean = v[disc].mean(axis=0) if has_d else np.zeros(shape.head_dim)
        for a, i in enumerate(qi):
            q = qn[h, a]
            diag = not in_kept[i]
            n_mean = len(disc) - (1 if diag else 0)
            s = [scale * (kK @ q)]
            vals = [vK]
            w = [np.ones(len(kept))]
            if diag:
                s.append(np.array([scale * (k[i] @ q)]))
                vals.append(v[i][None])
                w.append(np.ones(1))
            if n_mean > 0:
                s.append(np.array([scale * (k_mean @ q)]))
                vals.append(v_mean[None])
                w.append(np.array([float(n_mean)]))
            s = np.concatenate(s)
            w = np.concatenate(w)
            vv = np.concatenate(vals)
            m = s.max()
            p = w * np.exp(s - m)
            out[a, h] = (p @ vv) / p.sum()
    return out
