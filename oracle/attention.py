"""fp64 oracle functions (test infrastructure; see the package docstring).

Sources, cited by page title and section:
  [P1] VGGT-Omega Aggregator explainer -- section 2 (token recipe
       [1 camera][16 register][N patch], 16x16 patches), section 3
       (alternating frame / inter-frame attention, global and register
       modes, 2D RoPE, QK-norm).
  [P3] HTTM article, "04 method" -- RoPE re-applied at every attention layer
       of VGGT, applied identically to every frame.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence, Tuple

import numpy as np

HEAD_DIM = 64
ROPE_HALF = HEAD_DIM // 2        # dims per spatial axis (row, col)
ROPE_PAIRS = ROPE_HALF // 2      # rotation pairs per axis


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns, as float64."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def layer_norm(x: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float) -> np.ndarray:
    """LayerNorm over the last axis with biased variance ([P1] section 3, QK-norm).

    y = gamma * (x - mean) / sqrt(var + eps) + beta, var = mean((x - mean)^2).
    """
    x = np.asarray(x, dtype=np.float64)
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)
    return (x - mean) / np.sqrt(var + eps) * np.asarray(gamma, np.float64) + np.asarray(beta, np.float64)


def rope_frequencies(base: float) -> np.ndarray:
    """Angular frequency of each rotation pair inside one 32-dim half.

    omega_j = base^(-2j / 32) for j = 0..15 ([P1] section 3: 2D RoPE; base and
    the half-row/half-col split are fixed by the workload description).
    """
    j = np.arange(ROPE_PAIRS, dtype=np.float64)
    return np.power(float(base), -2.0 * j / ROPE_HALF)


def patch_row_col(t: np.ndarray, n_special: int, grid_w: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(is_patch, row, col) of in-frame token indices t ([P1] section 2).

    Tokens t < n_special are camera/register tokens; patch p = t - n_special
    sits at row p // grid_w, column p % grid_w (row-major patch grid).
    Row and col are returned as 0 for special tokens.
    """
    t = np.asarray(t, dtype=np.int64)
    is_patch = t >= n_special
    p = np.where(is_patch, t - n_special, 0)
    gw = grid_w if grid_w > 0 else 1          # a frame of special tokens only has no patch grid
    return is_patch, p // gw, p % gw


def _rotate_half_block(x: np.ndarray, pos: np.ndarray, omega: np.ndarray) -> np.ndarray:
    """Rotate pairs (j, j+16) of a 32-dim block by angle pos * omega_j."""
    ang = pos[..., None].astype(np.float64) * omega          # [..., 16]
    c, s = np.cos(ang), np.sin(ang)
    a = x[..., :ROPE_PAIRS]
    b = x[..., ROPE_PAIRS:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def rope_2d(x: np.ndarray, row: np.ndarray, col: np.ndarray, base: float) -> np.ndarray:
    """2D rotary embedding of 64-dim vectors x[..., 64] at (row, col).

    Dims [0, 32) rotate by the row position, dims [32, 64) by the column
    ([P1] section 3; [P3] "04 method").  ``row``/``col`` broadcast against
    x.shape[:-1].
    """
    omega = rope_frequencies(base)
    x = np.asarray(x, dtype=np.float64)
    row = np.broadcast_to(np.asarray(row, dtype=np.float64), x.shape[:-1])
    col = np.broadcast_to(np.asarray(col, dtype=np.float64), x.shape[:-1])
    return np.concatenate([_rotate_half_block(x[..., :ROPE_HALF], row, omega),
                           _rotate_half_block(x[..., ROPE_HALF:], col, omega)], axis=-1)


def normalized_tokens(shape, inputs, flat_tokens: np.ndarray, which: Sequence[str] = ("q", "k", "v")):
    """QK-LayerNorm + RoPE'd q, k and raw v of the listed tokens.

    ``flat_tokens`` are indices into the S*T token sequence (s*T + t).  q, k
    and v come from ``inputs["qkv"]`` (bf16 bits ``[S, T, 3, H, 64]``), or from
    ``inputs["qkv_f64"]`` (fp64, same shape) when the block's projection made them.
    Returns a dict of fp64 arrays ``[H, n, 64]`` for each name in ``which``.
    """
    flat_tokens = np.asarray(flat_tokens, dtype=np.int64)
    s, t = flat_tokens // shape.T, flat_tokens % shape.T
    is_patch, row, col = patch_row_col(t, shape.n_special, shape.grid_w)
    out = {}
    for c, name in enumerate(("q", "k", "v")):
        if name not in which:
            continue
        if "qkv_f64" in inputs:                              # projected in fp64 (attention block)
            x = np.asarray(inputs["qkv_f64"][s, t, c], dtype=np.float64)
        else:
            x = bf16_to_f64(inputs["qkv"][s, t, c])          # [n, H, 64]
        if name != "v":
            x = layer_norm(x, inputs[f"{name}_gamma"][None], inputs[f"{name}_beta"][None], shape.ln_eps)
            rot = rope_2d(x, row[:, None], col[:, None], shape.rope_base)
            x = np.where(is_patch[:, None, None], rot, x)
        out[name] = np.ascontiguousarray(x.transpose(1, 0, 2))  # [H, n, 64]
    return out


def resolved_scale(shape) -> float:
    return float(shape.softmax_scale) if shape.softmax_scale > 0 else 1.0 / math.sqrt(shape.head_dim)


def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                      mask: Optional[np.ndarray] = None, return_probs: bool = False,
                      chunk: int = 512):
    """Exact softmax attention of one head, fp64.

    s_ij = scale * q_i . k_j ; m_i = max_j s_ij ; p_ij = exp(s_ij - m_i);
    o_i = sum_j p_ij v_j / sum_j p_ij.  ``mask[i, j] == False`` removes key j
    for query i.  Queries are processed ``chunk`` rows at a time (each row is
    independent, so this is the definition, only less memory at once).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    out = np.empty((q.shape[0], v.shape[1]), dtype=np.float64)
    probs = np.empty((q.shape[0], k.shape[0]), dtype=np.float64) if return_probs else None
    for a in range(0, q.shape[0], chunk):
        b = min(a + chunk, q.shape[0])
        s = scale * (q[a:b] @ k.T)
        if mask is not None:
            s = np.where(mask[a:b], s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        den = p.sum(axis=1, keepdims=True)
        out[a:b] = (p @ v) / den
        if return_probs:
            probs[a:b] = p / den
    return (out, probs) if return_probs else out


def _queries_or_all(n: int, queries) -> np.ndarray:
    return np.arange(n, dtype=np.int64) if queries is None else np.asarray(queries, dtype=np.int64)


def attn_global(shape, inputs, queries=None) -> np.ndarray:
    """Global mode: every query attends over all S*T tokens ([P1] section 3, mode 1).

    ``queries``: flat token indices (default all).  Returns ``[n_q, H, 64]``.
    """
    N = shape.S * shape.T
    qi = _queries_or_all(N, queries)
    kv = normalized_tokens(shape, inputs, np.arange(N), ("k", "v"))
    qn = normalized_tokens(shape, inputs, qi, ("q",))["q"]
    scale = resolved_scale(shape)
    out = np.empty((len(qi), shape.H, shape.head_dim))
    for h in range(shape.H):
        out[:, h] = softmax_attention(qn[h], kv["k"][h], kv["v"][h], scale)
    return out


def attn_frame(shape, inputs, queries=None) -> np.ndarray:
    """Frame mode: each query attends over the T tokens of its own frame ([P1] section 3, step 1).

    ``queries``: flat token indices (default all).  Returns ``[n_q, H, 64]``.
    """
    qi = _queries_or_all(shape.S * shape.T, queries)
    frames = qi // shape.T
    scale = resolved_scale(shape)
    out = np.empty((len(qi), shape.H, shape.head_dim))
    for f in np.unique(frames):
        sel = np.nonzero(frames == f)[0]
        kv = normalized_tokens(shape, inputs, f * shape.T + np.arange(shape.T), ("k", "v"))
        qn = normalized_tokens(shape, inputs, qi[sel], ("q",))["q"]
        for h in range(shape.H):
            out[sel, h] = softmax_attention(qn[h], kv["k"][h], kv["v"][h], scale)
    return out


def register_tokens(shape) -> np.ndarray:
    """Flat indices of the camera + register tokens of every frame ([P1] section 3, mode 2)."""
    return (np.arange(shape.S)[:, None] * shape.T + np.arange(shape.n_special)[None, :]).reshape(-1)


def attn_register(shape, inputs, queries=None) -> np.ndarray:
    """Register mode: only the n_special special tokens of every frame attend, over each other.

    ``queries``: flat token indices of special tokens (default all of them).
    Returns ``[n_q, H, 64]``.  Patch tokens take no part (their output rows are
    not written by this mode).
    """
    keys = register_tokens(shape)
    qi = keys if queries is None else np.asarray(queries, dtype=np.int64)
    if np.any(qi % shape.T >= shape.n_special):
        raise ValueError("register-mode queries must be special tokens")
    kv = normalized_tokens(shape, inputs, keys, ("k", "v"))
    qn = normalized_tokens(shape, inputs, qi, ("q",))["q"]
    scale = resolved_scale(shape)
    out = np.empty((len(qi), shape.H, shape.head_dim))
    for h in range(shape.H):
        out[:, h] = softmax_attention(qn[h], kv["k"][h], kv["v"][h], scale)
    return out


def attn_mode(mode: str, shape, inputs, queries=None) -> np.ndarray:
    return {"frame": attn_frame, "global": attn_global, "register": attn_register}[mode](shape, inputs, queries)
