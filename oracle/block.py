"""fp64 oracle of the transformer blocks and the alternating-attention layer
schedule around the attention core (test infrastructure).

Source, cited by page title and section:
  [P1] VGGT-Omega Aggregator explainer -- section 3: the Aggregator is 24
       layers deep; every layer runs a frame block (attention within each
       frame, with 2D RoPE) and then an inter-frame block, global (all tokens
       of all frames) except at the layer indices [2, 6, 9, 14, 20], where
       only the 17 camera + register tokens of every frame take part and the
       patch tokens stay in their own frame's path; the attention layers use
       Q/K normalisation together with LayerScale (initial value 1e-5).
  [P1] section 2: the patch tokens come from a DINO-style ViT, whose block
       the Aggregator's blocks follow.
  [P1] section 4: only layers 4, 11, 17 and 23 are cached, each as the
       frame-block and inter-frame-block outputs concatenated along channels
       (2 x 1024); the camera head takes the first 17 tokens (camera +
       registers) of every frame from the last layer and mixes them across
       frames again with 4 self-attention blocks.

Readings where the page is silent:
  * A block is the pre-norm transformer block of a DINO-style ViT:
        x <- x + ls1 * proj(attention(qkv(norm1(x))))
        x <- x + ls2 * fc2(GELU(fc1(norm2(x))))
    norm1/norm2 are LayerNorms over the C channels of a token (biased
    variance, caller-given epsilon); the MLP hidden width is 4C; GELU is the
    exact form x * Phi(x); ls1, ls2 are per-channel LayerScale vectors.
  * In a register layer the whole inter-frame block (both residual branches)
    acts on the special tokens only; patch tokens pass through unchanged.
  * The attention inside a block is the core's (QK-LayerNorm, RoPE on patch
    tokens, softmax attention in the block's mode) on the block's own qkv.
  * The camera head's blocks are blocks of the same form over the S x 17
    special tokens of the last layer's features (all frames attend to each
    other; special tokens carry no RoPE position), of the features' width
    (2 x 1024 for the concatenated frame and global outputs) with 64-wide
    heads.
"""
from __future__ import annotations

import numpy as np
from scipy.special import erf

from .attention import HEAD_DIM, attn_mode, bf16_to_f64, register_tokens

REGISTER_LAYERS = (2, 6, 9, 14, 20)      # [P1] section 3
N_LAYERS = 24                            # [P1] section 3


def token_layer_norm(x: np.ndarray, gamma, beta, eps: float) -> np.ndarray:
    """LayerNorm over the last axis (the C channels of a token), biased variance."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(gamma, np.float64) + np.asarray(beta, np.float64)


def gelu(x: np.ndarray) -> np.ndarray:
    """x * Phi(x), Phi the standard normal distribution function."""
    return x * 0.5 * (1.0 + erf(x / np.sqrt(2.0)))


def _affine(x: np.ndarray, w_bits, b) -> np.ndarray:
    y = x @ bf16_to_f64(w_bits).T
    return y if b is None else y + np.asarray(b, np.float64)


def block_forward(mode: str, shape, x, w, norm_eps: float, rows=None) -> np.ndarray:
    """One block applied to token features x (bf16 bits or fp64, ``[S*T, C]``).

    Returns fp64 ``[S*T, C]``.  mode: "frame", "global" or "register"; in
    register mode only the rows of the special tokens change.  ``rows``
    (flat token indices; special tokens only in register mode): return just
    those output rows, ``[len(rows), C]`` (every token still provides keys).
    """
    x = bf16_to_f64(x) if x.dtype == np.uint16 else np.asarray(x, np.float64)
    C = shape.H * HEAD_DIM
    subset = rows is not None
    if not subset:
        rows = register_tokens(shape) if mode == "register" else np.arange(shape.S * shape.T, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    # Attention branch: qkv of the tokens the mode's attention reads (the keys
    # of the returned rows and the rows themselves); other entries stay 0 and
    # are never read.
    if mode == "register":
        need = register_tokens(shape)
    elif mode == "frame" and subset:
        frames = np.unique(rows // shape.T)
        need = (frames[:, None] * shape.T + np.arange(shape.T)[None, :]).reshape(-1)
    else:
        need = np.arange(shape.S * shape.T, dtype=np.int64)
    h = token_layer_norm(x[need], w["norm1_gamma"], w["norm1_beta"], norm_eps)
    qkv = np.zeros((shape.S * shape.T, 3 * C))
    qkv[need] = _affine(h, w["w_qkv"], w.get("b_qkv"))
    qkv = qkv.reshape(shape.S, shape.T, 3, shape.H, HEAD_DIM)
    inputs = {"qkv_f64": qkv}
    for name in ("q_gamma", "q_beta", "k_gamma", "k_beta"):
        inputs[name] = w[name]
    a = attn_mode(mode, shape, inputs, rows).reshape(len(rows), C)
    xr = x[rows] + np.asarray(w["ls1"], np.float64) * _affine(a, w["w_proj"], w.get("b_proj"))
    # MLP branch on the same rows.
    h2 = token_layer_norm(xr, w["norm2_gamma"], w["norm2_beta"], norm_eps)
    u = gelu(_affine(h2, w["w_fc1"], w.get("b_fc1")))
    yr = xr + np.asarray(w["ls2"], np.float64) * _affine(u, w["w_fc2"], w.get("b_fc2"))
    if subset:
        return yr
    y = x.copy()
    y[rows] = yr
    return y


CACHED_LAYERS = (4, 11, 17, 23)          # [P1] section 4


def aggregator_forward(shape, x, frame_blocks, inter_blocks, register_layers, norm_eps: float,
                       cache_layers=()) -> np.ndarray:
    """Layer l: the frame block frame_blocks[l], then the inter-frame block
    inter_blocks[l], in register mode if l is in register_layers, else global.

    With ``cache_layers``, returns ``(y, cache)`` where cache[l] is ``[S*T, 2C]``:
    the layer's frame-block output and inter-frame-block output side by side
    ([P1] section 4: the heads read the cached layers' concatenated outputs).
    """
    y = bf16_to_f64(x) if x.dtype == np.uint16 else np.asarray(x, np.float64)
    cache = {}
    for l, (fw, iw) in enumerate(zip(frame_blocks, inter_blocks)):
        y = block_forward("frame", shape, y, fw, norm_eps)
        frame_out = y
        y = block_forward("register" if l in register_layers else "global", shape, y, iw, norm_eps)
        if l in cache_layers:
            cache[l] = np.concatenate([frame_out, y], axis=1)
    return (y, cache) if cache_layers else y


CAMERA_TRUNK_BLOCKS = 4                  # [P1] section 4


def camera_trunk_forward(shape, feats, blocks, norm_eps: float) -> np.ndarray:
    """The special tokens of every frame of feats ``[S*T, C]``, then each block in
    turn with attention among all of them.  Returns fp64 ``[S*n_special, C]``."""
    x = bf16_to_f64(feats) if feats.dtype == np.uint16 else np.asarray(feats, np.float64)
    y = x[register_tokens(shape)]
    tok_shape = type(shape)(**{**shape.__dict__, "T": shape.n_special, "grid_h": 0, "grid_w": 0})
    for w in blocks:
        y = block_forward("global", tok_shape, y, w, norm_eps)
    return y
