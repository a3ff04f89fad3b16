"""Seeded synthetic workloads for the alternating-attention core.

This module only *draws* inputs; it holds none of the method's arithmetic
(no normalisation, no rotary positions, no attention).  Both the fp64 oracle
and the CUDA path consume exactly the arrays produced here:

  * ``qkv``  -- bf16 bit patterns (``numpy.uint16``) of shape ``[S, T, 3, H, 64]``,
    i.e. per frame ``s`` and token ``t`` the packed q, k and v vectors of every
    head.  Tokens ``t < n_special`` are the camera + register tokens, the rest
    are the patch tokens of a ``grid_h x grid_w`` patch grid in row-major order
    (VGGT-Omega Aggregator explainer, section 2 "Token recipe").
  * ``q_gamma, q_beta, k_gamma, k_beta`` -- float32 ``[H, 64]`` affine
    parameters of the per-head QK-LayerNorm (same page, section 3,
    "use_qk_norm=True").

Value recipe (no dataset is used; the shapes stand in for the pages'
624x416 images cut into 16x16 patches, 1 camera + 16 register tokens and
16 heads x 64 = 1024 channels):

  * qkv entries are N(0,1) float32 draws rounded to bf16 (round to nearest even).
  * the long global workload adds ``0.5 * u[t, c, h, d]`` to every frame, with
    ``u`` one more N(0,1) draw shared by all frames at the same token position
    (a stand-in for the temporal redundancy that HTTM's similarity analysis
    describes, "04 method").
  * gamma = 1 + 0.1 N(0,1), beta = 0.1 N(0,1), separately for q and k.

Seeds: frame ``s`` of qkv uses ``default_rng([seed, 0, s])``; the affine parameters use
``default_rng([seed, 1])``; query subsets use ``default_rng([seed, 2])``; the
shared low-rank component uses ``default_rng([seed, 3])``.  The seed of
workload ``i`` in ``WORKLOADS`` is ``1000 + i``.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import os
from typing import Dict, List, Optional

import numpy as np

HEAD_DIM = 64


@dataclasses.dataclass(frozen=True)
class Shape:
    """Problem shape shared by the oracle and the CUDA library.

    ``softmax_scale <= 0`` means ``1/sqrt(head_dim)``.
    """

    S: int
    T: int
    H: int
    n_special: int
    grid_h: int
    grid_w: int
    head_dim: int = HEAD_DIM
    ln_eps: float = 1e-5
    rope_base: float = 100.0
    softmax_scale: float = 0.0

    def __post_init__(self):
        if self.T != self.n_special + self.grid_h * self.grid_w:
            raise ValueError(
                f"T={self.T} must equal n_special + grid_h*grid_w = "
                f"{self.n_special + self.grid_h * self.grid_w}")

    @property
    def n_tokens(self) -> int:
        return self.S * self.T

    @property
    def n_register_tokens(self) -> int:
        return self.S * self.n_special


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    modes: tuple          # modes run on this input, in order
    shape: Shape
    lowrank: float = 0.0  # weight of the shared same-position component
    seed: int = 0


def _frame_shape(S: int, H: int = 16) -> Shape:
    # 624x416 pixels cut into 16x16 patches -> 39 columns x 26 rows,
    # plus 1 camera + 16 register tokens = 1031 tokens per frame.
    return Shape(S=S, T=17 + 26 * 39, H=H, n_special=17, grid_h=26, grid_w=39)


WORKLOADS: List[Workload] = [
    Workload("global_tiny_S2_T69_H4", ("global",),
             Shape(S=2, T=69, H=4, n_special=5, grid_h=8, grid_w=8), 0.0, 1000),
    Workload("frame_S24_T1031_H16", ("frame",), _frame_shape(24), 0.0, 1001),
    Workload("global_S24_N24744_H16", ("global",), _frame_shape(24), 0.0, 1002),
    Workload("global_S100_N103100_H16_lowrank", ("global",), _frame_shape(100), 0.5, 1003),
    Workload("register_frame_layer_S500_T1031_H16", ("register", "frame"),
             _frame_shape(500), 0.0, 1004),
]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return the bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def make_norm_params(H: int, seed: int, head_dim: int = HEAD_DIM) -> Dict[str, np.ndarray]:
    rng = np.random.default_rng([seed, 1])
    out = {}
    for name in ("q", "k"):
        out[f"{name}_gamma"] = (1.0 + 0.1 * rng.standard_normal((H, head_dim))).astype(np.float32)
        out[f"{name}_beta"] = (0.1 * rng.standard_normal((H, head_dim))).astype(np.float32)
    return out


def make_qkv(shape: Shape, seed: int, lowrank: float = 0.0, frames: Optional[range] = None) -> np.ndarray:
    """Seeded bf16 ``qkv[S, T, 3, H, head_dim]`` bit patterns (uint16).

    Frame ``s`` is drawn from its own generator ``default_rng([seed, 0, s])``,
    so frames can be drawn in parallel and the result does not depend on the
    number of threads.  ``frames`` (a range of frame indices) draws only those
    frames, ``[len(frames), T, 3, H, head_dim]``, equal to the same frames of
    the whole draw (a rank's share of a scene split by frames).
    """
    S, T, H, D = shape.S, shape.T, shape.H, shape.head_dim
    frames = range(S) if frames is None else frames
    shared = None
    if lowrank:
        shared = (lowrank * np.random.default_rng([seed, 3]).standard_normal(
            (T, 3, H, D), dtype=np.float32)).astype(np.float32)
    bits = np.empty((len(frames), T, 3, H, D), dtype=np.uint16)

    def draw(i: int) -> None:
        z = np.random.default_rng([seed, 0, frames[i]]).standard_normal((T, 3, H, D), dtype=np.float32)
        if shared is not None:
            z += shared
        bits[i] = f32_to_bf16_bits(z)

    if len(frames) * T * 3 * H * D >= (1 << 22):
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(draw, range(len(frames))))
    else:
        for i in range(len(frames)):
            draw(i)
    return bits


def make_inputs(workload: Workload) -> Dict[str, np.ndarray]:
    inputs = make_norm_params(workload.shape.H, workload.seed, workload.shape.head_dim)
    inputs["qkv"] = make_qkv(workload.shape, workload.seed, workload.lowrank)
    return inputs


def make_random_inputs(shape: Shape, seed: int, lowrank: float = 0.0) -> Dict[str, np.ndarray]:
    """Inputs for an arbitrary (test) shape with the same recipe."""
    inputs = make_norm_params(shape.H, seed, shape.head_dim)
    inputs["qkv"] = make_qkv(shape, seed, lowrank)
    return inputs


def make_block_inputs(shape: Shape, seed: int) -> Dict[str, np.ndarray]:
    """Seeded inputs of one attention block on token features (projections included).

    x: bf16 bits ``[S*T, C]`` ~ N(0, 1), C = H * head_dim (frame s from
    ``default_rng([seed, 4, s])``); w_qkv ``[3C, C]`` and w_out ``[C, C]``: bf16
    bits ~ N(0, 1/C), so projected values are ~ N(0, 1); b_qkv ``[3C]`` and b_out
    ``[C]``: fp32 ~ 0.1 N(0, 1); q/k gamma/beta as for the attention core.
    """
    S, T, C = shape.S, shape.T, shape.H * shape.head_dim
    out = make_norm_params(shape.H, seed, shape.head_dim)
    x = np.empty((S * T, C), dtype=np.uint16)
    for s in range(S):
        x[s * T:(s + 1) * T] = f32_to_bf16_bits(
            np.random.default_rng([seed, 4, s]).standard_normal((T, C), dtype=np.float32))
    out["x"] = x
    sd = np.float32(1.0 / np.sqrt(C))
    out["w_qkv"] = f32_to_bf16_bits(np.random.default_rng([seed, 5]).standard_normal((3 * C, C), dtype=np.float32) * sd)
    out["b_qkv"] = (0.1 * np.random.default_rng([seed, 6]).standard_normal(3 * C)).astype(np.float32)
    out["w_out"] = f32_to_bf16_bits(np.random.default_rng([seed, 7]).standard_normal((C, C), dtype=np.float32) * sd)
    out["b_out"] = (0.1 * np.random.default_rng([seed, 8]).standard_normal(C)).astype(np.float32)
    return out


def make_tokens(shape: Shape, seed: int) -> np.ndarray:
    """Seeded token features x: bf16 bits ``[S*T, C]`` ~ N(0, 1), frame s from ``default_rng([seed, 4, s])``."""
    S, T, C = shape.S, shape.T, shape.H * shape.head_dim
    x = np.empty((S * T, C), dtype=np.uint16)
    for s in range(S):
        x[s * T:(s + 1) * T] = f32_to_bf16_bits(
            np.random.default_rng([seed, 4, s]).standard_normal((T, C), dtype=np.float32))
    return x


def make_transformer_block_weights(H: int, seed: int, head_dim: int = HEAD_DIM) -> Dict[str, np.ndarray]:
    """Seeded weights of one pre-norm transformer block, C = H * head_dim, hidden width 4C.

    Matrices are bf16 bits in nn.Linear layout ``[out][in]`` ~ N(0, 1/in) (each
    product then has unit variance): w_qkv ``[3C, C]``, w_proj ``[C, C]``, w_fc1
    ``[4C, C]``, w_fc2 ``[C, 4C]``.  Vectors are fp32: norm gammas and LayerScales
    1 + 0.1 N(0, 1) (LayerScale drawn near 1, not at its 1e-5 initial value, so
    that both branches of the block show in its output), norm betas and biases
    0.1 N(0, 1); q/k gamma/beta as for the attention core.  Item k uses
    ``default_rng([seed, 20 + k])``.
    """
    C = H * head_dim
    out = make_norm_params(H, seed, head_dim)

    def rng(k):
        return np.random.default_rng([seed, 20 + k])

    def mat(k, n_out, n_in):
        sd = np.float32(1.0 / np.sqrt(n_in))
        return f32_to_bf16_bits(rng(k).standard_normal((n_out, n_in), dtype=np.float32) * sd)

    def vec(k, n, centre):
        return (centre + 0.1 * rng(k).standard_normal(n)).astype(np.float32)

    out["norm1_gamma"], out["norm1_beta"] = vec(0, C, 1.0), vec(1, C, 0.0)
    out["w_qkv"], out["b_qkv"] = mat(2, 3 * C, C), vec(3, 3 * C, 0.0)
    out["w_proj"], out["b_proj"] = mat(4, C, C), vec(5, C, 0.0)
    out["ls1"] = vec(6, C, 1.0)
    out["norm2_gamma"], out["norm2_beta"] = vec(7, C, 1.0), vec(8, C, 0.0)
    out["w_fc1"], out["b_fc1"] = mat(9, 4 * C, C), vec(10, 4 * C, 0.0)
    out["w_fc2"], out["b_fc2"] = mat(11, C, 4 * C), vec(12, C, 0.0)
    out["ls2"] = vec(13, C, 1.0)
    return out


def query_subset(n_queries: int, count: int, seed: int) -> np.ndarray:
    """Sorted seeded subset of query indices (all of them if count >= n)."""
    if count >= n_queries:
        return np.arange(n_queries, dtype=np.int64)
    rng = np.random.default_rng([seed, 2])
    return np.sort(rng.choice(n_queries, size=count, replace=False)).astype(np.int64)


def workload(index_or_name) -> Workload:
    if isinstance(index_or_name, int):
        return WORKLOADS[index_or_name]
    for w in WORKLOADS:
        if w.name == index_or_name:
            return w
    raise KeyError(index_or_name)
