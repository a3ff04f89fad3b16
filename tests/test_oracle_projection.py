"""Pins of the projection oracle (oracle/projection.py) -- CPU only.

The attention block of the VGGT-Omega Aggregator explainer (section 3)
projects token features to q, k, v and the attention output back; the oracle
writes that out in fp64.  These tests pin it to things other than itself: a
permutation weight (a transposed W would give the inverse permutation), torch's
fp64 linear (alone, and for both random projections around the pinned
attention oracle), and identity projections that reduce the block to that
attention oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.filterwarnings("ignore")


def _bits(a):
    return W.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def test_linear_permutation_weight_selects_columns():
    rng = np.random.default_rng(3)
    M, K, N = 5, 12, 7
    x = _bits(rng.integers(-8, 8, (M, K)))                 # small integers: exact in bf16
    perm = rng.permutation(K)[:N]
    w = np.zeros((N, K), dtype=np.float32)
    w[np.arange(N), perm] = 1.0
    b = np.arange(N, dtype=np.float32) * 0.5
    y = oracle.linear(x, _bits(w), b)
    expect = oracle.bf16_to_f64(x)[:, perm] + b
    np.testing.assert_array_equal(y, expect)


def test_linear_matches_torch_fp64():
    rng = np.random.default_rng(4)
    x = _bits(rng.standard_normal((9, 64)))
    w = _bits(rng.standard_normal((32, 64)))
    b = rng.standard_normal(32).astype(np.float32)
    got = oracle.linear(x, w, b)
    ref = torch.nn.functional.linear(torch.from_numpy(oracle.bf16_to_f64(x)), torch.from_numpy(oracle.bf16_to_f64(w)),
                                     torch.from_numpy(b.astype(np.float64))).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-12)


def _identity_block(shape, seed):
    """Block whose projections copy: q = k = v = x (per head), out = attention output."""
    C = shape.H * shape.head_dim
    base = W.make_random_inputs(shape, seed)
    x_qkv = base["qkv"][:, :, 0]                           # [S, T, H, 64] bf16 bits
    block = {k: base[k] for k in ("q_gamma", "q_beta", "k_gamma", "k_beta")}
    block["x"] = x_qkv.reshape(shape.S * shape.T, C)
    eye = np.eye(C, dtype=np.float32)
    block["w_qkv"] = _bits(np.concatenate([eye, eye, eye], axis=0))
    block["b_qkv"] = np.zeros(3 * C, np.float32)
    block["w_out"] = _bits(eye)
    block["b_out"] = np.zeros(C, np.float32)
    qkv = np.repeat(x_qkv[:, :, None], 3, axis=2)          # [S, T, 3, H, 64]
    attn_inputs = {k: base[k] for k in ("q_gamma", "q_beta", "k_gamma", "k_beta")}
    attn_inputs["qkv"] = qkv
    return block, attn_inputs


@pytest.mark.parametrize("mode", ["frame", "global", "register"])
def test_block_with_identity_projections_is_the_attention_core(mode):
    shape = W.Shape(S=2, T=13, H=2, n_special=4, grid_h=3, grid_w=3)
    block, attn_inputs = _identity_block(shape, 21)
    q = oracle.register_tokens(shape) if mode == "register" else None
    got = oracle.attention_block(mode, shape, block, q)
    ref = oracle.attn_mode(mode, shape, attn_inputs, q)
    np.testing.assert_allclose(got, ref.reshape(ref.shape[0], -1), rtol=1e-12, atol=1e-12)


def test_block_output_bias_shifts_every_row():
    shape = W.Shape(S=1, T=9, H=2, n_special=1, grid_h=2, grid_w=4)
    block = W.make_block_inputs(shape, 5)
    y0 = oracle.attention_block("global", shape, dict(block, b_out=None))
    y1 = oracle.attention_block("global", shape, block)
    np.testing.assert_allclose(y1 - y0, np.broadcast_to(block["b_out"].astype(np.float64), y0.shape), atol=1e-12)


def test_projected_qkv_orders_q_k_v_then_heads():
    shape = W.Shape(S=1, T=3, H=2, n_special=3, grid_h=0, grid_w=1)
    C = 128
    x = _bits(np.eye(3, C))                                # token t has a 1 in channel t
    w = np.zeros((3 * C, C), dtype=np.float32)
    for c in range(3):
        for h in range(2):
            w[c * C + h * 64 + 5, 1] = 100 * c + 10 * h + 1   # output (c, h, dim 5) reads channel 1
    qkv = oracle.projected_qkv(shape, {"x": x, "w_qkv": _bits(w), "b_qkv": None})
    assert qkv.shape == (1, 3, 3, 2, 64)
    for c in range(3):
        for h in range(2):
            assert qkv[0, 1, c, h, 5] == 100 * c + 10 * h + 1
            assert qkv[0, 0, c, h, 5] == 0 and qkv[0, 2, c, h, 5] == 0
    assert np.count_nonzero(qkv) == 6


@pytest.mark.parametrize("mode", ["frame", "global", "register"])
def test_block_matches_torch_linear_around_the_attention_core(mode):
    """Random (non-symmetric) projections: torch's fp64 linear for both maps around
    the pinned attention oracle.  An untransposed output weight or the q/k/v
    channel blocks taken in another order change the result."""
    shape = W.Shape(S=2, T=11, H=2, n_special=3, grid_h=2, grid_w=4)
    block = W.make_block_inputs(shape, 6)
    q = oracle.register_tokens(shape) if mode == "register" else None
    x = torch.from_numpy(oracle.bf16_to_f64(block["x"]))
    qkv = torch.nn.functional.linear(x, torch.from_numpy(oracle.bf16_to_f64(block["w_qkv"])),
                                     torch.from_numpy(block["b_qkv"].astype(np.float64)))
    inputs = {"qkv_f64": qkv.numpy().reshape(shape.S, shape.T, 3, shape.H, 64),
              **{k: block[k] for k in ("q_gamma", "q_beta", "k_gamma", "k_beta")}}
    a = oracle.attn_mode(mode, shape, inputs, q)
    want = torch.nn.functional.linear(torch.from_numpy(a.reshape(a.shape[0], -1)),
                                      torch.from_numpy(oracle.bf16_to_f64(block["w_out"])),
                                      torch.from_numpy(block["b_out"].astype(np.float64))).numpy()
    np.testing.assert_allclose(oracle.attention_block(mode, shape, block, q), want, rtol=1e-11, atol=1e-11)
