"""Pins of the transformer-block and layer-schedule oracle (oracle/block.py)
against library routines (torch fp64 layer_norm, linear, gelu), closed forms
and structural identities, not against itself."""
import dataclasses

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O
import workloads as W

EPS = 1e-6


def shp(S, H, ns, gh, gw):
    return W.Shape(S=S, T=ns + gh * gw, H=H, n_special=ns, grid_h=gh, grid_w=gw)


def t64(a):
    return torch.from_numpy(np.asarray(a, np.float64))


def tw(bits):
    return t64(O.bf16_to_f64(bits))


SHAPE = shp(2, 4, 3, 3, 4)      # C = 256, 15 tokens per frame


@pytest.fixture(scope="module")
def wts():
    return W.make_transformer_block_weights(SHAPE.H, 41)


@pytest.fixture(scope="module")
def x():
    return W.make_tokens(SHAPE, 42)


def test_token_layer_norm_matches_torch():
    a = np.random.default_rng(0).standard_normal((7, 256)) * 3 + 1
    g, b = np.random.default_rng(1).standard_normal((2, 256))
    want = F.layer_norm(t64(a), (256,), t64(g), t64(b), eps=1e-5).numpy()
    np.testing.assert_allclose(O.token_layer_norm(a, g, b, 1e-5), want, rtol=1e-12, atol=1e-12)


def test_gelu_matches_torch_and_closed_forms():
    a = np.linspace(-8, 8, 1001)
    np.testing.assert_allclose(O.gelu(a), F.gelu(t64(a), approximate="none").numpy(), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(O.gelu(a) - O.gelu(-a), a, rtol=0, atol=1e-14)   # x Phi(x) + x Phi(-x) = x
    assert O.gelu(np.zeros(1))[0] == 0.0
    assert abs(O.gelu(np.array([1.0]))[0] - 0.8413447460685429) < 1e-15         # Phi(1)


@pytest.mark.parametrize("mode", ["frame", "global", "register"])
def test_zero_layerscale_is_identity(mode, wts, x):
    w = dict(wts, ls1=np.zeros_like(wts["ls1"]), ls2=np.zeros_like(wts["ls2"]))
    np.testing.assert_array_equal(O.block_forward(mode, SHAPE, x, w, EPS), O.bf16_to_f64(x))


@pytest.mark.parametrize("mode", ["frame", "global"])
def test_attention_branch_alone(mode, wts, x):
    """ls2 = 0: x + ls1 * proj(attention(qkv(norm1 x))), norm and projections by torch."""
    w = dict(wts, ls2=np.zeros_like(wts["ls2"]))
    C = SHAPE.H * 64
    xf = tw(x)
    h = F.layer_norm(xf, (C,), t64(w["norm1_gamma"]), t64(w["norm1_beta"]), eps=EPS)
    qkv = F.linear(h, tw(w["w_qkv"]), t64(w["b_qkv"])).numpy().reshape(SHAPE.S, SHAPE.T, 3, SHAPE.H, 64)
    inputs = {"qkv_f64": qkv, **{k: w[k] for k in ("q_gamma", "q_beta", "k_gamma", "k_beta")}}
    a = t64(O.attn_mode(mode, SHAPE, inputs).reshape(-1, C))
    want = xf + t64(w["ls1"]) * F.linear(a, tw(w["w_proj"]), t64(w["b_proj"]))
    np.testing.assert_allclose(O.block_forward(mode, SHAPE, x, w, EPS), want.numpy(), rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("mode", ["frame", "global"])
def test_mlp_branch_alone(mode, wts, x):
    """ls1 = 0: x + ls2 * fc2(gelu(fc1(norm2 x))), every step by torch."""
    w = dict(wts, ls1=np.zeros_like(wts["ls1"]))
    C = SHAPE.H * 64
    xf = tw(x)
    h = F.layer_norm(xf, (C,), t64(w["norm2_gamma"]), t64(w["norm2_beta"]), eps=EPS)
    u = F.gelu(F.linear(h, tw(w["w_fc1"]), t64(w["b_fc1"])), approximate="none")
    want = xf + t64(w["ls2"]) * F.linear(u, tw(w["w_fc2"]), t64(w["b_fc2"]))
    np.testing.assert_allclose(O.block_forward(mode, SHAPE, x, w, EPS), want.numpy(), rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("mode", ["frame", "global"])
def test_full_block_runs_the_mlp_on_the_attention_branch_output(mode, wts, x):
    """Both branches on: the MLP reads x + ls1 * attention branch (sequential
    residuals, not two parallel branches on x), every step by torch."""
    C = SHAPE.H * 64
    xf = tw(x)
    h = F.layer_norm(xf, (C,), t64(wts["norm1_gamma"]), t64(wts["norm1_beta"]), eps=EPS)
    qkv = F.linear(h, tw(wts["w_qkv"]), t64(wts["b_qkv"])).numpy().reshape(SHAPE.S, SHAPE.T, 3, SHAPE.H, 64)
    inputs = {"qkv_f64": qkv, **{k: wts[k] for k in ("q_gamma", "q_beta", "k_gamma", "k_beta")}}
    a = t64(O.attn_mode(mode, SHAPE, inputs).reshape(-1, C))
    xr = xf + t64(wts["ls1"]) * F.linear(a, tw(wts["w_proj"]), t64(wts["b_proj"]))
    h2 = F.layer_norm(xr, (C,), t64(wts["norm2_gamma"]), t64(wts["norm2_beta"]), eps=EPS)
    u = F.gelu(F.linear(h2, tw(wts["w_fc1"]), t64(wts["b_fc1"])), approximate="none")
    want = xr + t64(wts["ls2"]) * F.linear(u, tw(wts["w_fc2"]), t64(wts["b_fc2"]))
    got = O.block_forward(mode, SHAPE, x, wts, EPS)
    np.testing.assert_allclose(got, want.numpy(), rtol=1e-11, atol=1e-11)
    # the test has teeth: with the block's LayerScale the MLP branch changes the output measurably
    assert np.abs(got - xr.numpy()).max() > 1e-8


def test_register_block_changes_only_special_rows_like_a_global_block_on_them(wts, x):
    y = O.block_forward("register", SHAPE, x, wts, EPS)
    sp = O.register_tokens(SHAPE)
    patch = np.setdiff1d(np.arange(SHAPE.S * SHAPE.T), sp)
    np.testing.assert_array_equal(y[patch], O.bf16_to_f64(x)[patch])
    compact = dataclasses.replace(SHAPE, T=SHAPE.n_special, grid_h=0, grid_w=0)
    want = O.block_forward("global", compact, x[sp], wts, EPS)
    np.testing.assert_allclose(y[sp], want, rtol=1e-12, atol=1e-12)


def test_frame_block_acts_on_each_frame_alone(wts, x):
    y = O.block_forward("frame", SHAPE, x, wts, EPS)
    one = dataclasses.replace(SHAPE, S=1)
    for s in range(SHAPE.S):
        r = slice(s * SHAPE.T, (s + 1) * SHAPE.T)
        np.testing.assert_allclose(y[r], O.block_forward("frame", one, x[r], wts, EPS), rtol=1e-12, atol=1e-12)


def test_global_block_commutes_with_frame_permutation(wts):
    shape = shp(3, 4, 3, 3, 4)
    x = W.make_tokens(shape, 43)
    perm = np.array([2, 0, 1])
    xp = x.reshape(3, shape.T, -1)[perm].reshape(x.shape)
    y = O.block_forward("global", shape, x, wts, EPS).reshape(3, shape.T, -1)
    yp = O.block_forward("global", shape, xp, wts, EPS).reshape(3, shape.T, -1)
    np.testing.assert_allclose(yp, y[perm], rtol=1e-11, atol=1e-11)


def test_aggregator_schedule(wts, x):
    w2 = W.make_transformer_block_weights(SHAPE.H, 44)
    np.testing.assert_array_equal(O.aggregator_forward(SHAPE, x, [], [], [], EPS), O.bf16_to_f64(x))
    got = O.aggregator_forward(SHAPE, x, [wts, w2], [w2, wts], [1], EPS)
    y = O.block_forward("frame", SHAPE, x, wts, EPS)
    y = O.block_forward("global", SHAPE, y, w2, EPS)
    y = O.block_forward("frame", SHAPE, y, w2, EPS)
    y = O.block_forward("register", SHAPE, y, wts, EPS)
    np.testing.assert_array_equal(got, y)
    assert O.REGISTER_LAYERS == (2, 6, 9, 14, 20) and O.N_LAYERS == 24


def test_camera_trunk_reduces_to_register_blocks(wts, x):
    sp = O.register_tokens(SHAPE)
    np.testing.assert_array_equal(O.camera_trunk_forward(SHAPE, x, [], EPS), O.bf16_to_f64(x)[sp])
    w2 = W.make_transformer_block_weights(SHAPE.H, 45)
    y = O.block_forward("register", SHAPE, x, wts, EPS)
    y = O.block_forward("register", SHAPE, y, w2, EPS)
    np.testing.assert_allclose(O.camera_trunk_forward(SHAPE, x, [wts, w2], EPS), y[sp], rtol=1e-12, atol=1e-12)
    assert O.CAMERA_TRUNK_BLOCKS == 4


@pytest.mark.parametrize("mode", ["frame", "global", "register"])
def test_row_subset_equals_rows_of_full_result(mode, wts, x):
    full = O.block_forward(mode, SHAPE, x, wts, EPS)
    pool = O.register_tokens(SHAPE) if mode == "register" else np.arange(SHAPE.S * SHAPE.T)
    rows = pool[[0, 3, len(pool) - 1]]
    np.testing.assert_allclose(O.block_forward(mode, SHAPE, x, wts, EPS, rows), full[rows], rtol=1e-12, atol=1e-12)


def test_cached_layers_concatenate_frame_and_inter_outputs(wts, x):
    w2 = W.make_transformer_block_weights(SHAPE.H, 46)
    y, cache = O.aggregator_forward(SHAPE, x, [wts, w2], [w2, wts], [1], EPS, cache_layers=(0, 1))
    f0 = O.block_forward("frame", SHAPE, x, wts, EPS)
    g0 = O.block_forward("global", SHAPE, f0, w2, EPS)
    f1 = O.block_forward("frame", SHAPE, g0, w2, EPS)
    np.testing.assert_array_equal(cache[0], np.concatenate([f0, g0], axis=1))
    np.testing.assert_array_equal(cache[1][:, :SHAPE.H * 64], f1)
    np.testing.assert_array_equal(cache[1][:, SHAPE.H * 64:], y)
    assert O.CACHED_LAYERS == (4, 11, 17, 23)
