"""Pins of the fp64 oracle against closed forms, invariants, library special
cases and brute force (CPU only).  Nothing here compares the oracle with
itself.  Sources are cited by page title and section."""
import cmath
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def unit(i, d=64):
    e = np.zeros(d)
    e[i] = 1.0
    return e


def tiny_shape(S=2, H=2, n_special=3, gh=3, gw=4, **kw):
    return W.Shape(S=S, T=n_special + gh * gw, H=H, n_special=n_special, grid_h=gh, grid_w=gw, **kw)


# ---------------------------------------------------------------- bf16 widening
def test_bf16_widening_exact_bit_patterns():
    bits = np.array([0x3F80, 0xC000, 0x3F81, 0x0001, 0x7F7F, 0x8000], dtype=np.uint16)
    want = [1.0, -2.0, 1.0 + 2.0 ** -7, 2.0 ** -133, (2 - 2.0 ** -7) * 2.0 ** 127, -0.0]
    got = O.bf16_to_f64(bits)
    assert list(got) == want


def test_input_rounding_is_nearest_even():
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> even (1); 1 + 3*2^-8 -> 1 + 2^-6 (even mantissa).
    x = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -20, -3.0], dtype=np.float32)
    assert list(O.bf16_to_f64(W.f32_to_bf16_bits(x))) == [1.0, 1 + 2 ** -6, 1 + 2 ** -7, -3.0]


# ---------------------------------------------------------------- LayerNorm
def test_layer_norm_golden_alternating():
    case = json.load(open(os.path.join(GOLDEN, "worked_examples.json")))["layer_norm"][0]
    x = np.array([3.0, 1.0] * 32)
    y = O.layer_norm(x, np.full(64, case["gamma"]), np.full(64, case["beta"]), case["eps"])
    assert np.all(y[0::2] == case["expected_even"]) and np.all(y[1::2] == case["expected_odd"])


def test_layer_norm_uses_biased_variance():
    case = json.load(open(os.path.join(GOLDEN, "worked_examples.json")))["layer_norm"][1]
    x = np.arange(64, dtype=np.float64)
    y = O.layer_norm(x, np.ones(64), np.zeros(64), 0.0)
    np.testing.assert_allclose(y, (x - case["mean"]) / math.sqrt(case["biased_var"]), rtol=0, atol=1e-14)


def test_layer_norm_moments_and_invariances():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 64)) * 3 + 2
    eps = 1e-5
    y = O.layer_norm(x, np.ones(64), np.zeros(64), eps)
    var = x.var(axis=1)
    np.testing.assert_allclose(y.mean(axis=1), 0, atol=1e-13)
    np.testing.assert_allclose(y.var(axis=1), var / (var + eps), rtol=1e-12)
    # invariant (up to the eps term) to a positive scale and a constant shift per vector
    y2 = O.layer_norm(x * 7.5 - 4.0, np.ones(64), np.zeros(64), 0.0)
    np.testing.assert_allclose(y2, O.layer_norm(x, np.ones(64), np.zeros(64), 0.0), atol=1e-12)


def test_layer_norm_matches_torch_fp64():
    rng = np.random.default_rng(1)
    x, g, b = rng.standard_normal((7, 64)), rng.standard_normal(64), rng.standard_normal(64)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (64,), torch.from_numpy(g), torch.from_numpy(b), 1e-5)
    np.testing.assert_allclose(O.layer_norm(x, g, b, 1e-5), ref.numpy(), rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- 2D RoPE
@pytest.mark.parametrize("idx", [0, 1, 2, 3, 4])
def test_rope_golden_unit_vectors(idx):
    case = json.load(open(os.path.join(GOLDEN, "worked_examples.json")))["rope"][idx]
    y = O.rope_2d(unit(case["x_unit_dim"]), case["row"], case["col"], case["base"])
    want = np.zeros(64)
    for dim, expr in case["expected"].items():
        want[int(dim)] = eval(expr, {"cos": math.cos, "sin": math.sin, "sqrt": math.sqrt})
    np.testing.assert_allclose(y, want, atol=1e-15)


def test_rope_frequencies_closed_form():
    om = O.rope_frequencies(100.0)
    np.testing.assert_allclose(om, [100.0 ** (-j / 16) for j in range(16)], rtol=1e-15)
    assert om[0] == 1.0 and abs(om[8] - 0.1) < 1e-16


@pytest.mark.parametrize("base,j,want", [(16.0, 4, 0.5), (16.0, 8, 0.25), (16.0, 12, 0.125),
                                         (10000.0, 8, 0.01), (10000.0, 4, 0.1), (10.0, 16 - 1, 10.0 ** (-15 / 16))])
def test_rope_frequencies_other_bases(base, j, want):
    # omega_j = base^(-2j/32): powers of two for base 16, powers of ten for base 10^4
    om = O.rope_frequencies(base)
    assert om[0] == 1.0
    assert abs(om[j] - want) <= 1e-15 * want


def test_rope_matches_complex_rotation():
    # Independent formulation: pair (x_j, x_{j+16}) as the complex number
    # x_j + i x_{j+16}, multiplied by exp(i * pos * omega_j).
    rng = np.random.default_rng(2)
    x = rng.standard_normal(64)
    row, col = 4, 11
    want = np.empty(64)
    for half, pos in ((0, row), (32, col)):
        for j in range(16):
            z = complex(x[half + j], x[half + j + 16]) * cmath.exp(1j * pos * 100.0 ** (-j / 16))
            want[half + j], want[half + j + 16] = z.real, z.imag
    np.testing.assert_allclose(O.rope_2d(x, row, col, 100.0), want, atol=1e-14)


def test_rope_zero_position_identity_and_norm():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((6, 64))
    np.testing.assert_array_equal(O.rope_2d(x, 0, 0, 100.0), x)
    y = O.rope_2d(x, np.arange(6), np.arange(6)[::-1], 100.0)
    pair_norm = lambda v: v[..., :16] ** 2 + v[..., 16:32] ** 2
    np.testing.assert_allclose(pair_norm(y), pair_norm(x), rtol=1e-12)
    np.testing.assert_allclose(pair_norm(y[..., 32:]), pair_norm(x[..., 32:]), rtol=1e-12)


def test_rope_dot_depends_only_on_relative_offset():
    # I4: (R(p) q) . (R(p') k) is a function of p - p' only.
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    base = O.rope_2d(q, 5, 9, 100.0) @ O.rope_2d(k, 2, 3, 100.0)
    for dr, dc in [(1, 0), (0, 1), (7, -3), (20, 30)]:
        shifted = O.rope_2d(q, 5 + dr, 9 + dc, 100.0) @ O.rope_2d(k, 2 + dr, 3 + dc, 100.0)
        assert abs(shifted - base) < 1e-12
    other = O.rope_2d(q, 6, 9, 100.0) @ O.rope_2d(k, 2, 3, 100.0)
    assert abs(other - base) > 1e-3


def test_patch_positions_row_major():
    is_patch, row, col = O.patch_row_col(np.array([0, 16, 17, 18, 17 + 38, 17 + 39, 1030]), 17, 39)
    assert list(is_patch) == [False, False, True, True, True, True, True]
    assert list(row[2:]) == [0, 0, 0, 1, 25] and list(col[2:]) == [0, 1, 38, 0, 38]


# ---------------------------------------------------------------- softmax attention
def test_attention_golden_cases():
    cases = json.load(open(os.path.join(GOLDEN, "worked_examples.json")))["attention"]
    q = 8 * math.log(3) * unit(0)
    out = O.softmax_attention(q[None], np.stack([np.zeros(64), unit(0)]),
                              np.stack([4 * unit(1), -4 * unit(1) + 8 * unit(2)]), cases[0]["scale"])[0]
    want = np.zeros(64)
    want[1], want[2] = cases[0]["expected"]["1"], cases[0]["expected"]["2"]
    np.testing.assert_allclose(out, want, atol=1e-13)
    out = O.softmax_attention((800 * unit(0))[None], np.stack([unit(0), unit(0), np.zeros(64)]),
                              np.stack([unit(3), 3 * unit(3), unit(5)]), cases[1]["scale"])[0]
    want = np.zeros(64)
    want[3] = cases[1]["expected"]["3"]
    np.testing.assert_allclose(out, want, atol=1e-14)


def test_attention_rows_sum_to_one_and_large_scores():
    # I1, plus max subtraction: scores of 1e4 must not overflow.
    rng = np.random.default_rng(5)
    q, k, v = rng.standard_normal((9, 64)) * 40, rng.standard_normal((33, 64)) * 40, rng.standard_normal((33, 64))
    out, p = O.softmax_attention(q, k, v, 0.125, return_probs=True)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=1e-14)
    assert np.all(np.isfinite(out)) and np.all(p >= 0)


def test_attention_constant_v_and_single_key():
    rng = np.random.default_rng(6)
    q, k = rng.standard_normal((10, 64)), rng.standard_normal((17, 64))
    c = rng.standard_normal(64)
    out = O.softmax_attention(q, k, np.tile(c, (17, 1)), 0.125)       # I2
    np.testing.assert_allclose(out, np.tile(c, (10, 1)), rtol=1e-13, atol=1e-14)
    out = O.softmax_attention(q, k[:1], c[None], 0.125)                # I3
    np.testing.assert_allclose(out, np.tile(c, (10, 1)), rtol=0, atol=0)


def test_attention_matches_torch_sdpa_fp64():
    rng = np.random.default_rng(7)
    q, k, v = (rng.standard_normal((n, 64)) for n in (23, 41, 41))
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(a)[None, None] for a in (q, k, v)))[0, 0].numpy()
    np.testing.assert_allclose(O.softmax_attention(q, k, v, 0.125), ref, rtol=1e-12, atol=1e-13)


def test_attention_mask_removes_keys():
    rng = np.random.default_rng(8)
    q, k, v = rng.standard_normal((4, 64)), rng.standard_normal((12, 64)), rng.standard_normal((12, 64))
    mask = np.zeros((4, 12), dtype=bool)
    mask[:, 3:7] = True
    np.testing.assert_allclose(O.softmax_attention(q, k, v, 0.3, mask=mask),
                               O.softmax_attention(q, k[3:7], v[3:7], 0.3), rtol=1e-13)


def test_explicit_softmax_scale_golden():
    case = json.load(open(os.path.join(GOLDEN, "worked_examples.json")))["pipeline_scale"][0]
    shape = W.Shape(**case["shape"])
    assert O.resolved_scale(shape) == 0.05
    assert O.resolved_scale(W.Shape(**{**case["shape"], "softmax_scale": 0.0})) == 0.125
    a = np.array([1.0, -1.0] * 32, dtype=np.float32)
    b = np.array([1.0, 1.0, -1.0, -1.0] * 16, dtype=np.float32)
    f = np.zeros((1, 2, 3, 1, 64), dtype=np.float32)
    f[0, 0, 0, 0] = f[0, 0, 1, 0] = a
    f[0, 1, 0, 0] = f[0, 1, 1, 0] = b
    f[0, 0, 2, 0] = 1.0
    x = {"qkv": W.f32_to_bf16_bits(f), "q_gamma": np.ones((1, 64), np.float32), "q_beta": np.zeros((1, 64), np.float32),
         "k_gamma": np.ones((1, 64), np.float32), "k_beta": np.zeros((1, 64), np.float32)}
    env = {"exp": math.exp}
    out = O.attn_global(shape, x)
    np.testing.assert_allclose(out[0, 0], eval(case["expected_out0"], env), rtol=1e-14)
    np.testing.assert_allclose(out[1, 0], eval(case["expected_out1"], env), rtol=1e-13)


# ---------------------------------------------------------------- whole pipeline (tiny)
def _torch_pipeline(shape, x, mode):
    """Independent restatement with torch ops + complex RoPE + SDPA (fp64)."""
    S, T, H = shape.S, shape.T, shape.H
    qkv = torch.from_numpy(O.bf16_to_f64(x["qkv"]))                     # [S,T,3,H,64]
    def norm(t, name):
        return torch.nn.functional.layer_norm(t, (64,), None, None, shape.ln_eps) * \
            torch.from_numpy(x[f"{name}_gamma"].astype(np.float64)) + torch.from_numpy(x[f"{name}_beta"].astype(np.float64))
    q, k, v = norm(qkv[:, :, 0], "q"), norm(qkv[:, :, 1], "k"), qkv[:, :, 2]
    # complex RoPE on patch tokens
    for t in range(shape.n_special, T):
        p = t - shape.n_special
        r, c = p // shape.grid_w, p % shape.grid_w
        for half, pos in ((0, r), (32, c)):
            ang = torch.tensor([pos * shape.rope_base ** (-j / 16) for j in range(16)], dtype=torch.float64)
            rot = torch.polar(torch.ones(16, dtype=torch.float64), ang)
            for arr in (q, k):
                z = torch.complex(arr[:, t, :, half:half + 16], arr[:, t, :, half + 16:half + 32]) * rot
                arr[:, t, :, half:half + 16], arr[:, t, :, half + 16:half + 32] = z.real, z.imag
    sdpa_kw = {"scale": shape.softmax_scale} if shape.softmax_scale > 0 else {}   # SDPA's default is 1/sqrt(64)
    if mode == "frame":
        o = torch.nn.functional.scaled_dot_product_attention(*(a.permute(0, 2, 1, 3) for a in (q, k, v)), **sdpa_kw)
        return o.permute(0, 2, 1, 3).reshape(S * T, H, 64).numpy()
    if mode == "global":
        o = torch.nn.functional.scaled_dot_product_attention(*(a.reshape(S * T, H, 64).permute(1, 0, 2) for a in (q, k, v)),
                                                             **sdpa_kw)
        return o.permute(1, 0, 2).numpy()
    ns = shape.n_special
    o = torch.nn.functional.scaled_dot_product_attention(*(a[:, :ns].reshape(S * ns, H, 64).permute(1, 0, 2) for a in (q, k, v)),
                                                         **sdpa_kw)
    return o.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("mode", ["frame", "global", "register"])
def test_pipeline_matches_torch_restatement(mode):
    shape = tiny_shape(S=3, H=2)
    x = W.make_random_inputs(shape, 11)
    np.testing.assert_allclose(O.attn_mode(mode, shape, x), _torch_pipeline(shape, x, mode), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("mode", ["frame", "global", "register"])
def test_pipeline_nondefault_scale_base_eps_matches_torch_restatement(mode):
    # explicit softmax scale, RoPE base 10 and LayerNorm epsilon 1e-3 (none of them the defaults)
    shape = tiny_shape(S=2, H=2, ln_eps=1e-3, softmax_scale=0.2, rope_base=10.0)
    x = W.make_random_inputs(shape, 12)
    np.testing.assert_allclose(O.attn_mode(mode, shape, x), _torch_pipeline(shape, x, mode), rtol=1e-11, atol=1e-12)


def test_workload0_pipeline_matches_torch_restatement():
    w = W.workload(0)
    x = W.make_inputs(w)
    np.testing.assert_allclose(O.attn_global(w.shape, x), _torch_pipeline(w.shape, x, "global"), rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- mode structure
def test_global_with_block_diagonal_mask_equals_frame():
    # I5
    shape = tiny_shape(S=3)
    x = W.make_random_inputs(shape, 12)
    N = shape.S * shape.T
    t = O.normalized_tokens(shape, x, np.arange(N))
    frame_of = np.arange(N) // shape.T
    mask = frame_of[:, None] == frame_of[None, :]
    masked = np.stack([O.softmax_attention(t["q"][h], t["k"][h], t["v"][h], 0.125, mask=mask)
                       for h in range(shape.H)], axis=1)
    np.testing.assert_allclose(masked, O.attn_frame(shape, x), rtol=1e-12, atol=1e-13)
    assert np.abs(masked - O.attn_global(shape, x)).max() > 1e-3


def test_permuting_frames_permutes_global_output():
    # I6 (positions are per frame, so a frame permutation is a token permutation)
    shape = tiny_shape(S=4)
    x = W.make_random_inputs(shape, 13)
    perm = np.array([2, 0, 3, 1])
    xp = dict(x)
    xp["qkv"] = x["qkv"][perm]
    a = O.attn_global(shape, x).reshape(shape.S, shape.T, shape.H, 64)
    b = O.attn_global(shape, xp).reshape(shape.S, shape.T, shape.H, 64)
    np.testing.assert_allclose(b, a[perm], rtol=1e-12, atol=1e-13)


def test_frame_equals_global_for_one_frame_and_register_for_specials_only():
    shape = tiny_shape(S=1)
    x = W.make_random_inputs(shape, 14)
    np.testing.assert_allclose(O.attn_frame(shape, x), O.attn_global(shape, x), rtol=1e-13, atol=1e-14)
    s2 = W.Shape(S=3, T=4, H=2, n_special=4, grid_h=0, grid_w=1)
    x2 = W.make_random_inputs(s2, 15)
    np.testing.assert_allclose(O.attn_register(s2, x2), O.attn_global(s2, x2), rtol=1e-13, atol=1e-14)


def test_register_mode_brute_force():
    # I7: explicit gather into plain lists + textbook loops, no numpy linear algebra.
    shape = tiny_shape(S=3, H=2, n_special=2, gh=2, gw=2)
    x = W.make_random_inputs(shape, 16)
    vals = O.bf16_to_f64(x["qkv"])
    eps = shape.ln_eps

    def ln(vec, g, b):
        m = sum(vec) / 64
        var = sum((a - m) ** 2 for a in vec) / 64
        return [(a - m) / math.sqrt(var + eps) * float(gg) + float(bb) for a, gg, bb in zip(vec, g, b)]

    got = O.attn_register(shape, x)
    toks = [(s, t) for s in range(shape.S) for t in range(shape.n_special)]
    for h in range(shape.H):
        K = [ln(list(vals[s, t, 1, h]), x["k_gamma"][h], x["k_beta"][h]) for s, t in toks]
        V = [list(vals[s, t, 2, h]) for s, t in toks]
        for qi, (s, t) in enumerate(toks):
            qv = ln(list(vals[s, t, 0, h]), x["q_gamma"][h], x["q_beta"][h])
            sc = [sum(a * b for a, b in zip(qv, kv)) / 8.0 for kv in K]
            mx = max(sc)
            w = [math.exp(z - mx) for z in sc]
            o = [sum(wj * V[j][d] for j, wj in enumerate(w)) / sum(w) for d in range(64)]
            np.testing.assert_allclose(got[qi, h], o, rtol=1e-11, atol=1e-12)


def test_register_rejects_patch_queries():
    shape = tiny_shape()
    x = W.make_random_inputs(shape, 17)
    with pytest.raises(ValueError):
        O.attn_register(shape, x, queries=[shape.n_special])


def test_query_subset_rows_match_full_run():
    shape = tiny_shape(S=2)
    x = W.make_random_inputs(shape, 18)
    sub = W.query_subset(shape.S * shape.T, 7, 18)
    for mode in ("frame", "global"):
        # BLAS may order the sums differently for a different row count
        np.testing.assert_allclose(O.attn_mode(mode, shape, x, sub), O.attn_mode(mode, shape, x)[sub], rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- workloads vs the pages
def test_workloads_follow_page_facts():
    f = json.load(open(os.path.join(GOLDEN, "page_facts.json")))
    gw = f["resolution"]["width"] // f["patch_size"]["value"]
    gh = f["resolution"]["height"] // f["patch_size"]["value"]
    ns = f["special_tokens_per_frame"]["camera"] + f["special_tokens_per_frame"]["register"]
    for w in W.WORKLOADS[1:]:
        s = w.shape
        assert (s.grid_w, s.grid_h, s.n_special, s.T) == (gw, gh, ns, ns + gw * gh) == (39, 26, 17, 1031)
        assert s.H * s.head_dim == f["feature_dim"]["value"]


# ------------------------------------------------------------------ property checks over random small shapes
from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=25, deadline=None)
@given(S=st.integers(1, 3), H=st.integers(1, 2), ns=st.integers(1, 4), gh=st.integers(0, 4), gw=st.integers(1, 4),
       seed=st.integers(0, 10_000))
def test_mode_identities_on_random_shapes(S, H, ns, gh, gw, seed):
    """For any small shape: each frame of frame mode is global attention over that frame alone, and
    register mode equals global attention over the special tokens taken as their own sequence."""
    import dataclasses
    shape = W.Shape(S=S, T=ns + gh * gw, H=H, n_special=ns, grid_h=gh, grid_w=gw)
    x = W.make_random_inputs(shape, seed)
    fr = O.attn_frame(shape, x)
    for s in range(S):
        one = dataclasses.replace(shape, S=1)
        xs = dict(x, qkv=x["qkv"][s:s + 1])
        np.testing.assert_allclose(fr[s * shape.T:(s + 1) * shape.T], O.attn_global(one, xs), rtol=1e-12, atol=1e-12)
    reg = O.attn_register(shape, x)
    sp = dataclasses.replace(shape, T=ns, grid_h=0, grid_w=0)
    xr = dict(x, qkv=np.ascontiguousarray(x["qkv"][:, :ns]))
    np.testing.assert_allclose(reg, O.attn_global(sp, xr), rtol=1e-12, atol=1e-12)
