"""Pins of the subsampled-global-attention oracle (oracle/sga.py) -- CPU only.

SGA (AVGGT article, section B, point 2) keeps a grid of keys, each token's
diagonal and one mean key/value pair for the discarded columns.  Pinned here
against exact global attention (no subsampling), against a brute force that
writes the mean pair out as n_i duplicate columns and calls the plain
softmax-attention routine, and against the constant-value invariant.
"""
import numpy as np
import pytest

import oracle
import workloads as W

SHAPE = W.Shape(S=3, T=14, H=2, n_special=2, grid_h=3, grid_w=4)


def test_no_subsampling_is_global_attention():
    inputs = W.make_random_inputs(SHAPE, 41)
    got = oracle.attn_global_sga(SHAPE, inputs, 1, 1)
    ref = oracle.attn_global(SHAPE, inputs)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_kept_tokens_grid():
    kept = oracle.sga_kept_tokens(SHAPE, 2, 3)
    # per frame: 2 special + patches at rows {0, 2} x cols {0, 3} of the 3 x 4 grid
    t = [0, 1, 2 + 0 * 4 + 0, 2 + 0 * 4 + 3, 2 + 2 * 4 + 0, 2 + 2 * 4 + 3]
    expect = np.array([s * SHAPE.T + x for s in range(SHAPE.S) for x in sorted(t)])
    np.testing.assert_array_equal(kept, expect)


@pytest.mark.parametrize("s_h,s_w", [(2, 2), (3, 2), (2, 4)])
def test_matches_brute_force_with_duplicated_mean_columns(s_h, s_w):
    inputs = W.make_random_inputs(SHAPE, 42)
    N = SHAPE.S * SHAPE.T
    kept = set(oracle.sga_kept_tokens(SHAPE, s_h, s_w).tolist())
    disc = [j for j in range(N) if j not in kept]
    kv = oracle.normalized_tokens(SHAPE, inputs, np.arange(N), ("k", "v"))
    qn = oracle.normalized_tokens(SHAPE, inputs, np.arange(N), ("q",))["q"]
    got = oracle.attn_global_sga(SHAPE, inputs, s_h, s_w)
    scale = oracle.resolved_scale(SHAPE)
    for h in range(SHAPE.H):
        k, v = kv["k"][h], kv["v"][h]
        k_mean = np.mean([k[j] for j in disc], axis=0)
        v_mean = np.mean([v[j] for j in disc], axis=0)
        for i in range(N):
            cols_k = [k[j] for j in sorted(kept)]
            cols_v = [v[j] for j in sorted(kept)]
            if i not in kept:
                cols_k.append(k[i])
                cols_v.append(v[i])
            n_mean = len(disc) - (0 if i in kept else 1)
            cols_k += [k_mean] * n_mean
            cols_v += [v_mean] * n_mean
            ref = oracle.softmax_attention(qn[h, i][None], np.array(cols_k), np.array(cols_v), scale)[0]
            np.testing.assert_allclose(got[i, h], ref, rtol=1e-10, atol=1e-12)


def test_constant_values_give_that_constant():
    inputs = W.make_random_inputs(SHAPE, 43)
    qkv = inputs["qkv"].copy()
    qkv[:, :, 2] = W.f32_to_bf16_bits(np.full(qkv[:, :, 2].shape, 0.75, np.float32))
    inputs["qkv"] = qkv
    got = oracle.attn_global_sga(SHAPE, inputs, 2, 2)
    np.testing.assert_allclose(got, 0.75, rtol=1e-12)
