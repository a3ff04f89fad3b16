"""Pins of the descriptor-attention oracle (oracle/descriptor.py): 1x1 windows
reduce it to the pinned global-attention oracle, a brute-force restatement with
explicit window loops, constant values, and the descriptor count."""
import math

import numpy as np
import pytest

import oracle as O
import workloads as W


def shp(S, H, ns, gh, gw):
    return W.Shape(S=S, T=ns + gh * gw, H=H, n_special=ns, grid_h=gh, grid_w=gw)


def test_unit_windows_are_global_attention():
    shape = shp(2, 2, 3, 4, 5)
    x = W.make_random_inputs(shape, 1)
    np.testing.assert_allclose(O.attn_global_desc(shape, x, 1, 1), O.attn_global(shape, x), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("s_h,s_w", [(2, 2), (3, 2), (4, 4)])
def test_descriptor_count_and_coverage(s_h, s_w):
    shape = shp(3, 1, 5, 7, 9)
    win = O.descriptor_windows(shape, s_h, s_w)
    assert len(win) == shape.S * (shape.n_special + math.ceil(7 / s_h) * math.ceil(9 / s_w))
    flat = np.sort(np.concatenate(win))
    np.testing.assert_array_equal(flat, np.arange(shape.S * shape.T))   # every token in exactly one descriptor


def test_brute_force_tiny():
    """Pooling written as explicit loops over the patch grid, softmax as a plain loop."""
    shape = shp(2, 1, 2, 3, 3)
    x = W.make_random_inputs(shape, 2)
    s_h = s_w = 2
    got = O.attn_global_desc(shape, x, s_h, s_w)
    N = shape.S * shape.T
    kv = O.normalized_tokens(shape, x, np.arange(N), ("q", "k", "v"))
    keys, vals = [], []
    for s in range(shape.S):
        for t in range(shape.n_special):
            keys.append(kv["k"][0, s * shape.T + t])
            vals.append(kv["v"][0, s * shape.T + t])
        for r0 in range(0, 3, 2):
            for c0 in range(0, 3, 2):
                ks, vs = [], []
                for r in range(r0, min(r0 + 2, 3)):
                    for c in range(c0, min(c0 + 2, 3)):
                        tok = s * shape.T + shape.n_special + r * 3 + c
                        ks.append(kv["k"][0, tok])
                        vs.append(kv["v"][0, tok])
                keys.append(sum(ks) / len(ks))
                vals.append(sum(vs) / len(vs))
    scale = 1 / 8
    for i in range(N):
        sc = [scale * float(np.dot(kv["q"][0, i], k)) for k in keys]
        m = max(sc)
        p = [math.exp(v - m) for v in sc]
        o = sum(pi * v for pi, v in zip(p, vals)) / sum(p)
        np.testing.assert_allclose(got[i, 0], o, rtol=1e-12, atol=1e-12)


def test_constant_values_give_constant_output():
    shape = shp(2, 2, 3, 4, 5)
    x = W.make_random_inputs(shape, 3)
    x["qkv"][:, :, 2] = x["qkv"][0, 0, 2]
    want = O.bf16_to_f64(x["qkv"][0, 0, 2])
    np.testing.assert_allclose(O.attn_global_desc(shape, x, 2, 3), np.broadcast_to(want, (shape.S * shape.T,) + want.shape),
                               rtol=1e-12, atol=1e-12)
