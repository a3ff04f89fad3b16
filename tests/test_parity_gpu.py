"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded bf16 inputs, element by element on every compared row.
Tolerance (the stated parity bar): max-abs <= 2e-2 and relative Frobenius <= 5e-3."""
import numpy as np
import pytest

import oracle as O
import workloads as W
from parity import MAX_ABS_TOL, REL_FRO_TOL, check_mode, rows, run_gpu, to_device

pytestmark = pytest.mark.gpu


def shp(S, H, ns, gh, gw, **kw):
    return W.Shape(S=S, T=ns + gh * gw, H=H, n_special=ns, grid_h=gh, grid_w=gw, **kw)


# ------------------------------------------------------------------ small / ragged (full oracle)
SMALL = [
    ("global", shp(2, 4, 5, 8, 8)),           # the tiny workload's shape: 138 tokens, 2 tiles, ragged
    ("frame", shp(3, 3, 17, 7, 13)),          # T = 108: one ragged tile per frame
    ("frame", shp(2, 2, 17, 10, 30)),         # T = 317: 3 tiles, ragged 61
    ("frame", shp(2, 2, 0, 16, 16)),          # no special tokens, T = 256 exactly 2 tiles
    ("global", shp(3, 2, 17, 6, 8)),          # N = 195
    ("global", shp(4, 2, 3, 16, 16)),         # N = 1036: 9 tiles, ragged 12
    ("global", shp(5, 1, 4, 0, 1)),           # specials only (T = n_special = 4)
    ("register", shp(40, 2, 17, 4, 4)),       # 680 special tokens: 6 tiles, ragged 40
    ("register", shp(3, 2, 5, 2, 3)),         # 15 special tokens: one small tile
    ("frame", shp(1, 1, 1, 1, 1)),            # T = 2
    ("frame", shp(2, 2, 17, 64, 64)),         # T = 4113: high-resolution frames, 33 tiles x 65 key steps
    ("register", shp(300, 2, 1, 2, 3)),       # camera token only: 300 special tokens
    ("global", shp(1, 3, 17, 30, 40)),        # one frame of 1217 tokens, odd head count
    ("frame", shp(2, 2, 5, 5, 15)),           # T = 80: exactly one frame-kernel key step (80 keys)
    ("frame", shp(2, 2, 1, 8, 10)),           # T = 81: one full step and a 1-key step
    ("frame", shp(2, 2, 5, 5, 31)),           # T = 160: exactly two steps
    ("frame", shp(2, 2, 1, 10, 16)),          # T = 161: two full steps and a 1-key step
]


@pytest.mark.parametrize("mode,shape", SMALL, ids=[f"{m}-S{s.S}T{s.T}H{s.H}" for m, s in SMALL])
def test_small_shapes_full_oracle(mode, shape):
    x = W.make_random_inputs(shape, 100 + shape.T)
    check_mode(mode, shape, x)


def test_workload0_global_tiny():
    w = W.workload(0)
    check_mode("global", w.shape, W.make_inputs(w))


def test_nondefault_softmax_scale_and_eps():
    shape = shp(2, 2, 5, 6, 7, ln_eps=1e-3, softmax_scale=0.2, rope_base=10.0)
    check_mode("global", shape, W.make_random_inputs(shape, 7))


# ------------------------------------------------------------------ exact special cases
def test_single_key_returns_v_exactly():
    shape = W.Shape(S=1, T=1, H=3, n_special=1, grid_h=0, grid_w=1)
    x = W.make_random_inputs(shape, 21)
    for mode in ("frame", "global", "register"):
        out = run_gpu(mode, shape, x)
        v = O.bf16_to_f64(x["qkv"][:, :, 2]).reshape(1, 3, 64)
        np.testing.assert_array_equal(rows(out, shape, [0]), v)


def test_constant_v_gives_constant_output():
    shape = shp(3, 2, 17, 10, 12)
    x = W.make_random_inputs(shape, 22)
    x["qkv"][:, :, 2] = x["qkv"][0, 0, 2]                   # every token's v = one bf16 vector per head
    out = run_gpu("global", shape, x)
    want = O.bf16_to_f64(x["qkv"][0, 0, 2])                  # [H, 64]
    got = out.float().cpu().numpy().reshape(-1, shape.H, 64)
    assert np.abs(got - want[None]).max() <= 2 ** -7 * np.abs(want).max()


# Frame mode runs persistent CTAs (two per SM) that each take several (tile, head, frame) units in turn;
# these shapes have more units than the grid has CTAs, with one key step per unit (T <= 64), a single
# ragged tile per unit, and a second tile holding only 2 rows.
MANY_UNITS = [
    shp(700, 1, 5, 4, 4),        # T = 21: 700 units of one key step
    shp(400, 2, 17, 7, 13),      # T = 108: 800 units of one ragged tile, two key steps
    shp(300, 1, 2, 8, 16),       # T = 130: 600 units, every second one with 2 valid rows
]


@pytest.mark.parametrize("shape", MANY_UNITS, ids=[f"S{s.S}T{s.T}H{s.H}" for s in MANY_UNITS])
def test_frame_more_units_than_ctas(shape):
    x = W.make_random_inputs(shape, 300 + shape.T)
    check_mode("frame", shape, x)


# ------------------------------------------------------------------ degenerate inputs
def test_zero_variance_rows_and_uniform_attention():
    """Rows whose q or k is constant over the head (zero variance: the LayerNorm output is beta, the
    epsilon alone keeps it finite), and one head whose keys are all equal (every score of a query equal:
    the output is the plain mean of v)."""
    import numpy as np
    shape = shp(2, 3, 5, 6, 7)
    x = W.make_random_inputs(shape, 31)
    qkv = x["qkv"]
    qkv[0, :10, 0, 1] = W.f32_to_bf16_bits(np.full(64, 0.75, np.float32))     # constant q rows, head 1
    qkv[1, 3:20, 1, 2] = W.f32_to_bf16_bits(np.full(64, -2.0, np.float32))    # constant k rows, head 2
    qkv[:, :, 1, 0] = qkv[0, 0, 1, 0]                                          # head 0: one key for all tokens
    x["k_gamma"][0] = 1.0
    x["k_beta"][0] = 0.0
    for mode in ("global", "frame", "register"):
        check_mode(mode, shape, x)
    # register mode has no RoPE: head 0's equal keys give every special query the mean of the special v
    out = run_gpu("register", shape, x).float().cpu().numpy()
    sp = O.register_tokens(shape)
    got = out.reshape(-1, shape.H, 64)[sp, 0]
    want = O.bf16_to_f64(qkv.reshape(-1, 3, shape.H, 64)[sp, 2, 0]).mean(axis=0)
    assert np.abs(got - want[None]).max() <= 2e-2


def _directional_inputs(shape, seed, angle_of_key):
    """Special tokens only (no rotation); per head q = u and k = cos(a_t) u + sin(a_t) w (u, w zero-mean,
    orthogonal, of equal norm, so LayerNorm keeps the angle) plus small noise, with gamma 2.5 so that the
    scores, 72 cos(a_t) in base 2, span about +-72: keys whose angle shrinks along the sequence move the
    running reference max by far more than its threshold after the first key step."""
    import numpy as np
    x = W.make_random_inputs(shape, seed)
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((shape.H, 64))
    u -= u.mean(-1, keepdims=True)
    w = rng.standard_normal((shape.H, 64))
    w -= w.mean(-1, keepdims=True)
    w -= (w * u).sum(-1, keepdims=True) / (u * u).sum(-1, keepdims=True) * u
    w *= np.linalg.norm(u, axis=-1, keepdims=True) / np.linalg.norm(w, axis=-1, keepdims=True)
    a = np.array([angle_of_key(t) for t in range(shape.T)])
    kdir = np.cos(a)[:, None, None] * u[None] + np.sin(a)[:, None, None] * w[None]        # [T, H, 64]
    noise = lambda: 0.02 * rng.standard_normal((shape.S, shape.T, shape.H, 64))
    x["qkv"][:, :, 0] = W.f32_to_bf16_bits((u[None, None] + noise()).astype(np.float32))
    x["qkv"][:, :, 1] = W.f32_to_bf16_bits((kdir[None] + noise()).astype(np.float32))
    for k in ("q_gamma", "k_gamma"):
        x[k][:] = 2.5
    for k in ("q_beta", "k_beta"):
        x[k][:] = 0.0
    return x


LATE_MAX = [
    ("step", lambda T: (lambda t: np.pi if t < 120 else 0.0)),      # one jump inside the second key step
    ("ramp", lambda T: (lambda t: np.pi * (1.0 - t / (T - 1)))),    # the max grows at every step
]


def _bf16_storage_rows(mode, shape, x, queries):
    """The attention of ``queries`` with the path's bf16 storage points applied to the fp64 computation
    (shapes without patch tokens, so no rotation): q-hat (LayerNorm, gamma/beta, times softmax_scale *
    log2(e)) and k-hat rounded to bf16, probabilities 2^(s - row max) rounded to bf16 for the product with v,
    their sum unrounded.  Frame mode attends within the query's frame, global and register mode over all
    tokens (every token is special here)."""
    from block_tolerance import bf16_round
    qkv = O.bf16_to_f64(x["qkv"])                                   # [S, T, 3, H, 64]
    def ln(v, g, b):
        m = v.mean(-1, keepdims=True)
        return (v - m) / np.sqrt(((v - m) ** 2).mean(-1, keepdims=True) + shape.ln_eps) * g + b
    scale = 0.125 * np.log2(np.e)
    q = bf16_round(ln(qkv[:, :, 0], x["q_gamma"], x["q_beta"]) * scale)
    k = bf16_round(ln(qkv[:, :, 1], x["k_gamma"], x["k_beta"]))
    v = qkv[:, :, 2]
    out = np.empty((len(queries), shape.H, 64))
    for n, i in enumerate(queries):
        f, t = divmod(int(i), shape.T)
        kk, vv = (k[f], v[f]) if mode == "frame" else (k.reshape(-1, shape.H, 64), v.reshape(-1, shape.H, 64))
        sc = np.einsum("hd,khd->hk", q[f, t], kk)
        p = np.exp2(sc - sc.max(1, keepdims=True))
        out[n] = np.einsum("hk,khd->hd", bf16_round(p), vv) / p.sum(1)[:, None]
    return out


@pytest.mark.parametrize("mode", ["frame", "global", "register"])
@pytest.mark.parametrize("kind,angle", LATE_MAX, ids=[k for k, _ in LATE_MAX])
def test_late_keys_move_the_reference_max(mode, kind, angle):
    """The online softmax's reference max moves (by tens of units, base 2) after the first key step; in
    frame mode the step's exponentials are then redone against the moved max.  Every query row is compared
    with the oracle.  Scores of +-72 magnify the bf16 rounding of q-hat and k-hat (a score's error grows with
    its size), so the bound is three times the error of the bf16 storage points alone on these inputs
    (about 2e-2 relative, against 5e-3 for the workloads); a wrong rescale would be off by O(1)."""
    from parity import errors
    shape = W.Shape(S=3, T=400, H=2, n_special=400, grid_h=0, grid_w=1)
    x = _directional_inputs(shape, 77, angle(shape.T))
    out = run_gpu(mode, shape, x)
    q = np.arange(shape.S * shape.T)
    want = O.attn_mode(mode, shape, x, q)
    got = rows(out, shape, q)
    assert np.all(np.isfinite(got))
    e_max, e_rel = errors(got, want)
    s_max, s_rel = errors(_bf16_storage_rows(mode, shape, x, q), want)
    assert e_max <= 3 * s_max and e_rel <= 3 * s_rel, (kind, mode, e_max, e_rel, s_max, s_rel)
    assert e_rel <= 0.05


# ------------------------------------------------------------------ the workloads at full size (sampled)
@pytest.mark.slow
def test_workload1_frame_full():
    """Frame mode, 24 frames x 1031 tokens: every one of the 24,744 query rows against the oracle."""
    w = W.workload(1)
    check_mode("frame", w.shape, W.make_inputs(w))


@pytest.mark.slow
def test_workload2_global_full():
    """Global mode over 24,744 tokens: every query row against the oracle (about a minute of oracle time
    on 16 host cores)."""
    w = W.workload(2)
    check_mode("global", w.shape, W.make_inputs(w))


@pytest.mark.slow
def test_workload3_global_long_sampled():
    w = W.workload(3)
    check_mode("global", w.shape, W.make_inputs(w), count=4096, seed=w.seed)


@pytest.mark.slow
def test_workload4_register_then_frame():
    w = W.workload(4)
    x = W.make_inputs(w)
    dev = to_device(x)
    from parity import assert_close, query_sample
    out_r = run_gpu("register", w.shape, dev_inputs=dev)
    q = query_sample("register", w.shape, 1 << 62, w.seed)  # all 8,500 special tokens
    assert_close(rows(out_r, w.shape, q), O.attn_register(w.shape, x, q), "register S=500")
    del out_r
    out_f = run_gpu("frame", w.shape, dev_inputs=dev)
    q = query_sample("frame", w.shape, 4096, w.seed)
    assert_close(rows(out_f, w.shape, q), O.attn_frame(w.shape, x, q), "frame S=500")


# ------------------------------------------------------------------ random small shapes
from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=30, deadline=None)
@given(mode=st.sampled_from(["frame", "global", "register"]), S=st.integers(1, 5), H=st.integers(1, 3),
       ns=st.integers(1, 17), gh=st.integers(0, 12), gw=st.integers(1, 12), seed=st.integers(0, 10_000))
def test_random_small_shapes_match_oracle(mode, S, H, ns, gh, gw, seed):
    shape = shp(S, H, ns, gh, gw)
    check_mode(mode, shape, W.make_random_inputs(shape, seed))
