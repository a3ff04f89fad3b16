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
