"""GPU parity of the transformer blocks and the alternating layer schedule
(vggt_block_forward, vggt_aggregator_forward) against the fp64 oracle
(oracle/block.py), through the C ABI binding.

Tolerance, derived per test from the arithmetic (tests/block_tolerance.py):
the CUDA path stores the norm outputs, qkv, the attention output, the
residual stream, the MLP hidden activations and the block output in bf16
(every GEMM accumulates in fp32).  The fp64 oracle with bf16 rounding at
exactly those points, run on the test's own inputs, gives the error that the
storage format alone makes (on these shapes a relative Frobenius error of
about 3e-3 on the block output, 5e-3 on its update output - input, and a
largest element error of 2-3e-2 where outputs reach |y| ~ 6 and one bf16 ulp
is 3.1e-2).  Each test allows ROOM = 3 times those three figures, for the
fp32 accumulation order and the attention core's own bf16 rounding of q, k
and P, which the emulation leaves out; chains of blocks are emulated as
chains."""
import numpy as np
import pytest

import oracle as O
import workloads as W
from block_tolerance import ROOM, block_with_storage_rounding, derived_bounds, errors

pytestmark = pytest.mark.gpu

EPS = 1e-6


def shp(S, H, ns, gh, gw):
    return W.Shape(S=S, T=ns + gh * gw, H=H, n_special=ns, grid_h=gh, grid_w=gw)


def _dev_bits(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def _dev_weights(w):
    import torch
    out = {}
    for k, v in w.items():
        if v.dtype == np.uint16:
            out[k] = _dev_bits(v)
        else:
            out[k] = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).cuda()
    return out


def _check(got, want, x0, rows, bounds):
    """got vs the oracle on ``rows``: output and update rel-Frobenius and max-abs within ``bounds``."""
    g, r, x = got[rows], want[rows], x0[rows]
    assert np.isfinite(g).all()
    e = errors(g, r, x)
    assert all(v <= b for v, b in zip(e, bounds)), f"errors {e} bounds {bounds}"


def _chain_bounds(want, emu, x0, rows):
    """ROOM x the errors of a chain of emulated blocks against the oracle's chain."""
    return tuple(ROOM * v for v in errors(emu[rows], want[rows], x0[rows]))


BLOCK_CASES = [
    ("frame", shp(3, 4, 5, 7, 9)),          # C = 256, T = 68: GEMM row tiles straddle frames, ragged tail
    ("global", shp(3, 4, 5, 7, 9)),
    ("register", shp(40, 4, 5, 2, 3)),      # 200 special tokens of 11-token frames
    ("frame", shp(2, 16, 17, 6, 8)),        # C = 1024, T = 65
    ("global", shp(2, 16, 17, 6, 8)),
    ("register", shp(9, 16, 17, 6, 8)),     # 153 special tokens
    ("global", shp(2, 32, 17, 3, 4)),       # C = 2048 (LayerNorm with 8 chunks per lane)
]


@pytest.mark.parametrize("mode,shape", BLOCK_CASES, ids=[f"{m}-S{s.S}T{s.T}H{s.H}" for m, s in BLOCK_CASES])
def test_block_matches_oracle(mode, shape):
    import torch
    import vit_attention_b200 as V
    w = W.make_transformer_block_weights(shape.H, 50 + shape.H)
    x = W.make_tokens(shape, 60 + shape.T)
    xd = _dev_bits(x).clone()
    ws = torch.empty(V.vggt_block_workspace_size(shape, mode), dtype=torch.uint8, device="cuda")
    V.vggt_block_forward(mode, shape, xd, _dev_weights(w), EPS, ws)
    assert V.vggt_attn_read_status(ws) == 0
    got = xd.float().cpu().numpy().astype(np.float64)
    want = O.block_forward(mode, shape, x, w, EPS)
    x0 = O.bf16_to_f64(x)
    rows = O.register_tokens(shape) if mode == "register" else np.arange(shape.S * shape.T)
    _check(got, want, x0, rows, derived_bounds(mode, shape, x, w, EPS, want=want))
    if mode == "register":   # patch rows untouched, bit for bit
        patch = np.setdiff1d(np.arange(shape.S * shape.T), rows)
        assert np.array_equal(xd.view(torch.int16).cpu().numpy().view(np.uint16)[patch], x[patch])


def test_zero_layerscale_leaves_x_bit_identical():
    import torch
    import vit_attention_b200 as V
    shape = shp(2, 4, 5, 7, 9)
    w = W.make_transformer_block_weights(shape.H, 70)
    w["ls1"] = np.zeros_like(w["ls1"])
    w["ls2"] = np.zeros_like(w["ls2"])
    x = W.make_tokens(shape, 71)
    xd = _dev_bits(x).clone()
    ws = torch.empty(V.vggt_block_workspace_size(shape, "global"), dtype=torch.uint8, device="cuda")
    V.vggt_block_forward("global", shape, xd, _dev_weights(w), EPS, ws)
    assert np.array_equal(xd.view(torch.int16).cpu().numpy().view(np.uint16), x)


def test_aggregator_two_layers_with_a_register_layer():
    import torch
    import vit_attention_b200 as V
    shape = shp(6, 4, 5, 4, 5)     # C = 256, T = 25
    fw = [W.make_transformer_block_weights(shape.H, 80 + l) for l in range(2)]
    iw = [W.make_transformer_block_weights(shape.H, 90 + l) for l in range(2)]
    x = W.make_tokens(shape, 99)
    xd = _dev_bits(x).clone()
    ws = torch.empty(V.vggt_aggregator_workspace_size(shape), dtype=torch.uint8, device="cuda")
    V.vggt_aggregator_forward(shape, xd, [_dev_weights(w) for w in fw], [_dev_weights(w) for w in iw], [1], EPS, ws)
    assert V.vggt_attn_read_status(ws) == 0
    got = xd.float().cpu().numpy().astype(np.float64)
    want = O.aggregator_forward(shape, x, fw, iw, [1], EPS)
    emu = x
    for l in range(2):
        emu = block_with_storage_rounding("frame", shape, emu, fw[l], EPS)
        emu = block_with_storage_rounding("register" if l == 1 else "global", shape, emu, iw[l], EPS)
    x0, rows = O.bf16_to_f64(x), np.arange(shape.S * shape.T)
    _check(got, want, x0, rows, _chain_bounds(want, emu, x0, rows))


def test_block_argument_errors():
    import torch
    import vit_attention_b200 as V
    shape = shp(2, 4, 5, 7, 9)
    w = _dev_weights(W.make_transformer_block_weights(shape.H, 70))
    x = _dev_bits(W.make_tokens(shape, 71))
    ws = torch.empty(V.vggt_block_workspace_size(shape, "frame"), dtype=torch.uint8, device="cuda")
    with pytest.raises(V.VggtAttnError) as e:        # C = 128: not a multiple of 256
        V.vggt_block_forward("frame", shp(2, 2, 5, 7, 9), x, w, EPS, ws)
    assert e.value.code == V.ERR_UNSUPPORTED_SHAPE
    with pytest.raises(V.VggtAttnError) as e:
        V.vggt_block_forward("frame", shape, x, w, EPS, ws, workspace_bytes=ws.numel() - 1)
    assert e.value.code == V.ERR_WORKSPACE_TOO_SMALL
    with pytest.raises(V.VggtAttnError) as e:
        V.vggt_block_forward("frame", shape, x, dict(w, ls1=None), EPS, ws)
    assert e.value.code == V.ERR_INVALID_ARG
    with pytest.raises(V.VggtAttnError) as e:        # x inside the workspace
        V.vggt_block_forward("frame", shape, ws, w, EPS, ws)
    assert e.value.code == V.ERR_INVALID_ARG


def test_camera_trunk_four_blocks():
    import torch
    import vit_attention_b200 as V
    shape = shp(10, 32, 17, 2, 3)     # features of width 2048, 17 special tokens in 23-token frames
    blocks = [W.make_transformer_block_weights(shape.H, 110 + b) for b in range(4)]
    feats = W.make_tokens(shape, 120)
    fd = _dev_bits(feats)
    tok = torch.empty((shape.S * shape.n_special, shape.H * 64), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(V.vggt_camera_trunk_workspace_size(shape), dtype=torch.uint8, device="cuda")
    V.vggt_camera_trunk_forward(shape, fd, tok, [_dev_weights(w) for w in blocks], EPS, ws)
    assert V.vggt_attn_read_status(ws) == 0
    got = tok.float().cpu().numpy().astype(np.float64)
    want = O.camera_trunk_forward(shape, feats, blocks, EPS)
    x0 = O.bf16_to_f64(feats)[O.register_tokens(shape)]
    tok_shape = W.Shape(S=shape.S, T=shape.n_special, H=shape.H, n_special=shape.n_special, grid_h=0, grid_w=0)
    emu = x0
    for w in blocks:
        emu = block_with_storage_rounding("global", tok_shape, emu, w, EPS)
    rows = np.arange(len(want))
    _check(got, want, x0, rows, _chain_bounds(want, emu, x0, rows))


@pytest.mark.parametrize("mode,idx,count", [("frame", 2, 256), ("global", 2, 256), ("register", 4, 512)])
def test_block_at_workload_size_sampled(mode, idx, count):
    """Blocks at the benchmark sizes (24 x 1031 tokens for frame and global, the 500-frame workload for
    register), compared with the oracle on sampled rows (every token still provides keys)."""
    import torch
    import vit_attention_b200 as V
    shape = W.workload(idx).shape
    w = W.make_transformer_block_weights(shape.H, 140 + idx)
    x = W.make_tokens(shape, 150 + idx)
    xd = _dev_bits(x)
    ws = torch.empty(V.vggt_block_workspace_size(shape, mode), dtype=torch.uint8, device="cuda")
    V.vggt_block_forward(mode, shape, xd, _dev_weights(w), EPS, ws)
    assert V.vggt_attn_read_status(ws) == 0
    pool = O.register_tokens(shape) if mode == "register" else np.arange(shape.S * shape.T)
    rows = pool[W.query_subset(len(pool), count, 160 + idx)]
    got = xd.view(shape.S * shape.T, -1)[torch.as_tensor(rows, device="cuda")].float().cpu().numpy().astype(np.float64)
    want = O.block_forward(mode, shape, x, w, EPS, rows)
    x0 = O.bf16_to_f64(x[rows])
    _check(got, want, x0, np.arange(len(rows)), derived_bounds(mode, shape, x, w, EPS, rows=rows, want=want))


def test_aggregator_caches_layers_for_the_heads():
    import torch
    import vit_attention_b200 as V
    shape = shp(4, 4, 5, 4, 5)     # C = 256
    fw = [W.make_transformer_block_weights(shape.H, 170 + l) for l in range(3)]
    iw = [W.make_transformer_block_weights(shape.H, 180 + l) for l in range(3)]
    x = W.make_tokens(shape, 190)
    xd = _dev_bits(x).clone()
    M, C = shape.S * shape.T, shape.H * 64
    cache = {l: torch.full((M, 2 * C), -9.0, dtype=torch.bfloat16, device="cuda") for l in (0, 2)}
    ws = torch.empty(V.vggt_aggregator_workspace_size(shape), dtype=torch.uint8, device="cuda")
    V.vggt_aggregator_forward_cached(shape, xd, [_dev_weights(w) for w in fw], [_dev_weights(w) for w in iw], [1],
                                     cache, EPS, ws)
    assert V.vggt_attn_read_status(ws) == 0
    y, want = O.aggregator_forward(shape, x, fw, iw, [1], EPS, cache_layers=(0, 2))
    # the last layer's inter-frame output is x itself
    assert torch.equal(cache[2][:, C:].view(torch.int16), xd.view(torch.int16))
    x0 = O.bf16_to_f64(x)
    emu, emu_cache = x, {}
    for l in range(3):
        emu = block_with_storage_rounding("frame", shape, emu, fw[l], EPS)
        frame_out = emu
        emu = block_with_storage_rounding("register" if l == 1 else "global", shape, emu, iw[l], EPS)
        emu_cache[l] = np.concatenate([frame_out, emu], axis=1)
    rows = np.arange(M)
    for l in (0, 2):
        got = cache[l].float().cpu().numpy().astype(np.float64)
        for half in (0, 1):
            sl = slice(half * C, (half + 1) * C)
            _check(got[:, sl], want[l][:, sl], x0, rows, _chain_bounds(want[l][:, sl], emu_cache[l][:, sl], x0, rows))


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=8, deadline=None)
@given(mode=st.sampled_from(["frame", "global", "register"]), S=st.integers(1, 4), H=st.sampled_from([4, 8]),
       ns=st.integers(1, 8), gh=st.integers(0, 8), gw=st.integers(1, 8), seed=st.integers(0, 10_000))
def test_random_block_shapes(mode, S, H, ns, gh, gw, seed):
    import torch
    import vit_attention_b200 as V
    shape = shp(S, H, ns, gh, gw)
    w = W.make_transformer_block_weights(H, seed)
    x = W.make_tokens(shape, seed + 1)
    xd = _dev_bits(x).clone()
    ws = torch.empty(V.vggt_block_workspace_size(shape, mode), dtype=torch.uint8, device="cuda")
    V.vggt_block_forward(mode, shape, xd, _dev_weights(w), EPS, ws)
    assert V.vggt_attn_read_status(ws) == 0
    got = xd.float().cpu().numpy().astype(np.float64)
    rows_ = O.register_tokens(shape) if mode == "register" else np.arange(shape.S * shape.T)
    want = O.block_forward(mode, shape, x, w, EPS)
    _check(got, want, O.bf16_to_f64(x), rows_, derived_bounds(mode, shape, x, w, EPS, want=want))
