"""GPU parity of the projections around the attention core (vggt_linear,
vggt_attn_qkv_proj, vggt_attn_block) against the fp64 oracle
(oracle/projection.py), through the C ABI binding."""
import numpy as np
import pytest

import oracle as O
import workloads as W
from parity import MAX_ABS_TOL, REL_FRO_TOL, assert_close, errors, query_sample

pytestmark = pytest.mark.gpu


def _dev_bits(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def _dev_f32(a):
    import torch
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _status_ws():
    import torch
    return torch.zeros(256, dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("M,N,K,with_bias", [(300, 512, 128, True), (129, 256, 64, False), (2 * 1031, 1024, 1024, True)])
def test_linear_matches_oracle(M, N, K, with_bias):
    import torch
    import vit_attention_b200 as V
    rng = np.random.default_rng([M, N, K])
    x = W.f32_to_bf16_bits(rng.standard_normal((M, K), dtype=np.float32))
    w = W.f32_to_bf16_bits(rng.standard_normal((N, K), dtype=np.float32) / np.float32(np.sqrt(K)))
    b = (0.1 * rng.standard_normal(N)).astype(np.float32) if with_bias else None
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = _status_ws()
    V.vggt_linear(_dev_bits(x), _dev_bits(w), _dev_f32(b), y, ws)
    assert V.vggt_attn_read_status(ws) == 0
    rows = W.query_subset(M, 512, 9)
    want = O.linear(x[rows], w, b)
    got = y.float().cpu().numpy().astype(np.float64)[rows]
    assert_close(got, want, f"linear {M}x{N}x{K}")


def _block_case(mode, shape, seed, count):
    import torch
    import vit_attention_b200 as V
    blk = W.make_block_inputs(shape, seed)
    C = shape.H * 64
    M = shape.S * shape.T
    dev = {k: _dev_bits(blk[k]) for k in ("x", "w_qkv", "w_out")}
    dev.update({k: _dev_f32(blk[k]) for k in ("b_qkv", "b_out", "q_gamma", "q_beta", "k_gamma", "k_beta")})
    ws = torch.empty(V.vggt_attn_workspace_size(shape, mode), dtype=torch.uint8, device="cuda")
    qkv = torch.empty((shape.S, shape.T, 3, shape.H, 64), dtype=torch.bfloat16, device="cuda")
    attn = torch.empty((M, C), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((M, C), dtype=torch.bfloat16, device="cuda")
    sentinel = -7.0
    y.fill_(sentinel)
    V.vggt_attn_block(mode, shape, dev["x"], dev["w_qkv"], dev["b_qkv"], dev["q_gamma"], dev["q_beta"],
                      dev["k_gamma"], dev["k_beta"], dev["w_out"], dev["b_out"], qkv, attn, y, ws)
    assert V.vggt_attn_read_status(ws) == 0
    q = query_sample(mode, shape, count, seed)
    idx = torch.as_tensor(q, device="cuda")
    if mode == "register":
        # patch rows untouched; special rows checked against the oracle block
        patch = torch.ones(M, dtype=torch.bool, device="cuda")
        patch[torch.as_tensor(O.register_tokens(shape), device="cuda")] = False
        assert bool((y[patch] == sentinel).all())
        want_y = O.attention_block(mode, shape, blk, q)
        got_y = y.index_select(0, idx).float().cpu().numpy().astype(np.float64)
        return assert_close(got_y, want_y, f"block output {mode} {shape}")
    # the attention output between the projections
    inputs = {"qkv_f64": O.projected_qkv(shape, blk)}
    inputs.update({k: blk[k] for k in ("q_gamma", "q_beta", "k_gamma", "k_beta")})
    want_attn = O.attn_mode(mode, shape, inputs, q).reshape(len(q), C)
    got_attn = attn.index_select(0, idx).float().cpu().numpy().astype(np.float64)
    assert_close(got_attn, want_attn, f"block attention {mode} {shape}")
    want_y = O.attention_block(mode, shape, blk, q)
    got_y = y.index_select(0, idx).float().cpu().numpy().astype(np.float64)
    return assert_close(got_y, want_y, f"block output {mode} {shape}")


@pytest.mark.parametrize("mode", ["frame", "global", "register"])
def test_block_small_matches_oracle(mode):
    _block_case(mode, W.workload(0).shape, 31, 1 << 62)


@pytest.mark.parametrize("mode", ["frame", "global", "register"])
def test_block_ragged_matches_oracle(mode):
    # 3 frames of 1031 tokens: 128-row tiles straddle frame boundaries.
    _block_case(mode, W.Shape(S=3, T=1031, H=16, n_special=17, grid_h=26, grid_w=39), 32, 512)


@pytest.mark.parametrize("mode", ["frame", "global"])
def test_block_wide_patch_grid_matches_oracle(mode):
    # grid 2 x 420: 422 RoPE positions, more than the normalising GEMM epilogue keeps in shared memory beside
    # its buffers, so the block takes the GEMM followed by the separate prologue instead.
    _block_case(mode, W.Shape(S=2, T=845, H=4, n_special=5, grid_h=2, grid_w=420), 33, 256)


def test_qkv_proj_matches_oracle_attention():
    """vggt_attn_qkv_proj (the QKV GEMM whose epilogue normalises and rotates q and k into the workspace and
    writes v into qkv) followed by vggt_attn_core: the attention output against the oracle on the projected
    qkv."""
    import torch
    import vit_attention_b200 as V
    for mode, shape in (("frame", W.Shape(S=3, T=1031, H=16, n_special=17, grid_h=26, grid_w=39)),
                        ("global", W.workload(0).shape)):
        blk = W.make_block_inputs(shape, 34)
        C, M = shape.H * 64, shape.S * shape.T
        dev = {k: _dev_bits(blk[k]) for k in ("x", "w_qkv")}
        dev.update({k: _dev_f32(blk[k]) for k in ("b_qkv", "q_gamma", "q_beta", "k_gamma", "k_beta")})
        ws = torch.empty(V.vggt_attn_workspace_size(shape, mode), dtype=torch.uint8, device="cuda")
        qkv = torch.empty((shape.S, shape.T, 3, shape.H, 64), dtype=torch.bfloat16, device="cuda")
        attn = torch.empty((shape.S, shape.T, shape.H, 64), dtype=torch.bfloat16, device="cuda")
        V.vggt_attn_qkv_proj(mode, shape, dev["x"], dev["w_qkv"], dev["b_qkv"], dev["q_gamma"], dev["q_beta"],
                             dev["k_gamma"], dev["k_beta"], qkv, ws)
        V.vggt_attn_core(mode, shape, qkv, attn, ws)
        assert V.vggt_attn_read_status(ws) == 0
        q = query_sample(mode, shape, 512, 35)
        inputs = {"qkv_f64": O.projected_qkv(shape, blk)}
        inputs.update({k: blk[k] for k in ("q_gamma", "q_beta", "k_gamma", "k_beta")})
        want = O.attn_mode(mode, shape, inputs, q)
        got = attn.view(M, shape.H, 64).index_select(0, torch.as_tensor(q, device="cuda")).float().cpu().numpy()
        assert_close(got.astype(np.float64), want, f"qkv_proj + core {mode}")


def test_qkv_proj_rejects_register_mode_and_odd_heads():
    import torch
    import vit_attention_b200 as V
    shape = W.workload(0).shape
    ws = torch.empty(V.vggt_attn_workspace_size(shape, "register"), dtype=torch.uint8, device="cuda")
    C = shape.H * 64
    x = torch.zeros((shape.S * shape.T, C), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((3 * C, C), dtype=torch.bfloat16, device="cuda")
    g = torch.ones((shape.H, 64), dtype=torch.float32, device="cuda")
    qkv = torch.empty((shape.S, shape.T, 3, shape.H, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(V.VggtAttnError) as e:
        V.vggt_attn_qkv_proj("register", shape, x, w, None, g, g, g, g, qkv, ws)
    assert e.value.code == V.ERR_INVALID_ARG
    odd = W.Shape(S=1, T=5, H=2, n_special=1, grid_h=2, grid_w=2)
    ws2 = torch.empty(V.vggt_attn_workspace_size(odd, "global"), dtype=torch.uint8, device="cuda")
    x2 = torch.zeros((5, 128), dtype=torch.bfloat16, device="cuda")
    w2 = torch.zeros((384, 128), dtype=torch.bfloat16, device="cuda")
    g2 = torch.ones((2, 64), dtype=torch.float32, device="cuda")
    qkv2 = torch.empty((1, 5, 3, 2, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(V.VggtAttnError) as e:
        V.vggt_attn_qkv_proj("global", odd, x2, w2, None, g2, g2, g2, g2, qkv2, ws2)
    assert e.value.code == V.ERR_UNSUPPORTED_SHAPE
