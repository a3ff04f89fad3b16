"""The oracle's pins catch plausible mistakes (CPU only).

Each case plants one mistake in the oracle -- a dropped term, a wrong sign,
index, axis or operand -- by replacing one of its functions for the duration of
the test, and checks that at least one pin of the module's pin file then fails:
tests/test_oracle.py for the attention core, test_oracle_projection.py,
test_oracle_block.py (blocks and the layer schedule), test_oracle_sga.py and
test_oracle_descriptor.py.  A pin set that some plausible mistake passes would
not pin the oracle; with no mistake planted every pin passes.  The mistakes
live only inside these tests: the oracle's own code is untouched."""
import numpy as np
import pytest
from scipy.special import erf

import oracle
import oracle.attention as OA
import oracle.block as OB
import oracle.descriptor as OD
import oracle.projection as OP
import oracle.sga as OS
import test_oracle as T
import test_oracle_block as TB
import test_oracle_descriptor as TD
import test_oracle_projection as TP
import test_oracle_sga as TS
import workloads as W

# Pins in the order they run; a case ends at its first failing pin.
PINS = [
    (T.test_bf16_widening_exact_bit_patterns, ()),
    (T.test_input_rounding_is_nearest_even, ()),
    (T.test_layer_norm_golden_alternating, ()),
    (T.test_layer_norm_uses_biased_variance, ()),
    (T.test_layer_norm_moments_and_invariances, ()),
    (T.test_layer_norm_matches_torch_fp64, ()),
    *[(T.test_rope_golden_unit_vectors, (i,)) for i in range(5)],
    (T.test_rope_frequencies_closed_form, ()),
    (T.test_rope_matches_complex_rotation, ()),
    (T.test_rope_zero_position_identity_and_norm, ()),
    (T.test_rope_dot_depends_only_on_relative_offset, ()),
    (T.test_patch_positions_row_major, ()),
    (T.test_attention_golden_cases, ()),
    (T.test_attention_rows_sum_to_one_and_large_scores, ()),
    (T.test_attention_constant_v_and_single_key, ()),
    (T.test_attention_matches_torch_sdpa_fp64, ()),
    (T.test_explicit_softmax_scale_golden, ()),
    *[(T.test_pipeline_matches_torch_restatement, (m,)) for m in ("frame", "global", "register")],
    (T.test_global_with_block_diagonal_mask_equals_frame, ()),
    (T.test_permuting_frames_permutes_global_output, ()),
    (T.test_frame_equals_global_for_one_frame_and_register_for_specials_only, ()),
    (T.test_register_mode_brute_force, ()),
]


def first_failing_pin(pins=PINS):
    for fn, args in pins:
        try:
            fn(*args)
        except Exception:   # an AssertionError, or an error the planted mistake provokes
            shown = tuple(a for a in args if isinstance(a, (str, int)))   # modes and sizes, not arrays
            return f"{fn.__name__}{shown if shown else ''}"
    return None


# ------------------------------------------------------------------ planted mistakes
_orig = {name: getattr(OA, name) for name in ("layer_norm", "rope_frequencies", "patch_row_col", "_rotate_half_block",
                                              "rope_2d", "normalized_tokens", "softmax_attention", "resolved_scale",
                                              "attn_frame", "attn_global", "register_tokens", "bf16_to_f64")}


def _ln(x, gamma, beta, eps, *, ddof=0, centre_numerator=True, eps_inside=True, swap_affine=False):
    x = np.asarray(x, np.float64)
    m = x.mean(axis=-1, keepdims=True)
    var = ((x - m) ** 2).sum(axis=-1, keepdims=True) / (x.shape[-1] - ddof)
    num = (x - m) if centre_numerator else x
    den = np.sqrt(var + eps) if eps_inside else np.sqrt(var) + eps
    g, b = np.asarray(gamma, np.float64), np.asarray(beta, np.float64)
    if swap_affine:
        g, b = b, g
    return num / den * g + b


def _rotate_minus_angle(x, pos, omega):
    return _orig["_rotate_half_block"](x, -np.asarray(pos), omega)


def _rotate_adjacent_pairs(x, pos, omega):
    ang = pos[..., None].astype(np.float64) * omega
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(np.asarray(x, np.float64))
    out[..., 0::2], out[..., 1::2] = a * c - b * s, b * c + a * s
    return out


def _rope_halves_swapped(x, row, col, base):
    return _orig["rope_2d"](x, col, row, base)


def _freq_half_exponent(base):
    j = np.arange(16, dtype=np.float64)
    return np.power(float(base), -j / 32.0)


def _positions_one_based(t, n_special, grid_w):
    is_patch, row, col = _orig["patch_row_col"](t, n_special, grid_w)
    return is_patch, row + is_patch, col + is_patch


def _specials_rotated(t, n_special, grid_w):
    t = np.asarray(t, dtype=np.int64)
    p = t - n_special                              # negative for the special tokens
    gw = grid_w if grid_w > 0 else 1
    return np.ones_like(t, dtype=bool), p // gw, p % gw


def _positions_over_sequence(shape, inputs, flat_tokens, which=("q", "k", "v")):
    # patch positions taken from the index in the whole S*T sequence instead of inside the frame
    flat = np.asarray(flat_tokens, dtype=np.int64)
    s, t = flat // shape.T, flat % shape.T
    is_patch = t >= shape.n_special
    _, row, col = _orig["patch_row_col"](flat, shape.n_special, shape.grid_w)
    out = {}
    for c, name in enumerate(("q", "k", "v")):
        if name not in which:
            continue
        x = OA.bf16_to_f64(inputs["qkv"][s, t, c])
        if name != "v":
            x = OA.layer_norm(x, inputs[f"{name}_gamma"][None], inputs[f"{name}_beta"][None], shape.ln_eps)
            x = np.where(is_patch[:, None, None], OA.rope_2d(x, row[:, None], col[:, None], shape.rope_base), x)
        out[name] = np.ascontiguousarray(x.transpose(1, 0, 2))
    return out


def _softmax_unnormalised(q, k, v, scale, mask=None, return_probs=False, chunk=512):
    q, k, v = (np.asarray(a, np.float64) for a in (q, k, v))
    s = scale * (q @ k.T)
    if mask is not None:
        s = np.where(mask, s, -np.inf)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    out = p @ v
    return (out, p) if return_probs else out


def _softmax_keys_as_values(q, k, v, scale, mask=None, return_probs=False, chunk=512):
    return _orig["softmax_attention"](q, k, k, scale, mask, return_probs, chunk)


def _softmax_over_queries(q, k, v, scale, mask=None, return_probs=False, chunk=512):
    q, k, v = (np.asarray(a, np.float64) for a in (q, k, v))
    s = scale * (q @ k.T)
    if mask is not None:
        s = np.where(mask, s, -np.inf)
    p = np.exp(s - s.max(axis=0, keepdims=True))
    p = p / p.sum(axis=0, keepdims=True)
    out = p @ v
    return (out, p) if return_probs else out


MISTAKES = {
    "layer norm: unbiased variance": ("layer_norm", lambda x, g, b, e: _ln(x, g, b, e, ddof=1)),
    "layer norm: mean not subtracted in the numerator": ("layer_norm", lambda x, g, b, e: _ln(x, g, b, e, centre_numerator=False)),
    "layer norm: epsilon outside the square root": ("layer_norm", lambda x, g, b, e: _ln(x, g, b, e, eps_inside=False)),
    "layer norm: gamma and beta swapped": ("layer_norm", lambda x, g, b, e: _ln(x, g, b, e, swap_affine=True)),
    "rope: rotation by minus the angle": ("_rotate_half_block", _rotate_minus_angle),
    "rope: adjacent pairs (2j, 2j+1)": ("_rotate_half_block", _rotate_adjacent_pairs),
    "rope: row and column halves swapped": ("rope_2d", _rope_halves_swapped),
    "rope: frequencies base^(-j/32)": ("rope_frequencies", _freq_half_exponent),
    "rope: 1-based patch positions": ("patch_row_col", _positions_one_based),
    "rope: special tokens rotated too": ("patch_row_col", _specials_rotated),
    "rope: positions counted over the whole sequence": ("normalized_tokens", _positions_over_sequence),
    "softmax: scale 1/64 instead of 1/sqrt(64)": (
        "resolved_scale", lambda shape: float(shape.softmax_scale) if shape.softmax_scale > 0 else 1.0 / 64),
    "softmax: no division by the row sum": ("softmax_attention", _softmax_unnormalised),
    "softmax: keys multiplied instead of values": ("softmax_attention", _softmax_keys_as_values),
    "softmax: normalised over the query axis": ("softmax_attention", _softmax_over_queries),
    "frame mode attends over every frame": ("attn_frame", lambda shape, inputs, queries=None:
                                            _orig["attn_global"](shape, inputs, queries)),
    "register mode takes a patch token as well": ("register_tokens", lambda shape: np.sort(np.concatenate(
        [_orig["register_tokens"](shape), [shape.n_special]])) if shape.T > shape.n_special else _orig["register_tokens"](shape)),
    "bf16 widening: one bit short": ("bf16_to_f64", lambda bits: (np.asarray(bits, np.uint16).astype(np.uint32)
                                                                  << np.uint32(15)).view(np.float32).astype(np.float64)),
}


# ------------------------------------------------------------------ the other oracle modules
# Block pins take the module's fixtures; these are the same seeded draws.
_WTS = W.make_transformer_block_weights(TB.SHAPE.H, 41)
_X = W.make_tokens(TB.SHAPE, 42)
_MODES3 = ("frame", "global", "register")

PIN_SETS = {
    "attention": PINS,
    "projection": [
        (TP.test_linear_permutation_weight_selects_columns, ()),
        (TP.test_linear_matches_torch_fp64, ()),
        *[(TP.test_block_with_identity_projections_is_the_attention_core, (m,)) for m in _MODES3],
        (TP.test_block_output_bias_shifts_every_row, ()),
        (TP.test_projected_qkv_orders_q_k_v_then_heads, ()),
        *[(TP.test_block_matches_torch_linear_around_the_attention_core, (m,)) for m in _MODES3],
    ],
    "block": [
        (TB.test_token_layer_norm_matches_torch, ()),
        (TB.test_gelu_matches_torch_and_closed_forms, ()),
        *[(TB.test_zero_layerscale_is_identity, (m, _WTS, _X)) for m in _MODES3],
        *[(TB.test_attention_branch_alone, (m, _WTS, _X)) for m in ("frame", "global")],
        *[(TB.test_mlp_branch_alone, (m, _WTS, _X)) for m in ("frame", "global")],
        *[(TB.test_full_block_runs_the_mlp_on_the_attention_branch_output, (m, _WTS, _X)) for m in ("frame", "global")],
        (TB.test_register_block_changes_only_special_rows_like_a_global_block_on_them, (_WTS, _X)),
        (TB.test_frame_block_acts_on_each_frame_alone, (_WTS, _X)),
        (TB.test_global_block_commutes_with_frame_permutation, (_WTS,)),
        (TB.test_aggregator_schedule, (_WTS, _X)),
        (TB.test_camera_trunk_reduces_to_register_blocks, (_WTS, _X)),
        *[(TB.test_row_subset_equals_rows_of_full_result, (m, _WTS, _X)) for m in _MODES3],
        (TB.test_cached_layers_concatenate_frame_and_inter_outputs, (_WTS, _X)),
    ],
    "sga": [
        (TS.test_no_subsampling_is_global_attention, ()),
        (TS.test_kept_tokens_grid, ()),
        *[(TS.test_matches_brute_force_with_duplicated_mean_columns, a) for a in ((2, 2), (3, 2), (2, 4))],
        (TS.test_constant_values_give_that_constant, ()),
    ],
    "descriptor": [
        (TD.test_unit_windows_are_global_attention, ()),
        *[(TD.test_descriptor_count_and_coverage, a) for a in ((2, 2), (3, 2), (4, 4))],
        (TD.test_brute_force_tiny, ()),
        (TD.test_constant_values_give_constant_output, ()),
    ],
}

_orig_p = {n: getattr(OP, n) for n in ("linear", "projected_qkv", "attention_block")}
_orig_b = {n: getattr(OB, n) for n in ("token_layer_norm", "gelu", "block_forward", "aggregator_forward",
                                       "camera_trunk_forward")}
_orig_s = {n: getattr(OS, n) for n in ("sga_kept_tokens", "attn_global_sga")}
_orig_d = {n: getattr(OD, n) for n in ("descriptor_windows", "attn_global_desc")}


# projection
def _linear_no_bias(x, w, b=None):
    return _orig_p["linear"](x, w, None)


def _qkv_heads_outer(shape, block):
    # the 3C outputs read as [H][3][64] instead of [3][H][64]
    y = OP.linear(block["x"], block["w_qkv"], block.get("b_qkv"))
    return y.reshape(shape.S, shape.T, shape.H, 3, 64).transpose(0, 1, 3, 2, 4)


def _attention_block(mode, shape, block, queries=None, *, out_untransposed=False, no_out_bias=False, qk_norm_swapped=False):
    inputs = {"qkv_f64": OP.projected_qkv(shape, block)}
    names = {"q_gamma": "k_gamma", "q_beta": "k_beta", "k_gamma": "q_gamma", "k_beta": "q_beta"} if qk_norm_swapped else {}
    for name in ("q_gamma", "q_beta", "k_gamma", "k_beta"):
        inputs[name] = block[names.get(name, name)]
    attn = OA.attn_mode(mode, shape, inputs, queries)
    a = attn.reshape(attn.shape[0], -1)
    w = OA.bf16_to_f64(block["w_out"])
    y = a @ (w if out_untransposed else w.T)
    if block.get("b_out") is not None and not no_out_bias:
        y = y + np.asarray(block["b_out"], np.float64)
    return y


# block and schedule
def _token_ln_unbiased(x, gamma, beta, eps):
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).sum(axis=-1, keepdims=True) / (x.shape[-1] - 1)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(gamma, np.float64) + np.asarray(beta, np.float64)


def _gelu_tanh(x):
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))


def _gelu_without_x(x):
    return 0.5 * (1.0 + erf(x / np.sqrt(2.0)))


def _block(mode, shape, x, w, norm_eps, rows=None, *, parallel=False, norm1_for_mlp=False, ls_on_residual=False,
           mlp_on_every_token=False):
    """The block restated with one planted mistake (flags); otherwise as in oracle/block.py."""
    x = OA.bf16_to_f64(x) if x.dtype == np.uint16 else np.asarray(x, np.float64)
    C = shape.H * 64
    subset = rows is not None
    if not subset:
        rows = OA.register_tokens(shape) if mode == "register" else np.arange(shape.S * shape.T, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    if mode == "register":
        need = OA.register_tokens(shape)
    elif mode == "frame" and subset:
        frames = np.unique(rows // shape.T)
        need = (frames[:, None] * shape.T + np.arange(shape.T)[None, :]).reshape(-1)
    else:
        need = np.arange(shape.S * shape.T, dtype=np.int64)

    def aff(a, wn, bn):
        y = a @ OA.bf16_to_f64(w[wn]).T
        return y + np.asarray(w[bn], np.float64)

    h = OB.token_layer_norm(x[need], w["norm1_gamma"], w["norm1_beta"], norm_eps)
    qkv = np.zeros((shape.S * shape.T, 3 * C))
    qkv[need] = aff(h, "w_qkv", "b_qkv")
    inputs = {"qkv_f64": qkv.reshape(shape.S, shape.T, 3, shape.H, 64), **{k: w[k] for k in ("q_gamma", "q_beta", "k_gamma", "k_beta")}}
    a = OA.attn_mode(mode, shape, inputs, rows).reshape(len(rows), C)
    ls1, ls2 = np.asarray(w["ls1"], np.float64), np.asarray(w["ls2"], np.float64)
    branch1 = aff(a, "w_proj", "b_proj")
    xr = ls1 * x[rows] + branch1 if ls_on_residual else x[rows] + ls1 * branch1

    def mlp(z):
        g, b = ("norm1_gamma", "norm1_beta") if norm1_for_mlp else ("norm2_gamma", "norm2_beta")
        return aff(OB.gelu(aff(OB.token_layer_norm(z, w[g], w[b], norm_eps), "w_fc1", "b_fc1")), "w_fc2", "b_fc2")

    yr = xr + ls2 * mlp(x[rows] if parallel else xr)
    if subset:
        return yr
    y = x.copy()
    if mlp_on_every_token:
        y = y + ls2 * mlp(y)
    y[rows] = yr
    return y


def _schedule(shape, x, frame_blocks, inter_blocks, register_layers, norm_eps, cache_layers=(), *,
              inter_first=False, cache_swapped=False):
    y = OA.bf16_to_f64(x) if x.dtype == np.uint16 else np.asarray(x, np.float64)
    cache = {}
    for l, (fw, iw) in enumerate(zip(frame_blocks, inter_blocks)):
        steps = [("frame", fw), ("register" if l in register_layers else "global", iw)]
        if inter_first:
            steps.reverse()
        y = OB.block_forward(steps[0][0], shape, y, steps[0][1], norm_eps)
        first = y
        y = OB.block_forward(steps[1][0], shape, y, steps[1][1], norm_eps)
        if l in cache_layers:
            cache[l] = np.concatenate([y, first] if cache_swapped else [first, y], axis=1)
    return (y, cache) if cache_layers else y


def _trunk(shape, feats, blocks, norm_eps, *, per_frame=False, leading_tokens=False):
    x = OA.bf16_to_f64(feats) if feats.dtype == np.uint16 else np.asarray(feats, np.float64)
    y = x[:shape.S * shape.n_special] if leading_tokens else x[OA.register_tokens(shape)]
    tok_shape = type(shape)(**{**shape.__dict__, "T": shape.n_special, "grid_h": 0, "grid_w": 0})
    for w in blocks:
        y = OB.block_forward("frame" if per_frame else "global", tok_shape, y, w, norm_eps)
    return y


# SGA
def _kept_last_of_window(shape, s_h, s_w):
    t = np.arange(shape.T)
    is_patch, row, col = OA.patch_row_col(t, shape.n_special, shape.grid_w)
    keep_t = np.nonzero(~is_patch | ((row % s_h == s_h - 1) & (col % s_w == s_w - 1)))[0]
    return (np.arange(shape.S)[:, None] * shape.T + keep_t[None, :]).reshape(-1)


def _sga(shape, inputs, s_h, s_w, queries=None, *, mean_once=False, no_diag=False, mean_over_all=False,
         n_mean_full=False):
    """SGA restated with one planted mistake (flags); otherwise as in oracle/sga.py."""
    N = shape.S * shape.T
    qi = np.arange(N, dtype=np.int64) if queries is None else np.asarray(queries, dtype=np.int64)
    kept = OS.sga_kept_tokens(shape, s_h, s_w)
    in_kept = np.zeros(N, dtype=bool)
    in_kept[kept] = True
    disc = np.nonzero(~in_kept)[0]
    pool = np.arange(N) if mean_over_all else disc
    kv = OA.normalized_tokens(shape, inputs, np.arange(N), ("k", "v"))
    qn = OA.normalized_tokens(shape, inputs, qi, ("q",))["q"]
    scale = OA.resolved_scale(shape)
    out = np.empty((len(qi), shape.H, 64))
    for h in range(shape.H):
        k, v = kv["k"][h], kv["v"][h]
        k_mean, v_mean = (k[pool].mean(axis=0), v[pool].mean(axis=0)) if len(pool) else (np.zeros(64), np.zeros(64))
        for a, i in enumerate(qi):
            diag = (not in_kept[i]) and not no_diag
            n_mean = len(disc) - (1 if (not in_kept[i]) and not n_mean_full else 0)
            if mean_once:
                n_mean = min(n_mean, 1)
            keys, vals, wts = [k[kept]], [v[kept]], [np.ones(len(kept))]
            if diag:
                keys, vals, wts = keys + [k[i][None]], vals + [v[i][None]], wts + [np.ones(1)]
            if n_mean > 0:
                keys, vals, wts = keys + [k_mean[None]], vals + [v_mean[None]], wts + [np.array([float(n_mean)])]
            s = scale * (np.concatenate(keys) @ qn[h, a])
            p = np.concatenate(wts) * np.exp(s - s.max())
            out[a, h] = (p @ np.concatenate(vals)) / p.sum()
    return out


# descriptor attention
def _windows(shape, s_h, s_w, *, floor_edges=False, specials_pooled=False):
    ceil = (lambda n, d: n // d) if floor_edges else (lambda n, d: -(-n // d))
    nh, nw = ceil(shape.grid_h, s_h), ceil(shape.grid_w, s_w)
    out = []
    for s in range(shape.S):
        base = s * shape.T
        if specials_pooled:
            out.append(base + np.arange(shape.n_special))
        else:
            out.extend(np.array([base + t]) for t in range(shape.n_special))
        for wr in range(nh):
            for wc in range(nw):
                rows = np.arange(wr * s_h, min((wr + 1) * s_h, shape.grid_h))
                cols = np.arange(wc * s_w, min((wc + 1) * s_w, shape.grid_w))
                out.append(base + shape.n_special + (rows[:, None] * shape.grid_w + cols[None, :]).reshape(-1))
    return out


def _desc(shape, inputs, s_h, s_w, queries=None, *, sum_pool=False, first_value=False):
    N = shape.S * shape.T
    qi = np.arange(N, dtype=np.int64) if queries is None else np.asarray(queries, dtype=np.int64)
    kv = OA.normalized_tokens(shape, inputs, np.arange(N), ("k", "v"))
    qn = OA.normalized_tokens(shape, inputs, qi, ("q",))["q"]
    win = OD.descriptor_windows(shape, s_h, s_w)
    pool = (lambda a, w: a[:, w].sum(axis=1)) if sum_pool else (lambda a, w: a[:, w].mean(axis=1))
    kd = np.stack([pool(kv["k"], w) for w in win], axis=1)
    vd = np.stack([kv["v"][:, w[0]] if first_value else pool(kv["v"], w) for w in win], axis=1)
    out = np.empty((len(qi), shape.H, 64))
    for h in range(shape.H):
        out[:, h] = OA.softmax_attention(qn[h], kd[h], vd[h], OA.resolved_scale(shape))
    return out


NEXT_MISTAKES = {
    # (pin set, module, function, replacement)
    "projection: bias dropped": ("projection", OP, "linear", _linear_no_bias),
    "projection: qkv outputs read as [H][3][64]": ("projection", OP, "projected_qkv", _qkv_heads_outer),
    "projection: output weight untransposed": (
        "projection", OP, "attention_block", lambda *a, **k: _attention_block(*a, **k, out_untransposed=True)),
    "projection: output bias dropped": (
        "projection", OP, "attention_block", lambda *a, **k: _attention_block(*a, **k, no_out_bias=True)),
    "projection: q and k norm parameters swapped": (
        "projection", OP, "attention_block", lambda *a, **k: _attention_block(*a, **k, qk_norm_swapped=True)),
    "block: unbiased variance in the token LayerNorm": ("block", OB, "token_layer_norm", _token_ln_unbiased),
    "block: GELU in its tanh form": ("block", OB, "gelu", _gelu_tanh),
    "block: GELU without the factor x": ("block", OB, "gelu", _gelu_without_x),
    "block: MLP branch reads the block input (parallel residuals)": (
        "block", OB, "block_forward", lambda *a, **k: _block(*a, **k, parallel=True)),
    "block: MLP LayerNorm with norm1's parameters": (
        "block", OB, "block_forward", lambda *a, **k: _block(*a, **k, norm1_for_mlp=True)),
    "block: LayerScale on the residual instead of the branch": (
        "block", OB, "block_forward", lambda *a, **k: _block(*a, **k, ls_on_residual=True)),
    "block: register layer runs the MLP on the patch tokens too": (
        "block", OB, "block_forward", lambda *a, **k: _block(*a, **k, mlp_on_every_token=True)),
    "schedule: inter-frame block before the frame block": (
        "block", OB, "aggregator_forward", lambda *a, **k: _schedule(*a, **k, inter_first=True)),
    "schedule: cached halves in the wrong order": (
        "block", OB, "aggregator_forward", lambda *a, **k: _schedule(*a, **k, cache_swapped=True)),
    "schedule: register layers counted from one": ("block", OB, "REGISTER_LAYERS", (3, 7, 10, 15, 21)),
    "camera trunk: attention inside each frame only": (
        "block", OB, "camera_trunk_forward", lambda *a, **k: _trunk(*a, **k, per_frame=True)),
    "camera trunk: the sequence's first tokens instead of each frame's": (
        "block", OB, "camera_trunk_forward", lambda *a, **k: _trunk(*a, **k, leading_tokens=True)),
    "sga: kept token is the last of each window": ("sga", OS, "sga_kept_tokens", _kept_last_of_window),
    "sga: mean pair counted once": ("sga", OS, "attn_global_sga", lambda *a, **k: _sga(*a, **k, mean_once=True)),
    "sga: no diagonal term": ("sga", OS, "attn_global_sga", lambda *a, **k: _sga(*a, **k, no_diag=True)),
    "sga: mean over every token, kept ones included": (
        "sga", OS, "attn_global_sga", lambda *a, **k: _sga(*a, **k, mean_over_all=True)),
    "sga: mean pair counted |D| times beside the diagonal": (
        "sga", OS, "attn_global_sga", lambda *a, **k: _sga(*a, **k, n_mean_full=True)),
    "descriptor: partial edge windows dropped": (
        "descriptor", OD, "descriptor_windows", lambda *a, **k: _windows(*a, **k, floor_edges=True)),
    "descriptor: special tokens pooled into one descriptor": (
        "descriptor", OD, "descriptor_windows", lambda *a, **k: _windows(*a, **k, specials_pooled=True)),
    "descriptor: window keys and values summed": (
        "descriptor", OD, "attn_global_desc", lambda *a, **k: _desc(*a, **k, sum_pool=True)),
    "descriptor: a window's first value instead of the mean": (
        "descriptor", OD, "attn_global_desc", lambda *a, **k: _desc(*a, **k, first_value=True)),
}


def test_restatements_without_a_mistake_equal_the_oracle():
    """The restated functions above differ from the oracle only by their planted flag."""
    shape = TS.SHAPE
    inputs = W.make_random_inputs(shape, 7)
    np.testing.assert_allclose(_sga(shape, inputs, 2, 2), OS.attn_global_sga(shape, inputs, 2, 2), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(_desc(shape, inputs, 2, 3), OD.attn_global_desc(shape, inputs, 2, 3), rtol=1e-12, atol=1e-13)
    for a, b in zip(_windows(shape, 2, 3), OD.descriptor_windows(shape, 2, 3)):
        np.testing.assert_array_equal(a, b)
    for mode in _MODES3:
        np.testing.assert_allclose(_block(mode, TB.SHAPE, _X, _WTS, TB.EPS), OB.block_forward(mode, TB.SHAPE, _X, _WTS, TB.EPS),
                                   rtol=1e-12, atol=1e-12)
    block = W.make_block_inputs(TP_SHAPE, 6)
    np.testing.assert_allclose(_attention_block("global", TP_SHAPE, block), OP.attention_block("global", TP_SHAPE, block),
                               rtol=1e-12, atol=1e-12)
    y, c = _schedule(TB.SHAPE, _X, [_WTS], [_WTS], [], TB.EPS, cache_layers=(0,))
    y0, c0 = OB.aggregator_forward(TB.SHAPE, _X, [_WTS], [_WTS], [], TB.EPS, cache_layers=(0,))
    np.testing.assert_array_equal(y, y0)
    np.testing.assert_array_equal(c[0], c0[0])
    np.testing.assert_array_equal(_trunk(TB.SHAPE, _X, [_WTS], TB.EPS), OB.camera_trunk_forward(TB.SHAPE, _X, [_WTS], TB.EPS))


TP_SHAPE = W.Shape(S=2, T=11, H=2, n_special=3, grid_h=2, grid_w=4)


def test_every_pin_passes_without_a_planted_mistake():
    assert first_failing_pin() is None


@pytest.mark.parametrize("mistake", sorted(MISTAKES))
def test_planted_mistake_fails_a_pin(mistake, monkeypatch):
    name, fn = MISTAKES[mistake]
    monkeypatch.setattr(OA, name, fn)
    if hasattr(oracle, name):
        monkeypatch.setattr(oracle, name, fn)
    caught = first_failing_pin()
    assert caught is not None, f"no pin fails with the mistake '{mistake}'"


@pytest.mark.parametrize("pins", sorted(PIN_SETS))
def test_every_pin_set_passes_without_a_planted_mistake(pins):
    assert first_failing_pin(PIN_SETS[pins]) is None


@pytest.mark.parametrize("mistake", sorted(NEXT_MISTAKES))
def test_planted_mistake_in_the_other_modules_fails_a_pin(mistake, monkeypatch):
    pins, module, name, fn = NEXT_MISTAKES[mistake]
    monkeypatch.setattr(module, name, fn)
    if hasattr(oracle, name):
        monkeypatch.setattr(oracle, name, fn)
    caught = first_failing_pin(PIN_SETS[pins])
    assert caught is not None, f"no pin fails with the mistake '{mistake}'"
