"""The oracle's pins catch plausible mistakes (CPU only).

Each case plants one mistake in the oracle -- a dropped term, a wrong sign,
index, axis or operand -- by replacing one of its functions for the duration of
the test, and checks that at least one pin of tests/test_oracle.py then fails.
A pin set that some plausible mistake passes would not pin the oracle; with no
mistake planted every pin passes.  The mistakes live only inside these tests:
the oracle's own code is untouched."""
import numpy as np
import pytest

import oracle
import oracle.attention as OA
import test_oracle as T

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


def first_failing_pin():
    for fn, args in PINS:
        try:
            fn(*args)
        except Exception:   # an AssertionError, or an error the planted mistake provokes
            return f"{fn.__name__}{args if args else ''}"
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
