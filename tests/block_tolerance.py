"""Derivation of the transformer-block parity tolerance (test helper).

The CUDA path of a block stores these intermediates in bf16 (round to nearest
even), with fp32 accumulation inside every GEMM and kernel: the token
LayerNorm outputs, the QKV projection, the attention output, the residual
stream after the attention branch, the MLP hidden activations and the block
output.  ``block_with_storage_rounding`` is the fp64 oracle's block
(oracle/block.py) with exactly those roundings inserted; its distance from the
plain fp64 oracle is the error that the storage format alone makes.  The GPU
tests allow ``ROOM`` times that distance, computed on the same inputs: the
room covers what the emulation leaves out (fp32 accumulation order in the
GEMMs, the attention core's own bf16 rounding of q, k and P), which is of the
same order as one of the modelled roundings.

With ``rounding=None`` the emulation is the oracle's block step for step
(tests/test_block_tolerance.py checks that it then matches the oracle to fp64
rounding), so the derived error comes from the inserted roundings only.
"""
from __future__ import annotations

import numpy as np

import oracle as O
import workloads as W

ROOM = 3.0


def bf16_round(a):
    """fp64 -> nearest bf16 (ties to even) -> fp64."""
    return O.bf16_to_f64(W.f32_to_bf16_bits(np.asarray(a, dtype=np.float64).astype(np.float32)))


def _affine(x, w_bits, b):
    y = x @ O.bf16_to_f64(w_bits).T
    return y if b is None else y + np.asarray(b, np.float64)


def block_with_storage_rounding(mode, shape, x, w, eps, rows=None, rounding=bf16_round):
    """The oracle's block with ``rounding`` applied where the CUDA path stores bf16.

    Same arguments and result layout as ``oracle.block_forward``."""
    r = rounding if rounding is not None else (lambda a: a)
    x = O.bf16_to_f64(x) if x.dtype == np.uint16 else np.asarray(x, np.float64)
    C = shape.H * 64
    subset = rows is not None
    if not subset:
        rows = O.register_tokens(shape) if mode == "register" else np.arange(shape.S * shape.T, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    if mode == "register":
        need = O.register_tokens(shape)
    elif mode == "frame" and subset:
        frames = np.unique(rows // shape.T)
        need = (frames[:, None] * shape.T + np.arange(shape.T)[None, :]).reshape(-1)
    else:
        need = np.arange(shape.S * shape.T, dtype=np.int64)
    h = r(O.token_layer_norm(x[need], w["norm1_gamma"], w["norm1_beta"], eps))
    qkv = np.zeros((shape.S * shape.T, 3 * C))
    qkv[need] = r(_affine(h, w["w_qkv"], w.get("b_qkv")))
    inputs = {"qkv_f64": qkv.reshape(shape.S, shape.T, 3, shape.H, 64)}
    for name in ("q_gamma", "q_beta", "k_gamma", "k_beta"):
        inputs[name] = w[name]
    a = r(O.attn_mode(mode, shape, inputs, rows).reshape(len(rows), C))
    xr = r(x[rows] + np.asarray(w["ls1"], np.float64) * _affine(a, w["w_proj"], w.get("b_proj")))
    h2 = r(O.token_layer_norm(xr, w["norm2_gamma"], w["norm2_beta"], eps))
    u = r(O.gelu(_affine(h2, w["w_fc1"], w.get("b_fc1"))))
    yr = r(xr + np.asarray(w["ls2"], np.float64) * _affine(u, w["w_fc2"], w.get("b_fc2")))
    if subset:
        return yr
    y = x.copy()
    y[rows] = yr
    return y


def errors(got, want, x0):
    """(rel-Frobenius of the output, rel-Frobenius of the update output - input, max-abs)."""
    fro = np.linalg.norm(got - want) / np.linalg.norm(want)
    dfro = np.linalg.norm((got - x0) - (want - x0)) / np.linalg.norm(want - x0)
    return float(fro), float(dfro), float(np.abs(got - want).max())


def storage_errors(mode, shape, x, w, eps, rows=None, want=None):
    """Errors of the bf16-storage emulation against the fp64 oracle on these inputs."""
    if want is None:
        want = O.block_forward(mode, shape, x, w, eps, rows)
    emu = block_with_storage_rounding(mode, shape, x, w, eps, rows)
    x0 = O.bf16_to_f64(x) if x.dtype == np.uint16 else np.asarray(x, np.float64)
    if rows is None:
        sel = O.register_tokens(shape) if mode == "register" else np.arange(shape.S * shape.T)
        return errors(emu[sel], want[sel], x0[sel])
    return errors(emu, want, x0[np.asarray(rows)])


def derived_bounds(mode, shape, x, w, eps, rows=None, want=None, room=ROOM):
    """(out_fro, delta_fro, max_abs) bounds for a GPU block on these inputs: ``room`` x the storage errors."""
    return tuple(room * e for e in storage_errors(mode, shape, x, w, eps, rows, want))
