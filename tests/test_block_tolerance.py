"""The transformer-block tolerance is derived, not quoted (CPU only).

tests/block_tolerance.py inserts bf16 rounding into the oracle's block at the
points where the CUDA path stores bf16; the GPU block tests allow ROOM times
the error that this emulation shows on their own inputs.  These tests check
that the emulation is the oracle's block step for step when nothing is
rounded, that the rounding it models is nearest-even bf16, and that the
resulting bounds stay of the size the storage format explains."""
import numpy as np
import pytest

import oracle as O
import workloads as W
from block_tolerance import ROOM, bf16_round, block_with_storage_rounding, derived_bounds, storage_errors


def shp(S, H, ns, gh, gw):
    return W.Shape(S=S, T=ns + gh * gw, H=H, n_special=ns, grid_h=gh, grid_w=gw)


CASES = [("frame", shp(3, 4, 5, 7, 9)), ("global", shp(3, 4, 5, 7, 9)), ("register", shp(40, 4, 5, 2, 3)),
         ("global", shp(2, 16, 17, 6, 8))]


@pytest.mark.parametrize("mode,shape", CASES, ids=[f"{m}-T{s.T}H{s.H}" for m, s in CASES])
def test_emulation_without_rounding_is_the_oracle_block(mode, shape):
    w = W.make_transformer_block_weights(shape.H, 50 + shape.H)
    x = W.make_tokens(shape, 60 + shape.T)
    want = O.block_forward(mode, shape, x, w, 1e-6)
    got = block_with_storage_rounding(mode, shape, x, w, 1e-6, rounding=None)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    rows = np.array([0, shape.T + 1, shape.S * shape.T - 1]) if mode != "register" else O.register_tokens(shape)[:3]
    np.testing.assert_allclose(block_with_storage_rounding(mode, shape, x, w, 1e-6, rows=rows, rounding=None),
                               O.block_forward(mode, shape, x, w, 1e-6, rows), rtol=1e-12, atol=1e-12)


def test_bf16_round_is_nearest_even():
    # 1 + 2^-8 lies halfway between bf16 neighbours 1 and 1 + 2^-7: ties go to the even mantissa (1);
    # 1 + 3 * 2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6: ties go to 1 + 2^-6
    np.testing.assert_array_equal(bf16_round([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -20, -3.0]),
                                  [1.0, 1 + 2 ** -6, 1 + 2 ** -7, -3.0])


@pytest.mark.parametrize("mode,shape", CASES, ids=[f"{m}-T{s.T}H{s.H}" for m, s in CASES])
def test_storage_errors_are_of_the_bf16_size(mode, shape):
    # bf16 keeps 8 significant bits (unit roundoff 2^-9 ~ 2e-3): a handful of roundings in a row leave a
    # relative error of a few 1e-3 on the block output, never a 1e-2 one.
    w = W.make_transformer_block_weights(shape.H, 50 + shape.H)
    x = W.make_tokens(shape, 60 + shape.T)
    fro, dfro, mx = storage_errors(mode, shape, x, w, 1e-6)
    assert 5e-4 < fro < 6e-3 and 5e-4 < dfro < 1e-2
    assert 0 < mx < 6e-2
    b = derived_bounds(mode, shape, x, w, 1e-6)
    assert b == pytest.approx((ROOM * fro, ROOM * dfro, ROOM * mx))
