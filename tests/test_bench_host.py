"""Host arithmetic of the measurement: the algorithmic flop and minimum-I/O byte counts that the bench
divides by measured time, against figures worked out by hand from each workload's shape (4 N_q N_k 64
flop per head for QK^T + PV; q, k, v read and out written, 128 bytes each per token and head)."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
import workloads as W  # noqa: E402

# (workload index, mode, algorithmic flop, minimum HBM bytes)
CASES = [
    (0, "global", 1.950e7, 138 * 4 * 512),          # 138 tokens x 4 heads
    (1, "frame", 1.0449e11, 24 * 1031 * 16 * 512),  # 24 frames of 1031 tokens
    (2, "global", 2.5078e12, 24744 * 16 * 512),     # one sequence of 24,744 tokens
    (3, "global", 4.3539e13, 103100 * 16 * 512),    # one sequence of 103,100 tokens
    (4, "register", 2.9594e11, 8500 * 16 * 512),    # 500 frames x 17 special tokens
    (4, "frame", 2.1771e12, 500 * 1031 * 16 * 512),
]


@pytest.mark.parametrize("idx,mode,flop,nbytes", CASES, ids=[f"w{c[0]}-{c[1]}" for c in CASES])
def test_flop_and_byte_counts(idx, mode, flop, nbytes):
    shape = W.workload(idx).shape
    assert bench.attention_flops(mode, shape) == pytest.approx(flop, rel=2e-4)
    assert bench.io_bytes(mode, shape) == nbytes


def test_frame_flop_is_sum_over_frames_of_one_frame_problem():
    shape = W.workload(4).shape
    one = W.Shape(S=1, T=shape.T, H=shape.H, n_special=shape.n_special, grid_h=shape.grid_h, grid_w=shape.grid_w)
    assert bench.attention_flops("frame", shape) == shape.S * bench.attention_flops("global", one)
