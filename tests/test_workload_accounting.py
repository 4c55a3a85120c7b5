"""The work counts behind every bench figure, checked on CPU against the
oracle's own mask: allowed (query, key) pairs per mask and problem; and the
committed DRAM-traffic record the roofline line reports.

With Q = K = 0 every allowed logit is 0, so the oracle's log-sum-exp of a
row is log(number of keys that row may see); summing exp(lse) over all rows
counts the pairs the oracle's predicate allows.
"""
import numpy as np
import pytest

from helpers import orc
from video_dit_windowed_b200.workloads import Workload

# detail grid, cube, global grid
SHAPES = [
    ((4, 8, 8), (2, 4, 4), (2, 4, 4)),
    ((5, 7, 9), (2, 3, 4), (2, 3, 4)),
    ((6, 20, 30), (3, 8, 8), (4, 6, 7)),
    ((4, 8, 8), (2, 4, 4), (3, 10, 5)),
]


def workload(grid, cube, gg):
    return Workload("t", grid, cube, gg, 1, 8, "fp32", (2, 2, 4), (1.0, 1.0, 1.0),
                    (1.0, 1.0, 1.0))


def oracle_pairs(grid, cube, gg, aligned):
    N, G, D = grid[0] * grid[1] * grid[2], gg[0] * gg[1] * gg[2], 8
    z_d, z_g = np.zeros((N, D)), np.zeros((G, D))
    ids = np.arange(N + G, dtype=np.int64)
    q = np.zeros((N + G, D))
    if aligned:
        _, lse = orc().attention_head_aligned(grid, cube, gg, 1.0, z_d, z_d, 0, z_g, z_g, ids, q)
    else:
        from video_dit_windowed_b200 import atlas
        off = atlas.cube_window_offsets(grid, cube).numpy().astype(np.int64)
        _, lse = orc().attention_head(N, 1, G, 1.0, z_d, z_d, 0, z_g, z_g, ids, q, 1, off)
    return int(round(float(np.sum(np.exp(lse)))))


@pytest.mark.parametrize("grid,cube,gg", SHAPES)
@pytest.mark.parametrize("mask", ["all", "aligned"])
def test_allowed_pairs_match_oracle(grid, cube, gg, mask):
    assert workload(grid, cube, gg).allowed_pairs(mask) == \
        oracle_pairs(grid, cube, gg, mask == "aligned")


def test_aligned_boxes_partition_the_global_axes():
    for grid, cube, gg in SHAPES + [((8, 270, 480), (3, 16, 16), (8, 27, 48)),
                                     ((81, 90, 160), (27, 18, 32), (27, 18, 32))]:
        w = workload(grid, cube, gg)
        for a in range(3):
            boxes = w.aligned_boxes(a)
            assert sum(boxes) == gg[a] and min(boxes) >= 0


def test_traffic_record_is_current():
    """The committed ncu traffic record was taken on the attention kernel as
    it stands (bench.py reports it only then), and it is close to the
    algorithmic bytes: Q, K, V read once and O written once."""
    import argparse
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    w = bench.workload(argparse.Namespace(workload="720p", heads=0, shard="replicas"))
    t = bench.measured_traffic(w)
    assert t is not None, "profiles/attn_tc_traffic.txt is stale: capture the kernel again"
    algorithmic = 4 * (w.n_detail + w.n_global) * w.heads * w.head_dim * w.elem_bytes
    assert 0.9 * algorithmic <= t <= 1.1 * algorithmic
