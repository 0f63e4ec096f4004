"""CPU checks of the benchmark's algorithmic work: the FLOP and byte counts
that every reported TFLOP/s and GB/s divide by, recounted by brute force from
the scale geometry and the keep schedule."""
import numpy as np
import pytest

import bench
import oracle
import synth
from synth import SIDES_1024, SIDES_TINY


def _visible_keys_full(sides):
    """Keys a query of each scale sees under full block-causal attention, by
    enumerating every key's scale."""
    g = oracle.ScaleGeometry(sides)
    key_scale = np.concatenate([np.full(g.n[s], s) for s in range(g.S)])
    return [int((key_scale <= k).sum()) for k in range(g.S)]


def _visible_keys_pruned(sides, keep_h, k):
    """Keys a query of scale k of one head sees: its retained past scales plus
    its own scale."""
    g = oracle.ScaleGeometry(sides)
    return sum(g.n[s] for s in range(k) if keep_h[s]) + g.n[k]


@pytest.mark.parametrize("sides,B,H,D", [(SIDES_TINY, 4, 4, 64), (SIDES_1024, 16, 16, 128)])
def test_calibration_flops_count_every_query_key_pair(sides, B, H, D):
    g = oracle.ScaleGeometry(sides)
    vis = _visible_keys_full(sides)
    # QK^T and PV: 2 * D multiply-adds per (query, key) pair, 2 FLOP each
    brute = sum(4 * D * g.n[k] * vis[k] for k in range(g.S)) * B * H
    assert bench.calib_flops(sides, B, H, D) == brute


def test_calibration_flops_per_head_and_seed_at_1024():
    # 35.06 GFLOP per (head, seed) at head_dim 128 for the 1024^2 scale list
    assert abs(bench.calib_flops(SIDES_1024, 1, 1, 128) / 1e9 - 35.06) < 0.01


@pytest.mark.parametrize("sides,L,H,B,D", [(SIDES_TINY, 2, 3, 2, 64), (SIDES_1024, 4, 16, 8, 128)])
def test_pruned_flops_count_retained_keys(sides, L, H, B, D):
    g = oracle.ScaleGeometry(sides)
    keep = np.random.default_rng(L * H).integers(0, 2, size=(L, H, g.S)).astype(np.uint8)
    keep[:, :, :2] = 1
    brute = 0
    for l in range(L):
        for h in range(H):
            for k in range(g.S):
                brute += 4 * D * B * g.n[k] * _visible_keys_pruned(sides, keep[l, h], k)
    assert bench.pruned_flops(keep, sides, B, D) == brute
    # a 100% budget does exactly the full attention's work
    ones = np.ones_like(keep)
    assert bench.pruned_flops(ones, sides, B, D) == bench.calib_flops(sides, B, H, D) * L


def test_compaction_bytes_are_the_kept_rows_read_and_written():
    sides, L, H, B, D = SIDES_1024, 3, 16, 8, 128
    g = oracle.ScaleGeometry(sides)
    w = synth.WORKLOADS["pruned_32l"]
    scas = np.random.default_rng(4).uniform(size=(L, H, g.S))
    keep = oracle.build_schedule(scas, sides, w.budget_bp, w.n_sinks)
    _, _, _, layer_base = oracle.build_offsets(keep, sides, B, D)
    kept_rows = int((keep * np.array(g.n)[None, None, :]).sum()) * B
    # layer_base[L] counts the elements of one of K / V; the benchmark moves
    # that many elements read + written, for K and V, 2 bytes each
    assert int(layer_base[L]) == kept_rows * D
    # the schedule meets the budget it was built for
    assert int((keep * np.array(g.n)[None, None, :]).sum()) * 10000 <= w.budget_bp * L * H * g.T
