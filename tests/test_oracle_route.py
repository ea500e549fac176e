"""Pins of the oracle's expert sort and expert-aligned tile table (CPU only)."""

import json
import os

import numpy as np

import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_tile_table_mlx_pr_4567_worked_example():
    g = json.load(open(os.path.join(GOLD, "p2_tile_example.json")))
    keys = np.repeat(np.arange(len(g["counts"])), g["counts"])
    _, _, offsets = O.sort_by_expert(keys, len(g["counts"]))
    tiles = O.tile_table(offsets, g["bm"])
    assert [list(t) for t in tiles] == g["aligned_tiles"]
    assert len(tiles) == g["aligned_passes"]
    # Independent tiling: cut every bm rows and count the expert passes per tile.
    R = int(offsets[-1])
    indep = []
    for r0 in range(0, R, g["bm"]):
        rows = keys[r0:r0 + g["bm"]]
        indep.append([int((rows == e).sum()) for e in np.unique(rows)])
    assert indep == g["independent_tiles_expert_rows"]
    assert sum(len(t) for t in indep) == g["independent_passes"]


def test_sort_by_expert_matches_brute_force_stable_order():
    rng = np.random.default_rng(1)
    for R, E in [(0, 4), (1, 1), (37, 5), (200, 16), (64, 300)]:
        keys = rng.integers(0, E, size=R)
        order, inv, offsets = O.sort_by_expert(keys, E)
        brute = sorted(range(R), key=lambda r: (keys[r], r))
        assert order.tolist() == brute
        assert np.array_equal(inv[order], np.arange(R))
        assert np.array_equal(order[inv], np.arange(R))
        assert offsets[0] == 0 and offsets[-1] == R
        for e in range(E):
            assert offsets[e + 1] - offsets[e] == int((keys == e).sum())
            assert all(keys[order[p]] == e for p in range(offsets[e], offsets[e + 1]))


def test_tile_table_brute_force_cover_and_alignment():
    rng = np.random.default_rng(2)
    for _ in range(50):
        E = int(rng.integers(1, 12))
        counts = rng.integers(0, 40, size=E) * (rng.random(E) < 0.7)
        keys = np.repeat(np.arange(E), counts)
        _, _, offsets = O.sort_by_expert(keys, E)
        for bm in (1, 8, 16, 128):
            tiles = O.tile_table(offsets, bm)
            covered = np.zeros(len(keys), int)
            for r0, e, valid in tiles:
                assert 1 <= valid <= bm
                assert offsets[e] <= r0 and r0 + valid <= offsets[e + 1]
                covered[r0:r0 + valid] += 1
            assert np.all(covered == 1)
            assert len(tiles) == sum(-(-int(c) // bm) for c in counts)
