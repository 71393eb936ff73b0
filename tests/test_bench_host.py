"""Host-side pieces of bench.py that need no GPU: the count of distinct
cache rows a launch reads (shared blocks once) and the seeded beam survivors."""
import numpy as np

import bench


def test_unique_kv_bytes_counts_shared_blocks_once():
    bs, Hkv, D = 16, 2, 64
    # two sequences share blocks 7 and 3 (32 tokens), then private suffixes
    tables = np.array([[7, 3, 5, -1], [7, 3, 9, 4]], np.int32)
    lens = np.array([40, 60], np.int32)
    ub = bench.unique_kv_bytes(tables, lens, bs, Hkv, D)
    rows = 16 + 16 + 8 + 16 + 12          # 7, 3 once; 5: 8 rows; 9: 16; 4: 12
    assert ub == rows * Hkv * D * 4
    logical = bench.algorithmic_bytes(lens, 4, Hkv, D, bs, 1)[0]
    assert logical == (40 + 60) * Hkv * D * 4 > ub
    # a block shared with different fill counts once, at its fullest use
    t2 = np.array([[1], [1]], np.int32)
    assert bench.unique_kv_bytes(t2, np.array([5, 11]), bs, 1, 8, k_bytes=1) == 11 * 8 * 3


def test_beam_parents_fork_then_survivors_within_each_prompt():
    S, W = 3, 4
    ps = bench.beam_parents(S, W, 5, seed=11)
    assert ps[0].tolist() == [0] * W + [1] * W + [2] * W
    for p in ps[1:]:
        assert p.shape == (S * W,)
        for g in range(S):
            assert ((p[g * W:(g + 1) * W] // W) == g).all()
    again = bench.beam_parents(S, W, 5, seed=11)
    assert all((a == b).all() for a, b in zip(ps, again))
