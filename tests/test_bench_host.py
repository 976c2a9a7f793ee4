"""Host logic of bench.py: the work models match brute-force counts from the oracle's masks."""
import numpy as np
import pytest

import bench
from oracle import spark_oracle as O


@pytest.mark.parametrize("kind", [O.SLIDING, O.FULL])
@pytest.mark.parametrize("T,pos0,hist", [(1, 0, False), (700, 0, False), (300, 1000, True), (129, 5, True),
                                         (600, 200, False)])
def test_visible_pairs_match_mask_counts(kind, T, pos0, hist):
    qpos = np.arange(pos0, pos0 + T)
    kpos = np.arange(0 if hist else pos0, pos0 + T)
    assert bench.visible_pairs(T, pos0, kind, hist) == int(O.visible(qpos, kpos, kind).sum())


def test_headline_work_numbers():
    # B=4, T=8192: full 2.199 TFLOP, sliding 0.266 TFLOP; the tiny case 8.60 / 6.45 GFLOP
    assert abs(bench.prefill_flops(4, 8192, 0, O.FULL, False) / 1e12 - 2.199) < 0.001
    assert abs(bench.prefill_flops(4, 8192, 0, O.SLIDING, False) / 1e12 - 0.266) < 0.001
    assert abs(bench.prefill_flops(1, 1024, 0, O.FULL, False) / 1e9 - 8.60) < 0.01
    assert abs(bench.prefill_flops(1, 1024, 0, O.SLIDING, False) / 1e9 - 6.45) < 0.01
    # decode: B=64 with 32768 cached + 1 new, per step over 36 layers ~ 80.9 GB
    tot = sum(bench.decode_kv_bytes(64, 32768, O.layer_kind(l)) for l in range(36))
    assert abs(tot / 1e9 - 80.93) < 0.05
    assert bench.decode_kv_bytes(1, 1 << 20 - 0, O.FULL) >= 4 * 2 ** 30


@pytest.mark.parametrize("kind", [O.SLIDING, O.FULL])
@pytest.mark.parametrize("T", [1, 128, 129, 700, 8192])
def test_tile_flops_count_touched_tiles(kind, T):
    """Tile-executed FLOPs: every (128-query tile, 128-key tile) pair that holds a visible pair,
    counted by brute force over the oracle's mask, times 128 x 128 pairs x 4 x 256 FLOP x 16 heads."""
    n_qt = (T + 127) // 128
    touched = 0
    for qt in range(n_qt):
        q = np.arange(qt * 128, min(T, qt * 128 + 128))
        for kt in range(n_qt):
            k = np.arange(kt * 128, min(T, kt * 128 + 128))
            touched += bool(O.visible(q, k, kind).any())
    assert bench.prefill_tile_flops(2, T, kind) == 2 * 16 * touched * 128 * 128 * 4 * 256
    assert bench.prefill_tile_flops(2, T, kind) >= bench.prefill_flops(2, T, 0, kind, False)
