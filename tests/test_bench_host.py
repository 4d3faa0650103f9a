"""Host-side arithmetic of bench.py on CPU: the tile count its byte model
uses agrees with the library's own tile pairing, the plan stages' algorithmic
bytes on a hand-counted grid, and the clock-normalised fraction."""
import pytest

import bench
from dynamic_block_sparse_fractal_b200 import api, workloads as W


@pytest.mark.parametrize("w", list(W.WORKLOADS.values()), ids=list(W.WORKLOADS))
def test_union_tiles_matches_the_library_pairing(w):
    desc = api.desc_for(w)
    n = bench.union_tiles(w)
    api.tile_blocks(desc, n - 1)  # the last tile exists
    with pytest.raises(api.SparseAttnError):
        api.tile_blocks(desc, n)  # and there is no further one


def test_plan_stage_bytes_hand_counted():
    # TINY: 1 x 2 heads, 4 frames of 8 x 8 tokens, d = 64, 8 x 8 patches:
    # nb = 4 blocks per head, 1 bitmap word per row, 2 query tiles per head
    w = W.TINY
    assert (w.BH, w.nb, w.d, w.S) == (2, 4, 64, 256)
    b = bench.plan_stage_bytes(w, kept_pairs=20, union_entries=12)
    pooled = 2 * 2 * 4 * 64 * 4        # Qbar, Kbar (fp32)
    split = 4 * 2 * 4 * 64 * 4         # their tf32 hi and lo
    lists = 2 * 4 * 4 + 20 * 4 + 2 * 4 * 1 * 4
    assert b["pool"] == 2 * 2 * 256 * 64 * 2 + pooled + split
    assert b["logits"] == split + 2 * 4 * 4 * 4
    assert b["select"] == 2 * 4 * 4 * 4 + lists
    assert b["union"] == 2 * 4 * 1 * 4 + 2 * 2 * 4 + 12 * 4
    assert b["tile_order"] == 2 * 2 * 2 * 4


def test_clock_normalised_fraction():
    r = bench.clock_normalised(800.0, 1600.0, {"sm_mhz": 1500.0, "sm_max_mhz": 1950.0})
    assert r["frac_clock_normalised"] == round(800.0 * 1950.0 / 1500.0 / 1600.0, 4)
    assert r["sm_mhz_median"] == 1500.0 and r["sm_max_mhz"] == 1950.0
    assert bench.clock_normalised(800.0, 1600.0, {}) == {"frac_clock_normalised": None}
