"""3-D tiles on the HunyuanVideo-like grid (tile 1 x 4 x 16) through the C ABI,
two heads: the full mask against the oracle, outputs on sampled rows."""
import dataclasses

import numpy as np
import pytest
import torch

from dynamic_block_sparse_fractal_b200 import workloads as W
from tests import test_gpu_parity as P

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def test_hunyuan_grid_tile_1x4x16_two_heads():
    w = dataclasses.replace(W.HUNYUAN_T1416, H=2, name=W.HUNYUAN_T1416.name + "_heads2")
    out, gm, *_ = P.run(w)
    r = P.check_mask(w, gm)
    assert r["bad"] == 0
    P.check_out_sampled(w, out, gm, heads=range(w.BH), n_tok=96)
    kept = gm.sum() / gm.size
    assert 0.02 < kept < 0.5  # a sparse mask, as with the square patch
