"""The seeded input generator: deterministic, head-separable, bf16-exact."""
import numpy as np
import torch

from dynamic_block_sparse_fractal_b200 import workloads as W


def test_deterministic_and_head_separable():
    w = W.TINY
    a = W.make_inputs(w)
    b = W.make_inputs(w)
    for x, y in zip(a, b):
        assert x.shape == (w.B, w.H, w.S, w.d) and x.dtype == np.uint16
        assert np.array_equal(x, y)
    one = W.make_inputs(w, heads=range(1, 2))
    for x, y in zip(a, one):
        assert np.array_equal(x.reshape(w.BH, w.S, w.d)[1], y[0])


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 7
    x[:4] = [1.00390625, 1.01171875, -2.0039062, 3.0]  # ties and exact values
    ours = W.f32_to_bf16_bits(x)
    theirs = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs)
    assert np.array_equal(W.bf16_bits_to_f32(ours),
                          torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_sweep_variants():
    names = {W.sweep(k).name for k in range(W.N_SWEEP)}
    assert len(names) == W.N_SWEEP == 48
    w = W.sweep(0)
    assert w.thr == 0.0 and w.sta == (0, 0, 0) and w.scale == 0.0


def test_drift_inputs_is_a_small_seeded_bf16_step():
    w = W.TINY
    q, k, v = W.make_inputs(w)
    a = W.drift_inputs(w, (q, k, v), eps=0.05)
    b = W.drift_inputs(w, (q, k, v), eps=0.05)
    for x, y, z in zip((q, k, v), a, b):
        assert y.dtype == np.uint16 and y.shape == x.shape and np.array_equal(y, z)
        dx = W.bf16_bits_to_f32(y) - W.bf16_bits_to_f32(x)
        assert 0.03 < float(np.std(dx)) < 0.07  # eps, plus bf16 rounding of the sum
        assert not np.array_equal(x, y)
