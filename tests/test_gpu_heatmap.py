"""Block max-pooled full-attention map (the Veda page's reference target,
section 2.1) on the GPU vs the fp64 oracle, and the recall of the NABLA mask
measured against it.

Tolerance: the kernel forms the scores in fp32 from the same bf16 inputs
(exact products, fp32 sums over d <= 128 terms), takes exp2 with the
hardware approximation or a degree-5 polynomial (relative error <= 2^-22 or
1.5e-7), log2 with the hardware approximation, and sums a row's S terms in
fp32; the heat value 2^(x - lse2) then carries a relative error of order
1e-5 on these workloads. rtol 1e-3 leaves a wide margin while a wrong index,
pairing or reduction shows as an O(1) difference."""
import functools

import numpy as np
import pytest
import torch

import oracle
from dynamic_block_sparse_fractal_b200 import api, workloads as W
from tests.test_gpu_parity import host_inputs, to_dev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

RTOL, ATOL = 1e-3, 1e-9

# odd block counts leave the last q-block of a query tile and the last k-block
# of a key pair alone
CASES = [
    W.TINY,
    W.TINY.with_(name="odd_1x2x576x128", T=3, Hh=8, Ww=24, d=128),
    W.TINY.with_(name="odd_1x1x2880x64_sta", T=5, Hh=24, Ww=24, d=64, H=1, sta=(3, 3, 3)),
    W.W8K_T248.with_(name="tile2x4x8_1x2x4096x128", T=8, Hh=16, Ww=32, H=2),
    # one block per head: a lone q-block in a lone tile, a lone k-block
    W.TINY.with_(name="single_block_1x2x64x128", T=1, Hh=8, Ww=8, d=128),
    # 384 units of four q-blocks on at most 148 CTAs: several units per CTA
    W.TINY.with_(name="multi_1x48x2048x64", T=4, Hh=16, Ww=32, H=48),
]


def gpu_heat_and_mask(w, inputs=None):
    q, k, _ = inputs if inputs is not None else host_inputs(w)
    qd, kd = to_dev(q, w), to_dev(k, w)
    desc = api.desc_for(w)
    ws = api.alloc_workspace(desc)
    heat = api.block_heatmap(desc, qd, kd, ws)
    st = api.check(desc, ws)
    assert st == api.SA_OK, api.status_string(st)
    api.plan(desc, qd, kd, ws)
    views = api.get_mask(desc, ws)
    cnt, idx = views["cnt"].cpu().numpy(), views["idx"].cpu().numpy()
    nb = views["nb"]
    M = np.zeros((w.BH, nb, nb), dtype=bool)
    for bh in range(w.BH):
        for i in range(nb):
            M[bh, i, idx[bh, i, :cnt[bh, i]]] = True
    return heat.cpu().numpy().astype(np.float64), M


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_heatmap_matches_oracle(w):
    H, M = gpu_heat_and_mask(w)
    q, k, _ = host_inputs(w)
    for bh in range(w.BH):
        ref = oracle.block_heatmap(q[bh], k[bh], w.T, w.Hh, w.Ww, w.block, w.N)
        np.testing.assert_allclose(H[bh], ref, rtol=RTOL, atol=ATOL, err_msg=f"head {bh}")
        # the recall of the GPU mask is the same whether measured on the
        # GPU's heat map or on the oracle's
        assert abs(oracle.heat_recall(H[bh], M[bh]) - oracle.heat_recall(ref, M[bh])) < 1e-4


def test_heatmap_uniform_when_queries_are_zero():
    # Zero queries: every probability is 1/S, so is every block maximum
    # (exact in the kernel too: all scores 0, exp2(0) = 1, sum = S).
    w = W.TINY.with_(name="zero_q", T=3, Hh=8, Ww=24, d=128)
    q, k, v = host_inputs(w)
    H, _ = gpu_heat_and_mask(w, inputs=(np.zeros_like(q), k, v))
    np.testing.assert_allclose(H, 1.0 / w.S, rtol=2e-6, atol=0)


@functools.lru_cache(maxsize=1)
def hunyuan_two_heads():
    w = W.HUNYUAN.with_(name="hunyuan_1x2x126720x128", H=2)
    return w, gpu_heat_and_mask(w)


def test_heatmap_full_size_sampled_rows():
    # HunyuanVideo-like grid (126,720 tokens, nb = 1980), two heads: whole
    # rows of the map for a spread of q-blocks, from the oracle's per-row form.
    w, (H, M) = hunyuan_two_heads()
    q, k, _ = host_inputs(w)
    rows = [0, 1, 777, 1500, w.nb - 2, w.nb - 1]
    for bh in range(w.BH):
        ref = oracle.block_heatmap_rows(q[bh], k[bh], w.T, w.Hh, w.Ww, w.block, w.N, rows)
        np.testing.assert_allclose(H[bh, rows], ref, rtol=RTOL, atol=ATOL, err_msg=f"head {bh}")
    # properties at every entry: probabilities, and per q-block the block
    # maxima sum to at least 1/N (the row's probabilities sum to 1)
    assert (H >= 0).all() and (H <= 1).all()
    assert (H.sum(axis=-1) >= (1.0 / w.N) * (1 - 1e-4)).all()
    r = np.mean([oracle.heat_recall(H[bh], M[bh]) for bh in range(w.BH)])
    assert 0.0 < r <= 1.0
