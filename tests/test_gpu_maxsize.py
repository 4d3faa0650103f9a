"""The largest problem the entry points accept: nb = 2880 blocks per head
(20 frames of 96 x 96 tokens, 184,320 tokens; the attention kernel stages a
tile's union list of up to 2880 entries in shared memory, and the select
kernel holds a row of 2880 masses, 90 per lane). One head with the
HunyuanVideo-like recipe: the whole mask against the oracle, sampled output
rows, sampled rows of the block max-pooled map, and sampled blocks of the
gradients."""
import numpy as np
import pytest
import torch

import oracle
from dynamic_block_sparse_fractal_b200 import api, workloads as W
from tests.test_gpu_backward import LSE_ABS, REL_MAX, REL_MEAN, gpu_grads, rel_errors
from tests.test_gpu_parity import check_mask, check_out_sampled, host_inputs, run, to_dev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

W_MAX = W.HUNYUAN.with_(name="max_1x1x184320x128", H=1, T=20, Hh=96, Ww=96)


def test_max_blocks_forward():
    w = W_MAX
    assert w.nb == 2880
    out, gm, *_ = run(w)
    check_mask(w, gm)
    check_out_sampled(w, out, gm, heads=(0,), n_tok=64)


def test_max_blocks_heatmap_rows():
    w = W_MAX
    q, k, _ = host_inputs(w)
    desc = api.desc_for(w)
    ws = api.alloc_workspace(desc)
    heat = api.block_heatmap(desc, to_dev(q, w), to_dev(k, w), ws)
    assert api.check(desc, ws) == api.SA_OK
    rows = [0, 1439, w.nb - 1]
    ref = oracle.block_heatmap_rows(q[0], k[0], w.T, w.Hh, w.Ww, w.block, w.N, rows)
    np.testing.assert_allclose(heat[0, rows].cpu().numpy(), ref, rtol=1e-3, atol=1e-9)


def test_max_blocks_backward_sampled():
    w = W_MAX
    dq, dk, dv, lse, mask, _ = gpu_grads(w, False)
    q, k, v = (x.reshape(w.BH, w.S, w.d) for x in W.make_inputs(w))
    g = W.make_output_grad(w).reshape(w.BH, w.S, w.d)
    perm = oracle.fractal_order(w.T, w.Hh, w.Ww, w.block)
    qbs, kbs, N = [0, 1439, w.nb - 1], [1, 1500, w.nb - 2], w.N
    qp, kp, vp, dop = (oracle.flatten(oracle.widen_bf16(x[0]), perm) for x in (q, k, v, g))
    rq, rk, rv, rl = oracle.masked_attention_backward_blocks(qp, kp, vp, dop, mask[0], N, qbs, kbs)
    got_l = oracle.flatten(lse[0][:, None], perm)[:, 0]
    for i, b in enumerate(qbs):
        assert np.abs(got_l[b * N:(b + 1) * N] - rl[i]).max() < LSE_ABS
    for got, ref, blocks in ((dq, rq, qbs), (dk, rk, kbs), (dv, rv, kbs)):
        gp = oracle.flatten(got[0], perm)
        mx, mean = rel_errors(np.stack([gp[b * N:(b + 1) * N] for b in blocks]), ref)
        assert mx <= REL_MAX[False] and mean <= REL_MEAN[False], (mx, mean)
