"""The largest problems: nb = 2880 blocks per head (20 frames of 96 x 96,
184,320 tokens: the most union entries a tile stages in shared memory) and
nb = 5760 (40 frames of 96 x 96, 368,640 tokens, beyond the Veda page's
245K-token measurement): there the select kernel holds a row's 5760 masses in
shared memory, and in the dense case every union list (5760 entries) runs past
the 2880 staged entries into global memory, in the attention and the gradient
kernels. One head of the HunyuanVideo-like recipe each: whole masks, whole
q-blocks of the output, sampled map rows and sampled gradient blocks against
the oracle."""
import numpy as np
import pytest
import torch

import oracle
from dynamic_block_sparse_fractal_b200 import api, workloads as W
from tests import parity
from tests.test_gpu_backward import LSE_ABS, REL_MAX, REL_MEAN, gpu_grads, rel_errors
from tests.test_gpu_parity import (check_mask, check_out_qblocks, check_out_sampled, host_inputs,
                                   run, to_dev)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

W_2880 = W.HUNYUAN.with_(name="max_1x1x184320x128", H=1, T=20, Hh=96, Ww=96)
W_5760 = W.HUNYUAN.with_(name="big_1x1x368640x128", H=1, T=40, Hh=96, Ww=96)


def test_2880_blocks_forward():
    w = W_2880
    assert w.nb == 2880
    out, gm, views, desc, _ = run(w)
    check_mask(w, gm)
    check_out_qblocks(w, out, gm, views, desc, heads=(0,), per_head=16)


def test_2880_blocks_heatmap_rows():
    w = W_2880
    q, k, _ = host_inputs(w)
    desc = api.desc_for(w)
    ws = api.alloc_workspace(desc)
    heat = api.block_heatmap(desc, to_dev(q, w), to_dev(k, w), ws)
    assert api.check(desc, ws) == api.SA_OK
    rows = [0, 1439, w.nb - 1]
    ref = oracle.block_heatmap_rows(q[0], k[0], w.T, w.Hh, w.Ww, w.block, w.N, rows)
    np.testing.assert_allclose(heat[0, rows].cpu().numpy(), ref, rtol=1e-3, atol=1e-9)


def test_2880_blocks_backward_sampled():
    w = W_2880
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


def test_2880_blocks_dense_matches_sdpa():
    w = W_2880.with_(thr=0.0)
    out, gm, *_ = run(w, out_fp32=True)
    assert gm.all()
    q, k, v = (to_dev(x, w) for x in host_inputs(w))
    # fp32 SDPA on the same bf16 values (torch's own kernel, as a second anchor)
    ref = torch.nn.functional.scaled_dot_product_attention(q.float(), k.float(), v.float())
    r = parity.out_check(out, ref.cpu().numpy().reshape(w.BH, w.S, w.d).astype(np.float64), False)
    assert r["ok"], r
    check_out_sampled(w, out, gm, heads=(0,), bf16_out=False)


def test_5760_blocks_forward():
    w = W_5760
    assert w.nb == 5760
    out, gm, views, desc, _ = run(w)
    r = check_mask(w, gm)
    assert r["density"] < 0.2, r
    check_out_qblocks(w, out, gm, views, desc, heads=(0,), per_head=12)


def test_5760_blocks_dense_lists_past_the_staged_entries():
    # thr = 0: every union list holds all 5760 blocks, so the attention kernel
    # reads entries 2880.. from global memory
    w = W_5760.with_(thr=0.0)
    out, gm, views, desc, _ = run(w, out_fp32=True)
    assert gm.all() and int(views["tile_cnt"].min()) == w.nb
    check_out_qblocks(w, out, gm, views, desc, heads=(0,), per_head=4, bf16_out=False)
    q, k, v = (to_dev(x, w) for x in host_inputs(w))
    ref = torch.nn.functional.scaled_dot_product_attention(q.float(), k.float(), v.float())
    r = parity.out_check(out, ref.cpu().numpy().reshape(w.BH, w.S, w.d).astype(np.float64), False)
    assert r["ok"], r


@pytest.mark.parametrize("thr", [0.1, 0.0], ids=["sparse", "dense"])
def test_5760_blocks_backward_sampled(thr):
    # dense: the gradient kernel's key-tile lists (5760 q-blocks) also run
    # past the staged entries
    w = W_5760.with_(thr=thr)
    dq, dk, dv, lse, mask, _ = gpu_grads(w, False)
    q, k, v = (x.reshape(w.BH, w.S, w.d) for x in W.make_inputs(w))
    g = W.make_output_grad(w).reshape(w.BH, w.S, w.d)
    perm = oracle.fractal_order(w.T, w.Hh, w.Ww, w.block)
    N = w.N
    qbs, kbs = ([0, 2881, w.nb - 1], [2900]) if thr > 0 else ([3001], [])
    qp, kp, vp, dop = (oracle.flatten(oracle.widen_bf16(x[0]), perm) for x in (q, k, v, g))
    rq, rk, rv, rl = oracle.masked_attention_backward_blocks(qp, kp, vp, dop, mask[0], N, qbs, kbs)
    got_l = oracle.flatten(lse[0][:, None], perm)[:, 0]
    for i, b in enumerate(qbs):
        assert np.abs(got_l[b * N:(b + 1) * N] - rl[i]).max() < LSE_ABS
    pairs = [(dq, rq, qbs)] + ([(dk, rk, kbs), (dv, rv, kbs)] if kbs else [])
    for got, ref, blocks in pairs:
        gp = oracle.flatten(got[0], perm)
        mx, mean = rel_errors(np.stack([gp[b * N:(b + 1) * N] for b in blocks]), ref)
        print(f"{w.name} thr {thr}: max {mx:.2e} mean {mean:.2e}")
        assert mx <= REL_MAX[False] and mean <= REL_MEAN[False], (mx, mean)
