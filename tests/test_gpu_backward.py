"""Gradients of the block-sparse attention (through the C ABI) against the
fp64 oracle, on the GPU's own mask, and the row log-sum-exp of the forward.

Tolerances. The kernel recomputes P = 2^(s log2(e) - lse2) in fp32, rounds P
and dS = P (dP - D) to bf16 for the tensor cores (relative 2^-9 each) and
accumulates in fp32; D = rowsum(dO * O) uses the forward's output as stored
(bf16 unless out_fp32). Errors are measured relative to the largest reference
magnitude of each gradient: max |g - ref| <= REL_MAX * max |ref| and
mean |g - ref| <= REL_MEAN * mean |ref|. dQ and dK are the loosest: a row's dS
sums to about zero (sum_j P (dP - D) = 0), so the bf16 rounding of its terms
is large next to the sums they form. Seen on the multi-block cases: max
1.2e-2 (dQ), mean 6.0e-3 with bf16 outputs and 2.9e-3 with fp32 outputs; the
bounds leave a factor of about 2.

The stored output. Rounding O to bf16 moves it by up to 2^-9 |O|, so D moves
by up to 2^-9 sum_c |dO_c O_c|, and every dS_ij of the row by P_ij times that
shift. With many kept keys per row dP - D is large next to the shift; with a
single 64-key block per row (the one-block case) the row's 64 terms of dP - D
cancel to within a few times the shift, which is where the bf16 case's dQ
mean error of 1.27e-2 comes from (2.0e-3 with fp32 outputs). That case alone
is held to SINGLE_BLOCK_REL_MEAN_BF16. The error source is also isolated:
fed the GPU's own stored bf16 output for D (oracle o_stored), the oracle must
agree with every bf16 case to the fp32-output bounds.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
from dynamic_block_sparse_fractal_b200 import api, workloads as W
from tests import parity

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

REL_MAX = {False: 2.5e-2, True: 2.5e-2}    # keyed by out_fp32
REL_MEAN = {False: 1.2e-2, True: 6e-3}
SINGLE_BLOCK_REL_MEAN_BF16 = 2e-2          # one 64-key block per row, bf16 output
LSE_ABS = 1e-4

CASES = [
    W.TINY,
    W.TINY.with_(name="odd_1x2x576x128", T=3, Hh=8, Ww=24, d=128),
    W.W8K_T248.with_(name="tile2x4x8_1x2x4096x128", T=8, Hh=16, Ww=32, H=2),
    W.W8K.with_(name="8k_1x2x8192x128_sta3", H=2),
    # one block per head: a lone key tile with a one-entry list (a lone step)
    W.TINY.with_(name="single_block_1x2x64x128", T=1, Hh=8, Ww=8, d=128),
]


def to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@functools.lru_cache(maxsize=4)
def gpu_grads(w, out_fp32):
    q, k, v = W.make_inputs(w)
    g = W.make_output_grad(w)
    qd, kd, vd, gd = (to_dev(x) for x in (q, k, v, g))
    desc = api.desc_for(w, out_fp32=out_fp32)
    ws = api.alloc_workspace(desc)
    api.plan(desc, qd, kd, ws)
    out = torch.empty(qd.shape, device="cuda",
                      dtype=torch.float32 if out_fp32 else torch.bfloat16)
    lse = torch.empty(qd.shape[:3], dtype=torch.float32, device="cuda")
    api.fwd_lse(desc, qd, kd, vd, ws, out, lse)
    dq, dk, dv = api.bwd(desc, qd, kd, vd, out, gd, lse, ws)
    st = api.check(desc, ws)
    assert st == api.SA_OK, api.status_string(st)
    views = api.get_mask(desc, ws)
    mask = parity.lists_to_mask(views["cnt"].cpu().numpy(), views["idx"].cpu().numpy())
    host = lambda t: t.float().cpu().numpy().reshape(w.BH, w.S, w.d)
    return (host(dq), host(dk), host(dv), lse.cpu().numpy().reshape(w.BH, w.S), mask,
            host(out))


def rel_errors(got, ref):
    e = np.abs(got - ref)
    return e.max() / np.abs(ref).max(), e.mean() / np.abs(ref).mean()


def mean_bound(w, out_fp32):
    if not out_fp32 and w.nb == 1:
        return SINGLE_BLOCK_REL_MEAN_BF16
    return REL_MEAN[out_fp32]


@pytest.mark.parametrize("out_fp32", [False, True])
@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_backward_matches_oracle(w, out_fp32):
    dq, dk, dv, lse, mask, _ = gpu_grads(w, out_fp32)
    q, k, v = (x.reshape(w.BH, w.S, w.d) for x in W.make_inputs(w))
    g = W.make_output_grad(w).reshape(w.BH, w.S, w.d)
    for bh in range(w.BH):
        rq, rk, rv, rl = oracle.attention_backward_head(q[bh], k[bh], v[bh], g[bh], w.T, w.Hh,
                                                        w.Ww, w.block, w.N, mask[bh])
        assert np.abs(lse[bh] - rl).max() < LSE_ABS
        for name, got, ref in (("dq", dq[bh], rq), ("dk", dk[bh], rk), ("dv", dv[bh], rv)):
            mx, mean = rel_errors(got, ref)
            print(f"{w.name} fp32={out_fp32} head {bh} {name}: max {mx:.2e} mean {mean:.2e}")
            assert mx <= REL_MAX[out_fp32], (name, bh, mx)
            assert mean <= mean_bound(w, out_fp32), (name, bh, mean)


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_backward_bf16_output_with_stored_D_meets_fp32_bounds(w):
    # The same bf16-output gradients against the oracle whose D reads the
    # GPU's stored bf16 output: with the one error source the bf16 output adds
    # taken into the reference, the fp32-output bounds hold for every case.
    dq, dk, dv, _, mask, out = gpu_grads(w, False)
    q, k, v = (x.reshape(w.BH, w.S, w.d) for x in W.make_inputs(w))
    g = W.make_output_grad(w).reshape(w.BH, w.S, w.d)
    for bh in range(w.BH):
        rq, rk, rv, _ = oracle.attention_backward_head(q[bh], k[bh], v[bh], g[bh], w.T, w.Hh,
                                                       w.Ww, w.block, w.N, mask[bh],
                                                       o_stored=out[bh])
        for name, got, ref in (("dq", dq[bh], rq), ("dk", dk[bh], rk), ("dv", dv[bh], rv)):
            mx, mean = rel_errors(got, ref)
            print(f"{w.name} stored-O head {bh} {name}: max {mx:.2e} mean {mean:.2e}")
            assert mx <= REL_MAX[True], (name, bh, mx)
            assert mean <= REL_MEAN[True], (name, bh, mean)


def test_backward_full_size_sampled_blocks():
    # HunyuanVideo-like grid (126,720 tokens, nb = 1980), two heads, bf16 as in
    # the benchmark: dQ and the log-sum-exp of three q-blocks and dK, dV of
    # three k-blocks per head, from the oracle's per-block form.
    w = W.HUNYUAN.with_(name="hunyuan_1x2x126720x128", H=2)
    dq, dk, dv, lse, mask, _ = gpu_grads(w, False)
    q, k, v = (x.reshape(w.BH, w.S, w.d) for x in W.make_inputs(w))
    g = W.make_output_grad(w).reshape(w.BH, w.S, w.d)
    perm = oracle.fractal_order(w.T, w.Hh, w.Ww, w.block)
    qbs, kbs = [0, 777, w.nb - 1], [1, 990, w.nb - 2]
    N = w.N
    for bh in range(w.BH):
        qp, kp, vp, dop = (oracle.flatten(oracle.widen_bf16(x[bh]), perm) for x in (q, k, v, g))
        rq, rk, rv, rl = oracle.masked_attention_backward_blocks(qp, kp, vp, dop, mask[bh], N,
                                                                 qbs, kbs)
        got_q, got_k, got_v = (oracle.flatten(x[bh], perm) for x in (dq, dk, dv))
        got_l = oracle.flatten(lse[bh][:, None], perm)[:, 0]
        for i, b in enumerate(qbs):
            assert np.abs(got_l[b * N:(b + 1) * N] - rl[i]).max() < LSE_ABS
        for name, got, ref, blocks in (("dq", got_q, rq, qbs), ("dk", got_k, rk, kbs),
                                       ("dv", got_v, rv, kbs)):
            sample = np.stack([got[b * N:(b + 1) * N] for b in blocks])
            mx, mean = rel_errors(sample, ref)
            print(f"{w.name} head {bh} {name}: max {mx:.2e} mean {mean:.2e}")
            assert mx <= REL_MAX[False], (name, bh, mx)
            assert mean <= REL_MEAN[False], (name, bh, mean)


def test_nabla_attention_methods_match_functional_calls():
    w = W.TINY
    q, k, v = (to_dev(x) for x in W.make_inputs(w))
    g = to_dev(W.make_output_grad(w))
    attn = api.NablaAttention(w.B, w.H, w.T, w.Hh, w.Ww, w.d, w.thr, w.sta, out_fp32=True)
    attn.plan(q, k)
    out, lse = attn.forward_lse(q, k, v)
    grads = attn.backward(q, k, v, out, g, lse)
    heat = attn.heatmap(q, k)
    assert attn.check() == api.SA_OK
    desc = api.desc_for(w, out_fp32=True)
    ws = api.alloc_workspace(desc)
    api.plan(desc, q, k, ws)
    out2 = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    lse2 = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    api.fwd_lse(desc, q, k, v, ws, out2, lse2)
    grads2 = api.bwd(desc, q, k, v, out2, g, lse2, ws)
    heat2 = api.block_heatmap(desc, q, k, ws)
    assert api.check(desc, ws) == api.SA_OK
    assert torch.equal(out, out2) and torch.equal(lse, lse2) and torch.equal(heat, heat2)
    for a, b in zip(grads, grads2):  # fp32 reductions in any order: equal to rounding
        assert torch.allclose(a, b, rtol=1e-5, atol=1e-6)


def test_per_head_shapes_gradients_and_map_match_single_shape_runs():
    w = W.W8K  # 12 heads
    tiles = [(1, 8, 8)] * 4 + [(2, 4, 8)] * 4 + [(4, 4, 4)] * 2 + [(2, 4, 8)] * 2
    desc = api.desc_for(w, out_fp32=True)
    q, k, v = (to_dev(x) for x in W.make_inputs(w))
    g = to_dev(W.make_output_grad(w))
    ws = torch.empty(api.workspace_size_heads(desc, tiles), dtype=torch.uint8, device="cuda")
    api.plan_heads(desc, tiles, q, k, ws)
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    api.fwd_lse_heads(desc, tiles, q, k, v, ws, out, lse)
    grads = api.bwd_heads(desc, tiles, q, k, v, out, g, lse, ws)
    heat = api.block_heatmap_heads(desc, tiles, q, k, ws)
    assert api.check_heads(desc, tiles, ws) == api.SA_OK
    for sub, head0, _, _ in api.heads_runs(desc, tiles):
        sl = slice(head0, head0 + sub.H)
        qs, ks, vs, gs = (x[:, sl].contiguous() for x in (q, k, v, g))
        ws1 = api.alloc_workspace(sub)
        api.plan(sub, qs, ks, ws1)
        o1 = torch.empty(qs.shape, dtype=torch.float32, device="cuda")
        l1 = torch.empty(qs.shape[:3], dtype=torch.float32, device="cuda")
        api.fwd_lse(sub, qs, ks, vs, ws1, o1, l1)
        g1 = api.bwd(sub, qs, ks, vs, o1, gs, l1, ws1)
        h1 = api.block_heatmap(sub, qs, ks, ws1)
        assert api.check(sub, ws1) == api.SA_OK
        assert torch.equal(out[:, sl], o1) and torch.equal(lse[:, sl], l1)
        assert torch.equal(heat[sl], h1)
        for a, b in zip(grads, g1):  # fp32 reductions in any order: equal to rounding
            assert torch.allclose(a[:, sl], b, rtol=1e-5, atol=1e-6)
