"""Token Radius Attention mask (a second mask builder) through the C ABI
against the fp64 oracle (oracle/tra.py): the per-token entropies of the dense
warm-up pass, the block mask from given entropies, its lists in the format the
attention kernel reads, and the forward on it.

Mask tolerance. The kernel takes each keep decision d^2 <= r^2 f(delta) in
fp32 (r^2 from expf and fp32 tables built in fp64), about 5 ulp from the
oracle's fp64 value. A decision is therefore open only where some token's
squared distance lies within RADIUS_BAND (2^-16, relative) of its squared
radius: the GPU mask must contain the oracle's mask at r^2 (1 - band) and be
contained in the one at r^2 (1 + band), and equal the oracle's mask wherever
those two agree. Both sides read the same fp32 entropies, taken from the
oracle and rounded.
"""
import numpy as np
import pytest
import torch

import oracle
from dynamic_block_sparse_fractal_b200 import api, workloads as W
from tests import parity

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

RADIUS_BAND = 2.0 ** -16
ENTROPY_ABS = 2e-4  # nats; fp32 sums over up to 8192 keys and fp32 scores

CASES = [
    # workload, tau, gamma, vote_min
    (W.TINY, 1.0, 0.3, 1),
    (W.W8K.with_(H=4), 2.0, 0.25, 1),
    (W.W8K.with_(H=4), 0.5, 0.0, 8),
    (W.W8K.with_(H=4), 4.0, 0.6, 32),
    (W.W8K_T248.with_(H=2), 2.0, 0.25, 4),
    (W.Workload("radius_ragged", B=2, H=1, d=128, T=5, Hh=16, Ww=24, seed=7), 1.5, 0.4, 2),
]


def to_dev(bits, w):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.reshape(w.B, w.H, w.S, w.d).cuda()


def oracle_entropy(w):
    q, k, _ = (x.reshape(w.BH, w.S, w.d) for x in W.make_inputs(w))
    return np.stack([oracle.token_entropy(q[bh], k[bh]) for bh in range(w.BH)])


def gpu_radius_mask(w, H32, tau, gamma, vmin):
    desc = api.desc_for(w)
    ws = api.alloc_workspace(desc)
    ent = torch.from_numpy(H32.reshape(w.B, w.H, w.S)).cuda()
    api.plan_radius(desc, tau, gamma, vmin, ent, ws)
    assert api.check(desc, ws) == api.SA_OK
    views = api.get_mask(desc, ws)
    gm = parity.lists_to_mask(views["cnt"].cpu().numpy(), views["idx"].cpu().numpy())
    return gm, views, desc, ws


def check_radius_mask(w, gm, H32, tau, gamma, vmin, band=RADIUS_BAND):
    flips = 0
    for bh in range(w.BH):
        H = H32[bh].astype(np.float64)
        M, _, r2 = oracle.tra_mask(H, w.T, w.Hh, w.Ww, w.block, w.N, tau, gamma, vmin)
        lo, _ = oracle.radius_block_mask(r2 * (1 - band), w.T, w.Hh, w.Ww, w.block, w.N,
                                         gamma, vmin)
        hi, _ = oracle.radius_block_mask(r2 * (1 + band), w.T, w.Hh, w.Ww, w.block, w.N,
                                         gamma, vmin)
        g = gm[bh]
        assert not (lo & ~g).any() and not (g & ~hi).any(), bh
        sure = lo == hi
        assert np.array_equal(g[sure], M[sure]), bh
        flips += int((g != M).sum())
        assert np.diag(g).all()  # every q-block keeps its own block
    return flips


@pytest.mark.parametrize("w,tau,gamma,vmin", CASES,
                         ids=[f"{c[0].name}_tau{c[1]}_g{c[2]}_v{c[3]}" for c in CASES])
def test_radius_mask_matches_oracle(w, tau, gamma, vmin):
    H32 = oracle_entropy(w).astype(np.float32)
    gm, views, desc, _ = gpu_radius_mask(w, H32, tau, gamma, vmin)
    flips = check_radius_mask(w, gm, H32, tau, gamma, vmin)
    print(f"{w.name} tau {tau} gamma {gamma} vote_min {vmin}: density {gm.mean():.4f}, "
          f"band flips {flips}")
    # the tile unions hold exactly the two q-blocks' kept blocks
    tc, ti = views["tile_cnt"].cpu().numpy(), views["tile_idx"].cpu().numpy()
    for bh in range(w.BH):
        for t in range(views["ntile"]):
            qa, qb = api.tile_blocks(desc, t)
            want = gm[bh, qa] | (gm[bh, qb] if qb >= 0 else False)
            ent = ti[bh, t, :tc[bh, t]]
            assert np.array_equal(np.sort(ent & 0xFFFF), np.nonzero(want)[0])


@pytest.mark.parametrize("w", [W.TINY, W.W8K.with_(H=4), W.W8K_T248.with_(H=2),
                               CASES[-1][0]], ids=lambda w: w.name)
def test_token_entropy_matches_oracle(w):
    q, k, _ = W.make_inputs(w)
    desc = api.desc_for(w)
    ws = api.alloc_workspace(desc)
    H = api.token_entropy(desc, to_dev(q, w), to_dev(k, w), ws)
    assert api.check(desc, ws) == api.SA_OK
    got = H.cpu().numpy().reshape(w.BH, w.S).astype(np.float64)
    ref = oracle_entropy(w)
    err = np.abs(got - ref)
    print(f"{w.name} entropy: max abs err {err.max():.3e}, range [{ref.min():.3f}, "
          f"{ref.max():.3f}] (ln S = {np.log(w.S):.3f})")
    assert err.max() <= ENTROPY_ABS


def test_forward_on_radius_mask_matches_oracle():
    w = W.W8K.with_(H=4)
    tau, gamma, vmin = 2.0, 0.25, 1
    H32 = oracle_entropy(w).astype(np.float32)
    gm, _, desc, ws = gpu_radius_mask(w, H32, tau, gamma, vmin)
    q, k, v = W.make_inputs(w)
    out = torch.empty((w.B, w.H, w.S, w.d), dtype=torch.bfloat16, device="cuda")
    api.fwd(desc, to_dev(q, w), to_dev(k, w), to_dev(v, w), ws, out)
    assert api.check(desc, ws) == api.SA_OK
    shape = (w.BH, w.S, w.d)
    ref, _ = oracle.nabla_attention(q.reshape(shape), k.reshape(shape), v.reshape(shape), w.T,
                                    w.Hh, w.Ww, w.block, w.N, w.thr, w.sta, mask=gm)
    r = parity.out_check(out.float().cpu().numpy().reshape(shape), ref, True)
    assert r["ok"], r


def test_radius_mask_from_gpu_entropy_is_stable_across_steps():
    # The page computes the entropies once, in the warm-up, and reuses them
    # at later steps: a plan from the GPU's own entropies, then the forward
    # of a drifted next step on that plan, against the oracle on that mask.
    w = W.W8K.with_(H=2)
    q, k, v = W.make_inputs(w)
    desc = api.desc_for(w)
    ws = api.alloc_workspace(desc)
    H = api.token_entropy(desc, to_dev(q, w), to_dev(k, w), ws)
    api.plan_radius(desc, 2.0, 0.25, 1, H, ws)
    views = api.get_mask(desc, ws)
    gm = parity.lists_to_mask(views["cnt"].cpu().numpy(), views["idx"].cpu().numpy())
    # against the oracle's own entropies: r^2 is proportional to exp(H), so an
    # entropy error of ENTROPY_ABS moves r^2 by that much, relatively
    check_radius_mask(w, gm, oracle_entropy(w).astype(np.float32), 2.0, 0.25, 1,
                      band=RADIUS_BAND + 2 * ENTROPY_ABS)
    q2, k2, v2 = W.drift_inputs(w, (q, k, v), eps=0.05)
    out = torch.empty((w.B, w.H, w.S, w.d), dtype=torch.bfloat16, device="cuda")
    api.fwd(desc, to_dev(q2, w), to_dev(k2, w), to_dev(v2, w), ws, out)
    assert api.check(desc, ws) == api.SA_OK
    shape = (w.BH, w.S, w.d)
    ref, _ = oracle.nabla_attention(q2.reshape(shape), k2.reshape(shape), v2.reshape(shape), w.T,
                                    w.Hh, w.Ww, w.block, w.N, w.thr, w.sta, mask=gm)
    r = parity.out_check(out.float().cpu().numpy().reshape(shape), ref, True)
    assert r["ok"], r
    assert 0.0 < gm.mean() < 1.0
