"""Pins for the fp64 CPU oracle, independent of the oracle's own code.

Each check fixes a part of the oracle against something other than itself:
hand-worked fixtures (tests/golden), closed forms, brute-force enumeration,
and special cases that reduce to a library routine (torch SDPA in fp64).
The mutation tests at the end plant plausible mistakes in the oracle and
confirm that some pin catches each of them.
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import nabla
from dynamic_block_sparse_fractal_b200 import workloads as W


# --- fixture readers ---------------------------------------------------------

def _rows(path):
    with open(path) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


def golden_orders(golden_dir):
    out = []
    for ln in _rows(os.path.join(golden_dir, "fractal_order.txt")):
        dims, perm = ln.split(":")
        out.append((tuple(int(x) for x in dims.split()), [int(x) for x in perm.split()]))
    return out


def golden_cdf(golden_dir):
    out = []
    for ln in _rows(os.path.join(golden_dir, "cdf_rows.txt")):
        thr, row, keep = ln.split(":")
        out.append((float(thr), np.array([float(x) for x in row.split()]),
                    np.array([bool(int(x)) for x in keep.split()])))
    return out


# --- pin functions (reused by the mutation tests) ----------------------------

def pin_fractal_golden(golden_dir):
    for (T, Hh, Ww, P), perm in golden_orders(golden_dir):
        assert oracle.fractal_order(T, Hh, Ww, P).tolist() == perm


def pin_fractal_reshape(T=3, Hh=16, Ww=24, P=8):
    # Independent construction: view the natural-order index grid as
    # [T, Hh/P, P, Ww/P, P] and move the two in-patch axes innermost.
    idx = np.arange(T * Hh * Ww).reshape(T, Hh // P, P, Ww // P, P)
    expect = idx.transpose(0, 1, 3, 2, 4).reshape(-1)
    assert np.array_equal(oracle.fractal_order(T, Hh, Ww, P), expect)


def pin_cdf_golden(golden_dir):
    for thr, row, keep in golden_cdf(golden_dir):
        assert np.array_equal(oracle.cdf_keep(row[None], thr)[0], keep), (thr, row)


def pin_cdf_bruteforce(seed=7, rows=60):
    rng = np.random.default_rng(seed)
    for r in range(rows):
        n = int(rng.integers(2, 11))
        a = rng.dirichlet(np.full(n, 0.6))
        thr = float(rng.choice([0.01, 0.05, 0.1, 0.2, 0.3, 0.5]))
        keep = oracle.cdf_keep(a[None], thr)[0]
        target = 1.0 - thr
        best_k, best_mass = None, -1.0
        for k in range(1, n + 1):
            masses = [sum(a[list(c)]) for c in itertools.combinations(range(n), k)]
            if max(masses) >= target:
                best_k, best_mass = k, max(masses)
                break
        assert best_k is not None
        assert keep.sum() == best_k, (a, thr, keep)
        assert abs(a[keep].sum() - best_mass) < 1e-12


def pin_reduced_closed_form():
    # Two key blocks, d = 4: logits are (q.k0, q.k1)/sqrt(4) = (1, 0), so the
    # row is the logistic pair (e/(e+1), 1/(e+1)).
    q = np.array([[2.0, 0.0, 0.0, 0.0]])
    k = np.array([[1.0, 0.0, 0.0, 0.0], [0.0, 0.0, 0.0, 0.0]])
    A = oracle.reduced_map(q, k)
    e = math.e
    assert np.allclose(A, [[e / (e + 1), 1 / (e + 1)]], rtol=0, atol=1e-15)


def pin_sta_golden(golden_dir):
    expect = np.loadtxt(os.path.join(golden_dir, "sta_T2_H1_W3_win1x1x3.txt"),
                        comments="#").astype(bool)
    got = oracle.sta_keep(2, 8, 24, 8, (1, 1, 3))
    assert np.array_equal(got, expect)


def _sdpa64(q, k, v):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v)).numpy()


def _small_problem(seed=3, T=2, Hh=16, Ww=16, P=8, d=32, BH=2):
    rng = np.random.default_rng(seed)
    S = T * Hh * Ww
    q, k, v = (rng.standard_normal((BH, S, d)) for _ in range(3))
    return q, k, v, (T, Hh, Ww, P, P * P)


def pin_attention_dense_is_sdpa():
    q, k, v, (T, Hh, Ww, P, N) = _small_problem()
    out, mask = oracle.nabla_attention(q, k, v, T, Hh, Ww, P, N, 0.0, (0, 0, 0))
    assert mask.all()
    assert np.abs(out - _sdpa64(q, k, v)).max() < 1e-10


def pin_attention_own_patch():
    # Keep only the diagonal block: each query attends its own P x P patch of
    # its own frame, gathered here straight from the natural layout.
    q, k, v, (T, Hh, Ww, P, N) = _small_problem(seed=5)
    BH, S, d = q.shape
    nb = S // N
    mask = np.broadcast_to(np.eye(nb, dtype=bool), (BH, nb, nb)).copy()
    out, _ = oracle.nabla_attention(q, k, v, T, Hh, Ww, P, N, 0.3, (0, 0, 0), mask=mask)

    def patches(x):
        g = x.reshape(BH, T, Hh // P, P, Ww // P, P, d).transpose(0, 1, 2, 4, 3, 5, 6)
        return g.reshape(BH, -1, P * P, d)

    ref = _sdpa64(patches(q), patches(k), patches(v))  # [BH, nb, N, d]
    ref = ref.reshape(BH, T, Hh // P, Ww // P, P, P, d).transpose(0, 1, 2, 4, 3, 5, 6)
    assert np.abs(out - ref.reshape(BH, S, d)).max() < 1e-10


# --- the pins as tests -------------------------------------------------------

def pin_fractal_reshape_3d(T=4, Hh=8, Ww=16, tile=(2, 4, 8)):
    # Independent construction for a p_t x p_h x p_w tile: view the natural
    # index grid as [T/pt, pt, Hh/ph, ph, Ww/pw, pw] and move the three
    # in-tile axes innermost, in (t, h, w) order.
    pt, ph, pw = tile
    idx = np.arange(T * Hh * Ww).reshape(T // pt, pt, Hh // ph, ph, Ww // pw, pw)
    expect = idx.transpose(0, 2, 4, 1, 3, 5).reshape(-1)
    assert np.array_equal(oracle.fractal_order(T, Hh, Ww, tile), expect)


def test_fractal_order_golden(golden_dir):
    pin_fractal_golden(golden_dir)


def test_fractal_order_matches_reshape():
    pin_fractal_reshape()
    pin_fractal_reshape(T=1, Hh=8, Ww=8, P=8)
    pin_fractal_reshape(T=2, Hh=12, Ww=6, P=2)


def test_fractal_round_trip_and_patches():
    T, Hh, Ww, P = 3, 16, 24, 8
    perm = oracle.fractal_order(T, Hh, Ww, P)
    assert np.array_equal(np.sort(perm), np.arange(T * Hh * Ww))
    x = np.random.default_rng(0).standard_normal((2, T * Hh * Ww, 5))
    assert np.array_equal(oracle.unflatten(oracle.flatten(x, perm), perm), x)
    # every run of P*P positions is one patch of one frame
    t, h, w = perm // (Hh * Ww), (perm // Ww) % Hh, perm % Ww
    for b in range(perm.size // (P * P)):
        sl = slice(b * P * P, (b + 1) * P * P)
        assert len(set(t[sl])) == 1 and len(set(h[sl] // P)) == 1 and len(set(w[sl] // P)) == 1
        assert len(set(zip(h[sl], w[sl]))) == P * P
    assert np.array_equal(t, np.sort(t))  # time stays ordered


def test_fractal_order_3d_tiles_match_reshape():
    pin_fractal_reshape_3d()
    pin_fractal_reshape_3d(T=8, Hh=16, Ww=16, tile=(4, 4, 4))
    pin_fractal_reshape_3d(T=3, Hh=8, Ww=32, tile=(1, 4, 16))
    # the square patch of one frame is the tile (1, P, P)
    assert np.array_equal(oracle.fractal_order(3, 16, 24, (1, 8, 8)),
                          oracle.fractal_order(3, 16, 24, 8))


def test_fractal_3d_round_trip_and_tiles():
    T, Hh, Ww, tile = 8, 8, 16, (2, 4, 8)
    pt, ph, pw = tile
    n = pt * ph * pw
    perm = oracle.fractal_order(T, Hh, Ww, tile)
    assert np.array_equal(np.sort(perm), np.arange(T * Hh * Ww))
    t, h, w = perm // (Hh * Ww), (perm // Ww) % Hh, perm % Ww
    coords = oracle.block_coords(T, Hh, Ww, tile)
    for b in range(perm.size // n):
        sl = slice(b * n, (b + 1) * n)
        # each run of N positions is exactly one p_t x p_h x p_w tile ...
        assert set(zip(t[sl], h[sl], w[sl])) == {
            (coords[b, 0] * pt + i, coords[b, 1] * ph + j, coords[b, 2] * pw + k)
            for i in range(pt) for j in range(ph) for k in range(pw)}
    # ... and block coordinates ascend in (t, h, w) block order
    nt, nh, nw = T // pt, Hh // ph, Ww // pw
    assert [tuple(c) for c in coords] == [(a, b, c) for a in range(nt) for b in range(nh)
                                          for c in range(nw)]


def test_sta_3d_tiles_loop():
    T, Hh, Ww, tile, win = 8, 8, 16, (2, 4, 4), (3, 1, 3)
    pt, ph, pw = tile
    nt, nh, nw = T // pt, Hh // ph, Ww // pw
    got = oracle.sta_keep(T, Hh, Ww, tile, win)
    expect = np.zeros((nt * nh * nw,) * 2, dtype=bool)
    for t1, h1, w1 in itertools.product(range(nt), range(nh), range(nw)):
        for t2, h2, w2 in itertools.product(range(nt), range(nh), range(nw)):
            if abs(t1 - t2) <= 1 and h1 == h2 and abs(w1 - w2) <= 1:
                expect[(t1 * nh + h1) * nw + w1, (t2 * nh + h2) * nw + w2] = True
    assert np.array_equal(got, expect)


def pin_attention_own_tile_3d():
    # One kept block per row (the query's own tile): each output is plain
    # attention over the tokens of the query's p_t x p_h x p_w tile, computed
    # here from token coordinates alone.
    rng = np.random.default_rng(23)
    T, Hh, Ww, tile = 4, 8, 8, (2, 4, 8)
    pt, ph, pw = tile
    S, d = T * Hh * Ww, 8
    q, k, v = (rng.standard_normal((S, d)) for _ in range(3))
    nb = S // (pt * ph * pw)
    out = oracle.attention_head(q, k, v, T, Hh, Ww, tile, pt * ph * pw, np.eye(nb, dtype=bool))
    t, h, w = np.arange(S) // (Hh * Ww), (np.arange(S) // Ww) % Hh, np.arange(S) % Ww
    key = (t // pt) * 1000000 + (h // ph) * 1000 + (w // pw)
    for i in (0, 5, 77, 200, 255):
        cols = np.nonzero(key == key[i])[0]
        s_ = q[i] @ k[cols].T / np.sqrt(d)
        e = np.exp(s_ - s_.max())
        assert np.abs(out[i] - e @ v[cols] / e.sum()).max() < 1e-12


def test_attention_3d_tile_single_block_is_tile_attention():
    pin_attention_own_tile_3d()


def test_pool_closed_forms():
    x = np.full((3, 256, 4), 1.75)
    assert np.array_equal(oracle.pool(x, 64), np.full((3, 4, 4), 1.75))
    # a ramp along the sequence pools to the mean of each run: 64 b + 31.5
    r = np.arange(256, dtype=np.float64)[:, None] * np.ones((1, 2))
    assert np.array_equal(oracle.pool(r, 64)[:, 0], 64.0 * np.arange(4) + 31.5)


def test_pooled_head_is_patch_mean():
    T, Hh, Ww, P, d = 2, 16, 8, 8, 3
    x = np.random.default_rng(1).standard_normal((T * Hh * Ww, d))
    got = oracle.pooled_head(x, T, Hh, Ww, P, P * P)
    g = x.reshape(T, Hh // P, P, Ww // P, P, d).mean(axis=(2, 4)).reshape(-1, d)
    assert np.allclose(got, g, rtol=0, atol=1e-14)


def test_reduced_map_closed_form_and_invariants():
    pin_reduced_closed_form()
    rng = np.random.default_rng(2)
    qb, kb = rng.standard_normal((5, 16)), rng.standard_normal((7, 16))
    A = oracle.reduced_map(qb, kb)
    assert np.allclose(A.sum(-1), 1.0, rtol=0, atol=1e-12)
    # equal key blocks -> uniform rows; permuting key blocks permutes columns
    assert np.allclose(oracle.reduced_map(qb, np.ones((7, 16))), 1 / 7, atol=1e-15)
    p = rng.permutation(7)
    assert np.allclose(oracle.reduced_map(qb, kb[p]), A[:, p], atol=1e-15)


def test_cdf_golden(golden_dir):
    pin_cdf_golden(golden_dir)


def test_cdf_bruteforce():
    pin_cdf_bruteforce()


def test_cdf_invariants_on_tiny_workload():
    w = W.TINY
    q, k, _ = W.make_inputs(w)
    BH = w.BH
    m, mn, A = oracle.nabla_mask(q.reshape(BH, w.S, w.d), k.reshape(BH, w.S, w.d),
                                 w.T, w.Hh, w.Ww, w.P, w.N, w.thr, w.sta)
    A2, K2 = A.reshape(-1, w.nb), mn.reshape(-1, w.nb)
    for a, keep in zip(A2, K2):
        assert a[keep].sum() >= 1 - w.thr
        assert a[keep].sum() - a[keep].min() < 1 - w.thr
        assert (~keep).sum() == 0 or a[keep].min() >= a[~keep].max()
        # brute force on nb = 4 blocks
        best = min(k for k in range(1, w.nb + 1)
                   if max(a[list(c)].sum() for c in itertools.combinations(range(w.nb), k)) >= 1 - w.thr)
        assert keep.sum() == best


def test_sta_golden_and_loop(golden_dir):
    pin_sta_golden(golden_dir)
    T, Hh, Ww, P, win = 4, 24, 40, 8, (3, 1, 5)
    got = oracle.sta_keep(T, Hh, Ww, P, win)
    nh, nw = Hh // P, Ww // P
    nb = T * nh * nw
    expect = np.zeros((nb, nb), dtype=bool)
    for t1, h1, w1 in itertools.product(range(T), range(nh), range(nw)):
        for t2, h2, w2 in itertools.product(range(T), range(nh), range(nw)):
            if abs(t1 - t2) <= 1 and h1 == h2 and abs(w1 - w2) <= 2:
                expect[(t1 * nh + h1) * nw + w1, (t2 * nh + h2) * nw + w2] = True
    assert np.array_equal(got, expect)
    assert oracle.sta_keep(T, Hh, Ww, P, (9, 9, 11)).all()  # window covers the grid
    assert np.array_equal(oracle.sta_keep(T, Hh, Ww, P, (1, 1, 1)), np.eye(nb, dtype=bool))
    assert not oracle.sta_keep(T, Hh, Ww, P, (0, 0, 0)).any()


def test_attention_dense_equals_sdpa():
    pin_attention_dense_is_sdpa()


def test_attention_full_sta_window_equals_sdpa():
    q, k, v, (T, Hh, Ww, P, N) = _small_problem(seed=11)
    out, mask = oracle.nabla_attention(q, k, v, T, Hh, Ww, P, N, 0.5, (5, 5, 5))
    assert mask.all()
    assert np.abs(out - _sdpa64(q, k, v)).max() < 1e-10


def test_attention_single_block_is_patch_attention():
    pin_attention_own_patch()


def test_attention_rows_sample_matches_full():
    q, k, v, (T, Hh, Ww, P, N) = _small_problem(seed=13)
    out, mask = oracle.nabla_attention(q, k, v, T, Hh, Ww, P, N, 0.2, (1, 1, 3))
    toks = np.array([0, 7, 100, 511, 300])
    part = oracle.attention_head(q[1], k[1], v[1], T, Hh, Ww, P, N, mask[1], tokens=toks)
    assert np.abs(part - out[1][toks]).max() < 1e-12  # same rows, BLAS rounding order aside


def test_inner_patch_order_does_not_change_output():
    # The page fixes which tokens share a block, not their order inside it; with
    # a transposed in-patch order the result (natural order) must not change.
    q, k, v, (T, Hh, Ww, P, N) = _small_problem(seed=17)
    base, mask = oracle.nabla_attention(q, k, v, T, Hh, Ww, P, N, 0.2, (1, 3, 1))
    orig = nabla.fractal_order
    try:
        def transposed(T_, Hh_, Ww_, P_):
            idx = np.arange(T_ * Hh_ * Ww_).reshape(T_, Hh_ // P_, P_, Ww_ // P_, P_)
            return idx.transpose(0, 1, 3, 4, 2).reshape(-1)
        nabla.fractal_order = transposed
        alt, mask2 = oracle.nabla_attention(q, k, v, T, Hh, Ww, P, N, 0.2, (1, 3, 1))
    finally:
        nabla.fractal_order = orig
    assert np.array_equal(mask, mask2)
    assert np.abs(alt - base).max() < 1e-12


def test_widen_bf16_exact():
    x = np.array([1.0, -2.5, 3.140625, 0.0, 65280.0], dtype=np.float32)
    bits = W.f32_to_bf16_bits(x)
    assert np.array_equal(oracle.widen_bf16(bits), x.astype(np.float64))


# --- planted mistakes: each must be caught by some pin -----------------------

def _mut_fractal_inner_transposed(T, Hh, Ww, P):
    idx = np.arange(T * Hh * Ww).reshape(T, Hh // P, P, Ww // P, P)
    return idx.transpose(0, 1, 3, 4, 2).reshape(-1)


def _mut_fractal_patch_col_major(T, Hh, Ww, P):
    idx = np.arange(T * Hh * Ww).reshape(T, Hh // P, P, Ww // P, P)
    return idx.transpose(0, 3, 1, 2, 4).reshape(-1)


def _mut_fractal3d_tile_w_before_h(T, Hh, Ww, P):
    pt, ph, pw = nabla.tile_shape(P)
    idx = np.arange(T * Hh * Ww).reshape(T // pt, pt, Hh // ph, ph, Ww // pw, pw)
    return idx.transpose(0, 2, 4, 1, 5, 3).reshape(-1)


def _mut_fractal3d_time_inside_patch_last(T, Hh, Ww, P):
    pt, ph, pw = nabla.tile_shape(P)
    idx = np.arange(T * Hh * Ww).reshape(T // pt, pt, Hh // ph, ph, Ww // pw, pw)
    return idx.transpose(0, 2, 4, 3, 5, 1).reshape(-1)


def _mut_cdf_le(A, thr):
    if thr == 0.0:
        return np.ones(A.shape, dtype=bool)
    order = np.argsort(-A, axis=-1, kind="stable")
    s = np.take_along_axis(A, order, axis=-1)
    before = np.cumsum(s, axis=-1) - s
    keep = np.empty(A.shape, dtype=bool)
    np.put_along_axis(keep, order, before <= (1.0 - thr), axis=-1)
    return keep


def _mut_cdf_ascending(A, thr):
    if thr == 0.0:
        return np.ones(A.shape, dtype=bool)
    order = np.argsort(A, axis=-1, kind="stable")
    s = np.take_along_axis(A, order, axis=-1)
    before = np.cumsum(s, axis=-1) - s
    keep = np.empty(A.shape, dtype=bool)
    np.put_along_axis(keep, order, before < (1.0 - thr), axis=-1)
    return keep


def _mut_cdf_threshold_is_thr(A, thr):
    return _orig_cdf(A, 1.0 - thr if thr > 0 else 0.0)


def _mut_reduced_no_scale(qbar, kbar):
    logits = qbar @ np.swapaxes(kbar, -1, -2)
    e = np.exp(logits - logits.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def _mut_sta_window_too_wide(T, Hh, Ww, P, sta):
    st, sh, sw = sta
    return _orig_sta(T, Hh, Ww, P, (st, sh, sw + 2 if sw else sw))


def _mut_sta_strict_distance(T, Hh, Ww, P, sta):
    c = nabla.block_coords(T, Hh, Ww, P)
    diff = np.abs(c[:, None, :] - c[None, :, :])
    return ((diff[..., 0] < sta[0] // 2 + (sta[0] == 1)) & (diff[..., 1] < max(sta[1] // 2, 1))
            & (diff[..., 2] < max(sta[2] // 2, 1)))


def _mut_attention_strided_blocks(qp, kp, vp, mask, N, rows=None):
    S, d = qp.shape
    nb = S // N
    rows = np.arange(S) if rows is None else np.asarray(rows)
    out = np.empty((rows.size, d))
    for i, r in enumerate(rows):
        kept = np.nonzero(mask[r // N])[0]
        cols = (kept[:, None] + nb * np.arange(N)[None, :]).reshape(-1)
        s = qp[r] @ kp[cols].T / np.sqrt(d)
        e = np.exp(s - s.max())
        out[i] = e @ vp[cols] / e.sum()
    return out


def _mut_attention_no_scale(qp, kp, vp, mask, N, rows=None):
    return _orig_masked(qp * np.sqrt(qp.shape[-1]), kp, vp, mask, N, rows)


def pin_backward_finite_differences(seed=41):
    # Gradients of L = sum(O * G) against central differences of the forward
    # oracle (itself pinned above), on a tiny head with a random block mask.
    rng = np.random.default_rng(seed)
    T, Hh, Ww, P, N, d = 2, 8, 16, 8, 64, 4
    S = T * Hh * Ww
    nb = S // N
    q, k, v, g = (rng.standard_normal((S, d)) for _ in range(4))
    mask = rng.random((nb, nb)) < 0.5
    mask[np.arange(nb), np.arange(nb)] = True
    perm = oracle.fractal_order(T, Hh, Ww, P)

    def loss(q_, k_, v_):
        qp, kp, vp = (oracle.flatten(x, perm) for x in (q_, k_, v_))
        o = oracle.unflatten(oracle.masked_attention(qp, kp, vp, mask, N), perm)
        return float((o * g).sum())

    dq, dk, dv, _ = oracle.attention_backward_head(q, k, v, g, T, Hh, Ww, P, N, mask)
    eps = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for _ in range(10):
            i, c = int(rng.integers(S)), int(rng.integers(d))
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][i, c] += eps
            args_m[which][i, c] -= eps
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - grad[i, c]) < 1e-7 * max(1.0, abs(fd)), (which, i, c, fd, grad[i, c])


def pin_backward_dense_is_torch_autograd(seed=43):
    # With every block kept the gradients are those of plain softmax
    # attention: torch's fp64 autograd of scaled_dot_product_attention.
    import torch
    rng = np.random.default_rng(seed)
    T, Hh, Ww, P, N, d = 2, 8, 8, 8, 64, 8
    S = T * Hh * Ww
    q, k, v, g = (rng.standard_normal((S, d)) for _ in range(4))
    mask = np.ones((S // N, S // N), dtype=bool)
    dq, dk, dv, lse = oracle.attention_backward_head(q, k, v, g, T, Hh, Ww, P, N, mask)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq[None], tk[None], tv[None])[0]
    o.backward(torch.tensor(g))
    for got, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.abs(got - ref.numpy()).max() < 1e-10
    ref_lse = torch.logsumexp(torch.tensor(q) @ torch.tensor(k).T / np.sqrt(d), dim=-1)
    assert np.abs(lse - ref_lse.numpy()).max() < 1e-10


def pin_backward_uniform_rows():
    # Zero queries: every kept score is 0, so lse = log(kept keys), P is
    # uniform over the kept keys, dV of a key is the mean of dO over the rows
    # that keep its block divided by their kept-key counts.
    rng = np.random.default_rng(47)
    T, Hh, Ww, P, N, d = 2, 8, 16, 8, 64, 4
    S = T * Hh * Ww
    nb = S // N
    k, v, g = (rng.standard_normal((S, d)) for _ in range(3))
    mask = rng.random((nb, nb)) < 0.5
    mask[np.arange(nb), np.arange(nb)] = True
    perm = oracle.fractal_order(T, Hh, Ww, P)
    _, _, dv, lse = oracle.attention_backward_head(np.zeros((S, d)), k, v, g, T, Hh, Ww, P, N,
                                                   mask)
    kept_keys = mask.sum(axis=1) * N  # per q-block
    lse_p = oracle.flatten(lse[:, None], perm)[:, 0]
    assert np.allclose(lse_p, np.log(np.repeat(kept_keys, N)), rtol=0, atol=1e-12)
    gp = oracle.flatten(g, perm)
    expect = np.zeros((S, d))
    for i in range(nb):
        for j in np.nonzero(mask[i])[0]:
            expect[j * N:(j + 1) * N] += gp[i * N:(i + 1) * N].sum(axis=0) / kept_keys[i]
    assert np.abs(oracle.flatten(dv, perm) - expect).max() < 1e-12


_orig_cdf = nabla.cdf_keep
_orig_sta = nabla.sta_keep
_orig_masked = nabla.masked_attention
_orig_bwd = nabla.masked_attention_backward


def _mut_backward_no_D(qp, kp, vp, dop, mask, N, o_stored=None):
    # dS = P * dP (the -D term dropped): only dQ and dK change
    S, d = qp.shape
    o = _orig_masked(qp, kp, vp, mask, N)
    dq, dk, dv, lse = _orig_bwd(qp, kp, vp, dop, mask, N)
    D = (dop * o).sum(axis=-1, keepdims=True)
    # P * dP = dS + P * D: add the dropped term's contributions back
    for qb in range(S // N):
        r = slice(qb * N, (qb + 1) * N)
        kept = np.nonzero(mask[qb])[0]
        cols = (kept[:, None] * N + np.arange(N)[None, :]).reshape(-1)
        s = qp[r] @ kp[cols].T / np.sqrt(d)
        p = np.exp(s - s.max(axis=-1, keepdims=True))
        p /= p.sum(axis=-1, keepdims=True)
        dq[r] += (p * D[r]) @ kp[cols] / np.sqrt(d)
        dk[cols] += (p * D[r]).T @ qp[r] / np.sqrt(d)
    return dq, dk, dv, lse


def _mut_backward_dk_unscaled(qp, kp, vp, dop, mask, N, o_stored=None):
    dq, dk, dv, lse = _orig_bwd(qp, kp, vp, dop, mask, N)
    return dq, dk * np.sqrt(qp.shape[-1]), dv, lse


def golden_recall(golden_dir):
    out = []
    for ln in _rows(os.path.join(golden_dir, "heat_recall.txt")):
        h, m, r = (x.strip() for x in ln.split("|"))
        H = np.array([[float(x) for x in row.split()] for row in h.split(";")])
        M = np.array([[int(x) for x in row.split()] for row in m.split(";")], dtype=bool)
        out.append((H, M, float(Fraction(r))))
    return out


def pin_recall_golden(golden_dir):
    for H, M, expect in golden_recall(golden_dir):
        got = oracle.heat_recall(H, M)
        assert abs(got - expect) < 1e-12, (got, expect)


def _mut_recall_pooled(H, M):
    H = np.asarray(H, dtype=np.float64)
    return float((H * M).sum() / H.sum())


def _mut_recall_over_columns(H, M):
    H = np.asarray(H, dtype=np.float64)
    return float(np.mean((H * M).sum(axis=0) / H.sum(axis=0)))


MUTANTS = [
    ("fractal_order", _mut_fractal_inner_transposed, "fractal"),
    ("fractal_order", _mut_fractal_patch_col_major, "fractal"),
    ("fractal_order", _mut_fractal3d_tile_w_before_h, "fractal3d"),
    ("fractal_order", _mut_fractal3d_time_inside_patch_last, "fractal3d"),
    ("cdf_keep", _mut_cdf_le, "cdf"),
    ("cdf_keep", _mut_cdf_ascending, "cdf"),
    ("cdf_keep", _mut_cdf_threshold_is_thr, "cdf"),
    ("reduced_map", _mut_reduced_no_scale, "reduced"),
    ("sta_keep", _mut_sta_window_too_wide, "sta"),
    ("sta_keep", _mut_sta_strict_distance, "sta"),
    ("masked_attention", _mut_attention_strided_blocks, "attention"),
    ("masked_attention", _mut_attention_no_scale, "attention"),
    ("masked_attention_backward", _mut_backward_no_D, "backward"),
    ("masked_attention_backward", _mut_backward_dk_unscaled, "backward"),
    ("heat_recall", _mut_recall_pooled, "recall"),
    ("heat_recall", _mut_recall_over_columns, "recall"),
]


def test_backward_finite_differences():
    pin_backward_finite_differences()


def test_backward_dense_is_torch_autograd():
    pin_backward_dense_is_torch_autograd()


def test_backward_block_rows_match_full():
    # The per-block form (used for full-size samples) against the full form,
    # itself pinned by finite differences and autograd above.
    rng = np.random.default_rng(53)
    S, d, N = 512, 8, 64
    nb = S // N
    qp, kp, vp, dop = (rng.standard_normal((S, d)) for _ in range(4))
    mask = rng.random((nb, nb)) < 0.4
    mask[np.arange(nb), np.arange(nb)] = True
    dq, dk, dv, lse = oracle.masked_attention_backward(qp, kp, vp, dop, mask, N)
    qbs, kbs = [5, 0, 7], [3, 6]
    bq, bk, bv, bl = oracle.masked_attention_backward_blocks(qp, kp, vp, dop, mask, N, qbs, kbs)
    for i, b in enumerate(qbs):
        assert np.abs(bq[i] - dq[b * N:(b + 1) * N]).max() < 1e-12
        assert np.abs(bl[i] - lse[b * N:(b + 1) * N]).max() < 1e-12
    for i, b in enumerate(kbs):
        assert np.abs(bk[i] - dk[b * N:(b + 1) * N]).max() < 1e-12
        assert np.abs(bv[i] - dv[b * N:(b + 1) * N]).max() < 1e-12


def test_backward_uniform_rows():
    pin_backward_uniform_rows()


@pytest.mark.parametrize("name,mutant,area", MUTANTS, ids=[m[1].__name__ for m in MUTANTS])
def test_planted_mistake_is_caught(name, mutant, area, golden_dir, monkeypatch):
    monkeypatch.setattr(nabla, name, mutant)
    # oracle/__init__ re-exports the functions; route those through the mutant too
    monkeypatch.setattr(oracle, name, mutant)
    pins = {
        "fractal": [lambda: pin_fractal_golden(golden_dir), pin_fractal_reshape],
        "fractal3d": [pin_fractal_reshape_3d, pin_attention_own_tile_3d],
        "cdf": [lambda: pin_cdf_golden(golden_dir), pin_cdf_bruteforce],
        "reduced": [pin_reduced_closed_form],
        "sta": [lambda: pin_sta_golden(golden_dir)],
        "attention": [pin_attention_own_patch, pin_attention_dense_is_sdpa],
        "backward": [pin_backward_finite_differences, pin_backward_dense_is_torch_autograd],
        "recall": [lambda: pin_recall_golden(golden_dir)],
    }[area]
    caught = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin caught the planted mistake {mutant.__name__}"


# --- block max-pooled attention map -------------------------------------------

def test_block_heatmap_bruteforce_token_by_token():
    # Tiny problem: compute every probability by an explicit loop over tokens
    # (exp of the scaled dot product over the sum over all keys), then the
    # block max by looping over the positions of each block.
    rng = np.random.default_rng(29)
    T, Hh, Ww, P, N = 2, 8, 8, 8, 64
    S, d = T * Hh * Ww, 4
    q, k = rng.standard_normal((S, d)), rng.standard_normal((S, d))
    H = oracle.block_heatmap(q, k, T, Hh, Ww, P, N)
    perm = oracle.fractal_order(T, Hh, Ww, P)  # position -> natural token
    nb = S // N
    expect = np.zeros((nb, nb))
    for i in range(S):
        s = np.array([math.exp(float(q[i] @ k[j]) / math.sqrt(d)) for j in range(S)])
        prob = s / s.sum()
        pos = int(np.nonzero(perm == i)[0][0])
        for j in range(S):
            pj = int(np.nonzero(perm == j)[0][0])
            expect[pos // N, pj // N] = max(expect[pos // N, pj // N], prob[j])
    assert np.abs(H - expect).max() < 1e-12
    rows = [1, 0]  # the per-row form (only those q-blocks' softmax rows)
    Hr = oracle.block_heatmap_rows(q, k, T, Hh, Ww, P, N, rows)
    assert np.abs(Hr - expect[rows]).max() < 1e-12


def test_block_heatmap_closed_forms_and_bounds():
    T, Hh, Ww, P, N = 2, 16, 16, 8, 64
    S = T * Hh * Ww
    zero = np.zeros((S, 8))
    H = oracle.block_heatmap(zero, np.random.default_rng(1).standard_normal((S, 8)),
                             T, Hh, Ww, P, N)
    assert np.allclose(H, 1.0 / S, rtol=0, atol=1e-15)  # zero queries attend uniformly
    rng = np.random.default_rng(31)
    q, k = rng.standard_normal((S, 8)) * 2, rng.standard_normal((S, 8)) * 2
    H = oracle.block_heatmap(q, k, T, Hh, Ww, P, N)
    assert (H <= 1).all() and (H > 0).all()
    # a row's probabilities sum to 1 over nb blocks of N keys: the block
    # maxima of one q-block sum to at least 1/N
    assert (H.sum(axis=1) >= 1.0 / N - 1e-12).all()
    M = np.zeros(H.shape, dtype=bool)
    assert oracle.heat_recall(H, ~M) == 1.0 and oracle.heat_recall(H, M) == 0.0
    top = H >= np.sort(H, axis=1)[:, -2:-1]  # two largest per row
    assert 0.0 < oracle.heat_recall(H, top) < 1.0


def test_heat_recall_golden(golden_dir):
    pin_recall_golden(golden_dir)


def test_backward_stored_output_shifts_only_the_D_term():
    # D_i = sum_c dO_ic o_ic enters only through dS = P (dP - D). Replacing
    # the exact O by a stored copy moves D by delta_i = sum_c dO_ic
    # (stored - exact)_ic and therefore dQ_i by -delta_i / sqrt(d) times
    # sum_j P_ij k_j, which is the forward attention with K in place of V.
    rng = np.random.default_rng(61)
    S, d, N = 256, 8, 64
    nb = S // N
    qp, kp, vp, dop = (rng.standard_normal((S, d)) for _ in range(4))
    mask = rng.random((nb, nb)) < 0.5
    mask[np.arange(nb), np.arange(nb)] = True
    o = oracle.masked_attention(qp, kp, vp, mask, N)
    exact = oracle.masked_attention_backward(qp, kp, vp, dop, mask, N)
    same = oracle.masked_attention_backward(qp, kp, vp, dop, mask, N, o_stored=o)
    for a, b in zip(exact, same):
        assert np.abs(a - b).max() < 1e-12
    stored = o + 1e-3 * rng.standard_normal(o.shape)
    moved = oracle.masked_attention_backward(qp, kp, vp, dop, mask, N, o_stored=stored)
    delta = (dop * (stored - o)).sum(axis=-1)
    pk = oracle.masked_attention(qp, kp, kp, mask, N)
    expect_dq = exact[0] - delta[:, None] * pk / np.sqrt(d)
    assert np.abs(moved[0] - expect_dq).max() < 1e-12
    assert np.abs(moved[2] - exact[2]).max() < 1e-12 and np.abs(moved[3] - exact[3]).max() < 1e-12
    assert np.abs(moved[0] - exact[0]).max() > 1e-6  # the substitution is live
