"""Pins for the Token Radius Attention (TRA) mask oracle, independent of its
own code: a hand-worked vote matrix (tests/golden), closed forms of the
entropy, the budget and the frame weights, a token-by-token brute force of the
votes, limiting cases, and planted mistakes that some pin must catch."""
import math
import os

import numpy as np
import pytest

import oracle
from oracle import tra

GRID = (2, 4, 4, 2, 4)  # T, Hh, Ww, P, N of the hand-worked fixture


def golden_votes(golden_dir):
    out = []
    path = os.path.join(golden_dir, "tra_votes_T2_H4_W4_P2.txt")
    with open(path) as f:
        for ln in f:
            if ln.startswith("#") or not ln.strip():
                continue
            case, r2, decay, rows = (x.strip() for x in ln.split(":"))
            votes = np.array([[int(x) for x in r.split()] for r in rows.split(";")])
            gamma = -0.5 * math.log(float(decay))  # exp(-2 gamma) = decay
            out.append((case, float(r2), gamma, votes))
    return out


def pin_votes_golden(golden_dir):
    T, Hh, Ww, P, N = GRID
    for case, r2, gamma, expect in golden_votes(golden_dir):
        r2s = np.full(T * Hh * Ww, r2)
        for vmin in (1, 2, 3, 4):
            mask, votes = oracle.radius_block_mask(r2s, T, Hh, Ww, P, N, gamma, vmin)
            assert np.array_equal(votes, expect), (case, votes)
            assert np.array_equal(mask, expect >= vmin), (case, vmin)


def brute_votes(r2, T, Hh, Ww, P, N, gamma):
    """Votes by explicit loops over blocks, queries and keys (token
    coordinates read off the fractal order)."""
    perm = oracle.fractal_order(T, Hh, Ww, P)
    coords = [(n // (Hh * Ww), (n // Ww) % Hh, n % Ww) for n in range(T * Hh * Ww)]
    nb = T * Hh * Ww // N
    votes = np.zeros((nb, nb), dtype=np.int64)
    for a in range(nb):
        for qpos in range(a * N, (a + 1) * N):
            i = int(perm[qpos])
            ti, hi, wi = coords[i]
            for b in range(nb):
                for kpos in range(b * N, (b + 1) * N):
                    tj, hj, wj = coords[int(perm[kpos])]
                    rad2 = r2[i] * math.exp(-2.0 * gamma * abs(tj - ti))
                    if (hj - hi) ** 2 + (wj - wi) ** 2 <= rad2:
                        votes[a, b] += 1
                        break
    return votes


def pin_votes_bruteforce(seed=5):
    rng = np.random.default_rng(seed)
    for (T, Hh, Ww, P, N), gamma in ((( 3, 8, 8, 4, 16), 0.3), ((2, 8, 8, (2, 2, 4), 16), 0.7)):
        r2 = rng.uniform(0.0, 12.0, T * Hh * Ww)
        _, votes = oracle.radius_block_mask(r2, T, Hh, Ww, P, N, gamma, 1)
        assert np.array_equal(votes, brute_votes(r2, T, Hh, Ww, P, N, gamma))


def pin_pipeline_radius():
    # T = 2 frames and exp(-2 gamma) = 1/2 give Z(0) = Z(1) = 3/2, so an
    # entropy of ln(3 pi / 2) with tau = 1 budgets 3 pi / 2 keys and a squared
    # radius of exactly 1: the pipeline then reproduces golden case A.
    T, Hh, Ww, P, N = GRID
    gamma = 0.5 * math.log(2.0)
    H = np.full(T * Hh * Ww, math.log(1.5 * math.pi))
    mask, votes, r2 = oracle.tra_mask(H, T, Hh, Ww, P, N, 1.0, gamma, 2)
    assert np.allclose(r2, 1.0, rtol=1e-12, atol=0)
    assert votes[0].tolist() == [4, 2, 2, 0, 4, 0, 0, 0]
    assert mask[0].tolist() == [True, True, True, False, True, False, False, False]


def pin_entropy_closed_form():
    # one key scores c, the S - 1 others 0 (d = 1, q = c, k = e_0):
    # H = ln(e^c + S - 1) - c e^c / (e^c + S - 1)
    S = 37
    k = np.zeros((S, 1))
    k[0, 0] = 1.0
    for c in (0.0, 1.5, -2.0, 9.0):
        q = np.full((3, 1), c)
        z = math.exp(c) + S - 1
        expect = math.log(z) - c * math.exp(c) / z
        assert np.abs(oracle.token_entropy(q, k) - expect).max() < 1e-12
    # zero queries attend uniformly: ln S
    assert np.abs(oracle.token_entropy(np.zeros((4, 8)), np.ones((S, 8))) - math.log(S)).max() < 1e-12


def test_votes_golden(golden_dir):
    pin_votes_golden(golden_dir)


def test_votes_bruteforce():
    pin_votes_bruteforce()


def test_pipeline_reaches_golden_radius():
    pin_pipeline_radius()


def test_entropy_closed_forms_and_bruteforce():
    pin_entropy_closed_form()
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal((5, 4)), rng.standard_normal((9, 4))
    H = oracle.token_entropy(q, k)
    for i in range(5):
        s = [float(q[i] @ k[j]) / 2.0 for j in range(9)]
        z = sum(math.exp(x) for x in s)
        expect = -sum(math.exp(x) / z * math.log(math.exp(x) / z) for x in s)
        assert abs(H[i] - expect) < 1e-12


def test_budget_and_frame_weight_closed_forms():
    H = np.log(np.array([5.0, 1.0, 1e6]))
    assert np.allclose(oracle.entropy_budget(H, 100, 2.0), [10.0, 2.0, 100.0], rtol=1e-14)
    assert np.allclose(tra.frame_weight(4, 0.0), 4.0)
    Z = tra.frame_weight(3, 0.5 * math.log(2.0))  # terms 2^-|t - t'|
    assert np.allclose(Z, [1.75, 2.0, 1.75], rtol=1e-14)
    r2 = oracle.budget_radius2([math.pi * 1.75, math.pi * 4.0], [0, 1], 3, 0.5 * math.log(2.0))
    assert np.allclose(r2, [1.0, 2.0], rtol=1e-14)


def test_limits():
    T, Hh, Ww, P, N = 2, 8, 8, 4, 16
    S = T * Hh * Ww
    nb = S // N
    # zero radius: every query keeps only its own (h, w), in every frame ->
    # the blocks of the same patch in all frames, each with all N votes
    mask, votes = oracle.radius_block_mask(np.zeros(S), T, Hh, Ww, P, N, 0.4, 1)
    pf = (Hh // P) * (Ww // P)
    same_patch = (np.arange(nb)[:, None] % pf) == (np.arange(nb)[None, :] % pf)
    assert np.array_equal(mask, same_patch)
    assert np.array_equal(votes, same_patch * N)
    # a radius beyond the grid and no decay: dense, every token votes
    mask, votes = oracle.radius_block_mask(np.full(S, 1e6), T, Hh, Ww, P, N, 0.0, N)
    assert mask.all() and (votes == N).all()
    # the support grows with the radius: votes never decrease
    r2 = np.random.default_rng(1).uniform(0, 6, S)
    _, v1 = oracle.radius_block_mask(r2, T, Hh, Ww, P, N, 0.2, 1)
    _, v2 = oracle.radius_block_mask(r2 * 1.5, T, Hh, Ww, P, N, 0.2, 1)
    assert (v2 >= v1).all() and (v2 > v1).any()


# --- planted mistakes ----------------------------------------------------------

_orig_support = tra.radius_support


def _mut_decay_on_r2_not_r(r2, T, Hh, Wd, gamma, queries=None):
    # phi applied once to the squared radius (exp(-gamma delta) on r^2)
    return _orig_support(r2, T, Hh, Wd, gamma / 2.0, queries)


def _mut_chebyshev(r2, T, Hh, Wd, gamma, queries=None):
    t, h, w = tra.token_coords(T, Hh, Wd)
    qi = np.arange(t.size) if queries is None else np.asarray(queries)
    dt = np.abs(t[None, :] - t[qi][:, None])
    d = np.maximum(np.abs(h[None, :] - h[qi][:, None]), np.abs(w[None, :] - w[qi][:, None]))
    return d ** 2 <= np.asarray(r2)[qi][:, None] * np.exp(-2.0 * gamma * dt)


def _mut_votes_count_pairs(r2, T, Hh, Wd, P, N, gamma, vote_min):
    perm = oracle.fractal_order(T, Hh, Wd, P)
    nb = T * Hh * Wd // N
    votes = np.zeros((nb, nb), dtype=np.int64)
    for a in range(nb):
        sup = tra.radius_support(r2, T, Hh, Wd, gamma, queries=perm[a * N:(a + 1) * N])
        votes[a] = oracle.flatten(sup.T, perm).T.reshape(N, nb, N).sum(axis=(0, 2))
    return votes >= vote_min, votes


def _mut_frame_weight_one_sided(T, gamma):
    t = np.arange(T)
    return np.array([np.exp(-2.0 * gamma * np.arange(T - s)).sum() for s in t])


def _mut_budget_linear(H, S, tau):
    return np.minimum(float(tau) * np.asarray(H, dtype=np.float64), float(S))


TRA_MUTANTS = [
    ("radius_support", _mut_decay_on_r2_not_r),
    ("radius_support", _mut_chebyshev),
    ("radius_block_mask", _mut_votes_count_pairs),
    ("frame_weight", _mut_frame_weight_one_sided),
    ("entropy_budget", _mut_budget_linear),
]


@pytest.mark.parametrize("name,mutant", TRA_MUTANTS, ids=[m[1].__name__ for m in TRA_MUTANTS])
def test_planted_mistake_is_caught(name, mutant, golden_dir, monkeypatch):
    monkeypatch.setattr(tra, name, mutant)
    if hasattr(oracle, name):
        monkeypatch.setattr(oracle, name, mutant)
    caught = 0
    for pin in (lambda: pin_votes_golden(golden_dir), pin_votes_bruteforce, pin_pipeline_radius):
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin caught the planted mistake {mutant.__name__}"
