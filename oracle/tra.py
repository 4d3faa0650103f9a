"""Plain fp64 CPU oracle for the Token Radius Attention (TRA) block mask.

TEST INFRASTRUCTURE ONLY, like the rest of this package: the tests, the smoke
check and the benchmark's CPU leg are its only callers; the CUDA library never
imports it and shares no code with it.

It follows the page "Token Radius Attention per la Generazione di Video
Efficiente" (gist.science/it/paper/2608.02504), section 2 ("Metodologia:
Token Radius Attention (TRA)"), in the order of its pipeline ("La Pipeline
TRA"): the entropy of each query's full attention row, the entropy mapped to a
per-token key budget, the budget turned into a query-centred spatial radius
that shrinks with the temporal distance phi(delta) = exp(-gamma delta), and
the token-level disc masks turned into a block mask by token votes. The block
mask then feeds the same block-sparse attention as the NABLA mask.

Readings taken where the page is silent (each one is listed in the design
notes as well):

* Entropy: H_i = -sum_j p_ij ln p_ij over query i's full softmax row
  (all keys, scale 1/sqrt(d), no mask), in nats.
* Budget: the page writes B_hat ~ tau exp(H_i) / N with N the number of
  tokens, a fraction of the keys; the number of keys is then
  k_i = tau exp(H_i), capped at S.
* Budget to radius: the keys inside the support are counted as disc areas:
  sum over the frames t of the video of pi (r_i phi(|t - t_i|))^2 = k_i, so
  r_i^2 = k_i / (pi Z(t_i)) with Z(t) = sum_t' exp(-2 gamma |t' - t|).
* Support: key j is in query i's support iff
  (h_j - h_i)^2 + (w_j - w_i)^2 <= r_i^2 exp(-2 gamma |t_j - t_i|),
  distances in token units (a disc per frame, radius r_i phi(delta)).
* Token votes: query token i votes for key block b iff its support holds at
  least one key of b; block (a, b) is kept iff at least vote_min of the N
  query tokens of block a vote for b (1 <= vote_min <= N). A query's own
  position is always in its support, so every q-block keeps its own block.
"""
from __future__ import annotations

import numpy as np

from .nabla import _as_f64, fractal_order, flatten


def token_entropy(q, k):
    """Entropy (nats) of every query's full softmax attention row, one head.

    q, k: [S, d] (bf16 bit patterns or floats), any token order (the result
    follows q's order). Returns float64 [S].
    """
    q, k = _as_f64(q), _as_f64(k)
    s = q @ k.T / np.sqrt(q.shape[-1])
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    p = e / e.sum(axis=-1, keepdims=True)
    # 0 * log 0 = 0 for probabilities that underflow
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(p > 0, p * np.log(p), 0.0)
    return -t.sum(axis=-1)


def entropy_budget(H, S, tau):
    """Keys per query, k_i = tau exp(H_i), capped at the S keys there are."""
    return np.minimum(float(tau) * np.exp(np.asarray(H, dtype=np.float64)), float(S))


def frame_weight(T, gamma):
    """Z(t) = sum over the T frames t' of exp(-2 gamma |t' - t|): the area
    factor of the discs over the video, float64 [T]."""
    t = np.arange(T)
    return np.exp(-2.0 * gamma * np.abs(t[None, :] - t[:, None])).sum(axis=1)


def budget_radius2(budget, t_of_query, T, gamma):
    """Squared base radius r_i^2 = k_i / (pi Z(t_i)) per query (token units)."""
    Z = frame_weight(T, gamma)
    return np.asarray(budget, dtype=np.float64) / (np.pi * Z[np.asarray(t_of_query)])


def token_coords(T, Hh, Ww):
    """(t, h, w) of every natural-order token, int64 [S] each."""
    t, h, w = np.meshgrid(np.arange(T), np.arange(Hh), np.arange(Ww), indexing="ij")
    return t.reshape(-1), h.reshape(-1), w.reshape(-1)


def radius_support(r2, T, Hh, Ww, gamma, queries=None):
    """Token-level disc masks: bool [len(queries), S], natural order.

    r2: [S] squared base radius of every query (natural order); queries:
    natural-order query indices (default all).
    """
    t, h, w = token_coords(T, Hh, Ww)
    qi = np.arange(t.size) if queries is None else np.asarray(queries)
    dt = np.abs(t[None, :] - t[qi][:, None])
    d2 = (h[None, :] - h[qi][:, None]) ** 2 + (w[None, :] - w[qi][:, None]) ** 2
    return d2 <= np.asarray(r2, dtype=np.float64)[qi][:, None] * np.exp(-2.0 * gamma * dt)


def radius_block_mask(r2, T, Hh, Ww, P, N, gamma, vote_min):
    """Token votes -> block mask of one head (fractal block order).

    r2: [S] squared base radius per query, natural order. Returns
    (mask bool [nb, nb], votes int64 [nb, nb]): votes[a, b] = number of query
    tokens of block a whose support holds a key of block b.
    """
    perm = fractal_order(T, Hh, Ww, P)  # position -> natural token
    S = T * Hh * Ww
    nb = S // N
    votes = np.zeros((nb, nb), dtype=np.int64)
    for a in range(nb):
        sup = radius_support(r2, T, Hh, Ww, gamma, queries=perm[a * N:(a + 1) * N])
        sup_f = flatten(sup.T, perm).T  # keys in fractal order
        touches = sup_f.reshape(N, nb, N).any(axis=2)  # [query, key block]
        votes[a] = touches.sum(axis=0)
    return votes >= int(vote_min), votes


def tra_mask(H, T, Hh, Ww, P, N, tau, gamma, vote_min):
    """The whole TRA mask pipeline for one head from its per-query entropies
    H [S] (natural order): budget, radius, disc supports, token votes.
    Returns (mask [nb, nb], votes, r2 [S])."""
    S = T * Hh * Ww
    t, _, _ = token_coords(T, Hh, Ww)
    r2 = budget_radius2(entropy_budget(H, S, tau), t, T, gamma)
    mask, votes = radius_block_mask(r2, T, Hh, Ww, P, N, gamma, vote_min)
    return mask, votes, r2
