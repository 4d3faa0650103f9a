"""Plain fp64 CPU oracle for NABLA block-sparse video self-attention.

TEST INFRASTRUCTURE ONLY. The tests, the smoke check and the benchmark's
CPU-baseline leg are the only callers; the CUDA library never imports it and
shares no code with it.

Every function follows the method as described on the page
"NABLA - Neighborhood Adaptive Block-Level Attention per la Generazione
Efficiente di Video" (gist.science/it/paper/2507.13546), section
"Metodologia: NABLA", and is written for a reader to check by eye: fp64
throughout, library primitives (matmul, sort, cumsum) as single steps, no
blocking, fusion or reordering beyond what the method states.

Readings taken where the page is silent (each one is listed in the design
notes as well):

* Fractal order: time outermost, then patch row, then patch column; inside a
  P x P patch the tokens are row-major (h % P, then w % P).
* Three-dimensional tiles (the head-aware tiling of the page "Veda -
  Diffusione Video Scalabile tramite Attenzione Sparsa Distillata"
  (gist.science/it/paper/2605.30325), section 2.2, "Tiling Consapevole delle
  Teste"): a tile shape (p_t, p_h, p_w) with
  p_t * p_h * p_w = N makes each block p_t consecutive frames of a
  p_h x p_w patch. Blocks are ordered (t // p_t, h // p_h, w // p_w) and the
  tokens inside a block (t % p_t, h % p_h, w % p_w), both row-major; the
  square patch of one frame is the shape (1, P, P). Block coordinates and the
  STA window are then in units of blocks along each axis.
* Pooling "in N x N blocks" means the mean of N consecutive tokens of the
  reordered sequence; the N x N refers to the block of the attention map.
* The reduced map uses the same 1/sqrt(d) scale as the main attention and no
  causal mask.
* CDF thresholding keeps the shortest prefix of the row, sorted by descending
  probability (ties: smaller block index first), whose mass reaches 1 - thr:
  block j is kept iff the mass strictly before it is < 1 - thr. thr = 0 is
  defined as dense.
* The STA window is centred on the query block in block units, clipped at the
  grid edges; window sizes are odd; (0, 0, 0) means no STA.
"""
from __future__ import annotations

import numpy as np


def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u32.view(np.float32).astype(np.float64)


# --- Metodologia 1: "Riordinamento dei Token (Fractal Flattening)" ----------

def tile_shape(P) -> tuple:
    """(p_t, p_h, p_w) of a block: an int P is the P x P patch of one frame."""
    if isinstance(P, (tuple, list)):
        pt, ph, pw = (int(v) for v in P)
        return pt, ph, pw
    return 1, int(P), int(P)


def fractal_order(T: int, Hh: int, Ww: int, P) -> np.ndarray:
    """perm[i] = natural-order index of the token at position i of the
    fractally flattened sequence.

    Tokens of each block (a P x P spatial patch of one frame, or a
    p_t x p_h x p_w tile) become contiguous; blocks and the frames inside a
    block stay in time order. Natural order index of (t, h, w) is
    t*Hh*Ww + h*Ww + w. Position order is (t // p_t, h // p_h, w // p_w,
    t % p_t, h % p_h, w % p_w).
    """
    pt, ph, pw = tile_shape(P)
    if T % pt or Hh % ph or Ww % pw:
        raise ValueError("T, Hh, Ww must be multiples of the tile shape")
    nt, nh, nw = T // pt, Hh // ph, Ww // pw
    tb = np.arange(nt).reshape(nt, 1, 1, 1, 1, 1)
    hb = np.arange(nh).reshape(1, nh, 1, 1, 1, 1)
    wb = np.arange(nw).reshape(1, 1, nw, 1, 1, 1)
    ti = np.arange(pt).reshape(1, 1, 1, pt, 1, 1)
    hi = np.arange(ph).reshape(1, 1, 1, 1, ph, 1)
    wi = np.arange(pw).reshape(1, 1, 1, 1, 1, pw)
    natural = (tb * pt + ti) * (Hh * Ww) + (hb * ph + hi) * Ww + (wb * pw + wi)
    return natural.reshape(-1).astype(np.int64)


def flatten(x: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Reorder tokens (axis -2) from natural order into fractal order."""
    return x[..., perm, :]


def unflatten(xp: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Inverse of ``flatten``: scatter fractal-order rows back to natural order."""
    out = np.empty_like(xp)
    out[..., perm, :] = xp
    return out


# --- Metodologia 2: "Costruzione della Maschera Adattiva" -------------------

def pool(xp: np.ndarray, N: int) -> np.ndarray:
    """Sottocampionamento: mean of each run of N consecutive reordered tokens.

    [..., S, d] -> [..., S/N, d].
    """
    S, d = xp.shape[-2], xp.shape[-1]
    if S % N:
        raise ValueError("S must be a multiple of N")
    return xp.reshape(xp.shape[:-2] + (S // N, N, d)).mean(axis=-2)


def reduced_map(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """Attenzione Ridotta: full softmax(Qbar Kbar^T / sqrt(d)) between pooled
    blocks, row-wise, computed with max subtraction. [..., nb, nb]."""
    d = qbar.shape[-1]
    logits = qbar @ np.swapaxes(kbar, -1, -2) / np.sqrt(d)
    e = np.exp(logits - logits.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def cdf_keep(A: np.ndarray, thr: float) -> np.ndarray:
    """CDF Thresholding: per row, keep the smallest set of blocks, taken in
    order of descending probability, whose cumulative mass reaches 1 - thr.

    Block j is kept iff the mass of the blocks before it in that order is
    strictly below 1 - thr (so the first block is always kept). Equal
    probabilities are ordered by ascending block index. thr = 0 keeps all.
    """
    if not 0.0 <= thr < 1.0:
        raise ValueError("thr must lie in [0, 1)")
    if thr == 0.0:
        return np.ones(A.shape, dtype=bool)
    order = np.argsort(-A, axis=-1, kind="stable")
    a_sorted = np.take_along_axis(A, order, axis=-1)
    incl = np.cumsum(a_sorted, axis=-1)
    before = np.concatenate([np.zeros(A.shape[:-1] + (1,)), incl[..., :-1]], axis=-1)
    keep_sorted = before < (1.0 - thr)
    keep = np.empty(A.shape, dtype=bool)
    np.put_along_axis(keep, order, keep_sorted, axis=-1)
    return keep


def block_coords(T: int, Hh: int, Ww: int, P) -> np.ndarray:
    """(t, hp, wp) of every block in fractal order, in block units
    (t // p_t, h // p_h, w // p_w), shape [nb, 3]."""
    pt, ph, pw = tile_shape(P)
    nt, nh, nw = T // pt, Hh // ph, Ww // pw
    b = np.arange(nt * nh * nw)
    return np.stack([b // (nh * nw), (b // nw) % nh, b % nw], axis=1)


# --- Metodologia 3: "Integrazione Ibrida con STA" ---------------------------

def sta_keep(T: int, Hh: int, Ww: int, P, sta) -> np.ndarray:
    """Static sliding-tile window in block units: q-block and k-block are
    paired iff their distance along each of (t, hp, wp) is at most half the
    (odd) window size. (0, 0, 0) is no window. [nb, nb] bool."""
    st, sh, sw = sta
    c = block_coords(T, Hh, Ww, P)
    nb = c.shape[0]
    if (st, sh, sw) == (0, 0, 0):
        return np.zeros((nb, nb), dtype=bool)
    if min(st, sh, sw) < 1 or not (st % 2 and sh % 2 and sw % 2):
        raise ValueError("STA window sizes must be odd and positive")
    diff = np.abs(c[:, None, :] - c[None, :, :])
    return ((diff[..., 0] <= st // 2) & (diff[..., 1] <= sh // 2)
            & (diff[..., 2] <= sw // 2))


def _as_f64(x):
    return widen_bf16(x) if np.asarray(x).dtype == np.uint16 else np.asarray(x, dtype=np.float64)


def pooled_head(x, T, Hh, Ww, P, N):
    """Pooled blocks of one head: natural-order [S, d] -> [nb, d] float64."""
    return pool(flatten(_as_f64(x), fractal_order(T, Hh, Ww, P)), N)


def nabla_mask(q, k, T, Hh, Ww, P, N, thr, sta):
    """The final block mask M = M_nabla OR M_STA for every (batch, head).

    q, k: natural-order [BH, S, d] (bf16 bits as uint16, or floats), handled
    one head at a time. Returns (M, M_nabla, A): bool [BH, nb, nb] masks and
    the float64 reduced map.
    """
    pt, ph, pw = tile_shape(P)
    if N != pt * ph * pw:
        raise ValueError("this reading needs N == p_t * p_h * p_w (one block = one tile)")
    m_sta = sta_keep(T, Hh, Ww, P, sta)
    BH, nb = q.shape[0], q.shape[1] // N
    A = np.empty((BH, nb, nb))
    m_nabla = np.empty((BH, nb, nb), dtype=bool)
    for bh in range(BH):
        A[bh] = reduced_map(pooled_head(q[bh], T, Hh, Ww, P, N),
                            pooled_head(k[bh], T, Hh, Ww, P, N))
        m_nabla[bh] = cdf_keep(A[bh], thr)
    return m_nabla | m_sta[None], m_nabla, A


# --- Espansione + masked exact attention ------------------------------------

def masked_attention(qp, kp, vp, mask, N, rows=None):
    """Exact attention in fractal order with every dropped N x N block at -inf.

    qp, kp, vp: [S, d] float64 (one head, fractal order); mask: [nb, nb] bool.
    rows: fractal-order query positions to compute (default: all).
    Returns [len(rows), d] float64.
    """
    S, d = qp.shape
    rows = np.arange(S) if rows is None else np.asarray(rows)
    out = np.empty((rows.size, vp.shape[-1]))
    qb_of_row = rows // N
    for qb in np.unique(qb_of_row):
        sel = np.nonzero(qb_of_row == qb)[0]
        kept_blocks = np.nonzero(mask[qb])[0]
        cols = (kept_blocks[:, None] * N + np.arange(N)[None, :]).reshape(-1)
        s = qp[rows[sel]] @ kp[cols].T / np.sqrt(d)
        e = np.exp(s - s.max(axis=-1, keepdims=True))
        out[sel] = (e / e.sum(axis=-1, keepdims=True)) @ vp[cols]
    return out


def attention_head(q, k, v, T, Hh, Ww, P, N, mask, tokens=None):
    """One head of the whole path: fractal flatten, masked attention over the
    kept blocks of ``mask`` [nb, nb], inverse flatten.

    q, k, v: natural-order [S, d]. tokens: natural-order query indices to
    compute (default all); each output row is exact on its own, so a sample
    of rows equals the same rows of the full result. Returns [n, d] float64.
    """
    perm = fractal_order(T, Hh, Ww, P)
    qp, kp, vp = (flatten(_as_f64(x), perm) for x in (q, k, v))
    if tokens is None:
        return unflatten(masked_attention(qp, kp, vp, mask, N), perm)
    pos_of = np.empty_like(perm)
    pos_of[perm] = np.arange(perm.size)
    return masked_attention(qp, kp, vp, mask, N, rows=pos_of[np.asarray(tokens)])


def nabla_attention(q, k, v, T, Hh, Ww, P, N, thr, sta, mask=None):
    """Whole path for natural-order [BH, S, d] inputs: mask build (unless
    ``mask`` [BH, nb, nb] is given) then per-head masked attention.
    Returns (O natural order float64 [BH, S, d], mask)."""
    if mask is None:
        mask, _, _ = nabla_mask(q, k, T, Hh, Ww, P, N, thr, sta)
    out = np.stack([attention_head(q[bh], k[bh], v[bh], T, Hh, Ww, P, N, mask[bh])
                    for bh in range(q.shape[0])])
    return out, mask


# --- Gradients of the block-sparse attention (training use) -----------------
# The NABLA page reuses the same block mask when training (pre-training and
# fine-tuning a DiT, "Risultati Sperimentali"), which needs the gradients of
# the masked attention: those of softmax attention with every dropped block at
# -inf. With s = q.k / sqrt(d) on the kept blocks, P = softmax over a row's
# kept keys and O = P V, for a loss with output gradient dO:
#   dV = P^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic = sum_j P_ij dP_ij,
#   dS = P * (dP - D),  dQ = dS K / sqrt(d),  dK = dS^T Q / sqrt(d).

def masked_attention_backward(qp, kp, vp, dop, mask, N, o_stored=None):
    """Gradients of sum(O * dO) for O = masked_attention(qp, kp, vp, mask, N),
    and the rows' natural-log log-sum-exp of the kept scaled scores.

    qp, kp, vp, dop: [S, d] float64 (one head, fractal order); mask [nb, nb].
    o_stored: optional [S, d] fractal-order output as a forward pass stored
    it (for instance rounded to bf16). D_i then sums dO_i * o_stored_i
    instead of dO_i * O_i, as a backward pass that reads its stored output
    does; every other term is unchanged and exact.
    Returns (dq, dk, dv, lse): [S, d] x 3 and [S], fractal order.
    """
    S, d = qp.shape
    scale = 1.0 / np.sqrt(d)
    dq, dk, dv = np.zeros_like(qp), np.zeros_like(kp), np.zeros_like(vp)
    lse = np.empty(S)
    for qb in range(S // N):
        r = slice(qb * N, (qb + 1) * N)
        kept = np.nonzero(mask[qb])[0]
        cols = (kept[:, None] * N + np.arange(N)[None, :]).reshape(-1)
        s = qp[r] @ kp[cols].T * scale
        mx = s.max(axis=-1, keepdims=True)
        e = np.exp(s - mx)
        l = e.sum(axis=-1, keepdims=True)
        p = e / l
        lse[r] = (mx + np.log(l))[:, 0]
        o = p @ vp[cols] if o_stored is None else np.asarray(o_stored, dtype=np.float64)[r]
        dp = dop[r] @ vp[cols].T
        D = (dop[r] * o).sum(axis=-1, keepdims=True)
        ds = p * (dp - D)
        dq[r] = ds @ kp[cols] * scale
        dk[cols] += ds.T @ qp[r] * scale
        dv[cols] += p.T @ dop[r]
    return dq, dk, dv, lse


def masked_attention_backward_blocks(qp, kp, vp, dop, mask, N, qblocks, kblocks):
    """The rows of masked_attention_backward for some blocks only: dq of the
    q-blocks ``qblocks`` and dk, dv of the k-blocks ``kblocks``, from the
    q-blocks involved (those sampled, and those keeping a sampled k-block).
    Returns (dq [len(qblocks), N, d], dk, dv [len(kblocks), N, d], lse
    [len(qblocks), N]), fractal order within each block."""
    S, d = qp.shape
    scale = 1.0 / np.sqrt(d)
    qblocks, kblocks = list(qblocks), list(kblocks)
    dq = np.zeros((len(qblocks), N, d))
    lse = np.zeros((len(qblocks), N))
    dk = np.zeros((len(kblocks), N, d))
    dv = np.zeros((len(kblocks), N, d))
    rows = set(qblocks) | {int(i) for b in kblocks for i in np.nonzero(mask[:, b])[0]}
    for qb in sorted(rows):
        r = slice(qb * N, (qb + 1) * N)
        kept = np.nonzero(mask[qb])[0]
        cols = (kept[:, None] * N + np.arange(N)[None, :]).reshape(-1)
        s = qp[r] @ kp[cols].T * scale
        mx = s.max(axis=-1, keepdims=True)
        e = np.exp(s - mx)
        l = e.sum(axis=-1, keepdims=True)
        p = e / l
        o = p @ vp[cols]
        dp = dop[r] @ vp[cols].T
        ds = p * (dp - (dop[r] * o).sum(axis=-1, keepdims=True))
        if qb in qblocks:
            i = qblocks.index(qb)
            dq[i] = ds @ kp[cols] * scale
            lse[i] = (mx + np.log(l))[:, 0]
        for i, b in enumerate(kblocks):
            pos = np.nonzero(kept == b)[0]
            if pos.size:
                c = slice(int(pos[0]) * N, (int(pos[0]) + 1) * N)
                dk[i] += ds[:, c].T @ qp[r] * scale
                dv[i] += p[:, c].T @ dop[r]
    return dq, dk, dv, lse


def attention_backward_head(q, k, v, do, T, Hh, Ww, P, N, mask, o_stored=None):
    """One head in natural order: fractal flatten, masked_attention_backward,
    inverse flatten. q, k, v, do (and o_stored, if given, a natural-order
    [S, d] stored output): [S, d]. Returns (dq, dk, dv, lse) float64."""
    perm = fractal_order(T, Hh, Ww, P)
    qp, kp, vp, dop = (flatten(_as_f64(x), perm) for x in (q, k, v, do))
    os_p = None if o_stored is None else flatten(np.asarray(o_stored, dtype=np.float64), perm)
    dq, dk, dv, lse = masked_attention_backward(qp, kp, vp, dop, mask, N, o_stored=os_p)
    lse_nat = np.empty_like(lse)
    lse_nat[perm] = lse
    return unflatten(dq, perm), unflatten(dk, perm), unflatten(dv, perm), lse_nat


# --- Block max-pooled attention map (quality signal for a block mask) --------
# The reference target of the page "Veda - Diffusione Video Scalabile tramite
# Attenzione Sparsa Distillata" (gist.science/it/paper/2605.30325), section
# 2.1 ("Costruzione dell'Obiettivo"): the full
# attention matrix, max-pooled over the (query block, key block) regions.

def block_heatmap(q, k, T, Hh, Ww, P, N):
    """H[qb, kb] = max over the N x N block of the full softmax attention
    probabilities (all keys, no mask) of one head, blocks in fractal order.

    q, k: natural-order [S, d]. Returns float64 [nb, nb].
    """
    perm = fractal_order(T, Hh, Ww, P)
    qp, kp = flatten(_as_f64(q), perm), flatten(_as_f64(k), perm)
    S, d = qp.shape
    s = qp @ kp.T / np.sqrt(d)
    p = np.exp(s - s.max(axis=-1, keepdims=True))
    p /= p.sum(axis=-1, keepdims=True)
    nb = S // N
    return p.reshape(nb, N, nb, N).max(axis=(1, 3))


def block_heatmap_rows(q, k, T, Hh, Ww, P, N, qblocks):
    """Rows ``qblocks`` (fractal block ids) of block_heatmap, computed from
    the softmax rows of those blocks' queries only: float64 [len, nb]."""
    perm = fractal_order(T, Hh, Ww, P)
    qp, kp = flatten(_as_f64(q), perm), flatten(_as_f64(k), perm)
    S, d = kp.shape
    nb = S // N
    out = np.empty((len(qblocks), nb))
    for r, b in enumerate(qblocks):
        if not 0 <= b < nb:
            raise IndexError(f"q-block {b} outside [0, {nb})")
        s = qp[b * N:(b + 1) * N] @ kp.T / np.sqrt(d)
        p = np.exp(s - s.max(axis=-1, keepdims=True))
        p /= p.sum(axis=-1, keepdims=True)
        out[r] = p.reshape(N, nb, N).max(axis=(0, 2))
    return out


def heat_recall(H, M):
    """Per q-block row, the share of the row's max-pooled attention (sum of
    H over its key blocks) that the kept blocks of mask M cover; the mean
    over rows. 1.0 = the mask keeps every block that carries attention."""
    H = np.asarray(H, dtype=np.float64)
    return float(np.mean((H * M).sum(axis=-1) / H.sum(axis=-1)))
