"""GPU-vs-oracle comparison rules (test side).

Masks. The CUDA path must keep exactly the oracle's blocks except where the
decision is numerically ambiguous. Block j's decision is "keep iff the mass
ranked before it is < 1 - thr". That mass is uncertain in two ways:

  * the fp32 reduced map differs from the fp64 one by ~1e-6, so a block whose
    cumulative mass lies within MASK_BAND (1e-4) of 1 - thr may flip;
  * blocks whose probabilities agree to within the tie window (relative, per
    row, from the measured logit error; see LOGIT_REL) can be ranked either
    way, so block j's cumulative mass is only known to lie in [c_lo, c_hi],
    the mass of blocks surely above it vs. possibly above it.

A block is ambiguous when that interval, widened by MASK_BAND, straddles
1 - thr. Blocks forced in by the STA window are never ambiguous. In addition,
every row's kept set must hold at least 1 - thr - MASK_BAND of the oracle's
mass.

Outputs. max |gpu - oracle| <= 2e-2 and mean |gpu - oracle| <= 2e-3, with the
oracle's attention evaluated on the GPU's mask (so a band flip tests the
band, not the attention). For a bf16 output the max bound is widened by half
a bf16 unit in the last place of the oracle's value (2^-9 |ref|): no bf16
number can be closer to the exact result than that.
"""
from __future__ import annotations

import numpy as np
import torch

MASK_BAND = 1e-4
# Ranking ties. The GPU's reduced-map logits carry an error of at most
# 2.0e-6 of L1 = sum_c |qbar_c kbar_c| / sqrt(d) (measured on two heads each
# of the HunyuanVideo-like, 8k and two scale-4 sweep workloads: three TF32
# products of a hi/lo split, accumulated in fp32); LOGIT_REL doubles that. Two
# probabilities of one row can then swap order only if their ratio is within
# 2 * LOGIT_REL * (the row's largest L1) of 1, plus the fp32 exponential and
# normalisation (EXP_REL), or if they differ by less than the 2^-30 mass
# quantum the kernel ranks by (TIE_ABS).
LOGIT_REL = 4e-6
EXP_REL = 2.0 ** -21
TIE_ABS = 2.0 ** -30
TIE_REL = 1e-4  # the fallback when no pooled means are given
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3


def lists_to_mask(cnt: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """[BH, nb] counts + [BH, nb, nb] ascending lists -> bool [BH, nb, nb]."""
    BH, nb = cnt.shape
    valid = np.arange(nb)[None, None, :] < cnt[..., None]
    ids = np.where(valid, idx, nb)
    m = np.zeros((BH, nb, nb + 1), dtype=bool)
    np.put_along_axis(m, ids.astype(np.int64), True, axis=-1)
    return m[..., :nb]


def tie_rel_rows(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """Per-row relative tie window from the pooled means of one or more
    heads ([..., nb, d] each): 2 LOGIT_REL max_j L1[i, j] + EXP_REL."""
    qa, ka = np.abs(qbar), np.abs(kbar)
    L1 = np.matmul(qa, np.swapaxes(ka, -1, -2)) / np.sqrt(qbar.shape[-1])
    return 2.0 * LOGIT_REL * L1.max(axis=-1) + EXP_REL


def ambiguous(A: np.ndarray, thr: float, band: float = MASK_BAND,
              rel=TIE_REL) -> np.ndarray:
    """Bool mask of blocks whose keep decision the tolerances leave open.
    rel: a relative tie window, scalar or one per row (shape A.shape[:-1])."""
    if thr == 0.0:
        return np.zeros(A.shape, dtype=bool)
    shape = A.shape
    a = torch.from_numpy(np.ascontiguousarray(A.reshape(-1, shape[-1])))
    r = torch.from_numpy(np.broadcast_to(np.asarray(rel, dtype=np.float64),
                                         shape[:-1]).reshape(-1, 1).copy())
    asc, _ = torch.sort(a, dim=-1)
    n = a.shape[-1]
    top = torch.cumsum(torch.flip(asc, dims=[-1]), dim=-1)
    cs = torch.cat([torch.zeros(a.shape[0], 1, dtype=a.dtype), top], dim=-1)  # sum of k largest
    n_gt = n - torch.searchsorted(asc, a * (1 + r) + TIE_ABS, right=True)
    n_ge = n - torch.searchsorted(asc, a * (1 - r) - TIE_ABS, right=False)
    c_lo = torch.gather(cs, 1, n_gt)
    c_hi = torch.gather(cs, 1, n_ge) - a
    target = 1.0 - thr
    sure_keep = c_hi < target - band
    sure_drop = c_lo >= target + band
    return (~(sure_keep | sure_drop)).numpy().reshape(shape)


def compare_masks(gpu: np.ndarray, M: np.ndarray, M_nabla: np.ndarray, A: np.ndarray,
                  thr: float, rel=TIE_REL) -> dict:
    """Returns counts; 'bad' must be 0 and 'min_mass_margin' >= -MASK_BAND.
    rel: the tie window (tie_rel_rows of the heads' pooled means)."""
    sta_only = M & ~M_nabla
    amb = ambiguous(A, thr, rel=rel) & ~sta_only
    mismatch = gpu != M
    bad = mismatch & ~amb
    kept_mass = (A * gpu).sum(-1)
    return {
        "bad": int(bad.sum()),
        "band_flips": int((mismatch & amb).sum()),
        "band_blocks": int(amb.sum()),
        "min_mass_margin": float((kept_mass - (1.0 - thr)).min()) if thr > 0 else 0.0,
        "sta_missing": int((sta_only & ~gpu).sum()),
        "kept": int(gpu.sum()),
        "density": float(gpu.mean()),
    }


def max_band_flips(rows: int) -> int:
    """Flips inside the band are allowed, but they must stay rare: a flip
    needs the GPU's fp32 mass of a block to land on the other side of
    1 - thr from the fp64 one, within MASK_BAND. At most one row in a
    hundred (and at least 4 flips in all)."""
    return max(4, rows // 100)


def out_errors(gpu: np.ndarray, ref: np.ndarray) -> tuple:
    err = np.abs(np.asarray(gpu, dtype=np.float64) - ref)
    return float(err.max()), float(err.mean())


def out_check(gpu: np.ndarray, ref: np.ndarray, bf16_out: bool) -> dict:
    """Max/mean errors and whether they meet the bar (see module docstring)."""
    err = np.abs(np.asarray(gpu, dtype=np.float64) - ref)
    allowed = OUT_MAX_ABS + (np.abs(ref) * 2.0 ** -9 if bf16_out else 0.0)
    ok = bool((err <= allowed).all()) and float(err.mean()) <= OUT_MEAN_ABS
    return {"ok": ok, "max": float(err.max()), "mean": float(err.mean()),
            "worst_excess": float((err - allowed).max())}
