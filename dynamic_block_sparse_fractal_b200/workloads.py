"""Seeded synthetic video-attention workloads.

This module only makes inputs. It computes no step of the attention method:
no token reordering, no pooling, no masking, no attention. Both the CUDA path
and the CPU oracle consume the tensors it returns, bit for bit.

Recipe (the pages fix none of these constants; this is the stated reading):

* Token positions are normalised, x = (t/T, h/Hh, w/Ww); tokens are stored in
  the natural video order (t outermost, then h, then w).
* From a PCG64 generator seeded per workload, draw 16 frequency vectors
  w_f ~ N(0, sigma^2 I_3) (cycles per unit length) and 16 phases
  phi_f ~ U[0, 2 pi); per head, from that head's own seeded generator, an
  amplitude matrix A_h ~ N(0, 2 v / 16) of shape (d, 16), so each channel of
  F_h below has variance v.
* F_h(x)_c = sum_f A_h[c, f] * cos(2 pi w_f . x + phi_f).
* Q = N(0,1) + scale * F_h(x) and K = N(0,1) + scale * F_h(x) share F_h, so
  q . k is large for nearby positions and attention is spatially local.
  V = N(0,1) + scale * F_h(x) or plain N(0,1), per workload.
* Everything is rounded to bf16 (round to nearest even) and returned as the
  raw uint16 bit patterns, shape [B, H, T*Hh*Ww, d].

Two constants are calibrated: sigma = 1.5 keeps the field smooth over several
8 x 8 patches (attention is local in space; at a fixed place it reaches across
many frames), and v = 0.265 sets the logit scale so that the 126,720-token
HunyuanVideo-like workload at thr = 0.1 reaches 90% block sparsity (90.6%;
v = 0.26 gave 89.9%, v = 0.27 gives 91.3%).
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Tuple

import numpy as np

N_FEATURES = 16
# Bandwidth of the positional field, in cycles per unit of normalised position.
SIGMA = 1.5
# Per-channel variance of the positional field F_h (before ``scale``).
FIELD_VAR = 0.265


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, method parameters and generator knobs."""

    name: str
    B: int
    H: int
    d: int
    T: int
    Hh: int
    Ww: int
    P: int = 8
    N: int = 64
    thr: float = 0.1
    sta: Tuple[int, int, int] = (0, 0, 0)
    scale: float = 2.0
    v_positional: bool = False
    seed: int = 0
    sigma: float = SIGMA
    field_var: float = FIELD_VAR
    tile: Optional[Tuple[int, int, int]] = None  # block shape (pt, ph, pw); None = (1, P, P)

    @property
    def block(self):
        """The block shape as the oracle takes it: the tile, or the patch edge P."""
        return self.tile if self.tile is not None else self.P

    @property
    def S(self) -> int:
        return self.T * self.Hh * self.Ww

    @property
    def nb(self) -> int:
        return self.S // self.N

    @property
    def BH(self) -> int:
        return self.B * self.H

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def describe(self) -> dict:
        return {
            "workload": self.name, "B": self.B, "H": self.H, "d": self.d,
            "grid": [self.T, self.Hh, self.Ww], "tokens": self.S, "P": self.P,
            "N": self.N, "thr": self.thr, "sta": list(self.sta),
            "pos_scale": self.scale, "seed": self.seed,
            "tile": list(self.tile) if self.tile is not None else [1, self.P, self.P],
        }


TINY = Workload("tiny_1x2x256x64", B=1, H=2, d=64, T=4, Hh=8, Ww=8, thr=0.1,
                v_positional=True, seed=1000)
W8K = Workload("8k_1x12x8192x128_sta3", B=1, H=12, d=128, T=8, Hh=32, Ww=32,
               thr=0.2, sta=(3, 3, 3), v_positional=True, seed=1001)
WAN = Workload("wan_1x12x37632x128_sta3", B=1, H=12, d=128, T=21, Hh=32,
               Ww=56, thr=0.1, sta=(3, 3, 3), seed=1002)
HUNYUAN = Workload("hunyuan_1x24x126720x128", B=1, H=24, d=128, T=33, Hh=48,
                   Ww=80, thr=0.1, seed=1003)
SWEEP_BASE = Workload("sweep_1x24x61440x128", B=1, H=24, d=128, T=16, Hh=48,
                      Ww=80, thr=0.1, seed=1004)

SWEEP_THR = (0.0, 0.01, 0.05, 0.1, 0.2, 0.3)
SWEEP_STA = ((0, 0, 0), (3, 3, 3))
SWEEP_SCALE = (0.0, 1.0, 2.0, 4.0)


def sweep(k: int) -> Workload:
    """The k-th variant of the sparsity sweep (thr x STA x positional scale)."""
    n_thr, n_sta, n_sc = len(SWEEP_THR), len(SWEEP_STA), len(SWEEP_SCALE)
    if not 0 <= k < n_thr * n_sta * n_sc:
        raise IndexError(k)
    i_thr, rest = k % n_thr, k // n_thr
    i_sta, i_sc = rest % n_sta, rest // n_sta
    thr, sta, sc = SWEEP_THR[i_thr], SWEEP_STA[i_sta], SWEEP_SCALE[i_sc]
    return SWEEP_BASE.with_(
        name=f"sweep_1x24x61440x128_thr{thr}_sta{sta[0]}_s{sc:g}",
        thr=thr, sta=sta, scale=sc, seed=SWEEP_BASE.seed + 10 * k)


N_SWEEP = len(SWEEP_THR) * len(SWEEP_STA) * len(SWEEP_SCALE)

# The same inputs with three-dimensional blocks (head-aware tile shapes):
# pt frames x ph rows x pw columns, pt*ph*pw = 64.
W8K_T248 = dataclasses.replace(W8K, name="8k_1x12x8192x128_sta3_tile2x4x8", tile=(2, 4, 8))
W8K_T444 = dataclasses.replace(W8K, name="8k_1x12x8192x128_sta3_tile4x4x4", tile=(4, 4, 4))
HUNYUAN_T1416 = dataclasses.replace(HUNYUAN, name="hunyuan_1x24x126720x128_tile1x4x16",
                                    tile=(1, 4, 16))

WORKLOADS = {w.name: w for w in (TINY, W8K, WAN, HUNYUAN, W8K_T248, W8K_T444, HUNYUAN_T1416)}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns exactly to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _positional_basis(w: Workload, rng: np.random.Generator) -> np.ndarray:
    """cos(2 pi w_f . x + phi_f) for every token, shape [S, 16], float32."""
    omega = rng.standard_normal((N_FEATURES, 3)) * w.sigma
    phi = rng.uniform(0.0, 2.0 * np.pi, N_FEATURES)
    t = np.arange(w.T, dtype=np.float64) / w.T
    h = np.arange(w.Hh, dtype=np.float64) / w.Hh
    x = np.arange(w.Ww, dtype=np.float64) / w.Ww
    # Separable phase: omega_t * t + omega_h * h + omega_w * x, natural order.
    ph = (omega[:, 0][:, None, None, None] * t[None, :, None, None]
          + omega[:, 1][:, None, None, None] * h[None, None, :, None]
          + omega[:, 2][:, None, None, None] * x[None, None, None, :])
    ph = 2.0 * np.pi * ph + phi[:, None, None, None]
    basis = np.cos(ph).reshape(N_FEATURES, w.S).T
    return np.ascontiguousarray(basis, dtype=np.float32)


def make_inputs(w: Workload, heads: Optional[range] = None):
    """Return (q, k, v) bf16 bit arrays of shape [B, H, S, d] (uint16).

    ``heads`` restricts generation to a subset of the B*H flattened heads
    (returned with shape [len(heads), S, d]); the values of a head do not
    depend on which other heads are generated.
    """
    rng = np.random.Generator(np.random.PCG64(w.seed))
    basis = _positional_basis(w, rng)
    head_seeds = rng.integers(0, 2**63 - 1, size=w.BH)
    sel = range(w.BH) if heads is None else heads
    out = [np.empty((len(sel), w.S, w.d), dtype=np.uint16) for _ in range(3)]
    for i, bh in enumerate(sel):
        hr = np.random.Generator(np.random.PCG64(int(head_seeds[bh])))
        amp = (hr.standard_normal((w.d, N_FEATURES))
               * np.sqrt(2.0 * w.field_var / N_FEATURES)).astype(np.float32)
        field = basis @ amp.T  # [S, d]
        if w.scale != 1.0:
            field *= np.float32(w.scale)
        for j in range(3):
            x = hr.standard_normal((w.S, w.d), dtype=np.float32)
            if j < 2 or w.v_positional:
                x += field
            out[j][i] = f32_to_bf16_bits(x)
    if heads is None:
        return tuple(o.reshape(w.B, w.H, w.S, w.d) for o in out)
    return tuple(out)


def make_output_grad(w: Workload, heads: Optional[range] = None) -> np.ndarray:
    """A seeded upstream gradient dO for the workload's output: i.i.d. standard
    normal values as bf16 bits, [B, H, S, d] (or [len(heads), S, d]); a head's
    values do not depend on which other heads are generated."""
    rng = np.random.Generator(np.random.PCG64(w.seed ^ 0x5EED_0D0))
    head_seeds = rng.integers(0, 2**63 - 1, size=w.BH)
    sel = range(w.BH) if heads is None else heads
    out = np.empty((len(sel), w.S, w.d), dtype=np.uint16)
    for i, bh in enumerate(sel):
        hr = np.random.Generator(np.random.PCG64(int(head_seeds[bh])))
        out[i] = f32_to_bf16_bits(hr.standard_normal((w.S, w.d), dtype=np.float32))
    return out.reshape(w.B, w.H, w.S, w.d) if heads is None else out


def drift_inputs(w: Workload, tensors, eps: float = 0.05, seed: int = 1):
    """The next denoising step's inputs, as a slow drift of ``tensors``
    (bf16 bit arrays of any shape): each value plus eps times a seeded
    standard normal draw, rounded to bf16. Returns new bit arrays."""
    rng = np.random.Generator(np.random.PCG64((w.seed << 8) ^ seed))
    out = []
    for t in tensors:
        x = bf16_bits_to_f32(t) + np.float32(eps) * rng.standard_normal(t.shape, dtype=np.float32)
        out.append(f32_to_bf16_bits(x).reshape(t.shape))
    return tuple(out)
