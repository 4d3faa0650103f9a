"""Python binding of libsparse_attn.so (include/sparse_attn.h).

Argument marshalling only: every step of the attention path runs in the
library's CUDA kernels. PyTorch provides device memory and streams. If the
library has not been built, every call raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libsparse_attn.so")

SA_OK = 0
SA_ERR_INVALID_ARG = 1
SA_ERR_UNSUPPORTED = 2
SA_ERR_WORKSPACE = 3
SA_ERR_CUDA = 4
SA_ERR_DEVICE_TIMEOUT = 5
SA_DEBUG_STALL_LOADER = 1

SYMBOLS = (
    "sparse_attn_workspace_size", "sparse_attn_plan", "sparse_attn_fwd",
    "sparse_attn_permute", "sparse_attn_get_mask", "sparse_attn_tile_blocks",
    "sparse_attn_check", "sparse_attn_forward_noalloc", "sparse_attn_status_string",
    "sparse_attn_workspace_size_heads", "sparse_attn_plan_heads", "sparse_attn_fwd_heads",
    "sparse_attn_check_heads", "sparse_attn_heads_run", "sparse_attn_block_heatmap",
    "sparse_attn_block_heatmap_scratch_size", "sparse_attn_fwd_lse",
    "sparse_attn_bwd_scratch_size", "sparse_attn_bwd", "sparse_attn_graph_create",
    "sparse_attn_graph_launch", "sparse_attn_graph_destroy", "sparse_attn_fwd_lse_heads",
    "sparse_attn_bwd_scratch_size_heads", "sparse_attn_bwd_heads",
    "sparse_attn_block_heatmap_scratch_size_heads", "sparse_attn_block_heatmap_heads",
    "sparse_attn_plan_profile", "sparse_attn_plan_stage_name",
    "sparse_attn_token_entropy", "sparse_attn_plan_radius",
)
NOALLOC_SCRATCH_BYTES = 64 << 20


class SaDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int),
                ("Hh", ctypes.c_int), ("Ww", ctypes.c_int), ("d", ctypes.c_int),
                ("N", ctypes.c_int), ("P", ctypes.c_int), ("thr", ctypes.c_float),
                ("sta_t", ctypes.c_int), ("sta_h", ctypes.c_int), ("sta_w", ctypes.c_int),
                ("out_fp32", ctypes.c_int), ("debug_flags", ctypes.c_int),
                ("pt", ctypes.c_int), ("ph", ctypes.c_int), ("pw", ctypes.c_int)]


class SaRadius(ctypes.Structure):
    _fields_ = [("tau", ctypes.c_float), ("gamma", ctypes.c_float), ("vote_min", ctypes.c_int)]


class SaMaskViews(ctypes.Structure):
    _fields_ = [("qbar", ctypes.c_void_p), ("kbar", ctypes.c_void_p), ("cnt", ctypes.c_void_p),
                ("idx", ctypes.c_void_p), ("tile_cnt", ctypes.c_void_p),
                ("tile_idx", ctypes.c_void_p), ("nb", ctypes.c_int), ("ntile", ctypes.c_int),
                ("logits", ctypes.c_void_p), ("logits_ld", ctypes.c_int)]


class SparseAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing; build it with "
                "`python -m dynamic_block_sparse_fractal_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        dp = ctypes.POINTER(SaDesc)
        L.sparse_attn_workspace_size.argtypes = [dp, ctypes.POINTER(sz)]
        L.sparse_attn_plan.argtypes = [dp, vp, vp, vp, sz, vp]
        L.sparse_attn_fwd.argtypes = [dp, vp, vp, vp, vp, sz, vp, vp]
        L.sparse_attn_permute.argtypes = [dp, vp, vp, i32, vp]
        L.sparse_attn_get_mask.argtypes = [dp, vp, sz, ctypes.POINTER(SaMaskViews)]
        L.sparse_attn_tile_blocks.argtypes = [dp, i32, ctypes.POINTER(i32), ctypes.POINTER(i32)]
        L.sparse_attn_check.argtypes = [dp, vp, sz, vp]
        L.sparse_attn_forward_noalloc.argtypes = [dp, vp, vp, vp, vp, vp]
        ip = ctypes.POINTER(i32)
        L.sparse_attn_workspace_size_heads.argtypes = [dp, ip, ctypes.POINTER(sz)]
        L.sparse_attn_plan_heads.argtypes = [dp, ip, vp, vp, vp, sz, vp]
        L.sparse_attn_fwd_heads.argtypes = [dp, ip, vp, vp, vp, vp, sz, vp, vp]
        L.sparse_attn_check_heads.argtypes = [dp, ip, vp, sz, vp]
        L.sparse_attn_heads_run.argtypes = [dp, ip, i32, dp, ip, ctypes.POINTER(sz),
                                            ctypes.POINTER(sz)]
        L.sparse_attn_plan_profile.argtypes = [dp, vp, vp, vp, sz, i32,
                                               ctypes.POINTER(ctypes.c_float), i32, ip, vp]
        L.sparse_attn_token_entropy.argtypes = [dp, vp, vp, vp, sz, vp, vp]
        L.sparse_attn_plan_radius.argtypes = [dp, ctypes.POINTER(SaRadius), vp, vp, sz, vp]
        L.sparse_attn_status_string.argtypes = [i32]
        L.sparse_attn_status_string.restype = ctypes.c_char_p
        L.sparse_attn_plan_stage_name.argtypes = [i32]
        L.sparse_attn_plan_stage_name.restype = ctypes.c_char_p
        for name in SYMBOLS:
            if name not in ("sparse_attn_status_string", "sparse_attn_plan_stage_name"):
                getattr(L, name).restype = i32
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().sparse_attn_status_string(int(status)).decode()


def _ok(status: int, what: str) -> None:
    if status != SA_OK:
        raise SparseAttnError(status, what)


def make_desc(B: int, H: int, T: int, Hh: int, Ww: int, d: int, thr: float,
              sta=(0, 0, 0), N: int = 64, P: int = 8, out_fp32: bool = False,
              debug_flags: int = 0, tile=None) -> SaDesc:
    """tile: block shape (pt, ph, pw) with pt*ph*pw == N, or None for the
    P x P patch of one frame."""
    pt, ph, pw = (0, 0, 0) if tile is None else (int(v) for v in tile)
    return SaDesc(B, H, T, Hh, Ww, d, N, P, float(thr), int(sta[0]), int(sta[1]), int(sta[2]),
                  int(bool(out_fp32)), int(debug_flags), pt, ph, pw)


def desc_for(w, out_fp32: bool = False, debug_flags: int = 0) -> SaDesc:
    """Descriptor of a workload from ``workloads``."""
    return make_desc(w.B, w.H, w.T, w.Hh, w.Ww, w.d, w.thr, w.sta, w.N, w.P, out_fp32,
                     debug_flags, getattr(w, "tile", None))


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t: Optional[torch.Tensor]) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _check_qkv(desc: SaDesc, *ts: torch.Tensor) -> None:
    S = desc.T * desc.Hh * desc.Ww
    for t in ts:
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors")
        if tuple(t.shape) != (desc.B, desc.H, S, desc.d):
            raise ValueError(f"expected shape {(desc.B, desc.H, S, desc.d)}, got {tuple(t.shape)}")


def workspace_size(desc: SaDesc) -> int:
    n = ctypes.c_size_t(0)
    _ok(lib().sparse_attn_workspace_size(ctypes.byref(desc), ctypes.byref(n)), "workspace_size")
    return n.value


def alloc_workspace(desc: SaDesc, device=None) -> torch.Tensor:
    return torch.empty(workspace_size(desc), dtype=torch.uint8,
                       device=device if device is not None else "cuda")


def plan(desc: SaDesc, q: torch.Tensor, k: torch.Tensor, workspace: torch.Tensor,
         stream=None) -> None:
    _check_qkv(desc, q, k)
    _ok(lib().sparse_attn_plan(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(workspace),
                               workspace.numel(), _stream(stream)), "plan")


def token_entropy(desc: SaDesc, q: torch.Tensor, k: torch.Tensor, workspace: torch.Tensor,
                  entropy: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Entropy (nats) of every query's full attention row: fp32 [B, H, S]."""
    _check_qkv(desc, q, k)
    if entropy is None:
        entropy = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    if entropy.dtype != torch.float32 or entropy.shape != q.shape[:3] or \
            not entropy.is_contiguous():
        raise ValueError("entropy must be a contiguous float32 tensor shaped [B, H, S]")
    _ok(lib().sparse_attn_token_entropy(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(workspace),
                                        workspace.numel(), _ptr(entropy), _stream(stream)),
        "token_entropy")
    return entropy


def plan_radius(desc: SaDesc, tau: float, gamma: float, vote_min: int, entropy: torch.Tensor,
                workspace: torch.Tensor, stream=None) -> None:
    """Token Radius Attention block mask from per-token entropies (fp32
    [B, H, S], natural order) into ``workspace``, in sparse_attn_plan's format."""
    if entropy.dtype != torch.float32 or not entropy.is_contiguous() or \
            entropy.numel() != desc.B * desc.H * desc.T * desc.Hh * desc.Ww:
        raise ValueError("entropy must be a contiguous float32 tensor shaped [B, H, S]")
    r = SaRadius(float(tau), float(gamma), int(vote_min))
    _ok(lib().sparse_attn_plan_radius(ctypes.byref(desc), ctypes.byref(r), _ptr(entropy),
                                      _ptr(workspace), workspace.numel(), _stream(stream)),
        "plan_radius")


def plan_profile(desc: SaDesc, q: torch.Tensor, k: torch.Tensor, workspace: torch.Tensor,
                 reps: int = 5, stream=None) -> dict:
    """Mean device time (µs) of each stage of the plan over ``reps`` plans
    (blocks until they finish): {stage name: µs}."""
    _check_qkv(desc, q, k)
    cap = 16
    us = (ctypes.c_float * cap)()
    n = ctypes.c_int(0)
    _ok(lib().sparse_attn_plan_profile(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(workspace),
                                       workspace.numel(), int(reps), us, cap, ctypes.byref(n),
                                       _stream(stream)), "plan_profile")
    return {lib().sparse_attn_plan_stage_name(i).decode(): float(us[i]) for i in range(n.value)}


def fwd(desc: SaDesc, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
        workspace: torch.Tensor, out: torch.Tensor, stream=None) -> torch.Tensor:
    _check_qkv(desc, q, k, v)
    want = torch.float32 if desc.out_fp32 else torch.bfloat16
    if out.dtype != want or out.shape != q.shape or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous {want} tensor shaped like q")
    _ok(lib().sparse_attn_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(workspace),
                              workspace.numel(), _ptr(out), _stream(stream)), "fwd")
    return out


def permute(desc: SaDesc, x: torch.Tensor, y: torch.Tensor, inverse: bool = False,
            stream=None) -> torch.Tensor:
    _check_qkv(desc, x, y)
    _ok(lib().sparse_attn_permute(ctypes.byref(desc), _ptr(x), _ptr(y), int(inverse),
                                  _stream(stream)), "permute")
    return y


def forward_noalloc(desc: SaDesc, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                    out: torch.Tensor, stream=None) -> torch.Tensor:
    """Plan + forward with the library's built-in workspace (for callers that
    cannot allocate device memory); see include/sparse_attn.h."""
    _check_qkv(desc, q, k, v)
    _ok(lib().sparse_attn_forward_noalloc(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v),
                                          _ptr(out), _stream(stream)), "forward_noalloc")
    return out


def check(desc: SaDesc, workspace: torch.Tensor, stream=None) -> int:
    """Synchronises the stream; returns the status (SA_OK or an error code)."""
    return lib().sparse_attn_check(ctypes.byref(desc), _ptr(workspace), workspace.numel(),
                                   _stream(stream))


def fwd_lse(desc: SaDesc, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
            workspace: torch.Tensor, out: torch.Tensor, lse: torch.Tensor,
            stream=None) -> torch.Tensor:
    """fwd that also writes each query row's log-sum-exp (fp32 [B, H, S])."""
    _check_qkv(desc, q, k, v)
    want = torch.float32 if desc.out_fp32 else torch.bfloat16
    if out.dtype != want or out.shape != q.shape or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous {want} tensor shaped like q")
    if lse.dtype != torch.float32 or tuple(lse.shape) != tuple(q.shape[:3]) or \
            not lse.is_contiguous():
        raise ValueError(f"lse must be a contiguous float32 tensor of shape {tuple(q.shape[:3])}")
    _ok(lib().sparse_attn_fwd_lse(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(workspace),
                                  ctypes.c_size_t(workspace.numel()), _ptr(out), _ptr(lse),
                                  _stream(stream)), "fwd_lse")
    return out


def bwd_scratch_size(desc: SaDesc) -> int:
    n = ctypes.c_size_t(0)
    _ok(lib().sparse_attn_bwd_scratch_size(ctypes.byref(desc), ctypes.byref(n)),
        "bwd_scratch_size")
    return n.value


def bwd(desc: SaDesc, q, k, v, out, dout, lse, workspace, dq=None, dk=None, dv=None,
        scratch=None, stream=None):
    """Gradients (dq, dk, dv) of sum(out * dout) over the planned mask; see
    include/sparse_attn.h. Allocates the outputs and the scratch when None."""
    _check_qkv(desc, q, k, v, dout)
    want = torch.float32 if desc.out_fp32 else torch.bfloat16
    if out.dtype != want or out.shape != q.shape or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous {want} tensor shaped like q")
    if lse.dtype != torch.float32 or tuple(lse.shape) != tuple(q.shape[:3]) or \
            not lse.is_contiguous():
        raise ValueError(f"lse must be a contiguous float32 tensor of shape {tuple(q.shape[:3])}")
    grads = []
    for g in (dq, dk, dv):
        if g is None:
            g = torch.empty(q.shape, dtype=want, device=q.device)
        if g.dtype != want or g.shape != q.shape or not g.is_contiguous():
            raise ValueError(f"gradients must be contiguous {want} tensors shaped like q")
        grads.append(g)
    if scratch is None:
        scratch = torch.empty(bwd_scratch_size(desc), dtype=torch.uint8, device=q.device)
    _ok(lib().sparse_attn_bwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                              _ptr(dout), _ptr(lse), _ptr(workspace),
                              ctypes.c_size_t(workspace.numel()), _ptr(grads[0]), _ptr(grads[1]),
                              _ptr(grads[2]), _ptr(scratch), ctypes.c_size_t(scratch.numel()),
                              _stream(stream)), "bwd")
    return tuple(grads)


def heatmap_scratch_size(desc: SaDesc) -> int:
    n = ctypes.c_size_t(0)
    _ok(lib().sparse_attn_block_heatmap_scratch_size(ctypes.byref(desc), ctypes.byref(n)),
        "block_heatmap_scratch_size")
    return n.value


def block_heatmap(desc: SaDesc, q: torch.Tensor, k: torch.Tensor, workspace: torch.Tensor,
                  heat: Optional[torch.Tensor] = None, scratch: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    """Exact block max-pooled full-attention map [B*H, nb, nb] (fp32, fractal
    block order); see include/sparse_attn.h. ``scratch``: a uint8 device
    buffer of heatmap_scratch_size(desc) bytes (allocated when None)."""
    _check_qkv(desc, q, k)
    nb = desc.T * desc.Hh * desc.Ww // desc.N
    shape = (desc.B * desc.H, nb, nb)
    if heat is None:
        heat = torch.empty(shape, dtype=torch.float32, device=q.device)
    if heat.dtype != torch.float32 or tuple(heat.shape) != shape or not heat.is_contiguous():
        raise ValueError(f"heat must be a contiguous float32 tensor of shape {shape}")
    if scratch is None:
        scratch = torch.empty(heatmap_scratch_size(desc), dtype=torch.uint8, device=q.device)
    _ok(lib().sparse_attn_block_heatmap(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(workspace),
                                        ctypes.c_size_t(workspace.numel()), _ptr(heat),
                                        _ptr(scratch), ctypes.c_size_t(scratch.numel()),
                                        _stream(stream)),
        "block_heatmap")
    return heat


def tile_blocks(desc: SaDesc, tile: int) -> Tuple[int, int]:
    a, b = ctypes.c_int(0), ctypes.c_int(0)
    _ok(lib().sparse_attn_tile_blocks(ctypes.byref(desc), int(tile), ctypes.byref(a),
                                      ctypes.byref(b)), "tile_blocks")
    return a.value, b.value


def get_mask(desc: SaDesc, workspace: torch.Tensor) -> dict:
    """Tensor views (no copies) of the planned lists inside ``workspace``."""
    v = SaMaskViews()
    _ok(lib().sparse_attn_get_mask(ctypes.byref(desc), _ptr(workspace), workspace.numel(),
                                   ctypes.byref(v)), "get_mask")
    base = workspace.data_ptr()
    BH, nb, nt, d = desc.B * desc.H, v.nb, v.ntile, desc.d

    def view(ptr, count, dtype, shape):
        off = ptr - base
        nbytes = count * torch.tensor([], dtype=dtype).element_size()
        return workspace[off:off + nbytes].view(dtype).view(*shape)

    return {
        "nb": nb, "ntile": nt,
        "qbar": view(v.qbar, BH * nb * d, torch.float32, (BH, nb, d)),
        "kbar": view(v.kbar, BH * nb * d, torch.float32, (BH, nb, d)),
        "cnt": view(v.cnt, BH * nb, torch.int32, (BH, nb)),
        "idx": view(v.idx, BH * nb * nb, torch.int32, (BH, nb, nb)),
        "tile_cnt": view(v.tile_cnt, BH * nt, torch.int32, (BH, nt)),
        "tile_idx": view(v.tile_idx, BH * nt * nb, torch.int32, (BH, nt, nb)),
        "logits": view(v.logits, BH * nb * v.logits_ld, torch.float32,
                       (BH, nb, v.logits_ld))[:, :, :nb],
    }


# ---- per-head block shapes (head-aware tiling) -------------------------------

def _tiles_array(tiles):
    flat = [int(v) for t in tiles for v in t]
    return (ctypes.c_int * len(flat))(*flat)


def workspace_size_heads(desc: SaDesc, tiles) -> int:
    n = ctypes.c_size_t(0)
    _ok(lib().sparse_attn_workspace_size_heads(ctypes.byref(desc), _tiles_array(tiles),
                                               ctypes.byref(n)), "workspace_size_heads")
    return n.value


def plan_heads(desc: SaDesc, tiles, q, k, workspace, stream=None) -> None:
    _check_qkv(desc, q, k)
    _ok(lib().sparse_attn_plan_heads(ctypes.byref(desc), _tiles_array(tiles), _ptr(q), _ptr(k),
                                     _ptr(workspace), workspace.numel(), _stream(stream)),
        "plan_heads")


def fwd_heads(desc: SaDesc, tiles, q, k, v, workspace, out, stream=None):
    _check_qkv(desc, q, k, v)
    want = torch.float32 if desc.out_fp32 else torch.bfloat16
    if out.dtype != want or out.shape != q.shape or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous {want} tensor shaped like q")
    _ok(lib().sparse_attn_fwd_heads(ctypes.byref(desc), _tiles_array(tiles), _ptr(q), _ptr(k),
                                    _ptr(v), _ptr(workspace), workspace.numel(), _ptr(out),
                                    _stream(stream)), "fwd_heads")
    return out


def check_heads(desc: SaDesc, tiles, workspace, stream=None) -> int:
    return lib().sparse_attn_check_heads(ctypes.byref(desc), _tiles_array(tiles),
                                         _ptr(workspace), workspace.numel(), _stream(stream))


def fwd_lse_heads(desc: SaDesc, tiles, q, k, v, workspace, out, lse, stream=None):
    _check_qkv(desc, q, k, v)
    if lse.dtype != torch.float32 or tuple(lse.shape) != tuple(q.shape[:3]) or \
            not lse.is_contiguous():
        raise ValueError(f"lse must be a contiguous float32 tensor of shape {tuple(q.shape[:3])}")
    _ok(lib().sparse_attn_fwd_lse_heads(ctypes.byref(desc), _tiles_array(tiles), _ptr(q), _ptr(k),
                                        _ptr(v), _ptr(workspace),
                                        ctypes.c_size_t(workspace.numel()), _ptr(out), _ptr(lse),
                                        _stream(stream)), "fwd_lse_heads")
    return out


def bwd_heads(desc: SaDesc, tiles, q, k, v, out, dout, lse, workspace, stream=None):
    """(dq, dk, dv) with per-head block shapes; see include/sparse_attn.h."""
    _check_qkv(desc, q, k, v, dout)
    want = torch.float32 if desc.out_fp32 else torch.bfloat16
    grads = [torch.empty(q.shape, dtype=want, device=q.device) for _ in range(3)]
    n = ctypes.c_size_t(0)
    _ok(lib().sparse_attn_bwd_scratch_size_heads(ctypes.byref(desc), _tiles_array(tiles),
                                                 ctypes.byref(n)), "bwd_scratch_size_heads")
    scratch = torch.empty(n.value, dtype=torch.uint8, device=q.device)
    _ok(lib().sparse_attn_bwd_heads(ctypes.byref(desc), _tiles_array(tiles), _ptr(q), _ptr(k),
                                    _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(workspace),
                                    ctypes.c_size_t(workspace.numel()), _ptr(grads[0]),
                                    _ptr(grads[1]), _ptr(grads[2]), _ptr(scratch),
                                    ctypes.c_size_t(scratch.numel()), _stream(stream)),
        "bwd_heads")
    return tuple(grads)


def block_heatmap_heads(desc: SaDesc, tiles, q, k, workspace, stream=None) -> torch.Tensor:
    """The block max-pooled map [B*H, nb, nb] with per-head block shapes."""
    _check_qkv(desc, q, k)
    nb = desc.T * desc.Hh * desc.Ww // desc.N
    heat = torch.empty((desc.B * desc.H, nb, nb), dtype=torch.float32, device=q.device)
    n = ctypes.c_size_t(0)
    _ok(lib().sparse_attn_block_heatmap_scratch_size_heads(
        ctypes.byref(desc), _tiles_array(tiles), ctypes.byref(n)), "heatmap_scratch_size_heads")
    scratch = torch.empty(n.value, dtype=torch.uint8, device=q.device)
    _ok(lib().sparse_attn_block_heatmap_heads(ctypes.byref(desc), _tiles_array(tiles), _ptr(q),
                                              _ptr(k), _ptr(workspace),
                                              ctypes.c_size_t(workspace.numel()), _ptr(heat),
                                              _ptr(scratch), ctypes.c_size_t(scratch.numel()),
                                              _stream(stream)), "block_heatmap_heads")
    return heat


def heads_runs(desc: SaDesc, tiles):
    """[(sub_desc, head0, ws_offset, ws_bytes)] for the runs of equal shapes."""
    out, i = [], 0
    arr = _tiles_array(tiles)
    while True:
        sub, h0 = SaDesc(), ctypes.c_int(0)
        off, nbytes = ctypes.c_size_t(0), ctypes.c_size_t(0)
        st = lib().sparse_attn_heads_run(ctypes.byref(desc), arr, i, ctypes.byref(sub),
                                         ctypes.byref(h0), ctypes.byref(off), ctypes.byref(nbytes))
        if st == SA_ERR_INVALID_ARG and i > 0:
            return out
        _ok(st, "heads_run")
        out.append((sub, h0.value, off.value, nbytes.value))
        i += 1


class AttentionGraph:
    """Plan (optional) + forward captured once as a CUDA graph on fixed
    tensors; ``launch`` replays the whole path with one launch on whatever
    the tensors then hold. See include/sparse_attn.h."""

    def __init__(self, desc: SaDesc, q, k, v, workspace, out, with_plan: bool = True):
        _check_qkv(desc, q, k, v)
        want = torch.float32 if desc.out_fp32 else torch.bfloat16
        if out.dtype != want or out.shape != q.shape or not out.is_contiguous():
            raise ValueError(f"out must be a contiguous {want} tensor shaped like q")
        self.desc = desc
        self._buffers = (q, k, v, workspace, out)  # the graph holds their addresses
        h = ctypes.c_void_p()
        _ok(lib().sparse_attn_graph_create(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v),
                                           _ptr(workspace), ctypes.c_size_t(workspace.numel()),
                                           _ptr(out), int(bool(with_plan)), ctypes.byref(h)),
            "graph_create")
        self._h = h

    def launch(self, stream=None) -> None:
        if not self._h:
            raise ValueError("graph already destroyed")
        _ok(lib().sparse_attn_graph_launch(self._h, _stream(stream)), "graph_launch")

    def close(self) -> None:
        if getattr(self, "_h", None):
            lib().sparse_attn_graph_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class NablaAttention:
    """User-facing wrapper: owns a workspace; ``plan`` builds the block mask,
    ``forward`` runs the block-sparse attention; calling it does both."""

    def __init__(self, B, H, T, Hh, Ww, d, thr, sta=(0, 0, 0), out_fp32=False, device="cuda",
                 tile=None):
        self.desc = make_desc(B, H, T, Hh, Ww, d, thr, sta, out_fp32=out_fp32, tile=tile)
        self.workspace = alloc_workspace(self.desc, device)

    def plan(self, q, k, stream=None):
        plan(self.desc, q, k, self.workspace, stream)

    def forward(self, q, k, v, out=None, stream=None):
        if out is None:
            out = torch.empty(q.shape, device=q.device,
                              dtype=torch.float32 if self.desc.out_fp32 else torch.bfloat16)
        return fwd(self.desc, q, k, v, self.workspace, out, stream)

    def __call__(self, q, k, v, out=None, stream=None):
        self.plan(q, k, stream)
        return self.forward(q, k, v, out, stream)

    def forward_lse(self, q, k, v, out=None, lse=None, stream=None):
        """Forward over the current plan, also returning each row's log-sum-exp
        (what ``backward`` needs): (out, lse)."""
        if out is None:
            out = torch.empty(q.shape, device=q.device,
                              dtype=torch.float32 if self.desc.out_fp32 else torch.bfloat16)
        if lse is None:
            lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
        fwd_lse(self.desc, q, k, v, self.workspace, out, lse, stream)
        return out, lse

    def backward(self, q, k, v, out, dout, lse, stream=None):
        """(dq, dk, dv) of sum(out * dout) over the current plan's mask."""
        return bwd(self.desc, q, k, v, out, dout, lse, self.workspace, stream=stream)

    def heatmap(self, q, k, stream=None):
        """Exact block max-pooled full-attention map [B*H, nb, nb]."""
        return block_heatmap(self.desc, q, k, self.workspace, stream=stream)

    def check(self, stream=None) -> int:
        return check(self.desc, self.workspace, stream)
