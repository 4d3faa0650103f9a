"""sparse_attn_forward_noalloc: plan + forward for callers that cannot
allocate device memory (the library supplies the workspace from a fixed array
in its own device image). Its output must match the workspace entry points'
within the parity tolerance, on two calls in a row (the shared array keeps the
previous call's contents). This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from dynamic_block_sparse_fractal_b200 import api, workloads as W
from tests import parity

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _dev(bits, w):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).reshape(
        w.B, w.H, w.S, w.d).cuda()


# The built-in array's layout offsets differ with the problem: besides the
# two workloads, fp32 output with a three-dimensional tile, and a problem whose
# workspace fills 97% of the array (Wan-like grid, 27 frames, 8 heads).
CASES = [
    (W.TINY, False), (W.W8K, False), (W.W8K_T248, True),
    (W.WAN.with_(name="wan_1x8x48384x128_sta3", H=8, T=27), False),
]


@pytest.mark.parametrize("w,out_fp32", CASES, ids=[f"{c[0].name}_fp32{int(c[1])}" for c in CASES])
def test_noalloc_matches_workspace_entry_points(w, out_fp32):
    q, k, v = (_dev(x, w) for x in W.make_inputs(w))
    desc = api.desc_for(w, out_fp32=out_fp32)
    assert api.workspace_size(desc) <= api.NOALLOC_SCRATCH_BYTES
    ws = api.alloc_workspace(desc)
    dtype = torch.float32 if out_fp32 else torch.bfloat16
    ref = torch.empty(q.shape, dtype=dtype, device="cuda")
    api.plan(desc, q, k, ws)
    api.fwd(desc, q, k, v, ws, ref)
    assert api.check(desc, ws) == api.SA_OK
    ref_np = ref.float().cpu().numpy().astype(np.float64)
    stream = torch.cuda.current_stream()
    for _ in range(2):
        out = torch.full(q.shape, float("nan"), dtype=dtype, device="cuda")
        st = api.lib().sparse_attn_forward_noalloc(
            ctypes.byref(desc), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
            ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
            ctypes.c_void_p(stream.cuda_stream))
        assert st == api.SA_OK, api.status_string(st)
        torch.cuda.synchronize()
        r = parity.out_check(out.float().cpu().numpy(), ref_np, bf16_out=not out_fp32)
        assert r["ok"], r


def test_noalloc_rejects_problems_larger_than_its_scratch():
    desc = api.desc_for(W.HUNYUAN)
    assert api.workspace_size(desc) > api.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000000)
    st = api.lib().sparse_attn_forward_noalloc(ctypes.byref(desc), fake, fake, fake, fake, None)
    assert st == api.SA_ERR_WORKSPACE
