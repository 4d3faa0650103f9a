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


@pytest.mark.parametrize("w", [W.TINY, W.W8K], ids=["tiny", "8k"])
def test_noalloc_matches_workspace_entry_points(w):
    q, k, v = (_dev(x, w) for x in W.make_inputs(w))
    desc = api.desc_for(w)
    assert api.workspace_size(desc) <= api.NOALLOC_SCRATCH_BYTES
    ws = api.alloc_workspace(desc)
    ref = torch.empty_like(q)
    api.plan(desc, q, k, ws)
    api.fwd(desc, q, k, v, ws, ref)
    assert api.check(desc, ws) == api.SA_OK
    ref_np = ref.float().cpu().numpy().astype(np.float64)
    stream = torch.cuda.current_stream()
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        st = api.lib().sparse_attn_forward_noalloc(
            ctypes.byref(desc), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
            ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
            ctypes.c_void_p(stream.cuda_stream))
        assert st == api.SA_OK, api.status_string(st)
        torch.cuda.synchronize()
        r = parity.out_check(out.float().cpu().numpy(), ref_np, bf16_out=True)
        assert r["ok"], r


def test_noalloc_rejects_problems_larger_than_its_scratch():
    desc = api.desc_for(W.HUNYUAN)
    assert api.workspace_size(desc) > api.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000000)
    st = api.lib().sparse_attn_forward_noalloc(ctypes.byref(desc), fake, fake, fake, fake, None)
    assert st == api.SA_ERR_WORKSPACE
