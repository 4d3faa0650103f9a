"""Timeline of one CTA of the block-sparse attention kernel, from the
diagnostics build (compiled with SA_TRACE=1 into lib/libsparse_attn_trace.so):
clock64 stamps of the MMA issuer per unit (a unit is PV_X(j) followed by
S_X(j+1) of one query tile X) and of the eight softmax warps per step.

    python -m dynamic_block_sparse_fractal_b200.trace_attn [--workload NAME] [--cta X,Y]

Prints, for the traced CTA: cycles per round (one unit of each of its two
tiles), the MMA issuer's time per unit split into waiting (for the softmax's P
and the K/V slots) and issuing (the 16 MMAs and their commits, which block
while the tensor core's queue is full), and each softmax warp's time per step
from S complete to P stored.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

K_UNITS, K_STEPS, K_SOFTMAX = 1300, 500, 4096
K_WORDS = K_SOFTMAX + 8 * 2 * K_STEPS


def summarise(t: np.ndarray) -> dict:
    start = t[K_SOFTMAX - 1]
    mma = t[:3 * K_UNITS].reshape(-1, 3)
    nu = int((mma[:, 2] > 0).sum())
    mma = mma[:nu] - start
    steps = []
    for w in range(8):
        a = t[K_SOFTMAX + w * 2 * K_STEPS:K_SOFTMAX + (w + 1) * 2 * K_STEPS].reshape(-1, 2)
        n = int((a[:, 1] > 0).sum())
        steps.append(float((a[:n, 1] - a[:n, 0]).mean()) if n else None)
    body = slice(4, max(5, nu - 4))  # steady state: without the first and last units
    span = int(mma[-1, 2] - mma[0, 0]) if nu else 0
    return {
        "units": nu,
        "cycles_per_round": round(span / (nu / 2), 1) if nu else None,
        "unit_wait_cycles": round(float((mma[body, 1] - mma[body, 0]).mean()), 1),
        "unit_issue_cycles": round(float((mma[body, 2] - mma[body, 1]).mean()), 1),
        "softmax_step_cycles_per_warp": [round(x, 1) if x is not None else None for x in steps],
        "ideal_cycles_per_round": 2048,
    }


def main():
    import torch
    from dynamic_block_sparse_fractal_b200 import api, build, workloads as W
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default=W.HUNYUAN.name)
    ap.add_argument("--cta", default="100,3", help="blockIdx.x,blockIdx.y of the traced CTA")
    args = ap.parse_args()
    api.LIB_PATH = build.build(trace=True)
    L = api.lib()
    L.sparse_attn_trace_select.argtypes = [ctypes.c_int, ctypes.c_int]
    L.sparse_attn_trace_read.argtypes = [ctypes.POINTER(ctypes.c_longlong), ctypes.c_int]
    w = W.WORKLOADS[args.workload]
    bx, by = (int(v) for v in args.cta.split(","))
    q, k, v = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
               for x in W.make_inputs(w))
    desc = api.desc_for(w)
    ws = api.alloc_workspace(desc)
    api.plan(desc, q, k, ws)
    out = torch.empty_like(q)
    for _ in range(3):
        api.fwd(desc, q, k, v, ws, out)
    torch.cuda.synchronize()
    assert L.sparse_attn_trace_select(bx, by) == 0
    api.fwd(desc, q, k, v, ws, out)
    torch.cuda.synchronize()
    assert api.check(desc, ws) == api.SA_OK
    buf = (ctypes.c_longlong * K_WORDS)()
    assert L.sparse_attn_trace_read(buf, K_WORDS) == 0
    res = summarise(np.array(buf[:], dtype=np.int64))
    res.update({"workload": w.name, "cta": [bx, by]})
    print(json.dumps(res))


if __name__ == "__main__":
    main()
