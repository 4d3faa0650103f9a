"""The whole path as one CUDA graph (sparse_attn_graph_*): replays equal the
direct calls bit for bit, follow new data written into the captured buffers
(the plan is re-run), and a forward-only graph reuses the workspace's plan."""
import time

import numpy as np
import pytest
import torch

from dynamic_block_sparse_fractal_b200 import api, workloads as W

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def dev_inputs(w):
    return [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
            for x in W.make_inputs(w)]


def direct(desc, q, k, v, plan=True):
    ws = api.alloc_workspace(desc)
    out = torch.empty_like(q)
    if plan:
        api.plan(desc, q, k, ws)
    return ws, out


def test_graph_replay_equals_direct_calls_and_follows_new_data():
    w = W.W8K
    desc = api.desc_for(w)
    q, k, v = dev_inputs(w)
    ws, out = api.alloc_workspace(desc), torch.empty_like(q)
    graph = api.AttentionGraph(desc, q, k, v, ws, out, with_plan=True)
    graph.launch()
    assert api.check(desc, ws) == api.SA_OK
    ws_ref, ref = direct(desc, q, k, v)
    api.fwd(desc, q, k, v, ws_ref, ref)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    # new data in the captured buffers: the replay re-plans
    q2, k2, v2 = dev_inputs(w.with_(seed=w.seed + 17))
    q.copy_(q2), k.copy_(k2), v.copy_(v2)
    graph.launch()
    assert api.check(desc, ws) == api.SA_OK
    ws_ref2, ref2 = direct(desc, q2, k2, v2)
    api.fwd(desc, q2, k2, v2, ws_ref2, ref2)
    torch.cuda.synchronize()
    assert torch.equal(out, ref2)
    assert not torch.equal(ref, ref2)
    m1 = api.get_mask(desc, ws)["cnt"]
    m2 = api.get_mask(desc, ws_ref2)["cnt"]
    assert torch.equal(m1, m2)
    graph.close()


def test_forward_only_graph_reuses_the_plan():
    w = W.W8K
    desc = api.desc_for(w)
    q, k, v = dev_inputs(w)
    ws, out = api.alloc_workspace(desc), torch.empty_like(q)
    api.plan(desc, q, k, ws)
    graph = api.AttentionGraph(desc, q, k, v, ws, out, with_plan=False)
    _, _, v2 = dev_inputs(w.with_(seed=w.seed + 5))
    v.copy_(v2)
    graph.launch()
    ref = torch.empty_like(q)
    api.fwd(desc, q, k, v2, ws, ref)  # same plan, new values
    torch.cuda.synchronize()
    assert api.check(desc, ws) == api.SA_OK
    assert torch.equal(out, ref)
    graph.close()


def test_graph_launch_cost():
    # host time per step (launch-bound for this 8k-token workload) and device
    # time, direct calls vs one graph replay; reported, not asserted
    w = W.W8K
    desc = api.desc_for(w)
    q, k, v = dev_inputs(w)
    ws, out = api.alloc_workspace(desc), torch.empty_like(q)
    graph = api.AttentionGraph(desc, q, k, v, ws, out, with_plan=True)
    n = 50

    def run(step):
        for _ in range(3):
            step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        e0.record()
        for _ in range(n):
            step()
        host = (time.perf_counter() - t0) / n * 1e6
        e1.record()
        torch.cuda.synchronize()
        return host, e0.elapsed_time(e1) / n * 1e3

    def step_direct():
        api.plan(desc, q, k, ws)
        api.fwd(desc, q, k, v, ws, out)

    h_d, d_d = run(step_direct)
    h_g, d_g = run(graph.launch)
    print(f"8k workload per step: direct host {h_d:.1f} us device {d_d:.1f} us; "
          f"graph host {h_g:.1f} us device {d_g:.1f} us")
    assert api.check(desc, ws) == api.SA_OK
    graph.close()
