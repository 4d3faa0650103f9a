"""Multi-rank host logic of bench.py on CPU: world_size 2 over gloo.

The path shards by replica (every rank runs the whole workload on its own
GPU, no data-path collective); the only collectives are the barrier and the
max over ranks of the timed region, and the reported value aggregates every
rank's work over that max time.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, mode, out):
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    try:
        if mode == "fail" and rank == 1:
            return  # leaves between steps, before the collective
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        t = bench.max_over_ranks(ms, dist, torch.device("cpu"))
        v = bench.aggregate_tflops(world, 1e12, t)
        out.put((rank, "ok", t, v))
    except Exception as e:  # the surviving rank sees the missing peer as an error
        out.put((rank, "error", type(e).__name__, str(e)[:200]))
    finally:
        if not (mode == "fail" and rank == 1):
            try:
                dist.destroy_process_group()
            except Exception:
                pass


def _run(mode):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, mode, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
    res = []
    while not out.empty():
        res.append(out.get())
    return sorted(res)


def test_max_over_ranks_and_aggregate_two_ranks():
    res = _run("ok")
    assert [r[0] for r in res] == [0, 1]
    for _, status, t, v in res:
        assert status == "ok"
        assert t == 15.0  # the slower rank's time, on every rank
        assert v == pytest.approx(2 * 1e12 / 0.015 / 1e12)  # both ranks' work over that time


def test_missing_rank_is_an_error_not_a_hang():
    res = _run("fail")
    assert len(res) == 1 and res[0][0] == 0
    assert res[0][1] == "error"
