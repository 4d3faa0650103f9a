"""Benchmark of the block-sparse video attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--heads H] [--no-cpu-baseline] [--no-heatmap]
                    [--no-backward]

One step = one pass of the whole hot path over one batch: sparse_attn_plan
(block pooling, reduced map, CDF threshold, STA union, block lists) followed by
sparse_attn_fwd (block-sparse attention over the kept pairs, written back in
natural token order). The metric is attention TFLOP/s counted on kept blocks
only (4 * 64^2 * d per kept (q-block, k-block) pair), whole step; the JSON
also carries the mask-build time, the attention kernel's own TFLOP/s and its
fraction of the measured bf16 tensor peak. Measured outside the timed step and
reported beside it: the exact block max-pooled attention map (its kernel time
and the mask's recall against it) and the gradients over the mask (one
sparse_attn_bwd call).

With N > 1 (launched by torch.distributed.run) every rank runs its own copy of
the workload (heads are independent: weak scaling, no data-path collective);
the time is the max over ranks.

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from dynamic_block_sparse_fractal_b200 import workloads as W  # noqa: E402

METRIC = "sparse attn TFLOP/s on kept blocks + mask-build µs; % of BF16 tensor peak"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = W.HUNYUAN
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except OSError:
        return dict(FALLBACK_PEAKS), "fallback"


def pick_workload(name):
    if name is None:
        return DEFAULT_WORKLOAD
    if name in W.WORKLOADS:
        return W.WORKLOADS[name]
    if name.startswith("sweep:"):
        return W.sweep(int(name.split(":")[1]))
    raise SystemExit(f"unknown workload {name}; choose from {sorted(W.WORKLOADS)} or sweep:K")


def kept_flops_per_pair(w):
    return 4.0 * w.N * w.N * w.d


# DRAM bytes (read + write) of one attention launch on the HunyuanVideo-like
# workload: the ncu capture of this kernel on the same grid with 2 of the 24
# heads (384.5 MB read + 56.1 MB written per launch), scaled by the 12 times
# more heads (every head's tiles run in the same order, so per-head traffic is
# the same). Reported only while the attention kernel's sources are the ones
# that capture measured.
ATTN_TRAFFIC = {
    "workload": "hunyuan_1x24x126720x128",
    "bytes": 12 * (384.546560e6 + 56.089088e6),
    "sources_sha1": "7baed63701d00a72c1b8b1da8c994391f79cc9cc",
}
ATTN_SOURCES = ("k_attn.cu", "sm100.cuh", "exp2_poly.cuh", "layout.cuh")


def attn_sources_sha1():
    """Hash of what the attention kernel is compiled from: its source, the
    headers it includes, and its argument struct (the other structs of
    kernels.cuh belong to other kernels)."""
    import hashlib
    import re
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "dynamic_block_sparse_fractal_b200", "csrc")
    for f in ATTN_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    with open(os.path.join(csrc, "kernels.cuh")) as fh:
        args = re.search(r"struct AttnArgs \{.*?\};", fh.read(), re.S)
    h.update(args.group(0).encode() if args else b"")
    return h.hexdigest()


def attn_traffic(w):
    """Measured DRAM bytes per attention launch, or None if stale or another workload."""
    if w.name != ATTN_TRAFFIC["workload"]:
        return None
    return ATTN_TRAFFIC["bytes"] if attn_sources_sha1() == ATTN_TRAFFIC["sources_sha1"] else None


def max_over_ranks(ms, dist, device):
    """The slowest rank's time (every rank runs the same collective)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(world, flops_per_rank, ms):
    """Whole-job throughput: every rank processes flops_per_rank in (the max) ms."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def to_device(bits, w, device):
    import torch
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    return t.reshape(w.B, w.H, w.S, w.d).to(device)


def run_ours(args, w, rank, world):
    import torch
    from dynamic_block_sparse_fractal_b200 import api

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    q_h, k_h, v_h = W.make_inputs(w)
    q, k, v = (to_device(x, w, dev) for x in (q_h, k_h, v_h))
    desc = api.desc_for(w)
    ws = api.alloc_workspace(desc, dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        api.plan(desc, q, k, ws)
        api.fwd(desc, q, k, v, ws, out)
    st = api.check(desc, ws)
    if st != api.SA_OK:
        raise SystemExit(f"device status after warm-up: {api.status_string(st)}")

    views = api.get_mask(desc, ws)
    kept_pairs = int(views["cnt"].sum().item())
    union_entries = int(views["tile_cnt"].sum().item())
    kept_flops = kept_pairs * kept_flops_per_pair(w)
    computed_flops = union_entries * 2 * kept_flops_per_pair(w)  # 128-row tiles
    sparsity = 1.0 - kept_pairs / (w.BH * w.nb * w.nb)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            api.plan(desc, q, k, ws)
            ev[i][1].record(stream)
            api.fwd(desc, q, k, v, ws, out)
            ev[i][2].record(stream)
        t1.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    total_ms = t0.elapsed_time(t1)
    plan_ms = [e[0].elapsed_time(e[1]) for e in ev]
    fwd_ms = [e[1].elapsed_time(e[2]) for e in ev]
    st = api.check(desc, ws)
    if st != api.SA_OK:
        raise SystemExit(f"device status after timing: {api.status_string(st)}")
    total_ms = max_over_ranks(total_ms, dist, dev)

    # ---- end to end through the public API, host buffers, copies timed.
    # Every step copies its Q/K/V from pinned host memory and its output back;
    # as a serving loop would, consecutive steps are double-buffered on three
    # streams (step i+1's inputs travel while step i computes, step i's output
    # travels while step i+1 computes).
    pin = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).reshape(w.B, w.H, w.S, w.d)
           .pin_memory() for x in (q_h, k_h, v_h)]
    out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    e2e_steps = max(2, min(args.steps, 10))
    attn = api.NablaAttention(w.B, w.H, w.T, w.Hh, w.Ww, w.d, w.thr, w.sta, device=dev)
    s_h2d, s_cmp, s_d2h = (torch.cuda.Stream(dev) for _ in range(3))
    bufs = [[torch.empty_like(q) for _ in range(3)] for _ in range(2)]
    outs = [torch.empty_like(out) for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of buffer b landed
    ev_done = [torch.cuda.Event() for _ in range(2)]  # compute on buffer b finished
    ev_out = [torch.cuda.Event() for _ in range(2)]   # output of buffer b copied back

    def e2e_step(i):
        b = i & 1
        with torch.cuda.stream(s_h2d):
            if i >= 2:
                s_h2d.wait_event(ev_done[b])  # the previous user of buffer b read its inputs
            for dst, src in zip(bufs[b], pin):
                dst.copy_(src, non_blocking=True)
            ev_in[b].record(s_h2d)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[b])
            if i >= 2:
                s_cmp.wait_event(ev_out[b])  # outs[b] was copied back
            attn(bufs[b][0], bufs[b][1], bufs[b][2], out=outs[b], stream=s_cmp)
            ev_done[b].record(s_cmp)
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(ev_done[b])
            out_h[b].copy_(outs[b], non_blocking=True)
            ev_out[b].record(s_d2h)

    e2e_step(0)
    e2e_step(1)
    torch.cuda.synchronize(dev)
    barrier()
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    a0.record(s_h2d)
    for i in range(2, 2 + e2e_steps):
        e2e_step(i)
    a1.record(s_d2h)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = a0.elapsed_time(a1) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    st = attn.check(s_cmp)
    if st != api.SA_OK:
        raise SystemExit(f"device status after e2e: {api.status_string(st)}")

    plan_stages = measure_plan_stages(api, desc, w, q, k, ws, kept_pairs, union_entries,
                                      stream)
    heatmap = None if args.no_heatmap else measure_heatmap(api, desc, w, q, k, ws, views, dev,
                                                             stream)
    backward = None if args.no_backward else measure_backward(api, desc, w, q, k, v, ws,
                                                              kept_pairs, dev, stream)
    radius = None if args.no_radius else measure_radius(api, desc, w, q, k, dev, stream)

    peaks, src = load_peaks()
    ms_step = total_ms / args.steps
    fwd_avg = statistics.mean(fwd_ms)
    attn_tflops = kept_flops / (fwd_avg * 1e-3) / 1e12
    # The denominator is the burst bf16 GEMM figure: one attention launch
    # lasts tens of milliseconds, a short burst by that measurement's terms.
    # The sustained (power-capped) figure is context only, and so is the rate
    # normalised to the maximum SM clock by the clocks sampled here.
    peak = float(peaks["bf16_tflops"])
    sustained = float(peaks["bf16_tflops_sustained"]) if "bf16_tflops_sustained" in peaks \
        else None
    clk = clocks.summary()
    hbm = float(peaks["hbm_gbs"])
    for st in plan_stages.values():
        if st.get("gbs") is not None:
            st["frac_of_hbm"] = round(st["gbs"] / hbm, 4)
    line = {
        "metric": METRIC, "value": round(aggregate_tflops(world, kept_flops, ms_step), 2),
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**w.describe(), "per_gpu": "one full copy of the workload per GPU",
                   "l2": "inputs larger than L2 (3 x %.0f MB bf16)" % (w.BH * w.S * w.d * 2 / 1e6)},
        "mask_build_us": round(statistics.mean(plan_ms) * 1e3, 1),
        "plan_kernels": plan_stages,
        "attn_fwd_ms": round(fwd_avg, 4),
        "attn_kept_tflops": round(attn_tflops, 2),
        "pct_bf16_peak": round(100.0 * attn_tflops / peak, 2),
        "sparsity": round(sparsity, 4),
        "kept_pairs": kept_pairs,
        "computed_over_kept": round(computed_flops / kept_flops, 4),
        "roofline": {"bound": "tensor", "achieved": round(attn_tflops, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(attn_tflops / peak, 4),
                     "traffic": attn_traffic(w), "kernel": "sa::attn_kernel<128>",
                     "peak_source": f"{src} bf16 GEMM burst (bf16_tflops)",
                     "frac_of_sustained": round(attn_tflops / sustained, 4) if sustained
                     else None,
                     **clock_normalised(attn_tflops, peak, clk)},
        "e2e": {"value": round(aggregate_tflops(world, kept_flops, e2e_ms), 2), "unit": UNIT,
                "ms_per_step": round(e2e_ms, 3), "steps": e2e_steps,
                "overlap": "double-buffered: H2D of step i+1 and D2H of step i-1 overlap step i",
                "h2d_bytes_per_step": int(3 * q.numel() * 2),
                "d2h_bytes_per_step": int(out.numel() * out.element_size())},
        "gpu_launches": 6 * args.steps,  # pool, logits, select, union, tile order, attention
        "clocks": clk,
    }
    if heatmap is not None:
        heatmap["frac"] = round(heatmap["tensor_tflops"] / peak, 4)
        line["heatmap"] = heatmap
    if backward is not None:
        backward["frac"] = round(backward["kept_tflops"] / peak, 4)
        line["backward"] = backward
    if radius is not None:
        radius["entropy_frac"] = round(radius["entropy_tensor_tflops"] / peak, 4)
        line["radius_mask"] = radius
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return line


def clock_normalised(tflops, peak, clk):
    """The rate scaled to the maximum SM clock by the median clock sampled in
    the timed region, as a fraction of the peak (context: the kernel's
    cycles, whatever clock the power cap allowed)."""
    med, mx = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    if not med or not mx:
        return {"frac_clock_normalised": None}
    return {"frac_clock_normalised": round(tflops * (mx / med) / peak, 4),
            "sm_mhz_median": med, "sm_max_mhz": mx}


def plan_stage_bytes(w, kept_pairs, union_entries):
    """Algorithmic HBM bytes of each plan stage: what it must read and write
    once (fp32 pooled means and their tf32 hi/lo split; int32 lists)."""
    BH, nb, d, S = w.BH, w.nb, w.d, w.S
    words = (nb + 31) // 32
    ntile = union_tiles(w)
    pooled = 2 * BH * nb * d * 4          # Qbar, Kbar
    split = 4 * BH * nb * d * 4           # their hi and lo halves
    lists = BH * nb * 4 + kept_pairs * 4 + BH * nb * words * 4  # counts, ids, bitmaps
    return {
        "pool": 2 * BH * S * d * 2 + pooled + split,
        "logits": split + BH * nb * nb * 4,
        "select": BH * nb * nb * 4 + lists,
        "reduced_map_select": split + lists,
        "union": BH * nb * words * 4 + BH * ntile * 4 + union_entries * 4,
        "tile_order": 2 * BH * ntile * 4,
    }


def union_tiles(w):
    nt, nh, nw = w.T, w.Hh // w.P, w.Ww // w.P
    if w.tile is not None:
        nt, nh, nw = w.T // w.tile[0], w.Hh // w.tile[1], w.Ww // w.tile[2]
    return (nt // 2) * nh * nw + ((nh * ((nw + 1) // 2)) if nt % 2 else 0)


def measure_plan_stages(api, desc, w, q, k, ws, kept_pairs, union_entries, stream, reps=5):
    """Device time of each plan kernel (CUDA events between the plan's
    launches, mean of ``reps`` plans) with its algorithmic bytes and GB/s."""
    us = api.plan_profile(desc, q, k, ws, reps=reps, stream=stream)
    nbytes = plan_stage_bytes(w, kept_pairs, union_entries)
    out = {}
    for name, t in us.items():
        b = nbytes.get(name)
        out[name] = {"us": round(t, 1), "bytes": b,
                     "gbs": round(b / (t * 1e-6) / 1e9, 1) if b and t > 0 else None}
    return out


def measure_heatmap(api, desc, w, q, k, ws, views, dev, stream, reps=3):
    """Times the exact block max-pooled attention map (one launch of the heat
    kernel after its zeroing) outside the step, and reports the recall of the
    planned NABLA mask against it: per q-block, the share of the block maxima
    that the kept blocks cover, averaged over q-blocks and heads."""
    import torch
    heat = torch.empty((w.BH, w.nb, w.nb), dtype=torch.float32, device=dev)
    api.block_heatmap(desc, q, k, ws, heat)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(reps):
        api.block_heatmap(desc, q, k, ws, heat)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / reps
    st = api.check(desc, ws)
    if st != api.SA_OK:
        raise SystemExit(f"device status after the heat map: {api.status_string(st)}")
    cnt = views["cnt"].long()
    idx = views["idx"].long().clamp_(0, w.nb - 1)
    kept = torch.arange(w.nb, device=dev).view(1, 1, -1) < cnt.unsqueeze(-1)
    covered = (torch.gather(heat, 2, idx) * kept).sum(-1)
    recall = float((covered / heat.sum(-1)).mean().item())
    qk_flops = 2.0 * w.S * w.S * w.d * w.BH  # one dense Q K^T
    return {"kernel": "sa::heat_kernel<%d>" % w.d, "ms": round(ms, 3),
            "tensor_tflops": round(qk_flops / (ms * 1e-3) / 1e12, 2),
            "note": "one dense Q K^T pass (row log-sum-exp + raw block maxima, then per-row "
                    "reduction of the maxima); time includes zeroing the map",
            "mask_recall": round(recall, 4)}


def measure_radius(api, desc, w, q, k, dev, stream, tau=2.0, gamma=0.25, vote_min=1, reps=5):
    """Times the Token Radius Attention mask builder outside the step, in a
    workspace of its own: the per-token entropy pass (one dense Q K^T) and the
    radius plan (block votes, lists, tile unions, tile order) for one setting
    of the key budget tau, the temporal decay gamma and the vote threshold, and
    reports the density of the mask it builds."""
    import torch
    ws_r = api.alloc_workspace(desc)
    ent = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    api.token_entropy(desc, q, k, ws_r, ent)
    api.plan_radius(desc, tau, gamma, vote_min, ent, ws_r)
    e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    torch.cuda.synchronize(dev)
    e0.record(stream)
    api.token_entropy(desc, q, k, ws_r, ent)
    e1.record(stream)
    for _ in range(reps):
        api.plan_radius(desc, tau, gamma, vote_min, ent, ws_r)
    e2.record(stream)
    torch.cuda.synchronize(dev)
    ent_ms = e0.elapsed_time(e1)
    plan_us = e1.elapsed_time(e2) / reps * 1e3
    st = api.check(desc, ws_r)
    if st != api.SA_OK:
        raise SystemExit(f"device status after the radius mask: {api.status_string(st)}")
    cnt = api.get_mask(desc, ws_r)["cnt"]
    density = float(cnt.double().sum().item()) / (w.BH * w.nb * w.nb)
    qk_flops = 2.0 * w.S * w.S * w.d * w.BH  # one dense Q K^T
    return {"tau": tau, "gamma": gamma, "vote_min": vote_min,
            "entropy_ms": round(ent_ms, 3),
            "entropy_tensor_tflops": round(qk_flops / (ent_ms * 1e-3) / 1e12, 2),
            "plan_us": round(plan_us, 1), "density": round(density, 4),
            "mean_entropy_nats": round(float(ent.double().mean().item()), 4),
            "note": "entropy pass = the map kernel in entropy mode; plan = votes, lists, "
                    "tile unions and order"}


def measure_backward(api, desc, w, q, k, v, ws, kept_pairs, dev, stream, reps=3):
    """Times sparse_attn_bwd (prep, transposed lists, the gradient kernel, dQ
    conversion) on the planned mask with a seeded upstream gradient, outside
    the step. Kept FLOPs: five N x N x d GEMMs per kept (q-block, k-block) pair
    (S, dP, dV, dK, dQ)."""
    import torch
    g = to_device(W.make_output_grad(w), w, dev)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    api.fwd_lse(desc, q, k, v, ws, out, lse)
    grads = [torch.empty_like(q) for _ in range(3)]
    scratch = torch.empty(api.bwd_scratch_size(desc), dtype=torch.uint8, device=dev)
    api.bwd(desc, q, k, v, out, g, lse, ws, *grads, scratch=scratch)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(reps):
        api.bwd(desc, q, k, v, out, g, lse, ws, *grads, scratch=scratch)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / reps
    st = api.check(desc, ws)
    if st != api.SA_OK:
        raise SystemExit(f"device status after the backward: {api.status_string(st)}")
    flops = kept_pairs * 5 * kept_flops_per_pair(w) / 2  # kept_flops_per_pair counts 2 GEMMs
    return {"kernels": "bwd_prep, bwd_lists, sa::bwd_kernel<%d>, dq_convert" % w.d,
            "ms": round(ms, 3), "kept_tflops": round(flops / (ms * 1e-3) / 1e12, 2),
            "note": "one sparse_attn_bwd call: dQ, dK, dV over the planned mask"}


def oracle_sample(w, budget_s=20.0, seed=0):
    """Times the fp64 oracle on a bounded sample of workload w.

    Sample: heads 0..h-1 in full for the mask build (pool, reduced map, CDF,
    STA), then exact masked attention for whole q-blocks drawn at random from
    those heads until the time budget is spent. Returns kept-block TFLOP/s of
    the attention part, the mask-build seconds per head and a description."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max([p.get("num_threads", 1) for p in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        cores = 1
    heads = [0]
    q, k, v = W.make_inputs(w, heads=range(0, 1))
    t = time.perf_counter()
    M, _, _ = oracle.nabla_mask(q, k, w.T, w.Hh, w.Ww, w.block, w.N, w.thr, w.sta)
    mask_s = time.perf_counter() - t
    rng = np.random.default_rng(seed)
    order = rng.permutation(w.nb)
    perm = oracle.fractal_order(w.T, w.Hh, w.Ww, w.block)
    qp, kp, vp = (oracle.flatten(oracle.widen_bf16(x[0]), perm) for x in (q, k, v))
    pairs, spent, nq = 0, 0.0, 0
    t = time.perf_counter()
    for qb in order:
        rows = np.arange(qb * w.N, (qb + 1) * w.N)
        oracle.masked_attention(qp, kp, vp, M[0], w.N, rows=rows)
        pairs += int(M[0, qb].sum())
        nq += 1
        spent = time.perf_counter() - t
        if spent > budget_s:
            break
    tflops = pairs * kept_flops_per_pair(w) / spent / 1e12
    desc = (f"head 0 of {w.BH}: full mask build ({mask_s:.1f} s), then exact masked attention "
            f"on {nq} of {w.nb} q-blocks drawn at random ({spent:.1f} s); value = kept-block "
            f"TFLOP/s of that attention")
    return tflops, mask_s, cores, desc


def run_reference(args, w, rank, world):
    if rank != 0:
        return None
    vals = []
    budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for i in range(args.warmup + args.steps):
        tf, mask_s, cores, desc = oracle_sample(w, budget_s=budget, seed=i)
        if i >= args.warmup:
            vals.append(tf)
    value = statistics.mean(vals)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": w.describe(),
        "cpu_baseline": {"kind": "oracle", "cores": cores, "sample": desc, "value": value,
                         "unit": UNIT},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-heatmap", action="store_true",
                    help="skip the block max-pooled attention map measurement")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the gradient (backward) measurement")
    ap.add_argument("--no-radius", action="store_true",
                    help="skip the radius (TRA) mask measurement")
    ap.add_argument("--heads", type=int, default=None,
                    help="run the workload's grid with this many heads (small ncu captures); "
                         "the line's config then names the changed workload")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = pick_workload(args.workload)
    if args.heads is not None:
        import dataclasses
        w = dataclasses.replace(w, H=args.heads, name=f"{w.name}_heads{args.heads}")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus if args.gpus == 1 else 1)))
    if args.impl == "reference":
        line = run_reference(args, w, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    line = run_ours(args, w, rank, world)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            tf, mask_s, cores, desc = oracle_sample(w, budget_s=15.0)
            line["cpu_baseline"] = {"value": tf, "unit": UNIT, "cores": cores, "kind": "oracle",
                                    "sample": desc, "mask_build_s_per_head": round(mask_s, 2)}
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
