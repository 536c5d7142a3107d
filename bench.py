"""Benchmark: MoE dispatch / combine on B200, V3-shaped workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = the whole hot path over one batch: layout -> FP8 dispatch (bf16
x quantised to e4m3 with 1x128 scales) -> BF16 combine, on the workload of
the DeepEP V2 README, section "Performance" (8192 tokens, hidden 7168,
top-8 of 256 experts in 8 segments, expert_alignment 128), synthetic seeded
inputs.  Prints ONE JSON line on rank 0.

value = algorithmic bytes of the step (below) / device time of the step,
        summed over ranks / max-over-ranks time (weak scaling: every rank
        runs its own batch; there is no exchange on this path).
Algorithmic bytes (per step, from the layout the step produced):
  layout   : topk_idx + topk_weights read, slot_map + 3 per-row arrays written
  dispatch : x read once (T*H*2) + slot_map read + for each valid slot one
             e4m3 row (H) and its scales (H/128*4) written + for each padding
             row H + H/128*4 zero bytes written
  combine  : for each valid slot one bf16 row of y read (H*2) + slot_map and
             weights read + the bf16 output written (T*H*2)
The step touches ~1.8 GB, far more than the 126 MB L2, so no L2 flush is
needed between steps.

--impl reference times the CPU oracle (the only other implementation of
this path; single-threaded C) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "dispatch & combine GB/s and % of B200 HBM peak (V3 shape); decode µs/call"
WORKLOAD = "v3"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0   # the nominal HBM3e figure the target is stated against
DTYPE = "bf16->e4m3 (1x128 scales), f32 accumulation"   # what the path computes in


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=WORKLOAD, choices=sorted(W.WORKLOADS))
    p.add_argument("--tokens", type=int, default=None,
                   help="override the workload's token count (same shapes otherwise; for profiling)")
    p.add_argument("--decode-pairs", type=int, default=256)
    p.add_argument("--decode-replays", type=int, default=20)
    p.add_argument("--e2e-steps", type=int, default=8)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-mgpu", action="store_true")
    p.add_argument("--no-extra-workloads", action="store_true",
                   help="skip the mid and skewed lines")
    p.add_argument("--ep", action="store_true",
                   help="time the expert-parallel group across the torchrun ranks (one GPU each) instead of "
                        "the one-GPU step")
    return p.parse_args()


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------ byte counts

def step_bytes(w: W.Workload, T: int, V: int, P: int, R: int) -> dict:
    """Algorithmic bytes of one layout / dispatch / combine, given the valid
    slot count V, padding rows P and total rows R of the layout."""
    H, k = w.H, w.k
    B = H // 128
    layout = T * k * 8 + T * k * 4 + T * k * 4 + R * 12
    if w.x_mode == "fp8_quant":
        dispatch = T * H * 2 + T * k * 4 + V * (H + B * 4) + P * (H + B * 4)
    else:
        dispatch = T * H * 2 + T * k * 4 + (V + P) * H * 2
    combine = V * H * 2 + T * k * 8 + T * H * 2
    return {"layout": layout, "dispatch": dispatch, "combine": combine}


def step_config(w: W.Workload, T: int, world: int) -> dict:
    """The `config` object of the JSON line (both arms)."""
    return {"workload": f"{w.name}: T={T} hidden={w.H} experts={w.E} segments={w.S} "
                        f"topk={w.k} alignment={w.align} x={w.x_mode}",
            "T": T, "hidden": w.H, "experts": w.E, "segments": w.S, "topk": w.k, "alignment": w.align,
            "dispatch": "bf16 -> e4m3 1x128" if w.x_mode == "fp8_quant" else "bf16",
            "combine": "bf16, weighted, fp32 accumulation", "parallelism": f"replicas{world}",
            "l2": "no flush: each step touches ~1.8 GB, > 126 MB L2"}


def layout_launches(T: int, k: int) -> int:
    """Kernels per layout: one CTA does it all when the slots fit one chunk
    of 1024 (T <= 1024 // k), else a count and an assign kernel."""
    return 1 if T <= 1024 // k else 2


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest x over all ranks (the slowest rank's time); x itself at N=1."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_gbs(bytes_per_rank_step: int, world: int, ms_per_step: float) -> float:
    """Whole-job GB/s: every rank moves its own batch's bytes each step, and a
    step lasts as long as the slowest rank."""
    return bytes_per_rank_step * world / (ms_per_step * 1e-3) / 1e9


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str | None):
        self.proc = None
        self.device_id = device_id

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.device_id is not None:
            cmd += ["-i", self.device_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def nvsmi_device_id(dev) -> str | None:
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        return vis.split(",")[dev.index or 0] if vis else str(dev.index or 0)


# ----------------------------------------------------------- ncu traffic

def combine_traffic(workload: str, T: int):
    """Per-launch DRAM bytes of the combine kernel from the committed ncu
    record (profiles/traffic.json), if that record was taken on the current
    combine source and on this workload; else None."""
    src = os.path.join(ROOT, "combine_ep_get_06_b200", "csrc", "combine.cu")
    rec = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        r = json.load(open(rec))["combine_kernel"]
    except (OSError, ValueError, KeyError):
        return None
    if r.get("workload") != workload or int(r.get("T", -1)) != T or r.get("source_sha16") != sha:
        return None
    return int(r["dram_read_bytes"]) + int(r["dram_write_bytes"])


# ------------------------------------------------------------- our arm

def time_back_to_back(fn, n: int, stream) -> float:
    """Mean ms per call of n back-to-back calls of fn on `stream` (CUDA events), after 3 untimed ones."""
    import torch

    for _ in range(3):
        fn()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(1_000_000)   # let the host queue the calls before the start event
    a.record(stream)
    for _ in range(n):
        fn()
    b.record(stream)
    b.synchronize()
    return a.elapsed_time(b) / n


def run_ep(args, rank, world, dev):
    """Expert parallelism across the ranks (segments = ranks, one GPU each):
    each rank routes its own V3-shaped batch; ExpertParallelGroup.dispatch
    (layout, all-gather of counts, dispatch kernel storing into the owners'
    blocks over NVLink, barrier) then .combine (barrier, combine kernel
    loading from them).  Reported like the pages' logical bandwidth: the
    rows a rank sends (or pulls back), local ones included, over the time,
    summed over ranks, max time over ranks."""
    import torch
    import torch.distributed as dist

    import combine_ep_get_06_b200 as ep
    from combine_ep_get_06_b200 import mgpu

    w = W.WORKLOADS[args.workload]
    T = args.tokens if args.tokens is not None else w.T
    inp = W.make_inputs(w, seed=rank, T=T)
    x = torch.from_numpy(np.ascontiguousarray(inp["x"]).view(np.int16)).view(torch.bfloat16).to(dev)
    idx = torch.from_numpy(inp["topk_idx"]).to(dev)
    wts = torch.from_numpy(inp["topk_weights"]).to(dev)
    fp8 = w.x_mode == "fp8_quant"
    grp = mgpu.ExpertParallelGroup(T, w.k, w.E, w.H, expert_alignment=w.align,
                                   mode=ep.EP_X_BF16_TO_FP8 if fp8 else ep.EP_X_BF16, device=dev)
    try:
        grp.block.y.zero_()                      # stands in for the expert GEMMs' output
        out = torch.empty(T, w.H, dtype=torch.bfloat16, device=dev)
        for _ in range(args.warmup):
            h = grp.dispatch(x, idx, wts, use_fp8=fp8)
            grp.combine(h, wts, out)
        torch.cuda.synchronize(dev)
        stream = torch.cuda.current_stream(dev)
        K = args.steps
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        for i in range(K):
            ev[i][0].record(stream)
            h = grp.dispatch(x, idx, wts, use_fp8=fp8)
            ev[i][1].record(stream)
            grp.combine(h, wts, out)
            ev[i][2].record(stream)
        torch.cuda.synchronize(dev)
        d_ms = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in ev), world, dev)
        c_ms = max_over_ranks(statistics.mean(e[1].elapsed_time(e[2]) for e in ev), world, dev)
        grp.kernels.check_error()
        # valid slots summed over the ranks (each rank routes its own batch)
        V = (idx >= 0).sum().to(torch.int64).reshape(1)
        if world > 1:
            dist.all_reduce(V)
        V = int(V.item())
        row = w.H + (w.H // 128) * 4 if fp8 else 2 * w.H
        d_bytes = V * row                        # rows sent by all ranks
        c_bytes = V * w.H * 2                    # rows pulled back by all ranks
        res = {"metric": "expert-parallel dispatch & combine logical GB/s across ranks (V3 shape)",
               "value": round((d_bytes + c_bytes) / ((d_ms + c_ms) * 1e-3) / 1e9, 2), "unit": "GB/s",
               "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(d_ms + c_ms, 5),
               "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
               "dtype": DTYPE, "data": "synthetic",
               "config": {**step_config(w, T, world), "parallelism": f"ep{world}"},
               "dispatch": {"us": round(d_ms * 1e3, 2),
                            "logical_gbs_per_rank": round(d_bytes / world / (d_ms * 1e-3) / 1e9, 1),
                            "includes": "layout, all-gather of counts, dispatch kernel, barrier"},
               "combine": {"us": round(c_ms * 1e3, 2),
                           "logical_gbs_per_rank": round(c_bytes / world / (c_ms * 1e-3) / 1e9, 1),
                           "includes": "barrier, combine kernel"},
               "pages_sm100_nvlink_context": {"dispatch_gbs": 726, "combine_gbs": 740, "sms": 64}}
    finally:
        grp.close()
    return res


def run_ours(args, rank, world, dev):
    import torch
    import torch.distributed as dist

    import combine_ep_get_06_b200 as ep

    w = W.WORKLOADS[args.workload]
    if args.tokens is not None:
        w = dataclasses.replace(w, T=args.tokens)
    inp = W.make_inputs(w, seed=rank)
    y_np = W.make_y(w, seed=rank)
    T, k, H = w.T, w.k, w.H

    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    x = bf16(inp["x"])
    y = bf16(y_np)
    idx = torch.from_numpy(inp["topk_idx"]).to(dev)
    wts = torch.from_numpy(inp["topk_weights"]).to(dev)
    fp8 = w.x_mode == "fp8_quant"
    handle = ep.EPHandle(T, k, w.E, w.S, w.align, device=dev)
    rows = handle.max_recv_rows
    recv_idx = torch.empty(rows, dtype=torch.int32, device=dev)
    recv_w = torch.empty(rows, dtype=torch.float32, device=dev)
    if fp8:
        recv_x = torch.empty(rows, H, dtype=torch.float8_e4m3fn, device=dev)
        recv_s = torch.empty(rows, H // 128, dtype=torch.float32, device=dev)
    else:
        recv_x = torch.empty(rows, H, dtype=torch.bfloat16, device=dev)
        recv_s = None
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def layout():
        ep.get_layout(idx, w.E, num_segments=w.S, expert_alignment=w.align, topk_weights=wts,
                      handle=handle, recv_topk_idx=recv_idx, recv_topk_weights=recv_w)

    def dispatch():
        ep.dispatch_with_handle(x, handle, use_fp8=fp8, recv_x=recv_x, recv_scales=recv_s)

    def layout_dispatch():   # the pages' dispatch(x, topk_idx, ...): routes and sends in one call
        ep.dispatch(x, idx, wts, w.E, expert_alignment=w.align, num_segments=w.S, handle=handle,
                    use_fp8=fp8, recv_x=recv_x, recv_scales=recv_s, recv_topk_idx=recv_idx,
                    recv_topk_weights=recv_w)

    def combine():
        ep.combine(y, handle, wts, out=out)

    for _ in range(args.warmup):
        layout_dispatch(); combine()
    torch.cuda.synchronize(dev)
    V = int(handle.counts.sum())
    P = int(handle.num_pad_rows[0])
    R = handle.total_rows()
    nbytes = step_bytes(w, T, V, P, R)
    handle.check_error()

    # The timed region: K steps with nothing between the calls, so each
    # kernel may launch while the one before it drains (programmatic
    # dependent launch); an event recorded between two kernels would stop it.
    K = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(nvsmi_device_id(dev))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    # Hold the stream for ~0.5 ms (torch's bounded sleep kernel, before the
    # start event) so that the host has queued the first steps when timing
    # starts: the timed region then holds device time only.
    torch.cuda._sleep(1_000_000)
    start.record(stream)
    for _ in range(K):
        layout_dispatch()
        combine()
    end.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    total_ms = start.elapsed_time(end)

    # Per-kernel breakdown after the timed region: the same step with an
    # event between the calls (slightly slower for it).
    K3 = max(5, min(50, K))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K3)]
    for e in ev:
        e[0].record(stream); layout_dispatch()
        e[1].record(stream); combine()
        e[2].record(stream)
    torch.cuda.synchronize(dev)
    ld_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    com_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    handle.check_error()

    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / K
    step_total = sum(nbytes.values())
    value = weak_scaling_gbs(step_total, world, ms_per_step)
    peak, peak_kind = hbm_peak()

    # the same step as two calls (layout, then dispatch with the handle), and
    # the dispatch kernel alone back to back, both after the timed region
    K2 = max(5, min(50, K))
    ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K2)]
    for i in range(K2):
        e = ev2[i]
        e[0].record(stream); layout()
        e[1].record(stream); dispatch()
        e[2].record(stream); combine()
        e[3].record(stream)
    torch.cuda.synchronize(dev)
    lay_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev2)
    dis_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev2)
    two_step_ms = statistics.mean(e[0].elapsed_time(e[3]) for e in ev2)
    handle.check_error()

    def rate(nb, ms):
        gbs = nb / (ms * 1e-3) / 1e9
        return {"us": round(ms * 1e3, 2), "bytes": nb, "gbs": round(gbs, 1), "frac_of_peak": round(gbs / peak, 4),
                "frac_of_nominal_8tbs": round(gbs / NOMINAL_HBM_GBS, 4)}

    res = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": DTYPE, "data": "synthetic",
        "config": step_config(w, T, world),
        "gpu_launches": K * (layout_launches(T, k) + 2),
        "step": "ep_layout_dispatch (layout + FP8 dispatch, one call) -> ep_combine",
        "layout_dispatch": {**rate(nbytes["layout"] + nbytes["dispatch"], ld_ms),
                            "note": "layout kernels and the dispatch kernel of one call, inside the step (events "
                                    "between the calls, after the timed region)"},
        "combine": rate(nbytes["combine"], com_ms),
        "dispatch": {**rate(nbytes["dispatch"], dis_ms), "valid_rows": V, "padding_rows": P,
                     "note": "the dispatch kernel between the layout and the combine of a two-call step "
                             "(ep_get_layout, ep_dispatch, ep_combine), after the timed step"},
        "two_call": {"layout_us": round(lay_ms * 1e3, 2), "dispatch_us": round(dis_ms * 1e3, 2),
                     "step_us": round(two_step_ms * 1e3, 2),
                     "note": "ep_get_layout, ep_dispatch, ep_combine as separate calls"},
        "clocks": clocks,
    }
    achieved = nbytes["combine"] / (com_ms * 1e-3) / 1e9
    res["roofline"] = {"bound": "hbm", "kernel": "combine_kernel", "achieved": round(achieved, 1),
                       "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                       "frac": round(achieved / peak, 4), "traffic": combine_traffic(w.name, T),
                       "algorithmic_bytes": nbytes["combine"]}

    n_x = max(5, min(50, K))

    # FP8 dispatch with GEMM-ready (MN-major) scales, same workload
    if fp8:
        ld = (rows + 3) // 4 * 4
        sc_mn = torch.empty(H // 128, ld, dtype=torch.float32, device=dev)
        mn = lambda: ep.dispatch_mn_scales(x, handle, recv_x=recv_x, recv_scales_mn=sc_mn, scales_ld=ld)
        res["dispatch_mn_scales"] = rate(nbytes["dispatch"], time_back_to_back(mn, n_x, stream))

    # NVFP4 dispatch (E2M1 codes, one e4m3 scale per 1x16 block), same workload
    if H % 32 == 0:
        nv_x = torch.empty(rows, H // 2, dtype=torch.uint8, device=dev)
        nv_s = torch.empty(rows, H // 16, dtype=torch.uint8, device=dev)
        nv = lambda: ep.dispatch_with_handle(x, handle, use_nvfp4=True, recv_x=nv_x, recv_scales=nv_s)
        nv_bytes = T * H * 2 + T * k * 4 + (V + P) * (H // 2 + H // 16)
        res["dispatch_nvfp4"] = rate(nv_bytes, time_back_to_back(nv, n_x, stream))

    # combine of FP8 expert outputs (the dispatch's own e4m3 rows and scales stand in for them)
    if fp8:
        out8 = torch.empty_like(out)
        c8 = lambda: ep.combine_fp8(recv_x, recv_s, handle, wts, out=out8)
        c8_bytes = V * (H + (H // 128) * 4) + T * k * 8 + T * H * 2
        res["combine_fp8"] = rate(c8_bytes, time_back_to_back(c8, n_x, stream))

    # dispatch and combine on a bounded number of SMs (the pages' #SMs column), same workload
    res["sm_budget"] = {"note": "dispatch and combine kernels alone, each CTA filling one SM, at most n SMs"}
    for n_sms in (24, 64):
        with ep.sm_budget(n_sms):
            res["sm_budget"][str(n_sms)] = {"dispatch": rate(nbytes["dispatch"], time_back_to_back(dispatch, n_x, stream)),
                                            "combine": rate(nbytes["combine"], time_back_to_back(combine, n_x, stream))}

    # the backward of the weighted combine (training), same workload
    gy = torch.empty(rows, H, dtype=torch.bfloat16, device=dev)
    gw = torch.empty(T, k, dtype=torch.float32, device=dev)
    g_out = out  # any [T,H] bf16 gradient; the forward's output serves
    bwd = lambda: ep.combine_backward(g_out, y, handle, wts, grad_y=gy, grad_weights=gw)
    bwd_bytes = T * H * 2 + V * H * 2 + (V + P) * H * 2 + T * k * 12
    res["combine_backward"] = rate(bwd_bytes, time_back_to_back(bwd, n_x, stream))
    handle.check_error()

    if not args.no_extra_workloads and args.tokens is None and w.name == WORKLOAD:
        for name in ("mid", "skewed"):
            res[name] = run_workload_lines(args, dev, name, peak)
    if not args.no_mgpu and H % 128 == 0:
        res["mgpu_local"] = run_mgpu_local(args, dev, w, inp, nbytes)
    if not args.no_decode:
        res["decode"] = run_decode(args, dev)
    if not args.no_e2e:
        res["e2e"] = run_e2e(args, dev, w, inp, y_np, nbytes)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w, inp, y_np)
    return res


def run_workload_lines(args, dev, name: str, peak: float) -> dict:
    """Dispatch and combine GB/s on another workload (its own seeded inputs):
    the step (one-call layout + dispatch, then combine), and the dispatch and
    combine kernels timed inside a two-call step (layout, dispatch, combine)."""
    import torch

    import combine_ep_get_06_b200 as ep

    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, seed=0)
    T, k, H = w.T, w.k, w.H

    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    x = bf16(inp["x"])
    y = bf16(W.make_y(w, seed=0))
    idx = torch.from_numpy(inp["topk_idx"]).to(dev)
    wts = torch.from_numpy(inp["topk_weights"]).to(dev)
    fp8 = w.x_mode == "fp8_quant"
    handle = ep.EPHandle(T, k, w.E, w.S, w.align, device=dev)
    rows = handle.max_recv_rows
    recv_x = torch.empty(rows, H, dtype=torch.float8_e4m3fn if fp8 else torch.bfloat16, device=dev)
    recv_s = torch.empty(rows, H // 128, dtype=torch.float32, device=dev) if fp8 else None
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    one = lambda: ep.dispatch(x, idx, wts, w.E, expert_alignment=w.align, num_segments=w.S, handle=handle,
                              use_fp8=fp8, recv_x=recv_x, recv_scales=recv_s)
    lay = lambda: ep.get_layout(idx, w.E, num_segments=w.S, expert_alignment=w.align, topk_weights=wts,
                                handle=handle)
    dis = lambda: ep.dispatch_with_handle(x, handle, use_fp8=fp8, recv_x=recv_x, recv_scales=recv_s)
    com = lambda: ep.combine(y, handle, wts, out=out)
    n = max(5, min(50, args.steps))
    step_ms = time_back_to_back(lambda: (one(), com()), n, stream)
    # the kernels inside a two-call step, each between its neighbours (as in the timed V3 step)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
    for e in ev:
        e[0].record(stream); lay()
        e[1].record(stream); dis()
        e[2].record(stream); com()
        e[3].record(stream)
    torch.cuda.synchronize(dev)
    dis_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    com_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in ev)
    handle.check_error()
    V = int(handle.counts.sum())
    P = int(handle.num_pad_rows[0])
    nb = step_bytes(w, T, V, P, handle.total_rows())

    def line(b, ms):
        gbs = b / (ms * 1e-3) / 1e9
        return {"us": round(ms * 1e3, 2), "bytes": b, "gbs": round(gbs, 1), "frac_of_peak": round(gbs / peak, 4)}

    in_mb = (x.numel() * x.element_size() + y.numel() * y.element_size()) / 1e6
    return {"config": step_config(w, T, 1)["workload"], "valid_rows": V, "padding_rows": P,
            "l2": f"no flush: the step's inputs (x and y, {in_mb:.0f} MB) exceed the 126 MB L2",
            "step": line(sum(nb.values()), step_ms), "dispatch": line(nb["dispatch"], dis_ms),
            "combine": line(nb["combine"], com_ms)}


def run_mgpu_local(args, dev, w, inp, nbytes, world=8):
    """The multi-GPU dispatch / combine kernels with all `world` ranks'
    blocks on this GPU: the step's batch split evenly over the ranks, so
    the concatenated batch (and the algorithmic bytes) are the step's.
    Each rank's launches go on a stream of its own.  The dispatch phase
    (per-rank layouts, the counts exchange as device copies, per-rank
    dispatch kernels) and the combine phase are each captured in a CUDA
    graph and timed over replays, so host launch costs are not counted."""
    import torch

    import combine_ep_get_06_b200 as ep
    from combine_ep_get_06_b200 import mgpu

    def bf16(a, device):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)

    T = inp["x"].shape[0]
    if T % world:
        return None
    Tr = T // world
    lr = mgpu.LocalRanks(world, Tr, w.k, w.E, w.H, expert_alignment=w.align, mode=ep.EP_X_BF16_TO_FP8,
                         device=dev, concurrent=True)
    xs = [bf16(inp["x"][r * Tr:(r + 1) * Tr], dev) for r in range(world)]
    idxs = [torch.from_numpy(inp["topk_idx"][r * Tr:(r + 1) * Tr].copy()).to(dev) for r in range(world)]
    wts = [torch.from_numpy(inp["topk_weights"][r * Tr:(r + 1) * Tr].copy()).to(dev) for r in range(world)]
    outs = [torch.empty(Tr, w.H, dtype=torch.bfloat16, device=dev) for _ in range(world)]
    for b in lr.blocks:
        b.y.zero_()
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        for _ in range(3):
            hs = lr.dispatch(xs, idxs, wts, use_fp8=True)
            lr.combine(hs, wts, outs)
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize(dev)
    g_d, g_c = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_d):
        hs = lr.dispatch(xs, idxs, wts, use_fp8=True)
    with torch.cuda.graph(g_c):
        lr.combine(hs, wts, outs)
    stream = torch.cuda.current_stream(dev)
    for _ in range(3):
        g_d.replay()
        g_c.replay()
    n = max(5, min(50, args.steps))
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    d_ms = c_ms = 0.0
    for _ in range(n):
        e[0].record(stream)
        g_d.replay()
        e[1].record(stream)
        g_c.replay()
        e[2].record(stream)
        torch.cuda.synchronize(dev)
        d_ms += e[0].elapsed_time(e[1])
        c_ms += e[1].elapsed_time(e[2])
    d_ms, c_ms = d_ms / n, c_ms / n
    for r in lr.ranks:
        r.check_error()
    del g_d, g_c
    return {"config": f"{world} ranks x {Tr} tokens on one GPU, a stream per rank, CUDA graphs, "
                      "fp8 dispatch + bf16 combine",
            "dispatch_phase_us": round(d_ms * 1e3, 2), "combine_us": round(c_ms * 1e3, 2),
            "dispatch_phase_gbs": round((nbytes["layout"] + nbytes["dispatch"]) / (d_ms * 1e-3) / 1e9, 1),
            "combine_gbs": round(nbytes["combine"] / (c_ms * 1e-3) / 1e9, 1),
            "launches_per_step": 2 * world + world + world}


def run_decode(args, dev):
    """decode: T=128, hidden 7168, 256 experts, top-8, alignment 1, FP8
    dispatch + BF16 combine; `pairs` layout->dispatch->combine pairs
    captured in one CUDA graph (4 routings in turn, shared receive
    buffers, as one layer after another would reuse them)."""
    import torch

    import combine_ep_get_06_b200 as ep

    w = W.WORKLOADS["decode"]
    n_route = 4
    inps = [W.make_inputs(w, seed=1000 + i) for i in range(n_route)]

    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    rows = ep.max_recv_rows(w.T, w.k, w.E, w.align)
    y = bf16(W.make_y(w, seed=1000, rows=rows))
    idx = [torch.from_numpy(i["topk_idx"]).to(dev) for i in inps]
    wts = [torch.from_numpy(i["topk_weights"]).to(dev) for i in inps]
    xs = [bf16(i["x"]) for i in inps]
    hs = [ep.EPHandle(w.T, w.k, w.E, w.S, w.align, device=dev) for _ in range(n_route)]
    ri = torch.empty(rows, dtype=torch.int32, device=dev)
    rw = torch.empty(rows, dtype=torch.float32, device=dev)
    rq = torch.empty(rows, w.H, dtype=torch.float8_e4m3fn, device=dev)
    rs = torch.empty(rows, w.H // 128, dtype=torch.float32, device=dev)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=dev)

    def pairs(n, cached=False):
        for p in range(n):
            i = p % n_route
            if cached:
                ep.dispatch_with_handle(xs[i], hs[i], use_fp8=True, recv_x=rq, recv_scales=rs)
            else:   # layout + dispatch in one call
                ep.dispatch(xs[i], idx[i], wts[i], w.E, expert_alignment=w.align, num_segments=w.S,
                            handle=hs[i], use_fp8=True, recv_x=rq, recv_scales=rs,
                            recv_topk_idx=ri, recv_topk_weights=rw)
            ep.combine(y, hs[i], wts[i], out=out)

    result = {"config": "decode: T=128 hidden=7168 experts=256 topk=8 alignment=1 fp8 dispatch + "
                        "bf16 combine", "pairs_per_graph": args.decode_pairs}
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        pairs(n_route)
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize(dev)
    for cached in (False, True):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            pairs(args.decode_pairs, cached)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize(dev)
        times = []
        for _ in range(args.decode_replays):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            b.synchronize()
            times.append(a.elapsed_time(b))
        us = statistics.median(times) * 1e3 / args.decode_pairs
        result["cached_handle_us_per_pair" if cached else "us_per_pair"] = round(us, 3)
        del g
    for h in hs:
        h.check_error()
    return result


def run_e2e(args, dev, w, inp, y_np, nbytes):
    """Same metric through the public API with HOST inputs: every step
    copies x, topk_idx, topk_weights and y from pinned host memory, runs
    layout -> dispatch -> combine, and copies recv_x, recv_scales and the
    combined output back to pinned host memory.  Steps are pipelined the
    way a host-fed job runs them: two sets of device buffers, and the
    copies in (one stream), kernels (another) and copies out (a third)
    overlap across consecutive steps.  A set is refilled only after its
    previous step's kernels and copies out have finished (events)."""
    import torch

    import combine_ep_get_06_b200 as ep

    T, k, H = w.T, w.k, w.H
    fp8 = w.x_mode == "fp8_quant"
    hx = torch.from_numpy(np.ascontiguousarray(inp["x"]).view(np.int16)).view(torch.bfloat16).pin_memory()
    hi = torch.from_numpy(inp["topk_idx"]).pin_memory()
    hw = torch.from_numpy(inp["topk_weights"]).pin_memory()
    hy = torch.from_numpy(np.ascontiguousarray(y_np).view(np.int16)).view(torch.bfloat16).pin_memory()
    rows = ep.max_recv_rows(T, k, w.E, w.align)
    qdt = torch.float8_e4m3fn if fp8 else torch.bfloat16

    def device_set():
        return {"handle": ep.EPHandle(T, k, w.E, w.S, w.align, device=dev),
                "x": torch.empty_like(hx, device=dev), "i": torch.empty_like(hi, device=dev),
                "w": torch.empty_like(hw, device=dev), "y": torch.empty_like(hy, device=dev),
                "rq": torch.empty(rows, H, dtype=qdt, device=dev),
                "rs": torch.empty(rows, H // 128, dtype=torch.float32, device=dev) if fp8 else None,
                "out": torch.empty(T, H, dtype=torch.bfloat16, device=dev),
                "in_done": torch.cuda.Event(), "disp_done": torch.cuda.Event(),
                "comp_done": torch.cuda.Event(), "out_done": torch.cuda.Event()}

    sets = [device_set(), device_set()]
    h_rq = torch.empty(rows, H, dtype=qdt).pin_memory()
    h_rs = torch.empty(rows, H // 128, dtype=torch.float32).pin_memory() if fp8 else None
    h_out = torch.empty(T, H, dtype=torch.bfloat16).pin_memory()
    h2d = hx.numel() * 2 + hi.numel() * 8 + hw.numel() * 4 + hy.numel() * 2
    d2h = h_rq.numel() * h_rq.element_size() + (h_rs.numel() * 4 if fp8 else 0) + h_out.numel() * 2
    s_in, s_k, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def step(i):
        d = sets[i % 2]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(d["comp_done"])       # the set's last kernels have read its inputs
            d["x"].copy_(hx, non_blocking=True)
            d["i"].copy_(hi, non_blocking=True)
            d["w"].copy_(hw, non_blocking=True)
            d["y"].copy_(hy, non_blocking=True)
            d["in_done"].record(s_in)
        with torch.cuda.stream(s_k):
            s_k.wait_event(d["in_done"])
            if i >= 2:
                s_k.wait_event(d["out_done"])         # its outputs have been copied out
            ep.dispatch(d["x"], d["i"], d["w"], w.E, expert_alignment=w.align, num_segments=w.S,
                        handle=d["handle"], use_fp8=fp8, recv_x=d["rq"], recv_scales=d["rs"])
            d["disp_done"].record(s_k)
            ep.combine(d["y"], d["handle"], d["w"], out=d["out"])
            d["comp_done"].record(s_k)
        with torch.cuda.stream(s_out):
            s_out.wait_event(d["disp_done"])
            h_rq.copy_(d["rq"], non_blocking=True)
            if fp8:
                h_rs.copy_(d["rs"], non_blocking=True)
            s_out.wait_event(d["comp_done"])
            h_out.copy_(d["out"], non_blocking=True)
            d["out_done"].record(s_out)

    main = torch.cuda.current_stream(dev)
    for s_ in (s_in, s_k, s_out):
        s_.wait_stream(main)
    for i in range(2):
        step(i)
    for s_ in (s_in, s_k, s_out):
        main.wait_stream(s_)
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(main)
    for s_ in (s_in, s_k, s_out):
        s_.wait_stream(main)
    for i in range(args.e2e_steps):
        step(i)
    for s_ in (s_in, s_k, s_out):
        main.wait_stream(s_)
    b.record(main)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b) / args.e2e_steps
    total = sum(nbytes.values())
    return {"value": round(total / (ms * 1e-3) / 1e9, 2), "unit": "GB/s", "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
            "pipelined": "copies in / kernels / copies out on three streams, two buffer sets"}


# ------------------------------------------------------ CPU oracle timing

def time_oracle_step(w: W.Workload, inp, y_np):
    import oracle

    T = inp["x"].shape[0]
    t0 = time.perf_counter()
    lay = oracle.layout(inp["topk_idx"], w.E, w.S, w.align, inp["topk_weights"])
    oracle.dispatch(lay, inp["x"], oracle.X_BF16_QUANT_FP8 if w.x_mode == "fp8_quant" else oracle.X_BF16)
    oracle.combine(lay["slot_map"], T, w.k, y_np, inp["topk_weights"])
    dt = time.perf_counter() - t0
    V = int(lay["counts"].sum())
    R = lay["R"]
    nb = step_bytes(w, T, V, R - V, R)
    return dt, sum(nb.values())


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(w: W.Workload, inp, y_np, reps=3):
    runs = [time_oracle_step(w, inp, y_np) for _ in range(reps)]
    dt = statistics.median(r[0] for r in runs)
    nb = runs[0][1]
    return {"value": round(nb / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"the full {w.name} workload (T={inp['x'].shape[0]}), layout+dispatch+combine, "
                      f"median of {reps} runs ({dt:.2f} s each), single-threaded C",
            "host_cores_available": os.cpu_count(), "cpu_model": cpu_model()}


def run_reference(args):
    """The reference arm: the CPU oracle, timed as it stands, on a bounded
    token sample of the same workload per step (sized so that the whole
    run stays within about two minutes)."""
    w = W.WORKLOADS[args.workload]
    if args.tokens is not None:
        w = dataclasses.replace(w, T=args.tokens)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    probe_T = 64
    inp = W.make_inputs(w, seed=0, T=probe_T)
    y_np = W.make_y(w, seed=0, rows=W.y_rows(W.Workload(**{**w.__dict__, "T": probe_T})))
    dt, _ = time_oracle_step(w, inp, y_np)
    per_token = dt / probe_T
    budget = 100.0 / max(1, args.steps + args.warmup)
    T_s = int(max(16, min(w.T, budget / max(per_token, 1e-9))))
    inp = W.make_inputs(w, seed=0, T=T_s)
    y_np = W.make_y(w, seed=0, rows=W.y_rows(W.Workload(**{**w.__dict__, "T": T_s})))
    for _ in range(args.warmup):
        time_oracle_step(w, inp, y_np)
    tot_t, tot_b = 0.0, 0
    for _ in range(args.steps):
        dt, nb = time_oracle_step(w, inp, y_np)
        tot_t += dt
        tot_b += nb
    value = tot_b / tot_t / 1e9
    sample = (f"{T_s} of the {w.T} tokens of the {w.name} workload per step (same hidden, experts, "
              f"top-k, alignment), layout+dispatch+combine, single-threaded C oracle")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot_t / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": DTYPE,
        "data": "synthetic",
        "config": {**step_config(w, T_s, world), "sampled_from": f"{w.name} T={w.T}"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    import torch
    import torch.distributed as dist

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
    try:
        res = run_ep(args, rank, world, dev) if args.ep else run_ours(args, rank, world, dev)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
