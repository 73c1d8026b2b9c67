#!/usr/bin/env python
"""Benchmark of the padding-free MoE layer hot path (forward + RBD plan + backward).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = moe_route -> pft_build -> moe_dispatch -> moe_expert_ffn -> moe_combine
-> moe_backward over one batch of synthetic tokens, with rbd_plan on a side stream
after routing (PFTMoELayer.step); inputs and weights resident in HBM.  Rank 0 prints
one JSON line.  ``value`` comes from K timed steps with no per-kernel events; a second
pass of the same K steps records a CUDA event pair around every launch for the
per-kernel table and the roofline.  ``e2e`` runs the same steps with each step's
inputs copied from pinned host memory and its results copied back (double-buffered
on copy streams).  With N > 1 (torchrun, one process per GPU) every rank runs an
independent replica on its own tokens: the layer has no exchange step on one GPU,
so there is no data-path collective; the timed region is bracketed by barriers and
the reported time is the max over ranks.

``--impl reference`` times the float64 CPU oracle (test infrastructure) on the
host cores, on bounded token samples of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer fwd+bwd tokens/s; grouped-GEMM % of BF16 peak; dispatch/combine GB/s"
DEFAULT_WORKLOAD = "dsmoe16b_bf16"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    ap.add_argument("--no-sort-stress", action="store_true", help="skip the PFT / RBD stress-shape timing")
    ap.add_argument("--cpu-sample-tokens", type=int, default=512)
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "100"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------- algorithmic work per kernel
def kernel_work(cfg, name):
    """(kind, amount per launch): FLOPs for contractions, bytes for data movement."""
    T, d, E, h, k, N = cfg.T, cfg.d, cfg.E, cfg.h, cfg.k, cfg.N
    b = 2 if cfg.dtype == "bf16" else 4
    flops = {
        "ffn_gemm1_swiglu": 2.0 * N * d * 2 * h,
        "ffn_gemm2": 2.0 * N * h * d,
        "ffn_dgrad_act_swiglu_bwd": 2.0 * N * d * h,
        "ffn_dgrad_x": 2.0 * N * 2 * h * d,
        "ffn_wgrad_w1w3": 2.0 * N * d * 2 * h,
        "ffn_wgrad_w2": 2.0 * N * h * d,
        "gate_logits": 2.0 * T * d * E,
        "gate_wgrad": 2.0 * T * d * E,
    }
    if name in flops:
        return "tensor", flops[name]
    bytes_ = {
        "dispatch": (T + N) * d * b + 4 * N,
        "combine": N * d * b + T * d * b + 8 * N,
        "combine_bwd": T * d * b + 2 * N * d * b + 12 * N,
        "token_grad": N * d * b + T * d * b + T * E * (4 + 2) + 16 * N,
        "route_topk": T * E * 4 + 8 * N,
        "pft_hist": 4 * N,
        "pft_scan": 8 * E,
        "pft_scatter": 8 * N + 16 * N,
        "transpose": 2 * d * E * b,
    }
    if cfg.has_rbd:   # RBD plan kernels: ids in, pilot / replica lists out (P <= N)
        P = T * min(k, E // (cfg.rbd_epd * cfg.rbd_dpn))
        bytes_.update({"rbd_count": 4 * N + 8 * T, "rbd_scan_tokens": 12 * T, "rbd_emit": 4 * N + 16 * P,
                       "rbd_hist": 4 * P, "rbd_scan_nodes": 8 * T, "rbd_scatter": 24 * P,
                       "rbd_scan_replicas": 8 * P, "rbd_final": 12 * N + 8 * T})
    if name in bytes_:
        return "hbm", float(bytes_[name])
    return None, None


def gemm_names():
    return ["ffn_gemm1_swiglu", "ffn_gemm2", "ffn_dgrad_act_swiglu_bwd", "ffn_dgrad_x", "ffn_wgrad_w1w3",
            "ffn_wgrad_w2"]


def traffic_for(kernel):
    """DRAM bytes per launch from a committed ncu capture, if the kernel source has not changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    ent = t.get(kernel)
    if not ent:
        return None
    src = os.path.join(ROOT, ent["source"])
    if not os.path.exists(src):
        return None
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    if sha != ent.get("source_sha256"):
        return None
    return ent["dram_bytes_per_launch"]


# -------------------------------------------------------------- CPU oracle leg
def oracle_sample(inp_cpu64, cfg, n_tok, seed=0):
    """Time the float64 oracle's full layer (forward + backward) on n_tok tokens."""
    import numpy as np
    import oracle as O
    rng = np.random.default_rng(seed)
    toks = np.sort(rng.choice(cfg.T, size=min(n_tok, cfg.T), replace=False))
    x, wg, bias, w1, w3, w2, dy = inp_cpu64
    t0 = time.perf_counter()
    f = O.layer_forward(x[toks], wg, bias, w1, w3, w2, cfg.k)
    O.layer_backward(f, dy[toks], x[toks], wg, w1, w3, w2)
    if cfg.has_rbd:
        O.rbd_plan(f["ids"], cfg.E, cfg.rbd_epd, cfg.rbd_dpn)
    return len(toks), time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def inputs_to_cpu64(inp):
    import torch
    cv = lambda t: None if t is None else t.detach().to("cpu").to(torch.float64).numpy()
    return tuple(cv(t) for t in (inp.x, inp.wg, inp.bias, inp.w1, inp.w3, inp.w2, inp.dy))


def run_reference(args):
    """Reference arm: the CPU oracle as it stands, on bounded token samples of the workload."""
    from padding_free_moe_b200 import replicas
    info = replicas.rank_info()
    rank, world = info.rank, info.world
    if rank != 0:
        return 0
    from workloads import get_config, make_inputs
    cfg = get_config(args.workload)
    inp = make_inputs(cfg, seed=0, device="cpu")
    cpu = inputs_to_cpu64(inp)
    n_tok = max(1, min(args.cpu_sample_tokens // 4, cfg.T))
    for _ in range(args.warmup):
        oracle_sample(cpu, cfg, n_tok)
    tot_tok, tot_s = 0, 0.0
    for i in range(args.steps):
        n, s = oracle_sample(cpu, cfg, n_tok, seed=i + 1)
        tot_tok += n
        tot_s += s
    value = tot_tok / tot_s
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(cfg, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{n_tok} random tokens of {cfg.name} per step through the float64 oracle "
                                   f"(forward, RBD plan, backward)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_block(cfg, world):
    return {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "E": cfg.E, "h": cfg.h, "k": cfg.k,
            "tokens_per_gpu": cfg.T, "global_batch": cfg.T * world,
            "rbd_map": (f"{cfg.rbd_epd} experts/device, {cfg.rbd_dpn} devices/node" if cfg.has_rbd else None),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "inputs larger than L2 (expert weights alone exceed 126 MB)"}


# ------------------------------------------------------------------ our arm
def stress_sort(L, torch, dev, stream, hbm_gbs, reps=20):
    """PFT build and RBD plan on a scaled shape (T = 2^20, E = 256, k = 8, RBD map 8 experts per
    device, 4 devices per node): at the layer configs these kernels are launch-latency bound, so
    their HBM efficiency is measured here.  Synthetic ids, distinct per token: (r_t + 37 j) mod E.
    Algorithmic bytes: PFT reads ids + weights (8Tk) and writes token_ids, expert_ids, weights,
    pos (16Tk) plus 8E of counts; the RBD plan reads ids (4Tk) and writes its lists (about 36Tk)."""
    T, E, k, epd, dpn = 1 << 20, 256, 8, 8, 4
    N = T * k
    g = torch.Generator(device=dev).manual_seed(11)
    r = torch.randint(0, E, (T, 1), generator=g, device=dev, dtype=torch.int64)
    ids = ((r + 37 * torch.arange(k, device=dev)) % E).to(torch.int32).contiguous()
    w = torch.full((T, k), 1.0 / k, device=dev)
    i32 = dict(device=dev, dtype=torch.int32)
    tpe, off, tiles = torch.empty(E, **i32), torch.empty(E + 1, **i32), torch.empty(E + 1, **i32)
    tok, eid, pos = torch.empty(N, **i32), torch.empty(N, **i32), torch.empty(N, **i32)
    cw = torch.empty(N, device=dev)
    err = torch.zeros(1, **i32)
    pws_b = L.pft_build_workspace_size(T, E, k)
    pws = torch.empty(max(pws_b, 256), device=dev, dtype=torch.uint8)
    n_nodes = E // (epd * dpn)
    P = T * min(k, n_nodes)
    ppn, noff = torch.empty(n_nodes, **i32), torch.empty(n_nodes + 1, **i32)
    ptok, pnode, pdev = torch.empty(P, **i32), torch.empty(P, **i32), torch.empty(P, **i32)
    roff, rexp, apil, cnt = torch.empty(P + 1, **i32), torch.empty(N, **i32), torch.empty(N, **i32), torch.empty(2, **i32)
    rws_b = L.rbd_plan_workspace_size(T, k, E, epd, dpn)
    rws = torch.empty(max(rws_b, 256), device=dev, dtype=torch.uint8)

    def pft():
        L.pft_build(ids, w, T, E, k, tpe, off, tok, eid, cw, pos, tiles, pws, pws_b, err, stream)

    def rbd():
        L.rbd_plan(ids, T, k, E, epd, dpn, ppn, noff, ptok, pnode, pdev, roff, rexp, apil, cnt, rws, rws_b, err,
                   stream)

    out = {}
    for name, fn, alg in (("pft_build", pft, 24 * N + 8 * E), ("rbd_plan", rbd, 40 * N)):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) / reps * 1000
        gbs = alg / (us * 1e-6) / 1e9
        # one more pass with per-kernel events: where the time goes inside the plan
        L.moe_profile_reset()
        L.moe_profile_enable(True)
        fn()
        torch.cuda.synchronize()
        L.moe_profile_enable(False)
        kern = {nm: round(ms * 1000, 1) for nm, (c, ms) in L.moe_profile_read().items()}
        out[name] = {"T": T, "E": E, "k": k, "us": us, "algorithmic_bytes": alg, "gbs": gbs, "frac": gbs / hbm_gbs,
                     "kernel_us": kern}
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item()):#x} in the PFT / RBD stress shape")
    out["rbd_plan"]["pilots"] = int(cnt[0].item())
    return out


def run_ours(args):
    import torch
    from padding_free_moe_b200 import _lib as L
    from padding_free_moe_b200 import replicas
    from padding_free_moe_b200.layer import PFTMoELayer, Shape
    from workloads import get_config, make_inputs
    from workloads.generate import storage_dtype

    info = replicas.rank_info()
    rank, world, local_rank = info.rank, info.world, info.local_rank
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    replicas.init(info, "nccl", timeout_s=120, device=dev)
    cfg = get_config(args.workload)
    inp = make_inputs(cfg, seed=1000 + rank, device=dev)
    layer = PFTMoELayer(Shape(cfg.T, cfg.d, cfg.E, cfg.h, cfg.k, storage_dtype(cfg), cfg.rbd_epd, cfg.rbd_dpn), dev)
    stream = torch.cuda.current_stream()

    def step():
        layer.step(inp.x, inp.wg, inp.bias, inp.w1, inp.w3, inp.w2, inp.dy, stream)

    def barrier():
        replicas.barrier(info)

    def max_over_ranks(v: float) -> float:
        return replicas.max_over_ranks(v, info, device=dev)

    warm = max(3, args.warmup)
    for _ in range(warm):
        step()
    torch.cuda.synchronize()
    if layer.device_error() != 0:
        raise RuntimeError(f"device error word {layer.device_error():#x} after warm-up")

    # ---- device-timed region, inputs resident (no per-kernel events in it)
    clk = ClockSampler(replicas.physical_gpu_index(local_rank))
    barrier()
    torch.cuda.synchronize()
    clk.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = clk.stop()
    ms_total = max_over_ranks(ev0.elapsed_time(ev1))
    ms_step = ms_total / args.steps
    value = world * cfg.T / (ms_step * 1e-3)

    # ---- the same steps again with a CUDA event pair around every kernel launch (on the
    # stream it is launched on): per-kernel durations for the roofline and launch counts.
    # Kept out of the headline pass because the events add host-side gaps between kernels;
    # the RBD plan runs in line here so that each event pair times one kernel's own work.
    L.moe_profile_reset()
    barrier()
    torch.cuda.synchronize()
    L.moe_profile_enable(True)
    for _ in range(args.steps):
        layer.step(inp.x, inp.wg, inp.bias, inp.w1, inp.w3, inp.w2, inp.dy, stream, overlap_rbd=False)
    torch.cuda.synchronize()
    L.moe_profile_enable(False)
    barrier()
    kern = L.moe_profile_read()

    # ---- end to end through the public API: every step copies its inputs (x, dY) from pinned
    # host memory and reads its results (y, dx) back to pinned host memory.  Copies run on
    # their own streams, double-buffered, so step i+1's inputs travel while step i computes;
    # the timed region ends when the last step's results are on the host.
    x_h = inp.x.to("cpu").pin_memory()
    dy_h = inp.dy.to("cpu").pin_memory()
    x_d = [torch.empty_like(inp.x) for _ in range(2)]
    dy_d = [torch.empty_like(inp.dy) for _ in range(2)]
    y_st = [torch.empty_like(layer.y) for _ in range(2)]
    dx_st = [torch.empty_like(layer.dx) for _ in range(2)]
    y_h = [torch.empty_like(layer.y, device="cpu").pin_memory() for _ in range(2)]
    dx_h = [torch.empty_like(layer.dx, device="cpu").pin_memory() for _ in range(2)]
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of buffer b on the device
    ev_used = [torch.cuda.Event() for _ in range(2)]   # the step reading buffer b has finished
    ev_out = [torch.cuda.Event() for _ in range(2)]    # results of buffer b staged
    ev_read = [torch.cuda.Event() for _ in range(2)]   # staged results of buffer b on the host
    e2e_steps = max(3, min(args.steps, 50))

    def run_e2e(n, start_event=None):
        if start_event is not None:
            h2d_s.wait_event(start_event)

        def h2d(i):
            b = i % 2
            if i >= 2:
                h2d_s.wait_event(ev_used[b])
            with torch.cuda.stream(h2d_s):
                x_d[b].copy_(x_h, non_blocking=True)
                dy_d[b].copy_(dy_h, non_blocking=True)
            ev_in[b].record(h2d_s)

        h2d(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                h2d(i + 1)
            stream.wait_event(ev_in[b])
            layer.step(x_d[b], inp.wg, inp.bias, inp.w1, inp.w3, inp.w2, dy_d[b], stream)
            if i >= 2:
                stream.wait_event(ev_read[b])
            with torch.cuda.stream(stream):
                y_st[b].copy_(layer.y)
                dx_st[b].copy_(layer.dx)
            ev_used[b].record(stream)
            ev_out[b].record(stream)
            d2h_s.wait_event(ev_out[b])
            with torch.cuda.stream(d2h_s):
                y_h[b].copy_(y_st[b], non_blocking=True)
                dx_h[b].copy_(dx_st[b], non_blocking=True)
            ev_read[b].record(d2h_s)
        stream.wait_event(ev_read[(n - 1) % 2])

    run_e2e(3)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run_e2e(e2e_steps, start_event=e0)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1)) / e2e_steps
    h2d = x_h.numel() * x_h.element_size() + dy_h.numel() * dy_h.element_size()
    d2h = y_h[0].numel() * y_h[0].element_size() + dx_h[0].numel() * dx_h[0].element_size()
    if not (torch.equal(y_h[(e2e_steps - 1) % 2], layer.y.cpu()) and torch.equal(dx_h[(e2e_steps - 1) % 2], layer.dx.cpu())):
        raise RuntimeError("end-to-end results read back to the host differ from the device results")
    if layer.device_error() != 0:
        raise RuntimeError(f"device error word {layer.device_error():#x}")

    # ---- roofline of the dominant kernel + per-kernel table
    peaks, peak_src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]))
    tc_peak = float(peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"]))
    kernels = {}
    for nm, (n_launch, ms) in sorted(kern.items(), key=lambda kv: -kv[1][1]):
        per_ms = ms / n_launch
        kind, work = kernel_work(cfg, nm)
        ent = {"launches": n_launch, "ms_per_launch": per_ms, "share": ms / sum(v[1] for v in kern.values())}
        if kind == "tensor":
            ent["tflops"] = work / (per_ms * 1e-3) / 1e12
            ent["frac_of_peak"] = ent["tflops"] / tc_peak
        elif kind == "hbm":
            ent["gbs"] = work / (per_ms * 1e-3) / 1e9
            ent["frac_of_peak"] = ent["gbs"] / hbm
        kernels[nm] = ent
    known = {nm: v for nm, v in kern.items() if kernel_work(cfg, nm)[0] is not None}
    dom = max((known or kern).items(), key=lambda kv: kv[1][1])[0]
    kind, work = kernel_work(cfg, dom)
    dom_ms = kern[dom][1] / kern[dom][0]
    if kind == "tensor":
        ach = work / (dom_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": dom, "achieved": ach, "peak": tc_peak, "unit": "TFLOP/s",
                "frac": ach / tc_peak, "traffic": traffic_for(dom),
                "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a long step)",
                "work_per_launch": work}
    else:
        ach = work / (dom_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": dom, "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                "traffic": traffic_for(dom), "peak_source": f"{peak_src} hbm_gbs", "work_per_launch": work}
    gemm_ms = sum(kern[n][1] for n in gemm_names() if n in kern) / args.steps
    gemm_flops = 18.0 * cfg.N * cfg.d * cfg.h
    gemm_tflops = gemm_flops / (gemm_ms * 1e-3) / 1e12 if gemm_ms > 0 else None

    def gbs(nm):
        return kernels.get(nm, {}).get("gbs")

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": warm, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if cfg.dtype == "bf16" else "f32", "data": "synthetic",
        "config": config_block(cfg, world),
        "clocks": clocks,
        "e2e": {"value": world * cfg.T / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": int(sum(v[0] for v in kern.values())),
        "roofline": roof,
        "grouped_gemm": {"tflops": gemm_tflops, "pct_of_bf16_peak": (100 * gemm_tflops / tc_peak) if gemm_tflops else None,
                         "pct_of_burst_peak": (100 * gemm_tflops / float(peaks.get("bf16_tflops", 1590.0)))
                         if gemm_tflops else None,
                         "flops_per_step": gemm_flops, "ms_per_step": gemm_ms},
        "dispatch_gbs": gbs("dispatch"), "combine_gbs": gbs("combine"),
        "sort_stress": None if args.no_sort_stress else stress_sort(L, torch, dev, stream, hbm),
        "kernels": kernels,
    }

    # ---- CPU oracle baseline (rank 0, one GPU only)
    if world == 1 and not args.no_cpu_baseline:
        cpu = inputs_to_cpu64(inp)
        n, s = oracle_sample(cpu, cfg, args.cpu_sample_tokens)
        line["cpu_baseline"] = {"value": n / s, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"{n} random tokens of {cfg.name} through the float64 oracle "
                                          f"(forward, RBD plan, backward), {s:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    replicas.finish(info)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
