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

The headline workload is the DeepSeek-V3-like layer (T=8192, d=7168, E=256,
h=2048, k=8), the largest single-GPU configuration; the DeepSeek-MoE-16B-like,
skewed DeepSeek-V3-like and fine-grained layers are timed after it and reported
under ``workloads``; the headline layer's step with the dispatch gather fused into
the first expert GEMM (PFTMoELayer(fused_gather=True)) is reported under
``gathered_forward`` (``--no-gathered`` skips it), and ``sort_stress`` times the PFT
build and the RBD plan on a 2^20-token shape (``--sort-stress-only`` runs just that).
``--gpus N`` without a torchrun environment relaunches this script under torchrun
with N ranks.
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
DEFAULT_WORKLOAD = "dsv3_bf16"
EXTRA_WORKLOADS = "dsmoe16b_bf16,dsv3_zipf_bf16,finegrained_bf16"
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
    ap.add_argument("--cpu-sample-seconds", type=float, default=12.0,
                    help="oracle time the cpu_baseline leg spends on token samples")
    ap.add_argument("--ref-tokens", type=int, default=0,
                    help="reference arm: tokens per step (0 = sized from the workload)")
    ap.add_argument("--extra-workloads", default=EXTRA_WORKLOADS,
                    help="comma-separated workloads timed after the headline one ('' = none)")
    ap.add_argument("--extra-steps", type=int, default=10)
    ap.add_argument("--sort-stress-only", action="store_true",
                    help="time only the PFT build and RBD plan on the stress shape (T = 2^20, E = 256, k = 8)")
    ap.add_argument("--no-gathered", action="store_true",
                    help="skip the timing of the step with the gather fused into the first expert GEMM")
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
        # dense dz rows x Wg^T reduce-added into dx: dz and Wg^T read, dx read and written (in L2/HBM)
        "gate_dx": 2 * T * d * b + T * E * b + d * E * b,
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


def traffic_for(kernel, workload):
    """DRAM bytes per launch of `kernel` at `workload` from a committed ncu capture
    (profiles/traffic.json), if the kernel's source file has not changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    ent = t.get(workload, {}).get(kernel)
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
class LazyWeights:
    """Stacked expert weights [E, r, c] (torch, any device) handed to the oracle one expert at a
    time as float64 numpy: the largest layers' float64 stacks would need tens of GB of host
    memory.  The conversion time is recorded so that it can be left out of the oracle's time."""

    def __init__(self, t, clock):
        self.t = t
        self.shape = tuple(t.shape)
        self.clock = clock

    def __len__(self):
        return self.shape[0]

    def __getitem__(self, e):
        import torch
        t0 = time.perf_counter()
        a = self.t[int(e)].detach().to("cpu").to(torch.float64).numpy()
        self.clock[0] += time.perf_counter() - t0
        return a


class OracleSampler:
    """The float64 CPU oracle (as it stands) on samples of one workload's tokens.

    One sample = the oracle's gate, routing, PFT, dispatch, expert FFN, combine, the
    backward of each of those and (with a device map) the RBD plan, on n tokens.  The
    oracle's own layer_backward keeps weight gradients of all E experts in float64 (30 GB
    per matrix for the DeepSeek-V3-like layer), so the backward calls its steps directly,
    one expert at a time, as layer_backward does.  The time reported is the oracle's,
    without the conversion of the BF16 inputs to float64."""

    def __init__(self, inp, cfg):
        import torch
        self.cfg = cfg
        self.clock = [0.0]
        cv = lambda t: None if t is None else t.detach().to("cpu").to(torch.float64).numpy()
        self.x, self.wg, self.bias, self.dy = cv(inp.x), cv(inp.wg), cv(inp.bias), cv(inp.dy)
        self.w1 = LazyWeights(inp.w1, self.clock)
        self.w3 = LazyWeights(inp.w3, self.clock)
        self.w2 = LazyWeights(inp.w2, self.clock)

    def sample(self, n_tok, seed):
        """(tokens, oracle seconds) of one sample of n_tok random tokens."""
        import numpy as np
        import oracle as O
        cfg = self.cfg
        rng = np.random.default_rng(seed)
        toks = np.sort(rng.choice(cfg.T, size=min(n_tok, cfg.T), replace=False))
        x, dy = self.x[toks], self.dy[toks]
        self.clock[0] = 0.0
        t0 = time.perf_counter()
        f = O.layer_forward(x, self.wg, self.bias, self.w1, self.w3, self.w2, cfg.k)
        pft = f["pft"]
        dO, g = O.combine_backward(dy, f["O"], pft["pos"], f["w"])
        offs = pft["expert_offsets"]
        dX = np.zeros_like(f["x_pft"])
        for e in range(cfg.E):
            r0, r1 = int(offs[e]), int(offs[e + 1])
            if r1 > r0:
                gr = O.expert_backward(f["x_pft"][r0:r1], f["H1"][r0:r1], f["H3"][r0:r1], f["A"][r0:r1], dO[r0:r1],
                                       self.w1[e], self.w3[e], self.w2[e])
                dX[r0:r1] = gr["dX"]
        _, _, dx_gate = O.gate_backward(x, self.wg, f["ids"], f["w"], g, cfg.E)
        O.token_grad(dX, pft["pos"]) + dx_gate
        if cfg.has_rbd:
            O.rbd_plan(f["ids"], cfg.E, cfg.rbd_epd, cfg.rbd_dpn)
        return len(toks), time.perf_counter() - t0 - self.clock[0]

    def tokens_per_second(self, seconds, batch, seed0=0):
        """Samples of `batch` tokens until the oracle has spent `seconds`: (tokens/s, tokens, seconds)."""
        tot_n, tot_s, i = 0, 0.0, 0
        while tot_s < seconds and tot_n < self.cfg.T:
            n, dt = self.sample(batch, seed0 + i)
            tot_n += n
            tot_s += dt
            i += 1
        return tot_n / tot_s, tot_n, tot_s


def oracle_batch(cfg):
    """Tokens per oracle sample: about the same oracle work per sample for every workload
    (a token costs k expert passes over d x h weights)."""
    per_token = cfg.k * cfg.d * cfg.h
    return int(max(1, min(256, round(2.0e8 / per_token))))


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def run_reference(args):
    """Reference arm: the CPU oracle as it stands, on bounded token samples of the workload.
    The inputs are generated with torch's seeded generator (on the GPU when there is one: the
    DeepSeek-V3-like weights take minutes to draw on host cores); nothing else uses the GPU."""
    from padding_free_moe_b200 import replicas
    info = replicas.rank_info()
    rank, world = info.rank, info.world
    if rank != 0:
        return 0
    import torch
    from workloads import get_config, make_inputs
    cfg = get_config(args.workload)
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(cfg, seed=0, device=gen_dev)
    smp = OracleSampler(inp, cfg)
    n_tok = args.ref_tokens if args.ref_tokens > 0 else oracle_batch(cfg)
    for i in range(args.warmup):
        smp.sample(n_tok, 10_000 + i)
    tot_tok, tot_s = 0, 0.0
    for i in range(args.steps):
        n, sec = smp.sample(n_tok, i + 1)
        tot_tok += n
        tot_s += sec
    value = tot_tok / tot_s
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(cfg, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{n_tok} random tokens of {cfg.name} per step through the float64 oracle "
                                   f"(forward, RBD plan, backward; expert weights converted to float64 one "
                                   f"expert at a time, conversion not timed)"},
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


def build_layer(cfg, rank, dev):
    from padding_free_moe_b200.layer import PFTMoELayer, Shape
    from workloads import make_inputs
    from workloads.generate import storage_dtype
    inp = make_inputs(cfg, seed=1000 + rank, device=dev)
    layer = PFTMoELayer(Shape(cfg.T, cfg.d, cfg.E, cfg.h, cfg.k, storage_dtype(cfg), cfg.rbd_epd, cfg.rbd_dpn), dev)
    return layer, inp


def device_timed(fn, n, stream, torch):
    """Device milliseconds of n calls of fn() on `stream` (CUDA events on that stream)."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def per_kernel_pass(L, layer, inp, stream, steps, torch, barrier):
    """The same steps with a CUDA event pair around every kernel launch (on the stream it is
    launched on): per-kernel durations and launch counts.  The RBD plan runs in line here so
    that each event pair times one kernel's own work.  Returns (kernels, pass milliseconds)."""
    L.moe_profile_reset()
    barrier()
    torch.cuda.synchronize()
    L.moe_profile_enable(True)
    ms = device_timed(lambda: layer.step(inp.x, inp.wg, inp.bias, inp.w1, inp.w3, inp.w2, inp.dy, stream,
                                         overlap_rbd=False), steps, stream, torch)
    L.moe_profile_enable(False)
    barrier()
    return L.moe_profile_read(), ms


def tensor_peak(peaks, peak_src, pass_ms):
    """The burst GEMM peak for kernels timed in a pass shorter than a second, else the sustained one."""
    if pass_ms < 1000.0:
        return float(peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])), \
            f"{peak_src} bf16_tflops (burst: the per-kernel pass lasted {pass_ms:.0f} ms)"
    return float(peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"])), \
        f"{peak_src} bf16_tflops_sustained (the per-kernel pass lasted {pass_ms:.0f} ms)"


def gemm_summary(cfg, kern, steps, tc_peak):
    gemm_ms = sum(kern[n][1] for n in gemm_names() if n in kern) / steps
    gemm_flops = 18.0 * cfg.N * cfg.d * cfg.h
    tf = gemm_flops / (gemm_ms * 1e-3) / 1e12 if gemm_ms > 0 else None
    return {"tflops": tf, "frac_of_peak": (tf / tc_peak) if tf else None, "flops_per_step": gemm_flops,
            "ms_per_step": gemm_ms}


def run_ours(args):
    import torch
    from padding_free_moe_b200 import _lib as L
    from padding_free_moe_b200 import replicas
    from workloads import get_config

    info = replicas.rank_info()
    rank, world, local_rank = info.rank, info.world, info.local_rank
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    replicas.init(info, "nccl", timeout_s=120, device=dev)
    cfg = get_config(args.workload)
    layer, inp = build_layer(cfg, rank, dev)
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
    ms_total = device_timed(step, args.steps, stream, torch)
    barrier()
    clocks = clk.stop()
    ms_step = max_over_ranks(ms_total) / args.steps
    value = world * cfg.T / (ms_step * 1e-3)

    kern, pass_ms = per_kernel_pass(L, layer, inp, stream, args.steps, torch, barrier)

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
    del x_d, dy_d, y_st, dx_st

    # ---- roofline of the dominant kernel + per-kernel table
    peaks, peak_src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]))
    tc_peak, tc_src = tensor_peak(peaks, peak_src, pass_ms)
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
        burst = float(peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"]))
        roof = {"bound": "tensor", "kernel": dom, "achieved": ach, "peak": tc_peak, "unit": "TFLOP/s",
                "frac": ach / tc_peak, "traffic": traffic_for(dom, cfg.name), "peak_source": tc_src,
                "frac_of_burst": ach / burst, "work_per_launch": work, "ms_per_launch": dom_ms}
    else:
        ach = work / (dom_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": dom, "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                "traffic": traffic_for(dom, cfg.name), "peak_source": f"{peak_src} hbm_gbs",
                "work_per_launch": work, "ms_per_launch": dom_ms}

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
        "grouped_gemm": gemm_summary(cfg, kern, args.steps, tc_peak),
        "dispatch_gbs": gbs("dispatch"), "combine_gbs": gbs("combine"),
        "sort_stress": None if args.no_sort_stress else stress_sort(L, torch, dev, stream, hbm),
        "kernels": kernels,
    }

    # ---- CPU oracle baseline (rank 0, one GPU only), on the headline workload's inputs
    if world == 1 and not args.no_cpu_baseline:
        smp = OracleSampler(inp, cfg)
        batch = oracle_batch(cfg)
        tps, n, sec = smp.tokens_per_second(args.cpu_sample_seconds, batch)
        line["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"{n} random tokens of {cfg.name} in samples of {batch} through the "
                                          f"float64 oracle (forward, RBD plan, backward), {sec:.1f} s of oracle "
                                          f"time; expert weights converted to float64 one expert at a time, "
                                          f"conversion not timed"}
        del smp

    # ---- the other workloads: device-timed steps and their grouped-GEMM rate
    del layer, inp
    torch.cuda.empty_cache()
    extra = {}
    for name in [w for w in args.extra_workloads.split(",") if w and w != cfg.name]:
        c2 = get_config(name)
        lay2, inp2 = build_layer(c2, rank, dev)

        def step2():
            lay2.step(inp2.x, inp2.wg, inp2.bias, inp2.w1, inp2.w3, inp2.w2, inp2.dy, stream)

        for _ in range(warm):
            step2()
        torch.cuda.synchronize()
        barrier()
        ms2 = max_over_ranks(device_timed(step2, args.extra_steps, stream, torch)) / args.extra_steps
        barrier()
        k2, pass2 = per_kernel_pass(L, lay2, inp2, stream, args.extra_steps, torch, barrier)
        if lay2.device_error() != 0:
            raise RuntimeError(f"device error word {lay2.device_error():#x} in {name}")
        pk, src = tensor_peak(peaks, peak_src, pass2)
        extra[name] = {"ms_per_step": ms2, "tokens_per_s": world * c2.T / (ms2 * 1e-3), "steps": args.extra_steps,
                       "grouped_gemm": gemm_summary(c2, k2, args.extra_steps, pk), "peak_source": src,
                       "config": config_block(c2, world)}
        del lay2, inp2
        torch.cuda.empty_cache()
    line["workloads"] = extra

    # ---- the same step with the dispatch gather fused into the first expert GEMM (no x_pft in the forward)
    if cfg.dtype == "bf16" and not args.no_gathered:
        lay3, inp3 = build_layer(cfg, rank, dev)
        lay3.fused_gather = True

        def step3():
            lay3.step(inp3.x, inp3.wg, inp3.bias, inp3.w1, inp3.w3, inp3.w2, inp3.dy, stream)

        for _ in range(warm):
            step3()
        torch.cuda.synchronize()
        barrier()
        ms3 = max_over_ranks(device_timed(step3, args.extra_steps, stream, torch)) / args.extra_steps
        barrier()
        k3, _ = per_kernel_pass(L, lay3, inp3, stream, args.extra_steps, torch, barrier)
        if lay3.device_error() != 0:
            raise RuntimeError(f"device error word {lay3.device_error():#x} in the gathered step")
        per = {nm: k3[nm][1] / k3[nm][0] for nm in ("ffn_gemm1_swiglu", "dispatch") if nm in k3}
        line["gathered_forward"] = {
            "workload": cfg.name, "ms_per_step": ms3, "tokens_per_s": world * cfg.T / (ms3 * 1e-3),
            "steps": args.extra_steps, "ffn_gemm1_swiglu_ms": per.get("ffn_gemm1_swiglu"),
            "dispatch_ms_in_backward": per.get("dispatch"),
            "note": "moe_expert_ffn_gathered: the forward writes no [N, d] copy of x; the backward dispatches it"}
        del lay3, inp3
        torch.cuda.empty_cache()
    if rank == 0:
        print(json.dumps(line), flush=True)
    replicas.finish(info)
    return 0


def relaunch_under_torchrun(n: int) -> int:
    """`--gpus N` from a plain `python bench.py`: run the same command as N torchrun ranks."""
    import socket
    sk = socket.socket()
    sk.bind(("127.0.0.1", 0))
    port = sk.getsockname()[1]
    sk.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd, cwd=ROOT)


def run_sort_stress_only(args):
    """The PFT build and RBD plan on the stress shape alone (one GPU): one JSON object."""
    import torch
    from padding_free_moe_b200 import _lib as L
    dev = torch.device("cuda", 0)
    peaks, _ = load_peaks()
    out = stress_sort(L, torch, dev, torch.cuda.current_stream(), float(peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])))
    print(json.dumps({"sort_stress": out}), flush=True)
    return 0


def main():
    args = parse()
    if args.sort_stress_only:
        return run_sort_stress_only(args)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch_under_torchrun(args.gpus)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
