#!/usr/bin/env python
"""Throughput of the Stable-LatentMoE layer step on B200s, one JSON line on rank 0.

A step is one pass of the whole hot path over one batch of synthetic tokens already resident
in HBM: lmoe_forward with QB statistics recorded (RMSNorm, latent down-projection, sigmoid
router, biased top-k and gates, histogram, dispatch plan and permutation, routed SwiGLU
experts, shared SwiGLU expert, combine, up-projection) and the QB bias update.  On one rank the
update runs inside the forward (LMOE_UPDATE_BIAS: a graph branch that starts once routing is
done); with N > 1 ranks every rank runs its own tokens (weak scaling) and the ranks sum their QB
histograms with one NCCL all-reduce before lmoe_qb_update (lq.dp_qb_update), so every rank
keeps the same bias.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload wide_stress] [--tokens T]
    python bench.py --impl reference ...   # the CPU oracle on the host cores, same metric

The default workload is the largest single-GPU layer (wide_stress: T=16384, d=7168, l=2048,
E=896, k=16), where the grouped expert GEMM is judged against the bf16 tensor peak; on one GPU
the same call also measures the token sweep's largest point (T=262144 at mini_replica widths),
where the router/permute/combine kernels are judged against HBM bandwidth ("also" key).
--gpus N without a torch.distributed launcher re-runs this script under torch.distributed.run
with N ranks (one per GPU); under a launcher, WORLD_SIZE must equal N.

Timing: W untimed steps, then K steps each bracketed by CUDA events on the launching stream,
with a 256 MiB write between steps (outside the events) to flush the 126 MB L2; barrier and
synchronize on both sides; the per-step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import socket
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "LatentMoE layer fwd tokens/s on 1 B200; % BF16 tensor peak; router/permute GB/s"
UNIT = "tokens/s"
BETA = 0.01
FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return p, "measured (MEASURED_PEAKS.json)"
    return FALLBACK_PEAKS, "fallback"


# the sources that define and launch each kernel whose DRAM traffic profiles/traffic.json records:
# a recorded figure counts only while these files are the ones it was measured on
TRAFFIC_SOURCES = {
    "shared_swiglu": ("common.cuh", "tc_gemm.cuh", "lmoe.cu"),
    "expert_swiglu": ("common.cuh", "tc_gemm.cuh", "lmoe.cu"),
    "expert_down": ("common.cuh", "tc_gemm.cuh", "lmoe.cu"),
    "norm_down_router": ("common.cuh", "k1_router.cuh", "lmoe.cu"),
}


def csrc_digest(files=None) -> str:
    """sha256 (16 hex digits) of the named CUDA sources, or of all of them."""
    d = os.path.join(ROOT, "latent_routing_quantile_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(d)):
        if f.endswith((".cu", ".cuh")) and (files is None or f in files):
            h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def stage_work(shape, T):
    """Algorithmic FLOPs and HBM bytes of one launch of each stage on T tokens (bf16 storage)."""
    d, l, E, k, h, hs = shape.d, shape.l, shape.E, shape.k, shape.h, shape.hs
    w = 2 if shape.dtype == "bf16" else 4
    TK = T * k
    nblk = (T + 127) // 128
    return {
        "rms": (0, T * w * d + 4 * T),
        "down_proj": (2 * T * d * l, T * w * d + l * d * w + 4 * T * l),
        "router": (2 * T * l * E, 4 * T * l + 4 * E * l + 4 * T * E),
        "norm_down_router": (2 * T * d * l + 2 * T * l * E,
                             T * (w * d + 2 * l + 4 * E + 4) + l * d * w + 4 * E * l),
        "topk": (0, 4 * T * E + 12 * TK),
        "plan": (0, 3 * 4 * nblk * E),
        # compulsory: each h row read once (its k copies come from L2), A_perm written, idx read,
        # perm and inv written
        "gather": (0, T * w * l + TK * (w * l + 12)),
        "hist": (0, 2 * T * E + 8 * E * 4096),
        "shared_swiglu": (4 * T * d * hs, T * w * d + 2 * hs * d * w + T * w * hs),
        "expert_swiglu": (4 * TK * l * h, TK * w * l + 2 * E * h * l * w + TK * w * h),
        "expert_down": (2 * TK * h * l, TK * w * h + E * l * h * w + TK * w * l),
        "combine": (0, TK * (w * l + 8) + T * w * l),
        "up_proj": (2 * T * d * (l + hs), T * w * (l + hs) + d * (l + hs) * w + T * w * d),
        # the update counts the last forward's pending bins (2 B per score) itself
        "qb_update": (0, 2 * T * E + 16 * E),
    }


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons = [], 0
        self.period = period_s
        self.stop_ev = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.hnd = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.hnd, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        while not self.stop_ev.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.hnd, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.hnd)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.th = threading.Thread(target=self._run, daemon=True)
            self.th.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self.stop_ev.set()
            self.th.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples),
                "reasons": sorted(n for b, n in self.REASONS.items() if self.reasons & b)}


# ----------------------------------------------------------------------------------------- ours
def measure(shape, args, rank, world, local_rank, e2e=True, experts=0):
    """Device-timed steps (the headline), per-stage times (a second, eager pass) and, with e2e,
    the host-buffer entry point, for one workload on this rank.  Returns (summary on rank 0, or
    None; the number of kernels launched in the timed region)."""
    import torch
    import torch.distributed as dist

    import datagen
    import latent_routing_quantile_b200 as lq

    T = shape.T
    w = datagen.layer_weights(shape)
    x_cpu = datagen.tokens(shape, seed=shape.seed + 1000 * rank)
    layer = lq.layer_from_weights(shape, w, experts=experts)
    del w
    stream = torch.cuda.current_stream()
    x = x_cpu.cuda()
    y = torch.empty_like(x)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    # one rank: the update runs inside the forward, as a branch after routing
    layer.set_update(BETA)

    def step():
        if world == 1:
            layer.forward(x, y, update_bias=True)
            return
        layer.forward(x, y, record_stats=True)
        lq.dp_qb_update(layer, BETA)  # the one exchange step: the ranks' statistics summed

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        flush.zero_()
        step()
    barrier()
    # ---------------- timed region
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    launches0 = layer.launches()
    with ClockSampler(local_rank) as clk:
        barrier()
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        barrier()
    launches = layer.launches() - launches0
    ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends)) / args.steps
    # per-stage times: the same K steps again with an event before every stage (eager launches;
    # the timed region above replays each call as one CUDA graph)
    layer.profile(True)
    layer.profile_read()
    barrier()
    for i in range(args.steps):
        flush.zero_()
        step()
    barrier()
    stage_ms, nfwd = layer.profile_read()
    layer.profile(False)
    ms_t = torch.tensor([ms], dtype=torch.float64, device="cuda")
    if world > 1:
        dist.all_reduce(ms_t, op=dist.ReduceOp.MAX)
    ms_max = float(ms_t.item())
    assert layer.status() == 0, "device status word set during the bench"

    # ---------------- end to end through the host-buffer entry point
    e2e_ms, e2e_steps = None, 0
    if e2e:
        e2e_steps = max(3, min(args.steps, 50))
        xh = x_cpu.pin_memory()
        yh = torch.empty_like(xh).pin_memory()

        # the output copy of step i runs on the library's own copy stream and overlaps step i+1
        def step_host():
            if world == 1:
                layer.forward_host(xh, yh, update_bias=True, async_output=True)
                return
            layer.forward_host(xh, yh, record_stats=True, async_output=True)
            lq.dp_qb_update(layer, BETA)

        for _ in range(3):
            flush.zero_()
            step_host()
        layer.host_wait()
        barrier()
        # one region from the first step's start to the arrival of the last step's output in host
        # memory (the steps overlap, so per-step events would not cover each step's output copy);
        # the L2 flushes between steps fall inside it
        e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.zero_()
        barrier()  # nothing in flight: the first input copy (on the library's copy stream) starts after e_start
        e_start.record(stream)
        for i in range(e2e_steps):
            if i:
                flush.zero_()
            step_host()
        layer.host_wait()
        e_end.record(stream)
        barrier()
        e2e_ms = e_start.elapsed_time(e_end) / e2e_steps
        e2e_t = torch.tensor([e2e_ms], dtype=torch.float64, device="cuda")
        if world > 1:
            dist.all_reduce(e2e_t, op=dist.ReduceOp.MAX)
        e2e_ms = float(e2e_t.item())
    layer.close()
    del flush, x, y
    torch.cuda.empty_cache()
    if rank != 0:
        return None, launches

    peaks, peak_src = load_peaks()
    work = stage_work(shape, T)
    per_launch = {n: stage_ms[n] / max(1, nfwd) for n in stage_ms}
    # with l <= 256 and E <= 256 the library runs rms, down_proj and router as one kernel
    # (norm_down_router); their own markers then bracket no work, only event overhead
    fused = shape.l <= 256 and shape.E <= 256 and shape.dtype == "bf16"
    for n in (("rms", "down_proj", "router") if fused else ("norm_down_router",)):
        per_launch.pop(n, None)
    # one recorded forward per update: its bins are counted by the update, and the hist marker
    # brackets no kernel (it runs only when a second recorded forward arrives first)
    if world == 1:
        per_launch.pop("hist", None)
    step_stage_ms = sum(per_launch.values())
    kernels = {}
    for n, t in per_launch.items():
        fl, by = work[n]
        t_s = t / 1e3
        if t_s <= 0:
            continue
        t_tensor = fl / (peaks["bf16_tflops"] * 1e12) if fl else 0.0
        t_hbm = by / (peaks["hbm_gbs"] * 1e9)
        bound = "tensor" if t_tensor >= t_hbm else "hbm"
        kernels[n] = {"ms": round(t, 5), "share": round(t / step_stage_ms, 4), "bound": bound,
                      "tflops": round(fl / t_s / 1e12, 2), "gbs": round(by / t_s / 1e9, 1),
                      "frac": round(max(t_tensor, t_hbm) / t_s, 4)}
    gemm_flops = sum(work[n][0] for n in work if work[n][0] > 0 and n in per_launch)
    rp = ["norm_down_router"] if fused else ["rms", "down_proj", "router"]
    rp += ["topk", "plan", "gather"]
    rp_bytes = sum(work[n][1] for n in rp)
    rp_ms = sum(per_launch[n] for n in rp)
    rpc = rp + ["combine"]
    rpc_bytes = sum(work[n][1] for n in rpc)
    rpc_ms = sum(per_launch[n] for n in rpc)
    ex_flops = work["expert_swiglu"][0] + work["expert_down"][0]
    ex_ms = per_launch["expert_swiglu"] + per_launch["expert_down"]
    # 8-bit experts run at twice the bf16 tensor rate (the dense fp8 rate is twice bf16's)
    ex_peak = peaks["bf16_tflops"] * (2 if experts else 1)
    summary = {
        "workload": shape.name, "T": T, "ms_per_step": round(ms_max, 5),
        "value": round(T * world / (ms_max / 1e3), 1),
        "gpu_launches": launches,
        "kernels": kernels,
        "tensor_peak_frac_step": round(gemm_flops / (ms_max / 1e3) / (peaks["bf16_tflops"] * 1e12), 4),
        "router_permute_gbs": round(rp_bytes / (rp_ms / 1e3) / 1e9, 1) if rp_ms > 0 else None,
        "router_permute_combine_frac_of_hbm":
            round(rpc_bytes / (rpc_ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4) if rpc_ms > 0 else None,
        "expert_gemm_frac_of_bf16_peak": round(ex_flops / (ex_ms / 1e3) / 1e12 / peaks["bf16_tflops"], 4),
        "expert_gemm_tflops": round(ex_flops / (ex_ms / 1e3) / 1e12, 1),
        "expert_gemm_frac_of_format_peak": round(ex_flops / (ex_ms / 1e3) / 1e12 / ex_peak, 4),
        "experts": "mxfp8" if experts else "bf16",
        "clocks": clk.summary(),
        "e2e_ms": e2e_ms, "e2e_steps": e2e_steps, "stage_ms": per_launch, "work": work,
        "peaks": (peaks, peak_src),
    }
    return summary, launches


def train_flops(shape, T):
    """Algorithmic FLOPs of one training step's layer products: every forward product and its two
    backward products (the data gradient and the weight gradient), three times the forward's."""
    d, l, E, k, h, hs = shape.d, shape.l, shape.E, shape.k, shape.h, shape.hs
    fwd = 2 * T * d * l + 2 * T * l * E + 6 * T * k * l * h + 4 * T * d * hs + 2 * T * d * (l + hs)
    return 3 * fwd


def measure_train(shape, args, local_rank):
    """Device-timed training steps of one layer: lmoe_forward_backward (the forward, then every
    gradient for a fixed output gradient dy), L2 flushed between steps outside the events; and the
    forward alone the same way, so the backward's share is known."""
    import torch

    import datagen
    import latent_routing_quantile_b200 as lq

    T = shape.T
    w_dev = {n: t.cuda() for n, t in datagen.layer_weights(shape).items()}
    layer = lq.Layer(shape.d, shape.l, shape.E, shape.k, shape.h, shape.hs, lq.BF16, T, w_dev,
                     rms_eps=shape.rms_eps)
    x = datagen.tokens(shape).cuda()
    dy = datagen.output_grad(shape, seed=shape.seed + 100).cuda()
    y = torch.empty_like(x)
    _, g = layer.forward_backward(x, dy, w_dev, y=y)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(args.warmup):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        st = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        en = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        for i in range(args.steps):
            flush.zero_()
            st[i].record(stream)
            fn()
            en[i].record(stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in zip(st, en)) / args.steps

    l0 = layer.launches()
    with ClockSampler(local_rank) as clk:
        ms = timed(lambda: layer.forward_backward(x, dy, w_dev, y=y, grads=g))
    launches = (layer.launches() - l0) // (args.warmup + args.steps)
    ms_fwd = timed(lambda: layer.forward(x, y))
    assert layer.status() == 0, "device status word set during the training bench"
    layer.close()
    del g, w_dev, flush
    torch.cuda.empty_cache()
    peaks, peak_src = load_peaks()
    fl = train_flops(shape, T)
    return {"workload": shape.name, "T": T, "ms_per_step": round(ms, 5), "value": round(T / (ms / 1e3), 1),
            "unit": "tokens/s", "forward_ms": round(ms_fwd, 5), "backward_ms": round(ms - ms_fwd, 5),
            "gpu_launches_per_step": launches, "algorithmic_tflop": round(fl / 1e12, 4),
            "tflops": round(fl / (ms / 1e3) / 1e12, 1),
            "frac_of_bf16_peak": round(fl / (ms / 1e3) / 1e12 / peaks["bf16_tflops"], 4),
            "peak_source": f"{peak_src}, burst", "clocks": clk.summary(),
            "step": "lmoe_forward_backward: forward, then dL/dx and every weight gradient (fp32) for a fixed dy"}


def roofline(summary, shape, name):
    """The roofline object of one kernel (stage) of a measured workload."""
    peaks, peak_src = summary["peaks"]
    kd = summary["kernels"][name]
    fl, by = summary["work"][name]
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        tj = json.load(open(tpath))
        ent = tj.get("workloads", {}).get(shape.name, {}).get("kernels", {}).get(name)
        if ent and name in TRAFFIC_SOURCES and ent.get("src_digest") == csrc_digest(TRAFFIC_SOURCES[name]):
            traffic = ent["dram_bytes_per_launch"]
    if kd["bound"] == "tensor":
        roof = {"bound": "tensor", "achieved": kd["tflops"], "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": kd["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = round(roof["achieved"] / roof["peak"], 4)
    roof.update({"traffic": traffic, "kernel": name, "algorithmic_flops": fl, "algorithmic_bytes": by,
                 "peak_source": f"{peak_src}, burst"})
    return roof


def run_ours(args, rank, world, local_rank):
    import torch

    import datagen

    torch.cuda.set_device(local_rank)
    shape = datagen.WORKLOADS[args.workload]
    if args.tokens:
        shape = shape.with_tokens(args.tokens)
    main_s, launches = measure(shape, args, rank, world, local_rank, experts=1 if args.experts == "mxfp8" else 0)
    also, train = {}, {}
    if world == 1 and args.also and not args.tokens:
        for spec in args.also.split(","):
            parts = spec.split(":")
            sh = datagen.WORKLOADS[parts[0]].with_tokens(int(parts[1]))
            if len(parts) > 2 and parts[2] == "train":
                train[sh.name] = measure_train(sh, args, local_rank)
                continue
            mx = len(parts) > 2 and parts[2] == "mxfp8"
            s2, _ = measure(sh, args, rank, world, local_rank, e2e=False, experts=1 if mx else 0)
            also[sh.name + ("_mxfp8" if mx else "")] = s2
    if rank != 0:
        return None
    m = main_s
    dom = max(m["kernels"], key=lambda n: m["kernels"][n]["ms"])
    T = shape.T
    out = {
        "metric": METRIC, "value": m["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": shape.dtype, "data": "synthetic (seeded; x ~ N(0,1), weights ~ N(0,1/fan_in))",
        "config": {"workload": shape.name, "T": T, "d": shape.d, "l": shape.l, "E": shape.E, "k": shape.k,
                   "h": shape.h, "hs": shape.hs, "experts": args.experts, "tokens_per_gpu": T, "global_tokens": T * world,
                   "step": "forward with QB statistics + QB update"
                           + (" (update inside the forward, after routing)" if world == 1 else ""), "beta": BETA,
                   "l2": "flushed between steps (256 MiB write outside the timed events)",
                   "parallelism": f"dp{world}" + (" (histogram all-reduce)" if world > 1 else "")},
        "e2e": {"value": round(T * world / (m["e2e_ms"] / 1e3), 1), "unit": UNIT, "ms_per_step": round(m["e2e_ms"], 5),
                "h2d_bytes_per_step": T * shape.d * (2 if shape.dtype == "bf16" else 4),
                "d2h_bytes_per_step": T * shape.d * (2 if shape.dtype == "bf16" else 4),
                "api": ("lmoe_forward_host with LMOE_UPDATE_BIAS" if world == 1 else
                        "lmoe_forward_host + histogram all-reduce + lmoe_qb_update")
                       + " and LMOE_ASYNC_OUTPUT (step i's output copy overlaps step i+1), pinned host buffers",
                "timing": f"one CUDA-event region over {m['e2e_steps']} steps, from the first step's start to "
                          "lmoe_host_wait after the last (every input and output copy inside), divided by the steps"},
        "gpu_launches": launches,
        "kernel_timing": "CUDA events before every stage on the launching stream, in a second pass of the "
                         "same K steps with eager launches (the timed region replays each call as a CUDA graph)",
        "roofline": roofline(m, shape, dom),
        "roofline_expert_gemms": {n: roofline(m, shape, n) for n in ("expert_swiglu", "expert_down")},
        "expert_gemm_frac_of_bf16_peak": m["expert_gemm_frac_of_bf16_peak"],
        "tensor_peak_frac_step": m["tensor_peak_frac_step"],
        "router_permute_gbs": m["router_permute_gbs"],
        "router_permute_combine_frac_of_hbm": m["router_permute_combine_frac_of_hbm"],
        "kernels": m["kernels"],
        "clocks": m["clocks"],
    }
    if also:
        out["also"] = {
            n: {"value": a["value"], "unit": UNIT, "ms_per_step": a["ms_per_step"], "T": a["T"],
                "gpu_launches": a["gpu_launches"], "router_permute_gbs": a["router_permute_gbs"],
                "router_permute_combine_frac_of_hbm": a["router_permute_combine_frac_of_hbm"],
                "expert_gemm_frac_of_bf16_peak": a["expert_gemm_frac_of_bf16_peak"],
                "experts": a["experts"], "expert_gemm_tflops": a["expert_gemm_tflops"],
                "expert_gemm_frac_of_format_peak": a["expert_gemm_frac_of_format_peak"],
                "tensor_peak_frac_step": a["tensor_peak_frac_step"], "kernels": a["kernels"], "clocks": a["clocks"]}
            for n, a in also.items()}
    if train:
        out["train"] = train
    return out


# ------------------------------------------------------------------------------ CPU oracle legs
# Fixed token sample per workload: the first S tokens, about two to three seconds of the
# single-threaded oracle per pass on a server core.  The oracle loops over the experts its tokens
# use, so its cost per token depends on S; a fixed S makes the baseline one number.
ORACLE_SAMPLE = {"tiny_fp32": 256, "mini_replica": 2048, "qb_skewed": 1024, "sweep": 2048, "wide_stress": 32}


def oracle_pass(shape, w, x_sample, b):
    """One oracle pass (layer forward, then the QB update from its histogram) over the sample;
    returns (forward seconds, update seconds)."""
    import oracle
    t0 = time.perf_counter()
    out = oracle.layer_forward(x_sample, w, b, shape.k, shape.rms_eps)
    t1 = time.perf_counter()
    oracle.qb_update(b, oracle.score_histogram(out["s"]), x_sample.shape[0], shape.k, BETA)
    return t1 - t0, time.perf_counter() - t1


def oracle_sample(shape):
    base = shape.name.split("_T")[0]
    return min(shape.T, ORACLE_SAMPLE.get(base, ORACLE_SAMPLE.get(shape.name, 256)))


def cpu_baseline(shape, budget_s=12.0):
    """The oracle as it stands on one host core (BLAS limited to one thread): passes over the
    fixed sample until about budget_s of host time, forward and QB update timed apart."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    import datagen
    w = datagen.layer_weights(shape)
    b = np.zeros(shape.E)
    S = oracle_sample(shape)
    x = datagen.tokens(shape, rows=range(S))
    with threadpool_limits(limits=1):
        oracle_pass(shape, w, datagen.tokens(shape, rows=range(min(S, 16))), b)  # first-call costs
        fw, up = [], []
        t_all = time.perf_counter()
        while not fw or (time.perf_counter() - t_all < budget_s and len(fw) < 20):
            f, u = oracle_pass(shape, w, x, b)
            fw.append(f)
            up.append(u)
    f, u = statistics.median(fw), statistics.median(up)
    return {"value": round(S / (f + u), 3), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"first {S} tokens of the {shape.name} workload, {len(fw)} passes (median): float64 numpy "
                      f"layer forward + QB update, BLAS limited to 1 thread",
            "forward_s": round(f, 4), "qb_update_s": round(u, 5),
            "forward_tokens_per_s": round(S / f, 3), "seconds": round(sum(fw) + sum(up), 2)}


def run_reference(args, rank):
    if rank != 0:
        return None
    import numpy as np
    from threadpoolctl import threadpool_limits

    import datagen
    shape = datagen.WORKLOADS[args.workload]
    if args.tokens:
        shape = shape.with_tokens(args.tokens)
    w = datagen.layer_weights(shape)
    b = np.zeros(shape.E)
    S = oracle_sample(shape)
    x = datagen.tokens(shape, rows=range(S))
    with threadpool_limits(limits=1):
        oracle_pass(shape, w, datagen.tokens(shape, rows=range(min(S, 16))), b)  # first-call costs
        # the fixed sample, unless K + W passes of it would take more than about four minutes
        f, u = oracle_pass(shape, w, x, b)
        while S > 8 and (f + u) * (args.steps + args.warmup) > 240:
            S //= 2
            x = x[:S]
            f, u = oracle_pass(shape, w, x, b)
        for _ in range(args.warmup):
            oracle_pass(shape, w, x, b)
        ts = [sum(oracle_pass(shape, w, x, b)) for _ in range(args.steps)]
    sec = sum(ts) / len(ts)
    value = S / sec
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeded workload)",
        "config": {"workload": shape.name, "T": shape.T, "d": shape.d, "l": shape.l, "E": shape.E, "k": shape.k,
                   "h": shape.h, "hs": shape.hs, "sample_tokens_per_step": S},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"first {S} tokens of {shape.name} per step: float64 numpy forward + QB update, "
                                   "BLAS limited to 1 thread"},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="wide_stress")
    ap.add_argument("--tokens", type=int, default=0)
    ap.add_argument("--also", default="sweep:262144,wide_stress:16384:mxfp8,mini_replica:8192:train",
                    help="extra workloads (name:T[:mxfp8|:train], comma-separated) measured in the same call on one "
                         "GPU, ':mxfp8' with 8-bit routed experts, ':train' as training steps (forward + backward); "
                         "'' for none")
    ap.add_argument("--experts", choices=["bf16", "mxfp8"], default="bf16",
                    help="operand format of the routed experts of the main workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--train-only", default="",
                    help="name:T: time only training steps (lmoe_forward_backward) of that workload on one GPU and "
                         "print their summary (for profiling the backward)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    world_env = os.environ.get("WORLD_SIZE")
    if args.impl == "ours" and world_env is None and args.gpus > 1:
        # one process per GPU: re-run this script under the torch.distributed launcher, bounded
        cmd = ["timeout", "-k", "60", "1800", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
               f"--nproc-per-node={args.gpus}", "--master-addr=127.0.0.1", f"--master-port={_free_port()}",
               os.path.abspath(__file__), *sys.argv[1:]]
        sys.exit(subprocess.call(cmd))
    world = int(world_env or "1")
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "ours" and world != args.gpus:
        sys.exit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; launch one rank per GPU")

    if args.impl == "reference":
        out = run_reference(args, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    if args.train_only:
        import torch

        import datagen
        name, t = args.train_only.split(":")
        torch.cuda.set_device(local_rank)
        print(json.dumps({"train": {name: measure_train(datagen.WORKLOADS[name].with_tokens(int(t)), args,
                                                        local_rank)}}), flush=True)
        return

    import datetime

    import torch.distributed as dist
    if world > 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=__import__("torch").device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if out is not None:
        if world == 1 and not args.no_cpu_baseline:
            import datagen
            shape = datagen.WORKLOADS[args.workload]
            if args.tokens:
                shape = shape.with_tokens(args.tokens)
            out["cpu_baseline"] = cpu_baseline(shape)
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
