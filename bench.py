#!/usr/bin/env python
"""KDA prefill/decode benchmark on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kda|reference]
                    [--workload prefill_8k] [--no-decode] [--no-cpu-baseline]
                    [--more-workloads pretrain_64k,prefill_1m] [--small-footprint]

A step is one kda_chunk_fwd over one batch of the prefill workload (B=1,
H=32, T=8192, d=128, bf16 inputs, fp32 state).  Two independent input sets
of 269 MB each (together > 4x the 126 MB L2) alternate between steps, so no
step starts with its inputs in L2.  The decode workload (256 requests x 32
heads, 1000 successive kda_decode_step calls) is timed in the same run and
reported under "decode", and the other prefill workloads of the pages'
length range (a batch of four 64K pre-training sequences and a
million-token sequence, each 32 heads) under their own names, each with its
tokens/s, roofline and clock record.  "e2e" is the same prefill through the public API
with host buffers: every step uploads its inputs from pinned host memory and
downloads o and hT, pipelined across steps on two copy streams.  Multi-GPU:
one process per GPU (torchrun), every
rank runs the same per-GPU workload on its own seed with no collective on
the data path (weak scaling); the time is the max over ranks.

--impl reference times the fp64 CPU oracle (the correctness reference) on
this host's cores (one whole head per core) over a bounded sample of the same
workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

BYTES_BF16 = 2
METRIC = ("KDA prefill tokens/s on 1 B200 (workload in config; default B1 H32 T8192 "
          "d128 bf16); decode steps/s and both rooflines reported alongside")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ------------------------------------------------------------ accounting --

def prefill_alg_bytes(B, T, H, dk, dv, with_h0=True, with_hT=True, elem=BYTES_BF16):
    """Algorithmic HBM bytes of one prefill: q, k, g, v, beta read once, o
    written once (elem bytes each), h0 read and hT written once (fp32)."""
    per_token_head = (3 * dk + dv + 1) * elem + dv * elem
    state = dk * dv * 4
    return B * T * H * per_token_head + B * H * state * (int(with_h0) + int(with_hT))


def prefill_alg_flops(B, T, H, dk, dv, C=16):
    """Algorithmic flops of the chunked form (per token-head: W S, Q S and
    K^T U state products 6 dk dv; intra-tile products ~ C (4 dk + 2 dv);
    the triangular solve ~ C^2/3)."""
    per = 6 * dk * dv + C * (4 * dk + 2 * dv) + C * C / 3.0
    return B * T * H * per


def backward_alg_bytes(B, T, H, dk, dv):
    """Algorithmic HBM bytes of one backward: q, k, g, v, beta and dO read
    once, dq, dk, dg, dv and dbeta written once (bf16); h0 and dhT read and
    dh0 written (fp32)."""
    per_token_head = (3 * dk + dv + 1 + dv) * BYTES_BF16 + (3 * dk + dv + 1) * BYTES_BF16
    return B * T * H * per_token_head + 3 * B * H * dk * dv * 4


def backward_alg_flops(B, T, H, dk, dv, C=32):
    """Flops of the chunked backward as computed (32-token chunks; FMA = 2
    flops): per chunk, the operand preparation (pair products, W, U', P W:
    ~4 C^2 d), the forward state chain (2 C d^2), the reverse chain
    (3 C d^2) and the chunk-local products (7 C d^2 + ~10 C^2 d)."""
    per_chunk = 2 * (4 * C * C * dk + 2 * C * dk * dv + 3 * C * dk * dv + 7 * C * dk * dv + 10 * C * C * dk)
    return B * H * ((T + C - 1) // C) * per_chunk


def alu_peak_tflops(sm_mhz=1965.0, sms=148):
    """fp32 FMA peak of the CUDA cores: SMs x 128 lanes x 2 flops x clock."""
    return sms * 128 * 2 * sm_mhz * 1e6 / 1e12


def decode_alg_bytes(N, H, dk, dv):
    """Per decode step: state read + written (fp32), q, k, g, v, beta read,
    o written (bf16)."""
    return N * H * (2 * dk * dv * 4 + (3 * dk + dv + 1 + dv) * BYTES_BF16)


def code_only(text):
    """C/C++/CUDA source without comments and with whitespace collapsed: what
    decides whether a kernel has changed since its counters were taken."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def measured_traffic(kernel, workload):
    """DRAM bytes per launch for this kernel on this workload from the
    committed ncu summary, or None when there is no such line or when the
    kernel's sources have changed since the capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        with open(path) as f:
            for line in f:
                if line.startswith("#") or not line.strip():
                    continue
                parts = line.split()
                if parts[0] != kernel or parts[4] != workload:
                    continue
                h = hashlib.sha256()
                for rel in parts[1].split(","):        # every source the kernel is built from
                    with open(os.path.join(ROOT, rel), encoding="utf-8") as src:
                        h.update(code_only(src.read()).encode())
                return int(parts[3]) if h.hexdigest()[:16] == parts[2] else None
    except Exception:
        return None
    return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def prefill_state_flops(B, T, H, dk, dv):
    """Flops of the three state-sized products (W S, Q S, K^T U: 6 dk dv per
    token-head), the part of prefill_alg_flops the cluster kernel runs as
    fp16 MMAs."""
    return B * T * H * 6 * dk * dv


def tensor_fractions(alg_flops, state_flops, launch_ms, bf16_tflops, variant=""):
    """Algorithmic tensor throughput of a prefill launch against the peaks of
    its MMA types.  The cluster kernel runs the three state-sized products as
    kind::f16 (fp16 shares the bf16 peak) and the intra-chunk products as
    kind::tf32 (half that: the nominal tf32 : bf16 ratio, 1 : 2); the one-SM
    kernel runs every product as tf32.  tensor_frac_mma is the time these
    flops need at their own peaks over the launch time; tensor_frac_tf32 and
    tensor_frac_bf16 put all of them on one peak."""
    tf = alg_flops / (launch_ms / 1e3) / 1e12
    f16 = min(float(state_flops), float(alg_flops)) if variant.startswith("cluster") else 0.0
    t_need = ((alg_flops - f16) / (bf16_tflops / 2.0) + f16 / bf16_tflops) / 1e12
    return {"tensor_alg_tflops": round(tf, 2),
            "tensor_frac_mma": round(t_need / (launch_ms / 1e3), 4),
            "mma_kinds": ("state products fp16 (kind::f16), intra-chunk products tf32"
                          if f16 > 0 else "every product tf32 (kind::tf32)"),
            "tensor_frac_tf32": round(tf / (bf16_tflops / 2.0), 4),
            "tensor_peak_tf32": round(bf16_tflops / 2.0, 1),
            "tensor_peak_note": "tf32 peak = measured bf16 peak x 1/2 (nominal tf32:bf16 ratio)",
            "tensor_frac_bf16": round(tf / bf16_tflops, 4)}


# ---------------------------------------------------------------- ranks ---

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_seed(base: int, rank: int) -> int:
    """Every rank draws its own independent batch of the same shape."""
    return int(base) + 7919 * int(rank)


def max_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# --------------------------------------------------------------- clocks ---

def smi_gpu_id(cuda_index: int, visible=None) -> str:
    """The nvidia-smi `-i` selector of the GPU that CUDA calls `cuda_index`
    in this process: CUDA numbers only the devices in CUDA_VISIBLE_DEVICES
    (indices or UUIDs, in that order), nvidia-smi numbers every device."""
    if visible is None:
        visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    if visible is None or not visible.strip():
        return str(cuda_index)
    entries = [e.strip() for e in visible.split(",") if e.strip()]
    if 0 <= cuda_index < len(entries):
        return entries[cuda_index]
    return str(cuda_index)


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = smi_gpu_id(gpu_index)
        self.proc = None
        self.lines = []
        self._t = None

    def __enter__(self):
        # no sleep here: the caller keeps the GPU under load while the
        # sampler starts (keep_busy), so the samples see the loaded clocks
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            if self._t is not None:
                self._t.join(timeout=2)
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def keep_busy(step, seconds, sync, first=0, parity=2):
    """Run untimed `step(i)` calls for about `seconds` of wall time (waiting
    for the device every 8 calls, so the queue stays short), around a timed
    region, so that clock samples taken meanwhile see the GPU under the same
    load.  Makes a multiple of `parity` calls, indices first, first + 1, ...,
    so with first = 0 the next call, step(0), uses the other input set than
    the last one, as it does between timed steps.  Returns the number of
    calls."""
    t_end = time.perf_counter() + seconds
    i = first
    while time.perf_counter() < t_end or (i - first) % parity != 0:
        step(i)
        i += 1
        if (i - first) % 8 == 0:
            sync()
    sync()
    return i - first


# ------------------------------------------------------------- kda arm ----

def bench_kda(args, rank, world, local):
    import torch
    import linear_attention_07_b200 as kda
    from linear_attention_07_b200.inputs import WORKLOADS, prefill_inputs, decode_inputs

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    kda.load_library()
    w = WORKLOADS[args.workload]
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv

    # two independent input sets, alternated between steps (one set in the
    # small-footprint mode for profiler captures: the timing there is the
    # profiler's, not the bench's)
    n_sets = 1 if args.small_footprint else 2
    sets = [prefill_inputs(B, T, H, dk, dv, seed=rank_seed(w.seed + 17 * i, rank),
                           device=dev, h0_std=w.h0_std, pin_frac=w.pin_frac)
            for i in range(n_sets)]
    outs = [(torch.empty((B, T, H, dv), dtype=w.dtype, device=dev),
             torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)) for _ in range(n_sets)]
    fwd = kda.chunk_fwd_f32 if w.dtype == torch.float32 else kda.chunk_fwd
    set_bytes = sum(t.numel() * t.element_size() for t in sets[0].values() if t is not None)

    def step(i):
        x = sets[i % n_sets]
        o, hT = outs[i % n_sets]
        fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], o=o, hT=hT)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        keep_busy(step, 0.4, torch.cuda.synchronize)
        barrier(dev)
        torch.cuda.synchronize()
        n0 = kda.launch_count()
        ev[0].record(stream)
        for i in range(args.steps):
            step(i)
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        launches = kda.launch_count() - n0
        barrier(dev)
        keep_busy(step, 0.3, torch.cuda.synchronize, first=args.steps)
    per_step = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_ms = ev[0].elapsed_time(ev[-1])
    total_ms = max_over_ranks(total_ms, dev)
    ms_per_step = total_ms / args.steps
    tokens = B * T * world * args.steps
    value = tokens / (total_ms / 1e3)

    # roofline of the prefill kernel (one launch per step)
    hbm_gbs, bf16_tf, peak_src = load_peaks()
    alg_b = prefill_alg_bytes(B, T, H, dk, dv, with_h0=w.h0_std > 0,
                              elem=4 if w.dtype == torch.float32 else BYTES_BF16)
    alg_f = prefill_alg_flops(B, T, H, dk, dv)
    launch_ms = statistics.mean(per_step)
    achieved_gbs = alg_b / (launch_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved_gbs, 1),
                "peak": hbm_gbs, "unit": "GB/s",
                "frac": round(achieved_gbs / hbm_gbs, 4),
                "traffic": measured_traffic("kda_chunk_fwd", args.workload), "peak_source": peak_src + " hbm_gbs (burst copy)",
                "alg_bytes_per_launch": alg_b,
                "kernel": "kda_chunk_fwd",
                "variant": kda.prefill_path(B, T, H)}
    roofline.update(tensor_fractions(alg_f, prefill_state_flops(B, T, H, dk, dv), launch_ms, bf16_tf,
                                     roofline["variant"]))

    result = {
        "metric": METRIC,
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "ms_per_step_median": round(statistics.median(per_step), 4),
        "scaling": "weak", "vs_baseline": None,
        "dtype": "f32" if w.dtype == torch.float32 else "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "B": B, "T": T, "H": H, "dk": dk, "dv": dv,
                   "global_batch": B * world, "seq_len": T,
                   "parallelism": "dp%d" % world,
                   "l2": "%s %.0f MB input set%s (%s)" % (
                       "two" if n_sets == 2 else "one", set_bytes / 1e6,
                       "s alternate" if n_sets == 2 else "",
                       "inputs > L2" if set_bytes > 126e6 else "inputs fit in L2")},
        "roofline": roofline,
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }

    # end to end through the public API: pinned host inputs -> device ->
    # kda_chunk_fwd -> o and hT back to pinned host memory, every step
    # (pipelined across steps; see bench_e2e)
    if not args.small_footprint:
        result["e2e"] = bench_e2e(args, kda, sets, dev, B, T, world, fwd, w.dtype)
    del sets, outs
    torch.cuda.empty_cache()

    if args.decode:
        result["decode"] = bench_decode(args, kda, dev, rank, world, hbm_gbs, peak_src)
    if args.backward and not args.small_footprint:
        result["backward"] = bench_backward(args, kda, dev, rank, world, hbm_gbs, peak_src)
    # the other prefill workloads of the pages' length range, each timed the
    # same way on its own inputs (each input set is far larger than L2)
    if not args.small_footprint:
        for name in args.more_workloads:
            if name and name != w.name:
                result[name] = bench_prefill_workload(args, kda, dev, rank, world, name,
                                                      hbm_gbs, bf16_tf, peak_src)
    return result


def bench_backward(args, kda, dev, rank, world, hbm_gbs, peak_src):
    """kda_chunk_bwd on the 8K workload's shape (B1 H32 T8192, the shortest
    pre-training length), with both cotangents, timed like the prefill."""
    import torch
    from linear_attention_07_b200.inputs import WORKLOADS, prefill_inputs
    w = WORKLOADS["prefill_8k"]
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    x = prefill_inputs(B, T, H, dk, dv, seed=rank_seed(w.seed + 99, rank), device=dev, h0_std=w.h0_std)
    gen = torch.Generator(device=dev).manual_seed(rank_seed(w.seed + 98, rank))
    dO = torch.randn((B, T, H, dv), generator=gen, device=dev).to(torch.bfloat16)
    dhT = torch.randn((B, H, dk, dv), generator=gen, device=dev) * 0.1

    def step(i):
        kda.chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], dO, dhT)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    steps = max(3, min(args.steps, 10))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        keep_busy(step, 0.3, torch.cuda.synchronize)
        barrier(dev)
        torch.cuda.synchronize()
        n0 = kda.launch_count()
        ev[0].record(stream)
        for i in range(steps):
            step(i)
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        launches = kda.launch_count() - n0
        barrier(dev)
    per_step = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), dev)
    mean_ms = statistics.mean(per_step)
    alg_b = backward_alg_bytes(B, T, H, dk, dv)
    alg_f = backward_alg_flops(B, T, H, dk, dv)
    csum = clk.summary()
    sm_mhz = csum.get("sm_mhz") or 1965.0
    peak_alu = alu_peak_tflops(sm_mhz)
    ach_f = alg_f / (mean_ms / 1e3) / 1e12
    ach_b = alg_b / (mean_ms / 1e3) / 1e9
    out = {"metric": "KDA backward tokens/s (B1 H32 T8192 d128, bf16 in/out, fp32 arithmetic)",
           "value": round(B * T * world * steps / (total_ms / 1e3), 1), "unit": "tokens/s",
           "ms_per_step": round(total_ms / steps, 4), "steps": steps, "warmup": args.warmup,
           "roofline": {"bound": "alu", "achieved": round(ach_f, 2), "peak": round(peak_alu, 1),
                        "unit": "TFLOP/s", "frac": round(ach_f / peak_alu, 4), "traffic": None,
                        "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 flops x median SM clock",
                        "alg_flops_per_launch": alg_f, "kernel": "kda_chunk_bwd (3 launches)"},
           "hbm": {"achieved": round(ach_b, 1), "peak": hbm_gbs, "unit": "GB/s",
                   "frac": round(ach_b / hbm_gbs, 4), "alg_bytes_per_launch": alg_b,
                   "peak_source": peak_src + " hbm_gbs"},
           "gpu_launches": int(launches), "clocks": csum}
    del x, dO, dhT
    torch.cuda.empty_cache()
    return out


def bench_prefill_workload(args, kda, dev, rank, world, name, hbm_gbs, bf16_tf, peak_src):
    """One more prefill workload, timed like the main line (warm-up, CUDA
    events around `steps` back-to-back launches, clocks sampled under load),
    with one input set: each of these workloads is many times the size of
    L2, so no step finds its inputs there."""
    import torch
    from linear_attention_07_b200.inputs import WORKLOADS, prefill_inputs
    w = WORKLOADS[name]
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    x = prefill_inputs(B, T, H, dk, dv, seed=rank_seed(w.seed, rank), device=dev,
                       h0_std=w.h0_std, pin_frac=w.pin_frac)
    o = torch.empty((B, T, H, dv), dtype=w.dtype, device=dev)
    hT = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    set_bytes = sum(t.numel() * t.element_size() for t in x.values() if t is not None)

    def step(i):
        kda.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], o=o, hT=hT)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        keep_busy(step, 0.3, torch.cuda.synchronize)
        barrier(dev)
        torch.cuda.synchronize()
        n0 = kda.launch_count()
        ev[0].record(stream)
        for i in range(args.steps):
            step(i)
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        launches = kda.launch_count() - n0
        barrier(dev)
        keep_busy(step, 0.2, torch.cuda.synchronize)
    per_step = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), dev)
    launch_ms = statistics.mean(per_step)
    alg_b = prefill_alg_bytes(B, T, H, dk, dv, with_h0=w.h0_std > 0)
    ach = alg_b / (launch_ms / 1e3) / 1e9
    roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm_gbs, "unit": "GB/s",
            "frac": round(ach / hbm_gbs, 4), "traffic": measured_traffic("kda_chunk_fwd", name),
            "peak_source": peak_src + " hbm_gbs (burst copy)",
            "alg_bytes_per_launch": alg_b, "kernel": "kda_chunk_fwd",
            "variant": kda.prefill_path(B, T, H)}
    roof.update(tensor_fractions(prefill_alg_flops(B, T, H, dk, dv), prefill_state_flops(B, T, H, dk, dv),
                                 launch_ms, bf16_tf, roof["variant"]))
    out = {"metric": "KDA prefill tokens/s (%s)" % w.note,
           "value": round(B * T * world * args.steps / (total_ms / 1e3), 1), "unit": "tokens/s",
           "ms_per_step": round(total_ms / args.steps, 4),
           "ms_per_step_median": round(statistics.median(per_step), 4),
           "steps": args.steps, "warmup": args.warmup,
           "config": {"workload": w.name, "B": B, "T": T, "H": H, "dk": dk, "dv": dv,
                      "l2": "one %.2f GB input set (inputs > L2)" % (set_bytes / 1e9)},
           "roofline": roof, "gpu_launches": int(launches), "clocks": clk.summary()}
    del x, o, hT
    torch.cuda.empty_cache()
    return out


def bench_e2e(args, kda, sets, dev, B, T, world, fwd, dtype):
    """End to end through the public API: every step copies its inputs from
    pinned host memory to the device, runs the prefill and copies o and hT
    back to pinned host memory, all inside the timed region.  Steps are
    pipelined as a user loop would be: inputs go in on one copy stream and
    results come out on another, double-buffered, so step i+1's upload
    overlaps step i's kernel and download (PCIe moves both directions at
    once).  Buffer reuse is ordered by events.  If the pipelined loop fails
    to run, the plain serial loop is timed instead and says so."""
    import torch
    host = []
    for x in sets:
        host.append({k: (None if t is None else t.cpu().pin_memory()) for k, t in x.items()})
    s_shape = (tuple(sets[0]["h0"].shape) if sets[0]["h0"] is not None else
               (B, sets[0]["q"].shape[2], sets[0]["q"].shape[3], sets[0]["v"].shape[3]))
    dbufs, outs, o_hs, s_hs = [], [], [], []

    def add_slot():
        # one set of device inputs, device outputs and pinned host outputs
        dbufs.append({k: (None if t is None else torch.empty_like(t)) for k, t in sets[0].items()})
        outs.append((torch.empty_like(sets[0]["v"]),
                     torch.empty(s_shape, dtype=torch.float32, device=dev)))
        o_hs.append(torch.empty(tuple(sets[0]["v"].shape), dtype=dtype).pin_memory())
        s_hs.append(torch.empty(s_shape, dtype=torch.float32).pin_memory())

    add_slot()
    h2d = sum(t.numel() * t.element_size() for t in host[0].values() if t is not None)
    d2h = o_hs[0].numel() * o_hs[0].element_size() + s_hs[0].numel() * 4
    comp = torch.cuda.current_stream(dev)

    def run_fwd(j, i):
        d = dbufs[j]
        fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"], o=outs[j][0], hT=outs[j][1])

    def upload(j, i):
        for k2, t in host[i % 2].items():
            if t is not None:
                dbufs[j][k2].copy_(t, non_blocking=True)

    def download(j):
        o_hs[j].copy_(outs[j][0], non_blocking=True)
        s_hs[j].copy_(outs[j][1], non_blocking=True)

    def timed_pipelined():
        add_slot()                                   # the second buffer (may not fit: then serial)
        s_in = torch.cuda.Stream(device=dev)
        s_out = torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def step(i):
            j = i % 2
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_comp[j])          # step i-2's kernel has read dbufs[j]
                upload(j, i)
                ev_in[j].record(s_in)
            comp.wait_event(ev_in[j])
            comp.wait_event(ev_out[j])               # step i-2's results have left outs[j]
            run_fwd(j, i)
            ev_comp[j].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[j])
                download(j)
                ev_out[j].record(s_out)

        for i in range(max(2, args.warmup)):
            step(i)
        torch.cuda.synchronize()
        barrier(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(args.steps):
            step(i)
        for j in range(2):                           # every copy of every step is inside
            comp.wait_event(ev_in[j])
            comp.wait_event(ev_out[j])
        e1.record(comp)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    def timed_serial():
        def step(i):
            upload(0, i)
            run_fwd(0, i)
            download(0)

        for i in range(max(1, args.warmup)):
            step(i)
        torch.cuda.synchronize()
        barrier(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        for i in range(args.steps):
            step(i)
        e1.record(comp)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    mode = "pipelined: uploads, kernel and downloads overlap across steps (2 copy streams)"
    try:
        ms = timed_pipelined()
    except Exception as e:          # local; both loops take the same one barrier before timing
        torch.cuda.synchronize()
        del dbufs[1:], outs[1:], o_hs[1:], s_hs[1:]
        mode = "serial (pipelined loop failed: %s)" % (repr(e)[:160],)
        ms = timed_serial()
    ms = max_over_ranks(ms, dev)
    return {"value": round(B * T * world * args.steps / (ms / 1e3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(ms / args.steps, 4), "mode": mode}


def bench_decode(args, kda, dev, rank, world, hbm_gbs, peak_src):
    import torch
    from linear_attention_07_b200.inputs import WORKLOADS, decode_inputs
    w = WORKLOADS["decode_256"]
    N, H, dk, dv, steps = w.B, w.H, w.dk, w.dv, w.T
    if args.small_footprint:
        steps = 16            # profiler captures: 16 steps of inputs, not 1000 (8.4 GB)
    d = decode_inputs(N, H, dk, dv, steps, seed=rank_seed(w.seed, rank), device=dev,
                      state_std=w.h0_std)
    S = d["state"]
    o = torch.empty((N, H, dv), dtype=torch.bfloat16, device=dev)
    for t in range(3):
        kda.decode_step(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], S, o=o)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    barrier(dev)
    ev[0].record(stream)
    for t in range(steps):
        kda.decode_step(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], S, o=o)
        ev[t + 1].record(stream)
    torch.cuda.synchronize()
    per = sorted(ev[t].elapsed_time(ev[t + 1]) for t in range(steps))
    total = max_over_ranks(ev[0].elapsed_time(ev[-1]), dev)
    alg = decode_alg_bytes(N, H, dk, dv)
    mean_ms = statistics.mean(per)
    ach = alg / (mean_ms / 1e3) / 1e9
    out = {"metric": "KDA decode steps/s (256 requests x H32 d128, fp32 state)",
           "value": round(steps * world / (total / 1e3) / world, 1), "unit": "steps/s per GPU",
           "aggregate_steps_per_s": round(steps * world / (total / 1e3), 1),
           "steps": steps, "ms_per_step_p50": round(per[len(per) // 2], 5),
           "ms_per_step_p99": round(per[int(len(per) * 0.99) - 1], 5),
           "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm_gbs,
                        "unit": "GB/s", "frac": round(ach / hbm_gbs, 4),
                        "traffic": measured_traffic("kda_decode_step", "decode_256"),
                        "peak_source": peak_src + " hbm_gbs (burst copy)",
                        "alg_bytes_per_launch": alg, "kernel": "kda_decode_step"}}
    del d
    return out


# -------------------------------------------------------- oracle on CPU ---

class OracleSample:
    """`heads` whole (b, h) sequences of a prefill workload (its per-head
    recipe), generated once, for timing the fp64 oracle on the host cores:
    the oracle runs one head per thread.  Tokens/s counts full tokens (all H
    heads of the workload), i.e. sampled token-heads / H / seconds."""

    def __init__(self, workload_name, heads, seed):
        import oracle
        from linear_attention_07_b200.inputs import WORKLOADS, prefill_inputs
        self.w = w = WORKLOADS[workload_name]
        self.heads = heads
        self.x = prefill_inputs(1, w.T, heads, w.dk, w.dv, seed=seed, dtype=w.dtype,
                                h0_std=w.h0_std, pin_frac=w.pin_frac)
        self.threads = min(heads, oracle.num_cores())
        self.tokens = heads * w.T / w.H
        self.desc = ("%d heads x %d tokens with the per-head recipe of %s (H = %d), fp64 "
                     "token-by-token, one head per thread" % (heads, w.T, w.name, w.H))

    def time(self):
        """One timed oracle run over the whole sample: seconds."""
        import oracle
        x = self.x
        t0 = time.perf_counter()
        oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
        return time.perf_counter() - t0


def oracle_heads(requested):
    """Heads per oracle sample: as asked, else one per host core (at most
    256), so the oracle runs on every core as its thread pool is built to."""
    if requested:
        return int(requested)
    import oracle
    return max(1, min(256, oracle.num_cores()))


def cpu_model():
    """The host CPU's model name (Linux), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_baseline(args, min_seconds=10.0, max_runs=40):
    """The oracle, as it stands, timed on one sample of the workload, run
    repeatedly until about `min_seconds` of oracle time has been timed."""
    smp = OracleSample(args.workload, oracle_heads(args.cpu_heads), 4242)
    total_t, runs = 0.0, 0
    while runs < max_runs and (runs == 0 or total_t < min_seconds):
        total_t += smp.time()
        runs += 1
    return {"value": round(smp.tokens * runs / total_t, 2), "unit": "tokens/s",
            "cores": smp.threads, "kind": "oracle", "sample": "%d x (%s)" % (runs, smp.desc),
            "seconds": round(total_t, 2), "cpu_model": cpu_model()}


def bench_reference(args, rank, world):
    if rank != 0:
        return None
    smp = OracleSample(args.workload, oracle_heads(args.ref_heads), 199)
    w = smp.w
    for i in range(args.warmup):
        smp.time()
    total = sum(smp.time() for _ in range(args.steps))
    value = smp.tokens * args.steps / total
    cores, desc = smp.threads, smp.desc
    return {"metric": METRIC,
            "value": round(value, 2), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total / args.steps * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk,
                       "dv": w.dv, "global_batch": w.B, "seq_len": w.T,
                       "parallelism": "host threads"},
            "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": "each step: " + desc,
                             "cpu_model": cpu_model()},
            "e2e": {"value": round(value, 2), "unit": "tokens/s",
                    "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------- main ---

def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kda", choices=["kda", "reference"])
    ap.add_argument("--workload", default="prefill_8k")
    ap.add_argument("--no-decode", dest="decode", action="store_false")
    ap.add_argument("--no-cpu-baseline", dest="cpu_base", action="store_false")
    ap.add_argument("--more-workloads", default="pretrain_64k,prefill_1m",
                    type=lambda x: [y for y in x.split(",") if y],
                    help="other prefill workloads timed in the same run, reported as sub-objects "
                         "(comma-separated names; empty: none)")
    ap.add_argument("--no-backward", dest="backward", action="store_false",
                    help="skip the backward (kda_chunk_bwd) line")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only the backward (for profiler captures); prints its line alone")
    ap.add_argument("--small-footprint", action="store_true",
                    help="for profiler captures: one prefill input set, 16 decode steps, "
                         "no end-to-end leg and no other workloads")
    ap.add_argument("--cpu-heads", type=int, default=None,
                    help="heads per oracle sample (default: one per host core)")
    ap.add_argument("--ref-heads", type=int, default=None,
                    help="heads per reference-arm step (default: one per host core)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local = dist_env()

    if args.impl == "reference":
        res = bench_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0

    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        if args.backward_only:
            import linear_attention_07_b200 as kda
            dev = torch.device("cuda", local)
            torch.cuda.set_device(dev)
            kda.load_library()
            hbm_gbs, _, peak_src = load_peaks()
            res = bench_backward(args, kda, dev, rank, world, hbm_gbs, peak_src)
            if rank == 0:
                print(json.dumps(res), flush=True)
            return 0
        res = bench_kda(args, rank, world, local)
        if rank == 0 and args.cpu_base:
            res["cpu_baseline"] = cpu_baseline(args)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1 and dist.is_initialized():
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
