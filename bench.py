#!/usr/bin/env python
"""Benchmark of the Ring Self-Attention hot path (forward + backward) on B200.

One step = rsa_forward + rsa_backward over one batch (ring pass 1, slab softmax, ring pass 2,
then the backward ring), on synthetic inputs shaped like the method's transformer workloads.
Default workload: the BERT-base-shaped configuration (B=8, H=12, L=512, d=64, N=4, bf16,
non-causal). Prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload bert|gpt|long]
    python bench.py --impl reference ...   # the fp64 CPU oracle on the same workload

Timing: W untimed steps; then K steps, each preceded (outside the timed events) by an L2
flush (a 512 MiB write) and a short GPU spin that keeps the launch queue ahead of the GPU;
each step is bracketed by CUDA events on the launching stream, and the step times are summed.
Every library kernel is also bracketed by events (rsa_profile_*), which gives the per-kernel
durations for the roofline. Multi-GPU (torchrun): every rank runs its own batch (weak
scaling, no collective on the data path); the job time is the slowest rank's.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "RSA fwd+bwd TFLOP/s and tokens/s on 1 B200; % of tensor/HBM roofline"

WORKLOADS = {
    "bert": dict(B=8, H=12, L=512, d=64, N=4, causal=False, seed=2,
                 name="BERT-base-shaped RSA fwd+bwd: B=8 H=12 L=512 d=64 N=4 bf16 non-causal"),
    "gpt": dict(B=4, H=16, L=4096, d=64, N=8, causal=True, seed=3,
                name="GPT-style causal RSA fwd+bwd: B=4 H=16 L=4096 d=64 N=8 bf16"),
    "long": dict(B=1, H=16, L=16384, d=128, N=16, causal=False, seed=4,
                 name="long-sequence RSA fwd+bwd: B=1 H=16 L=16384 d=128 N=16 bf16 non-causal"),
}

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, bf16_tflops_sustained=1400.0)


# ----------------------------------------------------------------------------- work model

def live_entries(L: int, causal: bool) -> int:
    """Score entries per head that the method computes: L^2, or L(L+1)/2 under a causal mask."""
    return L * (L + 1) // 2 if causal else L * L


def step_flops(w) -> float:
    """Algorithmic fwd+bwd flops per step: 4pd forward (QK^T, PV) + 8pd backward (dV, dP,
    dQ, dK); the backward's recompute of S is executed work but not counted."""
    p = w["B"] * w["H"] * live_entries(w["L"], w["causal"])
    return 12.0 * p * w["d"]


def kernel_model(w):
    """Algorithmic flops and bytes of one launch of each bf16 kernel when a single group holds
    every head (the default plan for the default workload). p = live score entries."""
    B, H, L, d = w["B"], w["H"], w["L"], w["d"]
    BH = B * H
    p = BH * live_entries(L, w["causal"])
    t = BH * L * d * 2  # one [B,H,L,d] bf16 tensor
    row = BH * L * 4    # one fp32 per row (lse, D)
    return {
        "qk_slab": (2 * p * d, 4 * p + 2 * t),                 # S fp32 write; Q, K read
        # slab-free forward: pass 1 (QK^T; Q K read, lse write), pass 2 (PV, with S recomputed,
        # not counted; Q K V read, O write, lse read)
        "fwd_stats": (2 * p * d, 2 * t + row),
        "fwd_pv": (2 * p * d, 4 * t + row),
        "pv_softmax": (2 * p * d, 4 * p + 2 * t + row),         # S read, V read, O, lse write
        # query-major backward: dQ (+ the recomputed S and dP, not counted); Q dO O K V read,
        # dQ write, lse read, the rows' lse*log2(e) and D written
        "bwd_rows": (2 * p * d, 6 * t + 3 * row),
        # key-major backward: dP^T, dV, dK (+ the recomputed S^T, not counted); Q K V dO read,
        # dK dV write, the rows' lse*log2(e) and D read
        "bwd_keys": (6 * p * d, 6 * t + 2 * row),
    }


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every `period` seconds."""

    REASONS = [("GpuIdle", "gpu_idle"), ("ApplicationsClocksSetting", "applications_clocks"),
               ("SwPowerCap", "sw_power_cap"), ("HwSlowdown", "hw_slowdown"),
               ("SyncBoost", "sync_boost"), ("SwThermalSlowdown", "sw_thermal_slowdown"),
               ("HwThermalSlowdown", "hw_thermal_slowdown"),
               ("HwPowerBrakeSlowdown", "hw_power_brake_slowdown")]

    def __init__(self, index: int, period: float = 0.01):
        self.samples = []
        self.period = period
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.bits = []
            for name, label in self.REASONS:
                v = getattr(pynvml, "nvmlClocksEventReason" + name, None)
                if v is None:
                    v = getattr(pynvml, "nvmlClocksThrottleReason" + name, None)
                if v is not None:
                    self.bits.append((int(v), label))
            self.ok = True
        except Exception as e:  # NVML missing: the line reports no clock record
            self.err = str(e)

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                r = int(get_reasons(self.h))
                self.samples.append((time.perf_counter(), mhz, r))
            except Exception:
                pass
            self._stop.wait(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0: float, t1: float):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        note = f"{len(inside)} samples in the timed region"
        if not inside and self.samples:  # region shorter than the sampling period
            mid = 0.5 * (t0 + t1)
            inside = sorted(self.samples, key=lambda s: abs(s[0] - mid))[:3]
            note = "timed region shorter than the sampling period; nearest samples"
        reasons = set()
        for _, _, r in inside:
            for bit, label in self.bits:
                if r & bit and label != "gpu_idle":
                    reasons.add(label)
        mhz = [s[1] for s in inside]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "note": note}


# ----------------------------------------------------------------------------- CPU oracle

def _oracle_heads(w, heads: int):
    """Seconds the fp64 oracle takes for forward and for backward of `heads` heads."""
    from oracle import oracle
    from sequence_ring_self_b200.inputs import make_inputs

    x = make_inputs(1, heads, w["L"], w["d"], seed=w["seed"], dtype="bf16")
    t = time.perf_counter()
    oracle.forward(x.q, x.k, x.v, w["causal"])
    t1 = time.perf_counter()
    oracle.backward(x.q, x.k, x.v, x.do, w["causal"])
    return t1 - t, time.perf_counter() - t1


def oracle_plan(w, seconds: float):
    """Heads per sample so that one sample takes about `seconds`; returns (heads, threads)."""
    from oracle import oracle

    oracle.build()
    threads = oracle.max_threads()
    t_f, t_b = _oracle_heads(w, 1)
    # the forward is parallel over rows (cost ~ heads * t_f); the backward is parallel over
    # heads (cost ~ ceil(heads / threads) * t_b)
    heads = 1
    while heads < w["B"] * w["H"]:
        h = heads + 1
        if h * t_f + math.ceil(h / threads) * t_b > seconds:
            break
        heads = h
    return heads, threads


def oracle_sample(w, seconds: float):
    """Time the oracle on a bounded sample of heads: (flops done, seconds, heads, threads)."""
    heads, threads = oracle_plan(w, seconds)
    dt = sum(_oracle_heads(w, heads))
    return 12.0 * live_entries(w["L"], w["causal"]) * w["d"] * heads, dt, heads, threads


def run_reference(args, w):
    """The reference arm: the fp64 CPU oracle, as it stands, on bounded samples of the workload."""
    from sequence_ring_self_b200.dist import env_ranks

    rank, world, _ = env_ranks()
    if rank != 0:
        return 0
    steps, warmup = args.steps, args.warmup
    budget = args.ref_budget / max(1, steps + warmup)  # whole run within the budget
    heads, threads = oracle_plan(w, budget)
    flops_step = 12.0 * live_entries(w["L"], w["causal"]) * w["d"] * heads
    times = []
    for i in range(warmup + steps):
        dt = sum(_oracle_heads(w, heads))
        if i >= warmup:
            times.append(dt)
    total = sum(times)
    value = flops_step * steps / total / 1e12
    sample = (f"fp64 oracle forward+backward of {heads} of the {w['B'] * w['H']} heads per step "
              f"({w['name']})")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": steps, "warmup": warmup,
        "ms_per_step": 1e3 * total / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w["name"], "global_batch": w["B"], "seq_len": w["L"],
                   "chunks": w["N"], "heads": w["H"], "head_dim": w["d"], "causal": w["causal"],
                   "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "tokens_per_s": heads / (w["B"] * w["H"]) * w["B"] * w["L"] * steps / total,
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm

def run_gpu(args, w):
    import torch

    from sequence_ring_self_b200 import build, dist, rsa
    from sequence_ring_self_b200.inputs import make_inputs

    rank, world, local = dist.env_ranks()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist.init("nccl", device=dev)
    build.build()
    rsa.load_library()

    B, H, L, d, N, causal = w["B"], w["H"], w["L"], w["d"], w["N"], w["causal"]
    x = make_inputs(B, H, L, d, seed=w["seed"] + 1000 * rank, dtype="bf16")
    q, k, v, do = (x.torch(n, dev) for n in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, L), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    nf = rsa.workspace_size(B, H, L, d, N, causal, torch.bfloat16, False, args.ws_budget)
    nb = rsa.workspace_size(B, H, L, d, N, causal, torch.bfloat16, True, args.ws_budget)
    ws_f = torch.empty(nf, dtype=torch.uint8, device=dev)
    ws_b = torch.empty(nb, dtype=torch.uint8, device=dev)
    plan_f = rsa.plan_describe(B, H, L, d, N, causal, torch.bfloat16, False, nf)
    plan_b = rsa.plan_describe(B, H, L, d, N, causal, torch.bfloat16, True, nb)
    flush = torch.empty(max(1, args.flush_mib) << 20, dtype=torch.uint8, device=dev)

    def step():
        if args.forward == "recompute":
            rsa.forward_recompute(q, k, v, N, causal, out=o, lse=lse)
        else:
            rsa.forward(q, k, v, N, causal, workspace=ws_f, out=o, lse=lse)
        rsa.backward(q, k, v, o, do, lse, N, causal, workspace=ws_b, dq=dq, dk=dk, dv=dv)

    # warm-up; measure how long the host takes to enqueue one step
    host = []
    for _ in range(max(3, args.warmup)):
        flush.zero_()
        t = time.perf_counter()
        step()
        host.append(time.perf_counter() - t)
        torch.cuda.synchronize()
    if rsa.last_device_status() != rsa.RSA_OK:
        raise RuntimeError("a kernel reported a timeout during warm-up")
    # GPU spin before each timed step: a few times the host's enqueue time (capped at 4 ms)
    guard_cycles = int(min(8e6, max(2e5, 4.0 * statistics.median(host) * 2.0e9)))

    clocks = ClockSampler(local)
    clocks.start()
    K = args.steps

    def timed_steps(n, kernel_events):
        """n steps, each preceded (outside its events) by the L2 flush and a short GPU spin that
        keeps the launch queue ahead of the GPU; returns the per-step device times (ms)."""
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        rsa.profile_enable(kernel_events)
        for i in range(n):
            flush.zero_()
            torch.cuda._sleep(guard_cycles)
            starts[i].record()
            step()
            ends[i].record()
        torch.cuda.synchronize()
        return [s.elapsed_time(e) for s, e in zip(starts, ends)]

    # the timed region: K steps, no per-kernel events (kernels overlap their prologues with the
    # previous kernel's tail through programmatic dependent launch)
    dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    step_ms = timed_steps(K, False)
    t1 = time.perf_counter()
    dist.barrier()
    clocks.stop()
    if rsa.last_device_status() != rsa.RSA_OK:
        raise RuntimeError("a kernel reported a timeout")
    # per-kernel durations: the same steps again with every library kernel bracketed by CUDA
    # events on its stream (the events themselves add about 5 us per kernel to a step)
    kp = max(3, min(K, args.profile_steps))
    prof_step_ms = timed_steps(kp, not args.no_kernel_events)
    prof = rsa.profile_read()
    rsa.profile_enable(False)
    total_ms = sum(step_ms)
    slowest_ms = dist.max_over_ranks(total_ms, dev)
    flops = step_flops(w)
    value = dist.weak_scaling_throughput(flops * K, world, slowest_ms / 1e3) / 1e12
    tokens_s = dist.weak_scaling_throughput(B * L * K, world, slowest_ms / 1e3)

    # end to end through the public API from pinned host buffers
    e2e = None
    if not args.no_e2e:
        hq, hk, hv, hdo = (x.torch(n).pin_memory() for n in ("q", "k", "v", "do"))
        res = rsa.forward_backward_host(hq, hk, hv, hdo, N, causal, ws_budget=args.ws_budget,
                                        device=dev, recompute=args.forward == "recompute")
        torch.cuda.synchronize()
        e_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        e_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        dist.barrier()
        torch.cuda.synchronize()
        for i in range(K):
            flush.zero_()
            e_s[i].record()
            rsa.forward_backward_host(hq, hk, hv, hdo, N, causal, ws_budget=args.ws_budget,
                                      device=dev, results=res,
                                      recompute=args.forward == "recompute")
            e_e[i].record()
        torch.cuda.synchronize()
        dist.barrier()
        e2e_ms = sum(s.elapsed_time(e) for s, e in zip(e_s, e_e))
        e2e_slowest = dist.max_over_ranks(e2e_ms, dev)
        e2e = {"value": dist.weak_scaling_throughput(flops * K, world, e2e_slowest / 1e3) / 1e12,
               "unit": "TFLOP/s", "h2d_bytes_per_step": 4 * q.numel() * q.element_size(),
               "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in res.values()),
               "ms_per_step": e2e_slowest / K}

    peaks = load_peaks()
    model = kernel_model(w)
    phases = []
    step_kernel_ms = sum(ms for ms, _ in prof.values())
    single_group = plan_f["groups"] == 1 and plan_b["groups"] == 1
    for name, (ms, n) in sorted(prof.items(), key=lambda kv: -kv[1][0]):
        avg_s = ms / n / 1e3
        fl, by = model.get(name, (None, None)) if single_group else (None, None)
        ph = {"kernel": name, "launches": n, "avg_us": 1e6 * avg_s, "share": ms / step_kernel_ms}
        if by:
            ph["alg_bytes"] = by
            ph["alg_flops"] = fl
            ph["achieved_gbs"] = by / avg_s / 1e9
            ph["hbm_frac"] = ph["achieved_gbs"] / peaks["hbm_gbs"]
            if fl:
                ph["achieved_tflops"] = fl / avg_s / 1e12
                ph["tensor_frac"] = ph["achieved_tflops"] / peaks["bf16_tflops"]
        phases.append(ph)
    if not phases:
        phases = [{"kernel": "none (no per-kernel events)"}]
    top = phases[0]
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if os.path.exists(tpath):
        try:
            from sequence_ring_self_b200.build import source_digest

            t = json.load(open(tpath))
            ent = t.get("kernels", {}).get(top["kernel"])
            if ent and t.get("workload") == w["name"] and t.get("source_digest") == source_digest():
                traffic = ent["dram_bytes_per_launch"]
        except Exception:
            traffic = None
    roofline = {"kernel": top["kernel"], "bound": "hbm",
                "achieved": top.get("achieved_gbs"), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": top.get("hbm_frac"), "traffic": traffic,
                "peak_source": f"{peaks['source']} (HBM copy bandwidth)"}
    for ph in phases:
        fl, by = ph.get("alg_flops"), ph.get("alg_bytes")
        if fl and by and fl / by > peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9):
            ph["bound"] = "tensor"
        elif by:
            ph["bound"] = "hbm"
    if top.get("bound") == "tensor":
        roofline.update(bound="tensor", achieved=top["achieved_tflops"], peak=peaks["bf16_tflops"],
                        unit="TFLOP/s", frac=top["tensor_frac"],
                        peak_source=f"{peaks['source']} (bf16 dense burst)")

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": slowest_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w["name"], "global_batch": B * world, "seq_len": L, "heads": H,
                   "head_dim": d, "chunks": N, "causal": causal,
                   "parallelism": f"dp{world} (independent batches per GPU)",
                   "l2": f"flushed between steps ({args.flush_mib} MiB write)",
                   "forward": args.forward,
                   "slab_groups": {"forward": plan_f["groups"], "backward": plan_b["groups"],
                                   "workspace_bytes": [nf, nb]}},
        "tokens_per_s": tokens_s,
        "step_ms_median": statistics.median(step_ms),
        "e2e": e2e,
        "gpu_launches": int(round(sum(n for _, n in prof.values()) / kp * K)),
        "profiled_pass": {"steps": kp, "ms_per_step_with_kernel_events": statistics.median(prof_step_ms)},
        "roofline": roofline,
        "phases": phases,
        "clocks": clocks.summary(t0, t1),
        "peaks": peaks,
    }
    if world == 1 and not args.no_cpu_baseline:
        fl, sec, heads, threads = oracle_sample(w, args.cpu_seconds)
        line["cpu_baseline"] = {
            "value": fl / sec / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"fp64 oracle forward+backward of {heads} of {B * H} heads, {sec:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.finish()
    return 0


def run_sweep(args):
    """The sweep configuration (B=1, H=16, d=64, bf16; L x N x causal): one JSON line per point
    with the GPU step time and TFLOP/s (documentation numbers; the contract line is the default
    workload's)."""
    import torch

    from sequence_ring_self_b200 import build, rsa
    from sequence_ring_self_b200.inputs import make_inputs

    build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    Ls = [int(x) for x in args.sweep_L.split(",")]
    Ns = [int(x) for x in args.sweep_N.split(",")]
    for causal in (False, True):
        for L in Ls:
            for N in Ns:
                w = dict(B=1, H=16, L=L, d=64, N=N, causal=causal, seed=5)
                x = make_inputs(1, 16, L, 64, seed=5, dtype="bf16")
                q, k, v, do = (x.torch(n, dev) for n in ("q", "k", "v", "do"))
                o, lse = rsa.forward(q, k, v, N, causal)
                rsa.backward(q, k, v, o, do, lse, N, causal)
                torch.cuda.synchronize()
                times = []
                for _ in range(args.steps):
                    flush.zero_()
                    torch.cuda._sleep(2_000_000)
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    o, lse = rsa.forward(q, k, v, N, causal)
                    rsa.backward(q, k, v, o, do, lse, N, causal)
                    e1.record()
                    torch.cuda.synchronize()
                    times.append(e0.elapsed_time(e1))
                ms = statistics.median(times)
                print(json.dumps({"sweep_point": {"L": L, "N": N, "causal": causal}, "ms_per_step": ms,
                                  "tflops": step_flops(w) / ms / 1e9,
                                  "tokens_per_s": L / ms * 1e3}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + ["sweep"], default="bert")
    ap.add_argument("--forward", choices=["slab", "recompute"], default="slab",
                    help="slab: the method's forward (score slab in HBM, the headline path); "
                         "recompute: the slab-free two-pass forward")
    ap.add_argument("--sweep-L", default="1024,2048,4096,8192,16384,32768")
    ap.add_argument("--sweep-N", default="1,2,4,8,16")
    ap.add_argument("--ws-budget", type=int, default=0, help="workspace budget in bytes (0: default)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU seconds of the oracle sample reported as cpu_baseline")
    ap.add_argument("--ref-budget", type=float, default=120.0,
                    help="seconds the whole --impl reference run should take")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end timing")
    ap.add_argument("--no-kernel-events", action="store_true",
                    help="skip the per-kernel profiled pass (no phases / roofline)")
    ap.add_argument("--profile-steps", type=int, default=50,
                    help="steps of the per-kernel profiled pass that follows the timed region")
    ap.add_argument("--flush-mib", type=int, default=512, help="L2 flush buffer (MiB) written before each step")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.workload == "sweep":
        return run_sweep(args)
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
