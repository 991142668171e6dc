#!/usr/bin/env python
"""Benchmark of the Ring Self-Attention hot path (forward + backward) on B200.

One step = rsa_forward + rsa_backward over one batch (ring pass 1, slab softmax, ring pass 2,
then the backward ring), on synthetic inputs shaped like the method's transformer workloads.
Default workload: the long-sequence configuration (B=1, H=16, L=16384, d=128, N=16, bf16,
non-causal), the largest one that fits one GPU; its score slab (17 GB) is produced and consumed
in groups that fit the workspace budget. Prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long|gpt|bert|f32|sweep]
    python bench.py --impl reference ...   # the fp64 CPU oracle on the same workload
    python bench.py --ring P ...           # the ring across P GPUs, emulated on one GPU

Timing: W untimed steps; then K steps, each preceded (outside the timed events) by an L2
flush (a 512 MiB write) and a short GPU spin that keeps the launch queue ahead of the GPU;
each step is bracketed by CUDA events on the launching stream, and the step times are summed.
A second pass brackets every library kernel with events (rsa_profile_*), which gives each
kernel's duration for the per-kernel roofline. Multi-GPU (torchrun): every rank runs its own
batch (weak scaling, no collective on the data path); the job time is the slowest rank's.
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
    "long": dict(B=1, H=16, L=16384, d=128, N=16, causal=False, seed=4, dtype="bf16",
                 name="long-sequence RSA fwd+bwd: B=1 H=16 L=16384 d=128 N=16 bf16 non-causal"),
    "gpt": dict(B=4, H=16, L=4096, d=64, N=8, causal=True, seed=3, dtype="bf16",
                name="GPT-style causal RSA fwd+bwd: B=4 H=16 L=4096 d=64 N=8 bf16"),
    "bert": dict(B=8, H=12, L=512, d=64, N=4, causal=False, seed=2, dtype="bf16",
                 name="BERT-base-shaped RSA fwd+bwd: B=8 H=12 L=512 d=64 N=4 bf16 non-causal"),
    "f32": dict(B=1, H=2, L=256, d=32, N=4, causal=False, seed=0, dtype="f32",
                name="fp32 RSA fwd+bwd: B=1 H=2 L=256 d=32 N=4 non-causal (CUDA cores)"),
}
DEFAULT_WORKLOAD = "long"

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS)


# ----------------------------------------------------------------------------- work model

def live_entries(L: int, causal: bool) -> int:
    """Score entries per head that the method computes: L^2, or L(L+1)/2 under a causal mask."""
    return L * (L + 1) // 2 if causal else L * L


def step_flops(w) -> float:
    """Algorithmic fwd+bwd flops per step: 4pd forward (QK^T, PV) + 8pd backward (dV, dP,
    dQ, dK); recomputed products (S in the backward, S and dP a second time for dQ) are
    executed work but not counted."""
    p = w["B"] * w["H"] * live_entries(w["L"], w["causal"])
    return 12.0 * p * w["d"]


def kernel_model(w):
    """Per step and per kernel kind: (algorithmic flops, executed flops, algorithmic bytes).

    Totals over every launch of the kind in one step, so they hold whatever the slab grouping
    (a kind's launches together cover every head and row once). p = live score entries, t =
    one [B,H,L,d] tensor, row = one fp32 per query row. Algorithmic bytes are what the design
    must move through HBM: each tensor once, the fp32 score slab once each way, the per-row
    softmax partials (one (max, sum) pair per 128 scores) and the per-row statistics."""
    B, H, L, d = w["B"], w["H"], w["L"], w["d"]
    BH = B * H
    p = BH * live_entries(L, w["causal"])
    es = 4 if w.get("dtype") == "f32" else 2
    t = BH * L * d * es
    row = BH * L * 4
    part = p // 16  # 8 bytes per 128 scores
    pd = p * d
    return {
        # bf16 tensor-core path
        "qk_slab": (2 * pd, 2 * pd, 4 * p + part + 2 * t),           # S, partials write; Q K read
        "pv_softmax": (2 * pd, 2 * pd, 4 * p + part + 2 * t + row),  # S, partials, V read; O lse write
        "fwd_stats": (2 * pd, 2 * pd, 2 * t + row),                  # Q K read, lse write
        "fwd_pv": (2 * pd, 4 * pd, 4 * t + row),                     # Q K V read, O write, lse read
        # query-major backward: dQ (S and dP recomputed); Q dO O K V read, dQ write, lse read,
        # lse*log2(e) and D written
        "bwd_rows": (2 * pd, 6 * pd, 6 * t + 3 * row),
        # key-major backward: dP^T, dV, dK (S^T recomputed); Q K V dO read, dK dV write,
        # lse*log2(e) and D read
        "bwd_keys": (6 * pd, 8 * pd, 6 * t + 2 * row),
        # fp32 CUDA-core path
        "f32_qk_slab": (2 * pd, 2 * pd, 4 * p + 2 * t),               # S write; Q K read
        "slab_softmax": (0, 0, 8 * p + row),                         # S read, P write, lse
        "f32_pv_ring_rows": (2 * pd, 2 * pd, 4 * p + 2 * t),          # P, V read; O write
        "rowdot": (0, 0, 2 * t + row),                               # dO, O read; D write
        "f32_bwd_slab": (2 * pd, 4 * pd, 8 * p + 4 * t + 2 * row),    # dP (P recomputed); P dS write
        "f32_ring_keys": (4 * pd, 4 * pd, 8 * p + 4 * t),             # dV, dK (two launches)
        "f32_dq_ring_rows": (2 * pd, 2 * pd, 4 * p + 2 * t),          # dS, K read; dQ write
    }


F32_KINDS = {"f32_qk_slab", "slab_softmax", "f32_pv_ring_rows", "rowdot", "f32_bwd_slab",
             "f32_ring_keys", "f32_dq_ring_rows"}


def phases_from_profile(prof, steps, w, peaks, compute_peak):
    """Per-kernel phases from {kind: (total ms, launches)} over `steps` steps: per-launch
    duration, algorithmic work per launch, achieved rates and the fraction of the roofline
    that bounds the kernel (tensor or HBM for the bf16 kernels, FP32 ALU or HBM for the fp32
    ones). compute_peak(kind) -> (TFLOP/s, label)."""
    model = kernel_model(w)
    total_ms = sum(ms for ms, _ in prof.values()) or 1.0
    phases = []
    for name, (ms, n) in sorted(prof.items(), key=lambda kv: -kv[1][0]):
        per_step_s = ms / steps / 1e3
        per_launch_s = ms / n / 1e3
        launches_step = n / steps
        ph = {"kernel": name, "launches": n, "launches_per_step": launches_step,
              "avg_us": 1e6 * per_launch_s, "ms_per_step": 1e3 * per_step_s,
              "share": ms / total_ms}
        if name in model:
            fl, ex, by = model[name]
            peak_t, label = compute_peak(name)
            ph["alg_flops_per_launch"] = fl / launches_step
            ph["exec_flops_per_launch"] = ex / launches_step
            ph["alg_bytes_per_launch"] = by / launches_step
            ph["achieved_gbs"] = by / per_step_s / 1e9
            ph["hbm_frac"] = ph["achieved_gbs"] / peaks["hbm_gbs"]
            ph["achieved_tflops"] = fl / per_step_s / 1e12
            ph["executed_tflops"] = ex / per_step_s / 1e12
            ph["compute_peak"] = label
            ph["compute_frac"] = ph["achieved_tflops"] / peak_t
            ph["compute_frac_executed"] = ph["executed_tflops"] / peak_t
            ridge = peak_t * 1e12 / (peaks["hbm_gbs"] * 1e9)
            is_f32 = name in F32_KINDS
            if fl and fl / by > ridge:
                ph["bound"] = "alu" if is_f32 else "tensor"
            else:
                ph["bound"] = "hbm"
            # lower bound on the kernel's time: the slower of its compute and its HBM traffic
            ph["roof_ms_per_step"] = 1e3 * max(fl / (peak_t * 1e12), by / (peaks["hbm_gbs"] * 1e9))
        phases.append(ph)
    return phases


def roofline_of(phases, peaks, traffic):
    """The dominant kernel's roofline object (achieved / peak on the bound it sits against)."""
    top = phases[0]
    if "bound" not in top:
        return {"kernel": top["kernel"], "bound": None, "achieved": None, "peak": None,
                "unit": None, "frac": None, "traffic": traffic}
    if top["bound"] == "hbm":
        return {"kernel": top["kernel"], "bound": "hbm", "achieved": top["achieved_gbs"],
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": top["hbm_frac"],
                "traffic": traffic, "alg_bytes_per_launch": top["alg_bytes_per_launch"],
                "peak_source": f"{peaks['source']} (HBM copy bandwidth)"}
    peak = top["achieved_tflops"] / top["compute_frac"]
    return {"kernel": top["kernel"], "bound": top["bound"], "achieved": top["achieved_tflops"],
            "peak": peak, "unit": "TFLOP/s", "frac": top["compute_frac"], "traffic": traffic,
            "alg_flops_per_launch": top["alg_flops_per_launch"],
            "frac_executed": top["compute_frac_executed"], "peak_source": top["compute_peak"]}


def roofline_e2e(phases, step_ms):
    """End-to-end roofline fraction: sum over kernels of max(F/peak, B/BW), over the measured
    step time."""
    bound = sum(ph.get("roof_ms_per_step", 0.0) for ph in phases)
    return {"bound_ms": bound, "step_ms": step_ms, "frac": bound / step_ms if step_ms else None}


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

def _sample_rows(L: int, n: int):
    """n query rows spread evenly over the sequence (first and last included)."""
    n = max(1, min(n, L))
    if n == 1:
        return [0]
    return sorted({round(i * (L - 1) / (n - 1)) for i in range(n)})


def _row_flops(w, rows):
    """Algorithmic flops the oracle's row functions perform for these rows: QK^T and PV of the
    forward, dP and dQ of the backward (4 flops per live score and head dimension); the
    scores recomputed for dQ are not counted."""
    return sum(8.0 * ((i + 1) if w["causal"] else w["L"]) * w["d"] for i in rows)


def _oracle_heads(w, heads: int):
    """Seconds the fp64 oracle takes for forward and for backward of `heads` whole heads."""
    from oracle import oracle
    from sequence_ring_self_b200.inputs import make_inputs

    x = make_inputs(1, heads, w["L"], w["d"], seed=w["seed"], dtype=w["dtype"])
    t = time.perf_counter()
    oracle.forward(x.q, x.k, x.v, w["causal"])
    t1 = time.perf_counter()
    oracle.backward(x.q, x.k, x.v, x.do, w["causal"])
    return t1 - t, time.perf_counter() - t1


_ROW_INPUTS = {}


def _oracle_rows(w, rows):
    """Seconds the fp64 oracle takes for the forward rows and the dQ rows of head (0, 0)."""
    from oracle import oracle
    from sequence_ring_self_b200.inputs import make_inputs

    key = (w["L"], w["d"], w["seed"], w["dtype"])
    if key not in _ROW_INPUTS:
        _ROW_INPUTS.clear()
        _ROW_INPUTS[key] = make_inputs(1, 1, w["L"], w["d"], seed=w["seed"], dtype=w["dtype"])
    x = _ROW_INPUTS[key]
    t = time.perf_counter()
    oracle.forward_rows(x.q, x.k, x.v, 0, 0, rows, w["causal"])
    oracle.backward_rows(x.q, x.k, x.v, x.do, 0, 0, rows, w["causal"])
    return time.perf_counter() - t


def oracle_plan(w, seconds: float):
    """How to sample the oracle so that one sample takes about `seconds`.

    Whole heads (forward + backward) when one head fits the time; otherwise evenly spread query
    rows of one head (forward rows and dQ rows). Returns (kind, count, threads, flops)."""
    from oracle import oracle

    oracle.build()
    threads = oracle.max_threads()
    # whole-head cost estimate: 12pd flops of one head at the rate of a small row probe
    probe = _sample_rows(w["L"], 2 * threads)
    dt = max(_oracle_rows(w, probe), 1e-6)
    rate = _row_flops(w, probe) / dt
    head_flops = 12.0 * live_entries(w["L"], w["causal"]) * w["d"]
    if head_flops / rate < 0.5 * seconds:
        t_f, t_b = _oracle_heads(w, 1)
        heads = 1
        while heads < w["B"] * w["H"]:
            h = heads + 1
            # the forward is parallel over rows (cost ~ heads * t_f), the backward over heads
            if h * t_f + math.ceil(h / threads) * t_b > seconds:
                break
            heads = h
        return "heads", heads, threads, head_flops * heads
    n = max(1, min(w["L"], int(seconds * rate / (8.0 * w["L"] * w["d"]))))
    rows = _sample_rows(w["L"], n)
    return "rows", len(rows), threads, _row_flops(w, rows)


def oracle_sample(w, seconds: float):
    """Time the oracle on a bounded sample: (algorithmic flops, seconds, description, threads)."""
    kind, count, threads, flops = oracle_plan(w, seconds)
    if kind == "heads":
        dt = sum(_oracle_heads(w, count))
        desc = f"fp64 oracle forward+backward of {count} of {w['B'] * w['H']} heads"
    else:
        dt = _oracle_rows(w, _sample_rows(w["L"], count))
        desc = (f"fp64 oracle forward and dQ of {count} evenly spaced query rows of one head "
                f"(QK^T, PV, dP, dQ flops of those rows counted; heads are independent and rows "
                f"cost alike)")
    return flops, dt, desc, threads


def run_reference(args, w):
    """The reference arm: the fp64 CPU oracle, as it stands, on bounded samples of the workload."""
    from sequence_ring_self_b200.dist import env_ranks

    rank, world, _ = env_ranks()
    if rank != 0:
        return 0
    steps, warmup = args.steps, args.warmup
    budget = args.ref_budget / max(1, steps + warmup)  # whole run within the budget
    kind, count, threads, flops_step = oracle_plan(w, budget)
    rows = _sample_rows(w["L"], count) if kind == "rows" else None
    times = []
    for i in range(warmup + steps):
        dt = sum(_oracle_heads(w, count)) if kind == "heads" else _oracle_rows(w, rows)
        if i >= warmup:
            times.append(dt)
    total = sum(times)
    value = flops_step * steps / total / 1e12
    what = (f"forward+backward of {count} of the {w['B'] * w['H']} heads" if kind == "heads" else
            f"forward and dQ of {count} evenly spaced query rows of one head")
    sample = f"fp64 oracle, {what} per step ({w['name']})"
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
        "tokens_per_s": value * 1e12 / step_flops(w) * w["B"] * w["L"],
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm

def measure_ffma(dev, reps: int = 5):
    """FP32 FMA throughput of this GPU (TFLOP/s), from the library's FMA probe kernel timed with
    CUDA events (best of `reps`)."""
    import ctypes

    import torch

    from sequence_ring_self_b200 import rsa

    lib = rsa.load_library()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    blocks, iters = sms * 8, 4096
    out = torch.empty(blocks, dtype=torch.float32, device=dev)
    s = torch.cuda.current_stream(dev)
    best = None
    for _ in range(reps + 1):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        rc = lib.rsa_probe_ffma(ctypes.c_void_p(out.data_ptr()), blocks, iters,
                                ctypes.c_void_p(s.cuda_stream))
        e1.record(s)
        if rc != rsa.RSA_OK:
            raise rsa.RSAError(rc, "rsa_probe_ffma")
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1)
        best = ms if best is None else min(best, ms)
    flops = lib.rsa_probe_ffma_flops_per_thread(iters) * blocks * 256
    return flops / (best / 1e3) / 1e12


# the slab kernels' traffic is almost all one direction: scores written, or scores read
SLAB_DIRECTION = {"qk_slab": "write", "pv_softmax": "read"}


def measure_hbm(dev, reps: int = 5):
    """HBM read-only and write-only streaming rates of this GPU (GB/s), from the library's probe
    kernels over a buffer far above the L2 size, timed with CUDA events (best of `reps`)."""
    import ctypes

    import torch

    from sequence_ring_self_b200 import rsa

    lib = rsa.load_library()
    free, _ = torch.cuda.mem_get_info(dev)
    nbytes = min(2 << 30, (free // 4) // (1 << 20) * (1 << 20))
    if nbytes < (512 << 20):
        return None  # too little free memory for a buffer well above L2
    buf = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    blocks = sms * 8
    out = torch.empty(blocks, dtype=torch.int32, device=dev)
    s = torch.cuda.current_stream(dev)
    rates = {}
    for name, write in (("write", 1), ("read", 0)):
        best = None
        for _ in range(reps + 1):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            rc = lib.rsa_probe_hbm(ctypes.c_void_p(buf.data_ptr()), nbytes, write, blocks,
                                   ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(s.cuda_stream))
            e1.record(s)
            if rc != rsa.RSA_OK:
                raise rsa.RSAError(rc, "rsa_probe_hbm")
            torch.cuda.synchronize(dev)
            ms = e0.elapsed_time(e1)
            best = ms if best is None else min(best, ms)
        rates[name] = nbytes / (best / 1e3) / 1e9
    del buf, out
    return rates


def annotate_directions(phases, hbm_probe):
    """Each slab kernel's achieved GB/s against the probe rate of its traffic's direction."""
    if not hbm_probe:
        return
    for ph in phases:
        direction = SLAB_DIRECTION.get(ph["kernel"])
        if direction and "achieved_gbs" in ph:
            ph["hbm_frac_of_" + direction + "_probe"] = ph["achieved_gbs"] / hbm_probe[direction]


class Workload:
    """Device tensors, workspaces and the step function of one workload on one GPU."""

    def __init__(self, w, dev, seed_offset: int, ws_budget: int, forward: str):
        import torch

        from sequence_ring_self_b200 import rsa
        from sequence_ring_self_b200.inputs import make_inputs

        self.w, self.dev, self.forward = w, dev, forward
        B, H, L, d, N, causal = w["B"], w["H"], w["L"], w["d"], w["N"], w["causal"]
        tdt = torch.float32 if w["dtype"] == "f32" else torch.bfloat16
        self.x = make_inputs(B, H, L, d, seed=w["seed"] + seed_offset, dtype=w["dtype"])
        self.q, self.k, self.v, self.do = (self.x.torch(n, dev) for n in ("q", "k", "v", "do"))
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((B, H, L), dtype=torch.float32, device=dev)
        self.dq, self.dk, self.dv = (torch.empty_like(self.q) for _ in range(3))
        self.nf = rsa.workspace_size(B, H, L, d, N, causal, tdt, False, ws_budget)
        self.nb = rsa.workspace_size(B, H, L, d, N, causal, tdt, True, ws_budget)
        self.ws_f = torch.empty(self.nf, dtype=torch.uint8, device=dev)
        self.ws_b = torch.empty(self.nb, dtype=torch.uint8, device=dev)
        self.plan_f = rsa.plan_describe(B, H, L, d, N, causal, tdt, False, self.nf)
        self.plan_b = rsa.plan_describe(B, H, L, d, N, causal, tdt, True, self.nb)

    def step(self):
        from sequence_ring_self_b200 import rsa

        w = self.w
        if self.forward == "recompute":
            rsa.forward_recompute(self.q, self.k, self.v, w["N"], w["causal"], out=self.o, lse=self.lse)
        else:
            rsa.forward(self.q, self.k, self.v, w["N"], w["causal"], workspace=self.ws_f,
                        out=self.o, lse=self.lse)
        rsa.backward(self.q, self.k, self.v, self.o, self.do, self.lse, w["N"], w["causal"],
                     workspace=self.ws_b, dq=self.dq, dk=self.dk, dv=self.dv)


def timed_steps(step, n, flush, guard_cycles, kernel_events):
    """n steps, each preceded (outside its events) by the L2 flush and a short GPU spin that
    keeps the launch queue ahead of the GPU; returns the per-step device times (ms)."""
    import torch

    from sequence_ring_self_b200 import rsa

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


def warm_up(step, n, flush):
    """n untimed steps; returns the host time to enqueue one step (median, seconds)."""
    import torch

    from sequence_ring_self_b200 import rsa

    host = []
    for _ in range(n):
        flush.zero_()
        t = time.perf_counter()
        step()
        host.append(time.perf_counter() - t)
        torch.cuda.synchronize()
    if rsa.last_device_status() != rsa.RSA_OK:
        raise RuntimeError("a kernel reported a timeout during warm-up")
    return statistics.median(host)


def compute_peaks(peaks, clocks, ffma_tflops):
    """compute_peak(kind) for the phases: bf16 tensor kernels against the measured bf16 GEMM
    rate (the sustained one when the clock record shows the power cap, else the burst one),
    fp32 kernels against the FMA probe's rate measured in the same run."""
    capped = "sw_power_cap" in (clocks.get("reasons") or [])
    bf16 = peaks["bf16_tflops_sustained"] if capped else peaks["bf16_tflops"]
    bf16_label = (f"{peaks['source']} bf16 dense "
                  f"{'sustained (power cap seen)' if capped else 'burst'}: {bf16:.0f} TFLOP/s")

    def fn(kind):
        if kind in F32_KINDS:
            return ffma_tflops, f"FP32 FMA probe, this run: {ffma_tflops:.1f} TFLOP/s"
        return bf16, bf16_label

    return fn


def run_gpu(args, w):
    import torch

    from sequence_ring_self_b200 import build, dist, rsa

    rank, world, local = dist.env_ranks()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist.init("nccl", device=dev)
    build.build()
    rsa.load_library()

    wl = Workload(w, dev, 1000 * rank, args.ws_budget, args.forward)
    B, L, N, causal = w["B"], w["L"], w["N"], w["causal"]
    flush = torch.empty(max(1, args.flush_mib) << 20, dtype=torch.uint8, device=dev)
    host_s = warm_up(wl.step, max(3, args.warmup), flush)
    # GPU spin before each timed step: a few times the host's enqueue time (capped at 4 ms)
    guard_cycles = int(min(8e6, max(2e5, 4.0 * host_s * 2.0e9)))

    clocks = ClockSampler(local)
    clocks.start()
    K = args.steps
    # the timed region: K steps, no per-kernel events (kernels overlap their prologues with the
    # previous kernel's tail through programmatic dependent launch)
    dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    step_ms = timed_steps(wl.step, K, flush, guard_cycles, False)
    t1 = time.perf_counter()
    dist.barrier()
    clocks.stop()
    if rsa.last_device_status() != rsa.RSA_OK:
        raise RuntimeError("a kernel reported a timeout")
    # per-kernel durations: the same steps again with every library kernel bracketed by CUDA
    # events on its stream (the events themselves add about 5 us per kernel to a step)
    kp = max(3, min(K, args.profile_steps))
    prof_step_ms = timed_steps(wl.step, kp, flush, guard_cycles, not args.no_kernel_events)
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
        x = wl.x
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
               "unit": "TFLOP/s", "h2d_bytes_per_step": 4 * wl.q.numel() * wl.q.element_size(),
               "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in res.values()),
               "ms_per_step": e2e_slowest / K}

    peaks = load_peaks()
    ffma = measure_ffma(dev)
    hbm_probe = measure_hbm(dev)
    clock_rec = clocks.summary(t0, t1)
    phases = phases_from_profile(prof, kp, w, peaks, compute_peaks(peaks, clock_rec, ffma))
    annotate_directions(phases, hbm_probe)
    if not phases:
        phases = [{"kernel": "none (no per-kernel events)"}]
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if os.path.exists(tpath):
        try:
            from sequence_ring_self_b200.build import source_digest

            t = json.load(open(tpath))
            ent = t.get("kernels", {}).get(phases[0]["kernel"])
            if ent and t.get("workload") == w["name"] and t.get("source_digest") == source_digest():
                traffic = ent["dram_bytes_per_launch"]
        except Exception:
            traffic = None
    roofline = roofline_of(phases, peaks, traffic)
    step_ms_avg = slowest_ms / K

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": step_ms_avg, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w["dtype"], "data": "synthetic",
        "config": {"workload": w["name"], "global_batch": B * world, "seq_len": L, "heads": w["H"],
                   "head_dim": w["d"], "chunks": N, "causal": causal,
                   "parallelism": f"dp{world} (independent batches per GPU)",
                   "l2": f"flushed between steps ({args.flush_mib} MiB write)",
                   "forward": args.forward,
                   "slab_groups": {"forward": wl.plan_f["groups"], "backward": wl.plan_b["groups"],
                                   "workspace_bytes": [wl.nf, wl.nb]}},
        "tokens_per_s": tokens_s,
        "step_ms_median": statistics.median(step_ms),
        "step_ms_min": min(step_ms),
        "e2e": e2e,
        "gpu_launches": int(round(sum(n for _, n in prof.values()) / kp * K)),
        "profiled_pass": {"steps": kp, "ms_per_step_with_kernel_events": statistics.median(prof_step_ms)},
        "roofline": roofline,
        "roofline_e2e": roofline_e2e(phases, step_ms_avg),
        "phases": phases,
        "clocks": clock_rec,
        "peaks": dict(peaks, ffma_tflops_this_run=ffma,
                      hbm_read_gbs_this_run=hbm_probe and hbm_probe["read"],
                      hbm_write_gbs_this_run=hbm_probe and hbm_probe["write"]),
    }
    if world == 1 and not args.no_cpu_baseline:
        fl, sec, desc, threads = oracle_sample(w, args.cpu_seconds)
        line["cpu_baseline"] = {"value": fl / sec / 1e12, "unit": "TFLOP/s", "cores": threads,
                                "kind": "oracle", "sample": f"{desc}, {sec:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.finish()
    return 0


def run_sweep(args):
    """The sweep configuration (B=1, H=16, d=64, bf16; L x N x causal): one JSON line per point
    with the step time, TFLOP/s, tokens/s, the end-to-end roofline fraction and the dominant
    kernel's roofline fraction (extra lines; the contract line is the default workload's)."""
    import torch

    from sequence_ring_self_b200 import build, rsa

    build.build()
    rsa.load_library()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    peaks = load_peaks()
    ffma = measure_ffma(dev)
    cpeak = compute_peaks(peaks, {"reasons": []}, ffma)
    Ls = [int(x) for x in args.sweep_L.split(",")]
    Ns = [int(x) for x in args.sweep_N.split(",")]
    idx = 0
    for causal in (False, True):
        for L in Ls:
            for N in Ns:
                w = dict(B=1, H=16, L=L, d=64, N=N, causal=causal, seed=5 + idx, dtype="bf16",
                         name=f"sweep point B=1 H=16 L={L} d=64 N={N} bf16 "
                              f"{'causal' if causal else 'non-causal'}")
                idx += 1
                wl = Workload(w, dev, 0, args.ws_budget, args.forward)
                host_s = warm_up(wl.step, 3, flush)
                guard = int(min(8e6, max(2e5, 4.0 * host_s * 2.0e9)))
                times = timed_steps(wl.step, args.sweep_steps, flush, guard, False)
                timed_steps(wl.step, 3, flush, guard, True)
                prof = rsa.profile_read()
                rsa.profile_enable(False)
                ms = statistics.median(times)
                phases = phases_from_profile(prof, 3, w, peaks, cpeak)
                top = roofline_of(phases, peaks, None)
                print(json.dumps({
                    "sweep_point": {"L": L, "N": N, "causal": causal}, "ms_per_step": ms,
                    "tflops": step_flops(w) / ms / 1e9, "tokens_per_s": L / ms * 1e3,
                    "slab_groups": wl.plan_f["groups"],
                    "roofline": {k: top[k] for k in ("kernel", "bound", "achieved", "peak", "unit", "frac")},
                    "roofline_e2e": roofline_e2e(phases, ms)["frac"],
                    "kernels": {ph["kernel"]: {"avg_us": ph["avg_us"], "bound": ph.get("bound"),
                                               "frac": (ph["hbm_frac"] if ph.get("bound") == "hbm"
                                                        else ph.get("compute_frac"))}
                                for ph in phases}}), flush=True)
                del wl
                torch.cuda.empty_cache()
    return 0


def run_ring(args, w):
    """The ring across GPUs, emulated on one GPU: every rank's per-rank kernels (rsa_sp_*, the
    library's sequence-parallel steps) run in lockstep on this device and the exchange between
    neighbours is a device copy (no kernel waits for another rank's). One JSON line with the
    emulated step's time (all P ranks' work, the same 12pd flops as the single-device step),
    the per-rank share, each kernel's roofline fraction, and the bytes per rank that NCCL would
    move between GPUs (not timed here: every GPU run available has one GPU). Not the contract
    line: an extra measurement of the ring's kernels."""
    import torch

    from sequence_ring_self_b200 import build, ring, rsa
    from sequence_ring_self_b200.inputs import make_inputs

    build.build()
    rsa.load_library()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    P = args.ring
    B, H, L, d, causal = w["B"], w["H"], w["L"], w["d"], w["causal"]
    if L % P or (L // P) % 128:
        raise SystemExit(f"the ring needs L / P to be a multiple of 128 (L={L}, P={P})")
    c = L // P
    x = make_inputs(B, H, L, d, seed=w["seed"], dtype="bf16")
    q, k, v, do = (x.torch(n, dev) for n in ("q", "k", "v", "do"))
    comp = ring.Kernels()
    chunk = lambda t, r: t[:, :, r * c:(r + 1) * c].contiguous()
    states = [ring.RankState(q=chunk(q, r), kfull=ring.full_buffer(chunk(k, r), r, P),
                             vfull=ring.full_buffer(chunk(v, r), r, P), causal=causal, do=chunk(do, r))
              for r in range(P)]

    def step():
        rings = []
        rings.extend(ring.LocalRing(r, states, rings) for r in range(P))
        ring.run_lockstep([ring.forward_steps(states[r], rings[r], comp) for r in range(P)])
        ring.run_lockstep([ring.backward_steps(states[r], rings[r], comp) for r in range(P)])

    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    host_s = warm_up(step, max(3, args.warmup), flush)
    guard = int(min(8e6, max(2e5, 4.0 * host_s * 2.0e9)))
    times = timed_steps(step, args.steps, flush, guard, False)
    kp = max(3, min(args.steps, args.profile_steps))
    timed_steps(step, kp, flush, guard, True)
    prof = rsa.profile_read()
    rsa.profile_enable(False)
    if rsa.last_device_status() != rsa.RSA_OK:
        raise RuntimeError("a kernel reported a timeout")
    ms = sum(times) / len(times)
    peaks = load_peaks()
    phases = phases_from_profile({n: v for n, v in prof.items() if n != "sp_accumulate"}, kp, w, peaks,
                                 compute_peaks(peaks, {"reasons": []}, measure_ffma(dev)))
    acc = prof.get("sp_accumulate")
    acc_ms = acc[0] / kp if acc else 0.0
    kernel_ms = sum(ph["ms_per_step"] for ph in phases) + acc_ms
    chunk_bf16 = B * H * c * d * 2
    line = {
        "ring_emulated": {"ranks": P, "chunk_rows": c}, "workload": w["name"],
        # the device time of every rank's kernels in one step (CUDA events per kernel): one
        # GPU of a real P-GPU ring runs a P-th of it
        "kernel_ms_per_step_all_ranks": kernel_ms, "kernel_ms_per_rank": kernel_ms / P,
        "kernel_tflops_one_gpu": step_flops(w) / kernel_ms / 1e9,
        # wall time of the emulated step on one GPU: host-bound when the per-rank problems are
        # small (P * P steps of launches from one Python thread)
        "wall_ms_per_step_all_ranks": ms,
        "nccl_bytes_per_rank_step": {"forward_kv_chunks": 2 * (P - 1) * chunk_bf16,
                                     "backward_dkdv_fp32_accumulators": 2 * (P - 1) * 2 * chunk_bf16},
        "exchange": "device copies on one GPU (NCCL send/recv between GPUs: not measured here)",
        "kernels": {ph["kernel"]: {"ms_per_step": ph["ms_per_step"], "launches_per_step": ph["launches_per_step"],
                                   "bound": ph.get("bound"),
                                   "frac": ph["hbm_frac"] if ph.get("bound") == "hbm" else ph.get("compute_frac")}
                    for ph in phases},
        "sp_accumulate_ms_per_step": acc_ms,
        "roofline_e2e_of_kernel_time": roofline_e2e(phases, kernel_ms)["frac"],
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + ["sweep"], default=DEFAULT_WORKLOAD)
    ap.add_argument("--forward", choices=["slab", "recompute"], default="slab",
                    help="slab: the method's forward (score slab in HBM, the headline path); "
                         "recompute: the slab-free two-pass forward (bf16)")
    ap.add_argument("--sweep-L", default="1024,2048,4096,8192,16384,32768")
    ap.add_argument("--sweep-N", default="1,2,4,8,16")
    ap.add_argument("--sweep-steps", type=int, default=5)
    ap.add_argument("--ws-budget", type=int, default=0, help="workspace budget in bytes (0: default)")
    ap.add_argument("--cpu-seconds", type=float, default=20.0,
                    help="CPU seconds of the oracle sample reported as cpu_baseline")
    ap.add_argument("--ref-budget", type=float, default=120.0,
                    help="seconds the whole --impl reference run should take")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end timing")
    ap.add_argument("--no-kernel-events", action="store_true",
                    help="skip the per-kernel profiled pass (no phases / roofline)")
    ap.add_argument("--profile-steps", type=int, default=10,
                    help="steps of the per-kernel profiled pass that follows the timed region")
    ap.add_argument("--flush-mib", type=int, default=512, help="L2 flush buffer (MiB) written before each step")
    ap.add_argument("--shape", default=None,
                    help="B,H,L,d,N,causal: a bf16 workload of this shape instead of --workload")
    ap.add_argument("--ring", type=int, default=0,
                    help="emulate the ring across this many GPUs on one GPU (extra line)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.workload == "sweep":
        return run_sweep(args)
    w = WORKLOADS[args.workload]
    if args.shape:
        B, H, L, d, N, causal = (int(x) for x in args.shape.split(","))
        w = dict(B=B, H=H, L=L, d=d, N=N, causal=bool(causal), seed=4, dtype="bf16",
                 name=f"RSA fwd+bwd: B={B} H={H} L={L} d={d} N={N} bf16 "
                      f"{'causal' if causal else 'non-causal'}")
    if args.impl == "reference":
        return run_reference(args, w)
    if args.ring:
        return run_ring(args, w)
    if args.forward == "recompute" and w["dtype"] != "bf16":
        ap.error("--forward recompute is bf16 only")
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
