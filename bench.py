"""Benchmark of the KDA operator on B200: prefill tokens/s and decode steps/s.

One bench step = one chunkwise prefill (kda_chunk_fwd) over the long-context
workload: B=1, H=32, T=65536, d_k=d_v=128, bf16 inputs, fp32 state, N(0,0.1)
initial state, log_alpha = logsigmoid(N(4,1)).  The decode workload (B=256,
H=32, d=128, fp32 state updated in place, 1024 distinct tokens) is timed in
the same run and reported in the "decode" object.

Usage:
    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {kda,reference}]
For N > 1 launch one process per GPU with torch.distributed.run; every rank
runs its own copy of the workload (weak scaling: the (sequence, head) units are
independent, no data-path collective), the timed region is bracketed by a
barrier and cuda synchronize, and the step time is the max over ranks.

`--impl reference` times the fp64 CPU oracle (the reference arm: there is no
installable reference implementation) on a bounded sample of the same
workload on the host cores, rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s & % tensor roofline; decode steps/s & % HBM GB/s"
PREFILL_WORKLOAD = "long_bf16"
DECODE_WORKLOAD = "decode_bf16"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


LIB_SOURCES = ("gated_delta_rule_86_b200/csrc", "include")


# The csrc files that a profiled kernel's device code and launch come from (the kernel's header and
# the headers it includes): its DRAM traffic depends on these alone.
KERNEL_SOURCES = {
    "kda_chunk_tc_kernel": ("kda_chunk_tc.cuh", "kda_common.cuh", "kda_recurrent.cuh", "tc_utils.cuh"),
    "kda_decode_kernel": ("kda_decode.cuh", "kda_common.cuh"),
    "kda_bwd_kernel": ("kda_backward.cuh", "kda_common.cuh"),
}


def build_hash(kernel=None):
    """Hash of the library's sources (csrc/*.cu, *.cuh, include/*.h), or of one kernel's sources
    (KERNEL_SOURCES): names the build that a profile summary was captured on."""
    import glob
    import hashlib
    h = hashlib.sha256()
    files = []
    if kernel is not None:
        files = [os.path.join(ROOT, LIB_SOURCES[0], f) for f in KERNEL_SOURCES[kernel]]
    else:
        for d in LIB_SOURCES:
            for ext in ("*.cu", "*.cuh", "*.h"):
                files += glob.glob(os.path.join(ROOT, d, ext))
    for f in sorted(files):
        h.update(os.path.relpath(f, ROOT).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_record(kernel, workload):
    """The DRAM traffic record of `kernel` on `workload` from profiles/*.md (a line
    `traffic-record: {json}` written next to the ncu summary), if it was captured on the kernel's
    current sources (build_hash(kernel)); else None.  Keys: build, kernel, workload, dram_bytes,
    units."""
    import glob
    want = build_hash(kernel)
    for f in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        with open(f) as fh:
            for line in fh:
                if line.startswith("traffic-record:"):
                    try:
                        rec = json.loads(line.split(":", 1)[1])
                    except ValueError:
                        continue
                    if rec.get("kernel") == kernel and rec.get("workload") == workload and rec.get("build") == want:
                        rec["file"] = os.path.relpath(f, ROOT)
                        return rec
    return None


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(PEAKS_FALLBACK), "fallback"


# ---- algorithmic work per unit (d = 128, C = 64) ---------------------------------------------------

def prefill_alg_bytes(tokens_heads, heads_total, dk=128, dv=128, in_bytes=2, out_bytes=4):
    """q, k, log_alpha (d_k each), v (d_v), beta, out (d_v) per token-head, plus the
    fp32 state read and written once per sequence-head."""
    per_th = (3 * dk + dv + 1) * in_bytes + dv * out_bytes
    return tokens_heads * per_th + heads_total * 2 * dk * dv * 4


def prefill_alg_flops(tokens_heads, dk=128, dv=128, C=64):
    """Triangular products counted as triangular: A, P, W, U, P U~ give 5 C d; W S, Q S,
    Kd^T U~ give 6 d^2 (d_k = d_v = d) per token-head."""
    return tokens_heads * (5 * C * dk + 2 * dk * dv * 3)


def decode_alg_bytes(heads, dk=128, dv=128, in_bytes=2, out_bytes=4):
    return heads * (2 * dk * dv * 4 + (3 * dk + dv + 1) * in_bytes + dv * out_bytes)


# ---- clocks -----------------------------------------------------------------------------------------

class ClockSampler:
    """SM clock, power and clock-event reasons sampled while the timed region runs: through NVML
    (read-only queries) every 5 ms from a background thread, else through `nvidia-smi -lms 200`.
    `nvml` may be given (a module with the pynvml names) for tests."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))
    PERIOD_S = 0.005

    def __init__(self, device_index, nvml=None):
        self.proc = None
        self.path = None
        self.device_index = device_index
        self.nvml = nvml
        self.rows = None       # NVML samples: (sm_mhz, max_mhz, power_w, reason bits)
        self.thread = None

    def _uuid(self):
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.device_index).uuid)
            return uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            return None

    def _start_nvml(self):
        nv = self.nvml
        if nv is None:
            try:
                import pynvml as nv
            except ImportError:
                return False
        try:
            nv.nvmlInit()
            uuid = self._uuid()
            handle = nv.nvmlDeviceGetHandleByUUID(uuid) if uuid else nv.nvmlDeviceGetHandleByIndex(self.device_index)
            max_mhz = nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM)
        except Exception:
            return False
        reasons_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        self.rows = []
        self.stop = threading.Event()

        def run():
            while True:
                try:
                    self.rows.append((nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM), max_mhz,
                                      nv.nvmlDeviceGetPowerUsage(handle) / 1000.0, reasons_fn(handle)))
                except Exception:
                    pass
                if self.stop.wait(self.PERIOD_S):
                    return

        self.nv = nv
        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()
        return True

    def __enter__(self):
        if self._start_nvml():
            return self
        ident = self._uuid() or str(self.device_index)
        fd, self.path = tempfile.mkstemp(prefix="kda_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", ident], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            try:
                self.nv.nvmlShutdown()
            except Exception:
                pass
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.rows is not None:
            if not self.rows:
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "source": "nvml"}
            bits = 0
            for r in self.rows:
                bits |= int(r[3])
            return {"sm_mhz": statistics.median(r[0] for r in self.rows), "sm_max_mhz": max(r[1] for r in self.rows),
                    "reasons": sorted(n for n, b in self.REASONS if bits & b), "samples": len(self.rows),
                    "power_w_max": max(r[2] for r in self.rows), "source": "nvml, every 5 ms"}
        if self.proc is None or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max((num(r[3]) or 0.0) for r in rows), "source": "nvidia-smi, every 200 ms"}


# ---- distributed plumbing ---------------------------------------------------------------------------

def dist_setup(n_gpus):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}; launch with torch.distributed.run")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world, device="cuda"):
    import torch
    if world > 1:
        torch.distributed.barrier()
    if device == "cuda":
        torch.cuda.synchronize()


def max_over_ranks(x, world, device="cuda"):
    """Max of a per-rank scalar (the step time) over all ranks; every rank gets it."""
    import torch
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank, world, ms_step_max):
    """Whole-job throughput: units processed by all ranks / the slowest rank's step time."""
    return world * units_per_rank / (ms_step_max * 1e-3)


# ---- the reference arm: the fp64 oracle on the host ----------------------------------------------------

def time_oracle(workload, seed_offset=0, target_s=10.0, max_tokens=None):
    """Oracle tokens/s on the first T_s tokens of the prefill workload (all heads),
    doubling T_s until one run takes >= target_s.  Returns (tokens/s, sample text, threads)."""
    import numpy as np
    import torch

    import oracle
    from gated_delta_rule_86_b200 import inputs
    w = inputs.WORKLOADS[workload]
    threads = os.cpu_count() or 1
    T_s = 256
    while True:
        x = inputs.make_prefill(w, device="cpu", T=T_s, seed=inputs.BASE_SEED + w.wid + seed_offset)
        args = [x[n].float().numpy().astype(np.float64) for n in ("q", "k", "v", "log_alpha", "beta")]
        s0 = None if x["init_state"] is None else x["init_state"].numpy().astype(np.float64)
        t0 = time.perf_counter()
        oracle.recurrent(*args, init_state=s0, nthreads=threads)
        dt = time.perf_counter() - t0
        if dt >= target_s or T_s >= (max_tokens or w.T):
            break
        T_s = min(T_s * 2, max_tokens or w.T)
    del torch
    tok = w.B * T_s
    sample = f"first {T_s} of {w.T} tokens, all {w.H} heads, B={w.B} ({tok * w.H} token-heads), fp64 C oracle"
    return tok / dt, sample, threads, dt


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from gated_delta_rule_86_b200 import inputs
    w = inputs.WORKLOADS[PREFILL_WORKLOAD]
    per_step = []
    sample = threads = None
    for i in range(args.warmup + args.steps):
        tps, sample, threads, dt = time_oracle(PREFILL_WORKLOAD, seed_offset=i, target_s=args.ref_seconds)
        if i >= args.warmup:
            per_step.append(tps)
    value = statistics.median(per_step)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": w.B * w.T / value * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": PREFILL_WORKLOAD, "B": w.B, "T": w.T, "H": w.H, "d_k": w.dk, "d_v": w.dv,
                       "chunk": w.chunk},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---- the kda arm ----------------------------------------------------------------------------------------

def event_time_ms(fn, n):
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(n):
        fn(i)
    e1.record()
    e1.synchronize()
    return e0.elapsed_time(e1)


def flushed_time_ms(fn, n, flush):
    """Sum of n per-call CUDA-event times, with `flush` (a write of a buffer larger than L2)
    before each call and outside its timed interval."""
    import torch
    total = 0.0
    for i in range(n):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn(i)
        e1.record()
        e1.synchronize()
        total += e0.elapsed_time(e1)
    return total


def timed_steps(fn, args, world, flush=None):
    """Warm-up, then the device time of args.steps calls between barriers; the max over ranks of
    the per-call time in ms."""
    for _ in range(args.warmup):
        fn(0)
    barrier(world)
    ms = event_time_ms(fn, args.steps) if flush is None else flushed_time_ms(fn, args.steps, flush)
    barrier(world)
    return max_over_ranks(ms / args.steps, world)


def hbm_roofline(alg_bytes, ms, hbm_peak, kernel="kda_chunk_tc_kernel", traffic=None):
    gbs = alg_bytes / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
            "traffic": traffic, "kernel": kernel, "alg_bytes_per_launch": alg_bytes}


def prefill_block(args, world, x, hbm_peak, entry="kda_chunk_fwd", out_dtype=None, flush=None, label=None, chunk=64):
    """Time one prefill entry point on the inputs x (a make_prefill dict on the GPU)."""
    import torch

    import gated_delta_rule_86_b200 as kda
    fn = getattr(kda, entry)
    out_dtype = out_dtype or torch.float32
    a = [x[n] for n in ("q", "k", "v", "log_alpha", "beta")]
    B, T, H, dk = a[0].shape
    dv = a[2].shape[-1]
    N = B if x["cu_seqlens"] is None else x["cu_seqlens"].numel() - 1

    def step(_i):
        return fn(*a, initial_state=x["init_state"], cu_seqlens=x["cu_seqlens"], out_dtype=out_dtype, chunk_size=chunk)

    ms = timed_steps(step, args, world, flush)
    tokens = B * T
    alg = prefill_alg_bytes(tokens * H, N * H, dk, dv, out_bytes=4 if out_dtype == torch.float32 else 2)
    w = x["workload"]
    return {"entry": entry, "workload": label or w.name, "B": B, "T": T, "H": H, "N": N, "d_k": dk, "d_v": dv,
            "chunk": chunk,
            "out_dtype": "f32" if out_dtype == torch.float32 else "bf16", "ms_per_step": ms,
            "tokens_per_s": world * tokens / (ms * 1e-3), "roofline": hbm_roofline(alg, ms, hbm_peak),
            "l2": "flushed before each call" if flush is not None else "inputs larger than L2"}


def gdn_prefill_block(args, world, a, s0, tokens, token_heads, hbm_peak):
    """Time gdn_chunk_fwd on the bench workload's q, k, v, beta with the first key channel of its
    log_alpha as the per-head gate.  Algorithmic bytes: those of the KDA prefill less the
    per-channel gate (254 B per token-head)."""
    from gated_delta_rule_86_b200 import gdn_chunk_fwd
    log_g = a[3][..., 0].contiguous()

    def step(_i):
        return gdn_chunk_fwd(a[0], a[1], a[2], log_g, a[4], initial_state=s0)

    ms_step = timed_steps(step, args, world)
    heads = a[0].shape[0] * a[0].shape[2]
    alg = prefill_alg_bytes(token_heads, heads) - token_heads * (a[3].shape[-1] - 1) * 2
    return {"entry": "gdn_chunk_fwd", "gate": "log_g [B,T,H] = the first key channel of the workload's log_alpha",
            "ms_per_step": ms_step, "tokens_per_s": world * tokens / (ms_step * 1e-3),
            "roofline": hbm_roofline(alg, ms_step, hbm_peak)}


def bwd_alg_flops(token_heads, dk=128, dv=128):
    """Algorithmic flops of the gradient per token-head: the adjoint step (dS += q do^T, dq, du, dk's two
    terms, dS', dlog_alpha, dS_prev: 15 d_k d_v) plus the forward step it needs (S', w, S: 5 d_k d_v)."""
    return token_heads * 20 * dk * dv


FP32_PEAK_NOTE = "148 SMs x 128 fp32 FMA/clk x 2 flop x 1.965 GHz = 74.4 TFLOP/s (nominal CUDA-core peak)"
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def backward_block(args, world):
    """kda_chunk_bwd on the shape of the 4K prefill workload (B=2, H=16, T=4096, d=128)."""
    import torch

    from gated_delta_rule_86_b200 import inputs, kda_chunk_bwd
    w = inputs.WORKLOADS["prefill_bf16"]
    x = inputs.make_prefill(w, device="cuda", init_state=True)
    g = torch.Generator(device="cuda").manual_seed(5)
    d_out = torch.randn(x["v"].shape, generator=g, device="cuda")
    a = [x[n] for n in ("q", "k", "v", "log_alpha", "beta")]

    def step(_i, chunk=64):
        return kda_chunk_bwd(*a, d_out, initial_state=x["init_state"], chunk_size=chunk)

    ms = timed_steps(step, args, world)
    # the state before every token kept (chunk_size 0): no recompute pass, one state per token-head
    ms_all = timed_steps(lambda i: step(i, 0), args, world)
    th = w.B * w.T * w.H
    flops = bwd_alg_flops(th)
    tf = flops / (ms * 1e-3) / 1e12
    return {"entry": "kda_chunk_bwd", "workload": "prefill_bf16 shape (B2 H16 T4096 d128), N(0,0.1) initial state, "
            "N(0,1) upstream gradient", "chunk_size": 64, "ms_per_step": ms,
            "tokens_per_s": world * w.B * w.T / (ms * 1e-3),
            "roofline": {"bound": "alu", "achieved": tf, "peak": FP32_PEAK_TFLOPS, "unit": "TFLOP/s",
                         "frac": tf / FP32_PEAK_TFLOPS, "traffic": None, "kernel": "kda_bwd_kernel",
                         "alg_flops_per_launch": flops, "peak_source": FP32_PEAK_NOTE},
            "every_state": {"chunk_size": 0, "ms_per_step": ms_all, "tokens_per_s": world * w.B * w.T / (ms_all * 1e-3),
                            "workspace_bytes": w.H * w.B * w.T * w.dk * w.dv * 4,
                            "frac_of_fp32_peak": flops / (ms_all * 1e-3) / 1e12 / FP32_PEAK_TFLOPS}}


def oracle_single_thread(workload, T_s=4096):
    """Single-thread oracle tokens/s on one head of the workload (its first T_s tokens)."""
    import numpy as np

    import oracle
    from gated_delta_rule_86_b200 import inputs
    w = inputs.WORKLOADS[workload]
    x = inputs.make_prefill(w, device="cpu", T=T_s, H=1, B=1)
    args = [x[n].float().numpy().astype(np.float64) for n in ("q", "k", "v", "log_alpha", "beta")]
    s0 = None if x["init_state"] is None else x["init_state"].numpy().astype(np.float64)
    t0 = time.perf_counter()
    oracle.recurrent(*args, init_state=s0, nthreads=1)
    dt = time.perf_counter() - t0
    return T_s / dt, f"first {T_s} tokens of one head, 1 thread"


def run_kda(args):
    import torch

    from gated_delta_rule_86_b200 import device_error, inputs, kda_chunk_fwd, kda_chunk_fwd_fused, kda_decode_step
    rank, world, local = dist_setup(args.gpus)
    peaks, peaks_src = load_peaks()
    hbm_peak = peaks["hbm_gbs"]
    tc_peak_burst = peaks["bf16_tflops"]
    tc_peak_sust = peaks.get("bf16_tflops_sustained", tc_peak_burst)

    # ---------------- prefill (the headline: fp32 output, the accumulator precision) ----------------
    w = inputs.WORKLOADS[PREFILL_WORKLOAD]
    x = inputs.make_prefill(w, device="cuda", seed=inputs.BASE_SEED + w.wid + 1000 * rank)
    names = ("q", "k", "v", "log_alpha", "beta")
    a = [x[n] for n in names]
    s0 = x["init_state"]
    tokens = w.B * w.T
    token_heads = tokens * w.H

    def prefill_step(_i):
        return kda_chunk_fwd(*a, initial_state=s0)

    for _ in range(args.warmup):
        prefill_step(0)
    assert device_error() == 0, "device error during warm-up"
    with ClockSampler(local) as clk:
        barrier(world)
        ms = event_time_ms(prefill_step, args.steps)
        barrier(world)
    clocks = clk.summary()
    ms_step = max_over_ranks(ms / args.steps, world)
    value = weak_scaling_value(tokens, world, ms_step)
    alg_bytes = prefill_alg_bytes(token_heads, w.B * w.H)
    alg_flops = prefill_alg_flops(token_heads)
    dense_flops = token_heads * (12 * w.chunk * w.dk + 6 * w.dk * w.dv)
    # DRAM traffic per launch: from an ncu capture of this very kernel build (a traffic-record line in
    # profiles/, matched by the hash of the kernel's sources), scaled to this launch by the units it
    # processes; null when no capture of this build exists
    rec = traffic_record("kda_chunk_tc_kernel", PREFILL_WORKLOAD)
    traffic = None
    if rec is not None:
        traffic = rec["dram_bytes"] * token_heads / rec["units"]
    roofline = hbm_roofline(alg_bytes, ms_step, hbm_peak, traffic=traffic)
    roofline.update({
        "peak_source": f"{peaks_src} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
        if peaks_src == "measured" else "fallback 6650 GB/s",
        "traffic_source": None if rec is None else
        f"{rec['file']}: ncu dram__bytes_read.sum + dram__bytes_write.sum on {rec['units']} token-heads "
        f"(build {rec['build']}), scaled by token-heads",
        # the same capture's utilisation counters (tensor pipe, DRAM throughput; the 16K launch under ncu)
        "ncu_counters": None if rec is None else rec.get("ncu"),
        "build": build_hash("kda_chunk_tc_kernel"),
        "tensor": {"alg_flops_per_launch": alg_flops,
                   "achieved_tflops": alg_flops / (ms_step * 1e-3) / 1e12,
                   "frac_of_burst_peak": alg_flops / (ms_step * 1e-3) / 1e12 / tc_peak_burst,
                   "frac_of_sustained_peak": alg_flops / (ms_step * 1e-3) / 1e12 / tc_peak_sust,
                   "dense_tile_frac_of_burst_peak": dense_flops / (ms_step * 1e-3) / 1e12 / tc_peak_burst}})
    # the same launch with bf16 output: the byte count of the survey's roofline (1282 B per token-head)
    bf16_out = prefill_block(args, world, x, hbm_peak, out_dtype=torch.bfloat16)
    bf16_out["roofline"]["tensor_frac_of_burst_peak"] = alg_flops / (bf16_out["ms_per_step"] * 1e-3) / 1e12 / \
        tc_peak_burst
    # end to end through the public API from pinned host memory
    host = [t.cpu().pin_memory() for t in a]
    s0_h = s0.cpu().pin_memory()

    def e2e_step(_i):
        out, fs = kda_chunk_fwd(*host, initial_state=s0_h)
        return out

    e2e_step(0)
    barrier(world)
    e2e_ms = event_time_ms(e2e_step, max(1, args.steps // 2))
    barrier(world)
    e2e_ms = max_over_ranks(e2e_ms / max(1, args.steps // 2), world)
    h2d = sum(t.numel() * t.element_size() for t in host) + s0_h.numel() * 4
    d2h = token_heads * w.dv * 4 + w.B * w.H * w.dk * w.dv * 4
    # ---------------- Gated DeltaNet on the same workload (one log-decay per head and token) --------
    gdn = gdn_prefill_block(args, world, a, s0, tokens, token_heads, hbm_peak)
    del host, s0_h, x, a
    torch.cuda.empty_cache()

    # ---------------- the same prefill from the raw projections (fused prologue) ----------------
    xr = inputs.make_prefill(w, device="cuda", seed=inputs.BASE_SEED + w.wid + 1000 * rank, raw=True)
    fused = prefill_block(args, world, xr, hbm_peak, entry="kda_chunk_fwd_fused")
    fused["inputs"] = ("raw bf16 q, k (not normalised), g ~ N(4,1), b ~ N(0,1); normalisation, logsigmoid and "
                       "sigmoid inside the kernel's loads")
    # what a separate prologue pass would add: write and re-read the activated q, k, log_alpha and beta
    fused["separate_pass_bytes_saved"] = 2 * token_heads * (3 * w.dk * 2 + 2)
    del xr
    torch.cuda.empty_cache()

    # ---------------- chunk length ablation and key width 64 on the same workload ----------------
    ablation = {}
    xa = inputs.make_prefill(w, device="cuda", seed=inputs.BASE_SEED + w.wid + 1000 * rank)
    for C in (16, 32, 64):
        blk = prefill_block(args, world, dict(xa, workload=w), hbm_peak, chunk=C)
        ablation[f"C{C}"] = {"ms_per_step": blk["ms_per_step"], "tokens_per_s": blk["tokens_per_s"],
                             "chain_steps_per_head": -(-w.T // C), "roofline_frac": blk["roofline"]["frac"]}
    del xa
    x64 = inputs.make_prefill(w, device="cuda", seed=inputs.BASE_SEED + w.wid + 1000 * rank, dk=64)
    dk64 = prefill_block(args, world, x64, hbm_peak, label="long_bf16 with d_k = 64")
    del x64
    torch.cuda.empty_cache()
    bwd = backward_block(args, world)
    torch.cuda.empty_cache()

    # ---------------- the other prefill workloads ----------------
    others = {}
    flush_buf = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")

    def flush():
        flush_buf.zero_()

    for name, fl in (("prefill_bf16", flush), ("varlen_bf16", None)):
        wo = inputs.WORKLOADS[name]
        xo = inputs.make_prefill(wo, device="cuda", seed=inputs.BASE_SEED + wo.wid + 1000 * rank)
        others[name] = prefill_block(args, world, xo, hbm_peak, flush=fl)
        if wo.varlen:
            lens = (xo["cu_seqlens"][1:] - xo["cu_seqlens"][:-1]).tolist()
            others[name]["seq_lens"] = lens
            # the longest sequence's chain is the critical path of a longest-first schedule
            others[name]["longest_seq_tokens"] = max(lens)
        del xo
    del flush_buf
    torch.cuda.empty_cache()

    # ---------------- decode ----------------
    dw = inputs.WORKLOADS[DECODE_WORKLOAD]
    d = inputs.make_decode(dw, device="cuda", seed=inputs.BASE_SEED + dw.wid + 1000 * rank)
    state = d["state"]
    nsteps = dw.decode_steps

    def decode_step(i):
        return kda_decode_step(d["q"][i], d["k"][i], d["v"][i], d["log_alpha"][i], d["beta"][i], state)

    for i in range(3):
        decode_step(i)
    barrier(world)
    dms = event_time_ms(decode_step, nsteps)
    barrier(world)
    dms_step = max_over_ranks(dms / nsteps, world)
    heads = dw.B * dw.H
    d_bytes = decode_alg_bytes(heads)
    d_gbs = d_bytes / (dms_step * 1e-3) / 1e9
    drec = traffic_record("kda_decode_kernel", DECODE_WORKLOAD)   # units: head-steps of the capture
    d_traffic = None if drec is None else drec["dram_bytes"] * heads / drec["units"]
    decode = {"workload": DECODE_WORKLOAD, "B": dw.B, "H": dw.H, "d_k": dw.dk, "d_v": dw.dv, "steps": nsteps,
              "steps_per_s": world * 1e3 / dms_step, "tokens_per_s": world * dw.B * 1e3 / dms_step,
              "us_per_step": dms_step * 1e3,
              "roofline": {"bound": "hbm", "achieved": d_gbs, "peak": hbm_peak, "unit": "GB/s",
                           "frac": d_gbs / hbm_peak, "traffic": d_traffic, "kernel": "kda_decode_kernel",
                           "alg_bytes_per_launch": d_bytes,
                           "traffic_source": None if drec is None else
                           f"{drec['file']}: ncu dram__bytes_read.sum + dram__bytes_write.sum on {drec['units']} "
                           f"head-steps (build {drec['build']})",
                           "ncu_counters": None if drec is None else drec.get("ncu")}}
    # decode end to end: tokens from pinned host memory each step, output read back each step
    hq = [d[n][:64].cpu().pin_memory() for n in names]
    hout = torch.empty((dw.B, dw.H, dw.dv), dtype=torch.float32, pin_memory=True)

    def decode_e2e(i):
        kda_decode_step(hq[0][i], hq[1][i], hq[2][i], hq[3][i], hq[4][i], state, out=hout)

    barrier(world)
    de2e = event_time_ms(decode_e2e, 64) / 64
    barrier(world)
    de2e = max_over_ranks(de2e, world)
    decode["e2e"] = {"value": world * 1e3 / de2e, "unit": "steps/s",
                     "h2d_bytes_per_step": sum(t[0].numel() * t.element_size() for t in hq),
                     "d2h_bytes_per_step": hout.numel() * 4}
    assert device_error() == 0, "device error during the timed region"

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            tps, sample, threads, _ = time_oracle(PREFILL_WORKLOAD, target_s=args.ref_seconds)
            tps1, sample1 = oracle_single_thread(PREFILL_WORKLOAD)
            cpu = {"value": tps, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample,
                   "cpu_model": cpu_model(), "single_thread": {"value": tps1, "unit": "tokens/s (one head)",
                                                               "sample": sample1}}
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": PREFILL_WORKLOAD, "B": w.B, "T": w.T, "H": w.H, "d_k": w.dk, "d_v": w.dv,
                           "chunk": w.chunk, "io": "bf16 q/k/v/log_alpha/beta, fp32 out and state",
                           "init_state": "N(0,0.1)", "log_alpha": "logsigmoid(N(4,1))",
                           "l2": "inputs larger than L2 (2.1 GB of q/k/v/log_alpha per step)",
                           "parallelism": f"replicas x{world}"},
                "roofline": roofline, "cpu_baseline": cpu,
                "e2e": {"value": world * tokens / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                        "path": "kda_chunk_fwd on pinned host tensors: 8 token segments whose copies overlap the "
                                "kernels (copy streams for H2D and D2H)"},
                # per step: the schedule-table kernel and the chunk kernel
                "gpu_launches": 2 * args.steps, "clocks": clocks, "decode": decode, "bf16_output": bf16_out,
                "fused_prologue": fused, "gated_deltanet": gdn, "other_prefill_workloads": others,
                "chunk_length_ablation": ablation, "key_width_64": dk64, "backward": bwd}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def run_profile_case(args):
    """One small launch set for ncu: warm-up launches then the profiled ones.

    chunk:  kda_chunk_fwd on B=1, H=32, T=16384 (0.54 GB of bf16 inputs, above L2).
    decode: kda_decode_step on the full decode workload state (B=256, H=32, 512 MiB fp32).
    bwd:    kda_chunk_bwd on the backward block's shape (B=2, H=16, T=4096).
    """
    import torch

    from gated_delta_rule_86_b200 import inputs, kda_chunk_bwd, kda_chunk_fwd, kda_decode_step
    torch.cuda.set_device(0)
    if args.profile == "chunk":
        x = inputs.make_prefill(PREFILL_WORKLOAD, device="cuda", T=16384)
        a = [x[n] for n in ("q", "k", "v", "log_alpha", "beta")]
        for _ in range(3):
            kda_chunk_fwd(*a, initial_state=x["init_state"])
    elif args.profile == "bwd":
        x = inputs.make_prefill("prefill_bf16", device="cuda", init_state=True)
        g = torch.Generator(device="cuda").manual_seed(5)
        d_out = torch.randn(x["v"].shape, generator=g, device="cuda")
        a = [x[n] for n in ("q", "k", "v", "log_alpha", "beta")]
        for _ in range(3):
            kda_chunk_bwd(*a, d_out, initial_state=x["init_state"])
    else:
        d = inputs.make_decode(DECODE_WORKLOAD, device="cuda", steps=4)
        for i in range(4):
            kda_decode_step(d["q"][i], d["k"][i], d["v"][i], d["log_alpha"][i], d["beta"][i], d["state"])
    torch.cuda.synchronize()
    print(f"profile case {args.profile} done", flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["kda", "reference"], default="kda")
    ap.add_argument("--ref-seconds", type=float, default=10.0, help="target CPU seconds per oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=["chunk", "decode", "bwd"], default=None,
                    help="run a small fixed launch set for an ncu capture (no timing output)")
    args = ap.parse_args()
    if args.profile:
        return run_profile_case(args)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_kda(args)


if __name__ == "__main__":
    sys.exit(main())
