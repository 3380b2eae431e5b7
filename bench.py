#!/usr/bin/env python
"""Attention forward + backward throughput on B200.

One step = one pass of the whole path over one batch of synthetic input:
attn_fwd (O, LSE) followed by the three backward stages (prepare,
accumulate, finalize -> dQ, dK, dV), on the causal bf16 workload
B=2, H=32, N=8192, d=128 with Q, K, V, dO ~ N(0, 1) drawn from seed 1.

FLOPs follow the usual convention: forward 4*B*H*N^2*d, halved for causal;
backward 2.5x the forward.  `value` is whole-job TFLOP/s (all ranks), with
inputs resident in device memory; `e2e` is the same metric through the
public API with pinned host buffers, host<->device copies inside the timed
region.  Inputs (0.54 GB per step) exceed the 126 MB L2, so no flush is done
between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun each rank runs the same per-GPU workload (weak scaling, no
data-path collective); the time is the maximum over ranks.  `--impl
reference` times the float64 CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd/bwd TFLOP/s (bf16, causal, d=128, N=8K) and % of B200 BF16 peak"
UNIT = "TFLOP/s"
WORKLOAD = "causal_b2_h32_n8192_d128"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_BF16_TFLOPS = 2250.0
# The sources that decide the main kernels' DRAM traffic: the kernels and
# the host code that picks their launch order (scheduling groups).
KERNEL_SOURCES = ["io_aware_exact_33_b200/csrc/fwd_kernel.cuh",
                  "io_aware_exact_33_b200/csrc/bwd_kernel.cuh",
                  "io_aware_exact_33_b200/csrc/sm100.cuh",
                  "io_aware_exact_33_b200/csrc/attn_api.cu"]


# ---------------------------------------------------------------- accounting
def step_flops(w):
    """(forward, backward) FLOPs of one pass.  Without a window: the formula
    convention (4*B*H*Nq*Nk*d, halved for causal).  With a sliding window the
    halved-causal formula overstates the work, so the exact count of visible
    (query, key) pairs times 4*d is used instead.  Backward = 2.5 x forward;
    0 for forward-only workloads."""
    if w.window_left >= 0 or w.window_right >= 0:
        pairs = visible_pairs(w.seqlen_q, w.seqlen_k, w.causal, w.window_left, w.window_right)
        fwd = 4.0 * w.batch * w.nheads * pairs * w.headdim
    else:
        fwd = 4.0 * w.batch * w.nheads * w.seqlen_q * w.seqlen_k * w.headdim
        if w.causal:
            fwd /= 2.0
    return fwd, (2.5 * fwd if has_bwd(w) else 0.0)


def has_bwd(w):
    return "bwd" in w.passes


def exact_pair_flops(w):
    """(forward, backward) FLOPs counted on the exact visible (query, key)
    pairs (for a causal N x N problem N (N + 1) / 2 pairs, where the formula
    convention counts N^2 / 2)."""
    pairs = visible_pairs(w.seqlen_q, w.seqlen_k, w.causal, w.window_left, w.window_right)
    fwd = 4.0 * w.batch * w.nheads * pairs * w.headdim
    return fwd, (2.5 * fwd if has_bwd(w) else 0.0)


def environment(torch, dev):
    """GPU, driver and library versions for the result line (best effort)."""
    env = {}
    try:
        prop = torch.cuda.get_device_properties(dev)
        env.update(gpu=prop.name, sm_count=prop.multi_processor_count,
                   memory_gb=round(prop.total_memory / 1e9, 1))
    except Exception:
        pass
    env.update(torch=torch.__version__, cuda_runtime=torch.version.cuda)
    try:
        out = subprocess.run(["nvidia-smi", "--query-gpu=driver_version", "--format=csv,noheader",
                              "-i", str(dev.index or 0)], capture_output=True, text=True,
                             timeout=10).stdout.strip()
        if out:
            env["driver"] = out.splitlines()[0]
    except Exception:
        pass
    return env


def flops_convention(w):
    if w.window_left >= 0 or w.window_right >= 0:
        return "exact visible pairs x 4d (fwd), x 10d (bwd)"
    return "4*B*H*N^2*d, halved for causal (fwd); bwd = 2.5 x fwd"


def visible_pairs(nq, nk, causal, wl, wr, rows=None):
    """Exact count of visible (query, key) pairs for the given query rows."""
    off = nk - nq
    total = 0
    for i in (range(nq) if rows is None else rows):
        hi = nk - 1
        if causal:
            hi = min(hi, i + off)
        if wr >= 0:
            hi = min(hi, i + off + wr)
        lo = 0 if wl < 0 else max(0, i + off - wl)
        total += max(0, hi - lo + 1)
    return total


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"]))}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summary, or None if absent, taken on another workload or on different
    kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        ent = d.get(kernel)
        if not ent or ent.get("source_hash") != kernel_source_hash() or \
                ent.get("workload") != workload:
            return None
        return float(ent["bytes_per_launch"])
    except (OSError, ValueError, KeyError):
        return None


# ---------------------------------------------------------------- ranks
def world_info():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init_dist(backend, world):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def barrier(dist, device=None):
    if dist is not None:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(value, dist, device=None):
    """Maximum of a float over all ranks (identity on one rank)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region.

    The sampler runs every 20 ms from before the region starts (entering
    waits for its first sample, outside the region) and each sample carries
    its arrival time, so the summary keeps only the samples that arrived
    while the region ran (the nearest one if the region is shorter than the
    sampling period)."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    PERIOD_MS = 20

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.samples = []  # (monotonic time, line)
        self.t0 = self.t1 = None

    def _read(self):
        for ln in self.proc.stdout:
            if ln.strip():
                self.samples.append((time.monotonic(), ln))

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.PERIOD_MS)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
            deadline = time.monotonic() + 5.0
            while not self.samples and time.monotonic() < deadline:
                time.sleep(0.005)
        except OSError:
            self.proc = None
        self.t0 = time.monotonic()
        return self

    def __exit__(self, *exc):
        self.t1 = time.monotonic()
        if self.proc is not None:
            time.sleep(self.PERIOD_MS / 1000.0)  # the sample that closes the region
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
            self.reader.join(timeout=5)
        return False

    def summary(self):
        period = self.PERIOD_MS / 1000.0
        inside = [ln for t, ln in self.samples
                  if self.t0 is not None and self.t0 <= t <= self.t1 + period]
        if not inside and self.samples and self.t0 is not None:
            mid = 0.5 * (self.t0 + self.t1)
            inside = [min(self.samples, key=lambda x: abs(x[0] - mid))[1]]
        sm, smax, reasons = [], [], set()
        for ln in inside:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        window_ms = None if self.t0 is None else round((self.t1 - self.t0) * 1e3, 1)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "window_ms": window_ms}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm), "window_ms": window_ms}


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(w, rows, heads):
    """A bounded, exact slice of the workload for the float64 oracle: the last
    `rows` queries of `heads` heads of batch 0 against all keys.  With the
    bottom-right causal alignment these queries see exactly the keys they
    see in the full problem.  Returns (inputs, FLOPs by the 4d/10d convention)."""
    from attn_inputs import make_inputs
    q, k, v, do = make_inputs(w)
    hs = slice(0, heads)
    kv_heads = max(1, heads * w.nheads_kv // w.nheads)
    q_s = q[:1, -rows:, hs].contiguous()
    do_s = do[:1, -rows:, hs].contiguous()
    k_s = k[:1, :, :kv_heads].contiguous()
    v_s = v[:1, :, :kv_heads].contiguous()
    first = w.seqlen_q - rows
    pairs = visible_pairs(w.seqlen_q, w.seqlen_k, w.causal, w.window_left, w.window_right,
                          rows=range(first, w.seqlen_q))
    flops = pairs * heads * (4.0 + (10.0 if has_bwd(w) else 0.0)) * w.headdim
    return (q_s, k_s, v_s, do_s), flops


def oracle_step(w, inputs):
    import oracle
    q, k, v, do = inputs
    oracle.attention_fwd(q, k, v, w.scale, w.causal, w.window_left, w.window_right)
    if has_bwd(w):
        oracle.attention_bwd(q, k, v, do, w.scale, w.causal, w.window_left, w.window_right)


def cpu_baseline(w, target_s=12.0):
    import oracle
    oracle.build()
    threads = oracle.num_threads()
    heads = max(1, min(w.nheads, threads))
    probe_rows = 32
    inputs, flops = oracle_sample(w, probe_rows, heads)
    t0 = time.perf_counter()
    oracle_step(w, inputs)
    dt = time.perf_counter() - t0
    rows = int(min(w.seqlen_q, max(probe_rows, probe_rows * target_s / max(dt, 1e-3))))
    rows = max(probe_rows, rows // 32 * 32)
    inputs, flops = oracle_sample(w, rows, heads)
    t0 = time.perf_counter()
    oracle_step(w, inputs)
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": (f"float64 oracle {w.passes} on the last {rows} queries of {heads} heads "
                       f"(batch 0) against all {w.seqlen_k} keys of {w.name}; "
                       f"{flops / 1e9:.1f} GFLOP in {dt:.1f} s"),
            "seconds": dt}


def run_reference(args):
    """The reference arm: the oracle as it stands, timed on the host cores."""
    rank, _, world = world_info()
    if rank != 0:
        return 0
    import oracle
    from attn_inputs import WORKLOADS
    w = WORKLOADS[args.workload]
    if getattr(args, "passes", None):
        w = w.replace(passes=args.passes)
    if getattr(args, "seqlen", None):
        w = w.replace(seqlen_q=args.seqlen, seqlen_k=args.seqlen)
    oracle.build()
    threads = oracle.num_threads()
    heads = max(1, min(w.nheads, threads))
    rows = 64
    inputs, flops = oracle_sample(w, rows, heads)
    for _ in range(args.warmup):
        oracle_step(w, inputs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(w, inputs)
    dt = time.perf_counter() - t0
    value = flops * args.steps / dt / 1e12
    sample = (f"float64 oracle {w.passes} on the last {rows} queries of {heads} heads (batch 0) "
              f"against all {w.seqlen_k} keys of {w.name} per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def input_bytes(w):
    """Bytes of the inputs one step reads (Q, K, V and, with a backward, dO)."""
    es = 2
    q = w.batch * w.seqlen_q * w.nheads * w.headdim * es
    kv = 2 * w.batch * w.seqlen_k * w.nheads_kv * w.headdim * es
    return q + kv + (q if has_bwd(w) else 0)


def workload_config(w):
    names = "Q,K,V,dO" if has_bwd(w) else "Q,K,V"
    cfg = {"workload": w.name, "batch": w.batch, "nheads": w.nheads, "nheads_kv": w.nheads_kv,
           "seqlen": w.seqlen_q, "headdim": w.headdim, "causal": w.causal, "pass": w.passes,
           "dtype": w.dtype, "softmax_scale": w.scale,
           "inputs": f"{names} ~ N(0,{w.sigma:g}^2), seed {w.seed}",
           "l2": (f"no flush: inputs {input_bytes(w) / 1e9:.2f} GB per step exceed the "
                  "126 MB L2"),
           "flops": flops_convention(w),
           "parallelism": "replicas (weak scaling, no collective)"}
    if w.window_left >= 0 or w.window_right >= 0:
        cfg["window"] = [w.window_left, w.window_right]
    return cfg


# ---------------------------------------------------------------- GPU arm
def run_gpu(args):
    import torch
    import io_aware_exact_33_b200 as attn
    from attn_inputs import WORKLOADS, make_inputs

    rank, local_rank, world = world_info()
    dist = init_dist("nccl", world)
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    if getattr(args, "passes", None):
        w = w.replace(passes=args.passes)
    if getattr(args, "seqlen", None):
        w = w.replace(seqlen_q=args.seqlen, seqlen_k=args.seqlen)
    f_fwd, f_bwd = step_flops(w)
    bwd = has_bwd(w)

    q, k, v, do = make_inputs(w, with_dout=bwd)
    if do is None:
        do = torch.empty(0, dtype=q.dtype)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    p = attn.params_for(qd, kd, w.scale, w.causal, w.window_left, w.window_right)
    o = torch.empty_like(qd)
    lse = torch.empty(w.batch, w.nheads, w.seqlen_q, dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(t) if bwd else None for t in (qd, kd, vd))
    ws = torch.empty(attn.attn_bwd_workspace_size(p) if bwd else 0, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    nev = 5
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(args.steps)]

    def step(ev=None):
        if ev: ev[0].record(stream)
        attn.attn_fwd(qd, kd, vd, w.scale, w.causal, w.window_left, w.window_right, out=o, lse=lse)
        if ev: ev[1].record(stream)
        if not bwd:
            return
        attn.attn_bwd_prepare(p, o, lse, dod, ws)
        if ev: ev[2].record(stream)
        attn.attn_bwd_accumulate(p, qd, kd, vd, dod, dk, dv, ws)
        if ev: ev[3].record(stream)
        attn.attn_bwd_finalize(p, dq, ws)
        if ev: ev[4].record(stream)

    # forward; prepare, main (three kernels at head dim 256: dV, dK, dQ), convert
    launches_per_step = (1 + (5 if w.headdim == 256 else 3)) if bwd else 1
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if attn.attn_get_device_status() != 0:
        raise RuntimeError("device status word reports an error after warm-up")
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist, dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(gpu_id) as clk:
        start.record(stream)
        for i in range(args.steps):
            step(events[i])
        end.record(stream)
        torch.cuda.synchronize(dev)
    barrier(dist, dev)
    ms_local = start.elapsed_time(end)
    ms = max_over_ranks(ms_local, dist, dev)
    t_fwd = [e[0].elapsed_time(e[1]) for e in events]
    t_prep = [e[1].elapsed_time(e[2]) for e in events] if bwd else [0.0]
    t_main = [e[2].elapsed_time(e[3]) for e in events] if bwd else [0.0]
    t_fin = [e[3].elapsed_time(e[4]) for e in events] if bwd else [0.0]
    value = (f_fwd + f_bwd) * args.steps * world / (ms / 1e3) / 1e12

    # end to end through the public API with pinned host buffers: every step
    # uploads its inputs, runs forward and backward, and downloads its
    # results.  Two device buffer sets let step i+1's upload and step i-1's
    # download run on their own streams while step i computes; the timed
    # region spans the first upload to the last download.
    k_e2e = max(1, min(args.steps, args.e2e_steps))
    host_in = [t.pin_memory() for t in ((q, k, v, do) if bwd else (q, k, v))]
    dev_out0 = [o, lse] + ([dq, dk, dv] if bwd else [])
    host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in dev_out0]
    sets = [([qd, kd, vd] + ([dod] if bwd else []), dev_out0)]
    sets.append(([torch.empty_like(t) for t in sets[0][0]], [torch.empty_like(t) for t in dev_out0]))
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(n):
        ev = [[torch.cuda.Event() for _ in range(3)] for _ in range(n)]  # uploaded, computed, downloaded
        for i in range(n):
            d_in, d_out = sets[i % 2]
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(ev[i - 2][1])  # this set's inputs are no longer read
                for dst, src in zip(d_in, host_in):
                    dst.copy_(src, non_blocking=True)
                ev[i][0].record(up)
            stream.wait_event(ev[i][0])
            if i >= 2:
                stream.wait_event(ev[i - 2][2])  # this set's outputs have been downloaded
            qx, kx, vx = d_in[:3]
            attn.attn_fwd(qx, kx, vx, w.scale, w.causal, w.window_left, w.window_right,
                          out=d_out[0], lse=d_out[1])
            if bwd:
                attn.attn_bwd(qx, kx, vx, d_out[0], d_out[1], d_in[3], w.scale, w.causal,
                              w.window_left, w.window_right, dq=d_out[2], dk=d_out[3],
                              dv=d_out[4], workspace=ws)
            ev[i][1].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev[i][1])
                for dst, src in zip(host_out, d_out):
                    dst.copy_(src, non_blocking=True)
                ev[i][2].record(down)

    e2e_run(2)
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(up)
    with torch.cuda.stream(down):
        down.wait_event(s2)
    stream.wait_event(s2)
    e2e_run(k_e2e)
    e2.record(down)
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    ms_e2e = max_over_ranks(s2.elapsed_time(e2), dist, dev)
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    status = attn.attn_get_device_status()

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return 0

    peaks, peak_kind = load_peaks()
    mean = lambda xs: sum(xs) / len(xs)
    kernels = {"attn_fwd_kernel": {"ms": mean(t_fwd), "flops": f_fwd}}
    if bwd:
        # head dim 256: the accumulate stage's three kernels together
        kernels["attn_bwd_kernel" if w.headdim <= 128 else "attn_bwd256 (3 kernels)"] = {
            "ms": mean(t_main), "flops": f_bwd}
    dominant = max(kernels, key=lambda n: kernels[n]["ms"])
    # DRAM traffic is recorded per (kernel, workload at its own size)
    cfg_workload = None if getattr(args, "seqlen", None) else w.name
    rl = {}
    for name, kk in kernels.items():
        achieved = kk["flops"] / (kk["ms"] / 1e3) / 1e12
        traffic = recorded_traffic(name, cfg_workload)
        rl[name] = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                    "unit": UNIT, "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
                    "peak_source": f"bf16_tflops (burst) of {peak_kind}",
                    "ms_per_launch": kk["ms"], "flops_per_launch": kk["flops"]}
    cpu = cpu_baseline(w) if (world == 1 and not args.no_cpu_baseline) else None
    if cpu is not None:
        cpu.pop("seconds", None)
    clocks = clk.summary()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": f"synthetic ({workload_config(w)['inputs']})",
        "config": workload_config(w),
        "pct_of_peak": {"measured_bf16": value / world / peaks["bf16_tflops"],
                        "nominal_2250": value / world / NOMINAL_BF16_TFLOPS,
                        "peak_source": peak_kind},
        "fwd_tflops": f_fwd / (mean(t_fwd) / 1e3) / 1e12,
        "value_exact_pairs": (sum(exact_pair_flops(w)) * args.steps * world / (ms / 1e3) / 1e12),
        "bwd_tflops": (f_bwd / ((mean(t_prep) + mean(t_main) + mean(t_fin)) / 1e3) / 1e12
                       if bwd else None),
        "ms": {"fwd": mean(t_fwd), "bwd_prepare": mean(t_prep), "bwd_accumulate": mean(t_main),
               "bwd_finalize": mean(t_fin)},
        "roofline": dict(rl[dominant], kernel=dominant),
        "kernels": rl,
        "cpu_baseline": cpu,
        "e2e": {"value": (f_fwd + f_bwd) * k_e2e * world / (ms_e2e / 1e3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": k_e2e,
                "ms_per_step": ms_e2e / k_e2e,
                "copies": "pinned host buffers; uploads and downloads on their own streams, "
                          "two device buffer sets, overlapping the neighbouring steps' compute"},
        "clocks": clocks,
        "gpu_launches": launches_per_step * args.steps,
        "device_status": status,
        "env": environment(torch, dev),
    }
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------- packed arm
def varlen_flops(w):
    """(forward, backward) FLOPs of a packed workload: exact visible pairs of
    every sequence x 4d (forward), x 2.5 of that (backward)."""
    pairs = sum(visible_pairs(n, n, w.causal, w.window_left, w.window_right) for n in w.lens)
    fwd = 4.0 * w.nheads * w.headdim * pairs
    return fwd, (2.5 * fwd if "bwd" in w.passes else 0.0)


def varlen_config(w):
    return {"workload": w.name, "sequences": len(w.lens), "tokens": sum(w.lens),
            "lengths": list(w.lens), "nheads": w.nheads, "nheads_kv": w.nheads_kv,
            "headdim": w.headdim, "causal": w.causal, "pass": w.passes, "dtype": w.dtype,
            "softmax_scale": w.scale, "layout": "packed (cu_seqlens)",
            "inputs": f"Q,K,V,dO ~ N(0,{w.sigma:g}^2), seed {w.seed}",
            "l2": "no flush: inputs exceed the 126 MB L2",
            "flops": "exact visible pairs x 4d (fwd), x 10d (bwd)",
            "parallelism": "replicas (weak scaling, no collective)"}


def varlen_cpu_baseline(w, inputs, target_s=12.0):
    """The float64 oracle on the last rows of the longest sequence (its keys
    in full), sized to about ``target_s`` seconds."""
    import oracle
    oracle.build()
    q, k, v, do, cu_q, cu_k = inputs
    threads = oracle.num_threads()
    heads = max(1, min(w.nheads, threads))
    kvh = max(1, heads * w.nheads_kv // w.nheads)
    b = max(range(len(w.lens)), key=lambda i: w.lens[i])
    q0, n = int(cu_q[b]), w.lens[b]

    def run(rows):
        sl = slice(q0 + n - rows, q0 + n)
        qs = q[sl, :heads][None].contiguous()
        dos = do[sl, :heads][None].contiguous()
        ks = k[q0:q0 + n, :kvh][None].contiguous()
        vs = v[q0:q0 + n, :kvh][None].contiguous()
        t0 = time.perf_counter()
        oracle.attention_fwd(qs, ks, vs, w.scale, w.causal, w.window_left, w.window_right)
        oracle.attention_bwd(qs, ks, vs, dos, w.scale, w.causal, w.window_left, w.window_right)
        dt = time.perf_counter() - t0
        pairs = visible_pairs(n, n, w.causal, w.window_left, w.window_right,
                              rows=range(n - rows, n))
        return dt, pairs * heads * 14.0 * w.headdim

    dt, _ = run(16)
    rows = int(min(n, max(16, 16 * target_s / max(dt, 1e-3))))
    dt, flops = run(rows)
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": (f"float64 oracle fwd+bwd on the last {rows} queries of {heads} heads of "
                       f"the longest sequence ({n} tokens) of {w.name}; "
                       f"{flops / 1e9:.1f} GFLOP in {dt:.1f} s")}


def run_gpu_varlen(args, w):
    """The packed entry points on a length mix: attn_fwd_varlen then
    attn_bwd_varlen (its three kernels) per step."""
    import torch
    import io_aware_exact_33_b200 as attn
    from attn_inputs import make_varlen_inputs

    rank, local_rank, world = world_info()
    dist = init_dist("nccl", world)
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    f_fwd, f_bwd = varlen_flops(w)
    inputs = make_varlen_inputs(w.lens, w.lens, w.nheads, w.nheads_kv, w.headdim, w.dtype,
                                w.sigma, w.seed)
    q, k, v, do, cu_q, cu_k = inputs
    qd, kd, vd, dod, cqd, ckd = (t.to(dev) for t in inputs)
    mx = max(w.lens)
    args_m = (w.scale, w.causal, w.window_left, w.window_right)
    o = torch.empty_like(qd)
    lse = torch.empty((w.nheads, qd.shape[0]), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    p = attn.make_varlen_params(len(w.lens), qd.shape[0], kd.shape[0], mx, mx, w.nheads,
                                w.nheads_kv, w.headdim, attn._dtype_code(qd), w.scale, w.causal,
                                w.window_left, w.window_right)
    ws = torch.empty(attn.attn_bwd_varlen_workspace_size(p), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]

    def step(ev=None):
        if ev: ev[0].record(stream)
        attn.attn_fwd_varlen(qd, kd, vd, cqd, ckd, mx, mx, *args_m, out=o, lse=lse)
        if ev: ev[1].record(stream)
        attn.attn_bwd_varlen(qd, kd, vd, o, lse, dod, cqd, ckd, mx, mx, *args_m, dq=dq, dk=dk,
                             dv=dv, workspace=ws)
        if ev: ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if attn.attn_get_device_status() != 0:
        raise RuntimeError("device status word reports an error after warm-up")
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist, dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(gpu_id) as clk:
        start.record(stream)
        for i in range(args.steps):
            step(events[i])
        end.record(stream)
        torch.cuda.synchronize(dev)
    barrier(dist, dev)
    ms = max_over_ranks(start.elapsed_time(end), dist, dev)
    t_fwd = [e[0].elapsed_time(e[1]) for e in events]
    t_bwd = [e[1].elapsed_time(e[2]) for e in events]
    value = (f_fwd + f_bwd) * args.steps * world / (ms / 1e3) / 1e12

    k_e2e = max(1, min(args.steps, args.e2e_steps))
    host = [t.pin_memory() for t in (q, k, v, do, cu_q, cu_k)]
    ho, hlse = torch.empty_like(host[0]).pin_memory(), torch.empty(lse.shape).pin_memory()
    hg = [torch.empty_like(t).pin_memory() for t in host[:3]]

    def e2e_step():
        for dst, src in zip((qd, kd, vd, dod, cqd, ckd), host):
            dst.copy_(src, non_blocking=True)
        attn.attn_fwd_varlen(qd, kd, vd, cqd, ckd, mx, mx, *args_m, out=o, lse=lse)
        attn.attn_bwd_varlen(qd, kd, vd, o, lse, dod, cqd, ckd, mx, mx, *args_m, dq=dq, dk=dk,
                             dv=dv, workspace=ws)
        for dst, src in zip([ho, hlse] + hg, (o, lse, dq, dk, dv)):
            dst.copy_(src, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(stream)
    for _ in range(k_e2e):
        e2e_step()
    e2.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    ms_e2e = max_over_ranks(s2.elapsed_time(e2), dist, dev)
    h2d = sum(t.numel() * t.element_size() for t in host)
    d2h = sum(t.numel() * t.element_size() for t in [ho, hlse] + hg)
    status = attn.attn_get_device_status()
    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return 0
    peaks, peak_kind = load_peaks()
    mean = lambda xs: sum(xs) / len(xs)
    rl = {}
    for name, ms_k, fl in (("attn_fwd_varlen", mean(t_fwd), f_fwd),
                           ("attn_bwd_varlen (3 kernels)", mean(t_bwd), f_bwd)):
        a = fl / (ms_k / 1e3) / 1e12
        rl[name] = {"bound": "tensor", "achieved": a, "peak": peaks["bf16_tflops"], "unit": UNIT,
                    "frac": a / peaks["bf16_tflops"], "traffic": None,
                    "peak_source": f"bf16_tflops (burst) of {peak_kind}", "ms_per_launch": ms_k,
                    "flops_per_launch": fl}
    dominant = max(rl, key=lambda n: rl[n]["ms_per_launch"])
    cpu = varlen_cpu_baseline(w, inputs) if (world == 1 and not args.no_cpu_baseline) else None
    line = {
        "metric": "packed variable-length attention fwd/bwd TFLOP/s", "value": value,
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": f"synthetic ({varlen_config(w)['inputs']})",
        "config": varlen_config(w),
        "fwd_tflops": rl["attn_fwd_varlen"]["achieved"],
        "bwd_tflops": rl["attn_bwd_varlen (3 kernels)"]["achieved"],
        "ms": {"fwd": mean(t_fwd), "bwd": mean(t_bwd)},
        "roofline": dict(rl[dominant], kernel=dominant), "kernels": rl, "cpu_baseline": cpu,
        "e2e": {"value": (f_fwd + f_bwd) * k_e2e * world / (ms_e2e / 1e3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": k_e2e},
        "clocks": clk.summary(), "gpu_launches": 4 * args.steps, "device_status": status,
    }
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------- extra entry points
def run_gpu_extra(args, w):
    """The decode path (CUDA cores, HBM-bound: GB/s of K, V, Q read and O, LSE
    written, against the measured copy bandwidth) or the FP8 forward (TFLOP/s
    of the exact visible pairs against the measured bf16 peak times the
    nominal FP8 / BF16 ratio of 2).  Inputs resident in HBM; every step
    reads more than the L2 holds."""
    import torch
    import io_aware_exact_33_b200 as attn
    from attn_inputs import make_inputs

    rank, local_rank, world = world_info()
    dist = init_dist("nccl", world)
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    decode = w.name.startswith("decode")
    q, k, v, _ = make_inputs(w, with_dout=False)
    pairs = visible_pairs(w.seqlen_q, w.seqlen_k, w.causal, w.window_left, w.window_right)
    flops = 4.0 * w.batch * w.nheads * w.headdim * pairs
    o = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.batch, w.nheads, w.seqlen_q), dtype=torch.float32, device=dev)
    mask = (w.scale, w.causal, w.window_left, w.window_right)
    if decode:
        qd, kd, vd = (t.to(dev) for t in (q, k, v))
        p = attn.params_for(qd, kd, w.scale, w.causal, w.window_left, w.window_right)
        fn = attn._lib.attn_fwd_decode_workspace_size
        fn.argtypes = [ctypes.POINTER(attn.AttnParams)]
        fn.restype = ctypes.c_size_t
        ws = torch.empty(max(int(fn(ctypes.byref(p))), 1), dtype=torch.uint8, device=dev)

        def call(qx):
            attn.attn_fwd_decode(qx, kd, vd, *mask, out=o, lse=lse, workspace=ws)
        launches, qdev, host_q = 2, qd, q.pin_memory()
        alg_bytes = sum(t.numel() * t.element_size() for t in (q, k, v)) + 2 * o.numel() + 4 * lse.numel()
    else:
        scales = [float(t.double().abs().max()) / 448.0 for t in (q, k, v)]
        q8, k8, v8 = ((t.float() / sc).to(torch.float8_e4m3fn) for t, sc in zip((q, k, v), scales))
        qd8, kd8, vd8 = (t.to(dev) for t in (q8, k8, v8))

        def call(qx):
            attn.attn_fwd_e4m3(qx, kd8, vd8, *scales, *mask, out=o, lse=lse)
        launches, qdev, host_q = 1, qd8, q8.pin_memory()
        alg_bytes = sum(t.numel() for t in (q8, k8, v8)) + 2 * o.numel() + 4 * lse.numel()
    stream = torch.cuda.current_stream(dev)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for _ in range(args.warmup):
        call(qdev)
    torch.cuda.synchronize(dev)
    if attn.attn_get_device_status() != 0:
        raise RuntimeError("device status word reports an error after warm-up")
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist, dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(gpu_id) as clk:
        start.record(stream)
        for i in range(args.steps):
            events[i][0].record(stream)
            call(qdev)
            events[i][1].record(stream)
        end.record(stream)
        torch.cuda.synchronize(dev)
    barrier(dist, dev)
    ms = max_over_ranks(start.elapsed_time(end), dist, dev)
    ms_call = sum(e[0].elapsed_time(e[1]) for e in events) / args.steps
    # end to end: the step's queries up from pinned host memory (the K / V
    # operands stay resident, as a cache or weights-like inputs would), the
    # output down
    host_o = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    k_e2e = max(1, min(args.steps, args.e2e_steps))
    barrier(dist, dev)
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(stream)
    for _ in range(k_e2e):
        qdev.copy_(host_q, non_blocking=True)
        call(qdev)
        host_o.copy_(o, non_blocking=True)
    e2.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    ms_e2e = max_over_ranks(s2.elapsed_time(e2), dist, dev)
    status = attn.attn_get_device_status()
    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return 0
    peaks, peak_kind = load_peaks()
    if decode:
        unit, value = "GB/s", alg_bytes * args.steps * world / (ms / 1e3) / 1e9
        achieved = alg_bytes / (ms_call / 1e3) / 1e9
        rl = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": unit,
              "frac": achieved / peaks["hbm_gbs"], "traffic": None, "kernel": "attn_fwd_decode",
              "peak_source": f"hbm_gbs of {peak_kind}", "bytes_per_launch": alg_bytes}
        metric, e2e_value = "decode attention HBM GB/s", alg_bytes * k_e2e * world / (ms_e2e / 1e3) / 1e9
    else:
        unit, value = UNIT, flops * args.steps * world / (ms / 1e3) / 1e12
        achieved = flops / (ms_call / 1e3) / 1e12
        peak = 2.0 * peaks["bf16_tflops"]
        rl = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": unit,
              "frac": achieved / peak, "traffic": None, "kernel": "attn_fwd_e4m3_kernel",
              "peak_source": f"2 x bf16_tflops (burst) of {peak_kind}: the nominal FP8/BF16 ratio",
              "flops_per_launch": flops}
        metric, e2e_value = "FP8 (E4M3) attention forward TFLOP/s", flops * k_e2e * world / (ms_e2e / 1e3) / 1e12
    cfg = workload_config(w)
    cfg["l2"] = f"no flush: {alg_bytes / 1e9:.2f} GB read and written per step exceed the 126 MB L2"
    line = {
        "metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if not decode else w.dtype,
        "data": f"synthetic ({cfg['inputs']})", "config": cfg, "roofline": rl,
        "cpu_baseline": None,
        "e2e": {"value": e2e_value, "unit": unit, "steps": k_e2e,
                "h2d_bytes_per_step": host_q.numel() * host_q.element_size(),
                "d2h_bytes_per_step": host_o.numel() * host_o.element_size()},
        "clocks": clk.summary(), "gpu_launches": launches * args.steps, "device_status": status,
    }
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--workload", default=WORKLOAD,
                    help=f"attn_inputs workload to time (default {WORKLOAD}, the headline)")
    ap.add_argument("--passes", choices=["fwd", "fwd+bwd"], default=None,
                    help="time these passes instead of the workload's own (for example the "
                         "backward of a forward-only workload)")
    ap.add_argument("--seqlen", type=int, default=None,
                    help="query and key length instead of the workload's (a smaller case of "
                         "the same kernels, for profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    from attn_inputs import EXTRA_WORKLOADS, VARLEN_WORKLOADS, WORKLOADS
    if args.workload in EXTRA_WORKLOADS:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable":
                              "the reference arm times the dense headline workload only"}))
            return 0
        return run_gpu_extra(args, EXTRA_WORKLOADS[args.workload])
    if args.workload in VARLEN_WORKLOADS:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable":
                              "the reference arm times the dense headline workload only"}))
            return 0
        return run_gpu_varlen(args, VARLEN_WORKLOADS[args.workload])
    if args.workload not in WORKLOADS:
        ap.error(f"unknown workload {args.workload}; choose from "
                 f"{sorted(WORKLOADS) + sorted(VARLEN_WORKLOADS) + sorted(EXTRA_WORKLOADS)}")
    wk = WORKLOADS[args.workload]
    if args.seqlen:
        wk = wk.replace(seqlen_q=args.seqlen, seqlen_k=args.seqlen)
    if input_bytes(wk) < 2 * 126e6:
        ap.error(f"{args.workload} fits in L2; it is a parity case, not a bench workload")
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
