"""Benchmark: fresh-partition attention TFLOP/s (and state-compose GB/s) on B200.

One step = one ``as_step`` over the FLUX-like image-DiT attention workload
(B=1, H=24, S=4608 = 4096 image + 512 text tokens, d=128, bf16 in / fp32
states, P=8 partitions of 576, every pair fresh and composed): plan
resolution, the partition states of all eight KV partitions and their
composition, on the tensor cores.  FLOPs counted: 4*B*H*S*S*d per step (QK^T
and PV, fresh pairs only).  Inputs are resident in HBM; the L2 is flushed
(a 256 MiB write) before every timed step, outside the timed events.

Also reported on the same line (same run):
* ``e2e``: the same step through the public API from pinned HOST buffers,
  with the host->device copy of Q, K, V and the device->host copy of OUT and
  LSE inside the timed region;
* ``roofline``: the attention kernel against the measured dense bf16 peak;
* ``secondary``: the state-compose kernel on the compose-bound workload (GB/s
  against measured HBM copy bandwidth) and the two-step video reuse workload
  (fresh TFLOP/s, reuse-compose GB/s, reuse MSE against full attention);
* ``cpu_baseline``: the float64 oracle on the host cores on a sample of rows.

``--impl reference`` times the float64 oracle instead (the only reference
implementation of this method available here), on the host cores, on samples
of the same workload, and prints the same metric.

Multi-GPU: every rank runs its own replica of the workload (the path shards
by heads and batches with no exchange step); value = all ranks' FLOPs / the
slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from attention_state_reuse_partition_b200 import workloads as W  # noqa: E402

METRIC = "fresh-partition attn TFLOP/s & compose GB/s at 1 B200; % of bf16/HBM roofline"
WORKLOAD = "flux_image"
WORKLOAD_TEXT = (f"{WORKLOAD}: B=1 H=24 S=4608 (4096 image + 512 text) d=128, P=8 partitions of 576, "
                 "all pairs fresh and composed")
L2_FLUSH_BYTES = 256 << 20


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


CSRC = os.path.join(ROOT, "attention_state_reuse_partition_b200", "csrc")
KERNEL_SOURCES = {
    "attn_tc_kernel<128>": ("attn_tc_bf16.cu", "as_device.cuh", "as_kernels.h"),
    "compose_strided_kernel<128>": ("compose.cu", "as_device.cuh", "as_kernels.h"),
}


def kernel_source_hash(kernel: str) -> str:
    """First 16 hex digits of the SHA-256 of the sources a kernel is built from."""
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, units_scale: float = 1.0):
    """DRAM bytes (read + write) per launch from the committed ncu summary
    (profiles/ncu_traffic.txt), scaled by units_scale when the capture ran a
    smaller case; None if absent or if the kernel's sources changed since."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        entry = json.load(f).get(kernel)
    if not entry or entry.get("source_sha256_16") != kernel_source_hash(kernel):
        return None
    return entry["dram_bytes_per_launch"] * units_scale


def attn_flops(s) -> float:
    return 4.0 * s.B * s.H * s.S * s.S * s.d


def max_over_ranks(x: float, device) -> float:
    """The maximum of a per-rank scalar over all ranks (identity at one rank).
    Every rank must call it at the same point (a collective)."""
    if not torch.distributed.is_available() or not torch.distributed.is_initialized() \
            or torch.distributed.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank processed units_per_rank in at most
    ms_max milliseconds (the slowest rank's time)."""
    return units_per_rank * world / (ms_max * 1e-3)


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML (read-only
    queries) every 2 ms in a background thread, so that even a timed region of
    a few milliseconds holds samples.  Samples taken inside the timed region
    are marked via ``mark_timed``."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, gpu_index: int, interval: float = 0.002):
        import threading
        self.gpu, self.interval = gpu_index, interval
        self.samples = []
        self.timed = False
        self.stop = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.error = None

    def _run(self):
        try:
            import pynvml as N
            N.nvmlInit()
            h = N.nvmlDeviceGetHandleByIndex(self.gpu)
            smax = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
            while not self.stop.is_set():
                sm = N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)
                try:
                    reasons = N.nvmlDeviceGetCurrentClocksEventReasons(h)
                except AttributeError:
                    reasons = N.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                power = N.nvmlDeviceGetPowerUsage(h) / 1000.0
                self.samples.append((self.timed, sm, smax, power, reasons))
                time.sleep(self.interval)
            N.nvmlShutdown()
        except Exception as e:  # noqa: BLE001
            self.error = repr(e)

    def __enter__(self):
        self.thread.start()
        return self

    def mark_timed(self, on: bool):
        self.timed = on

    def __exit__(self, *exc):
        self.stop.set()
        self.thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [f"no samples ({self.error})"]}
        timed = [x for x in self.samples if x[0]]
        use = timed if timed else self.samples
        reasons = sorted({name for x in use for bit, name in self.REASONS.items() if x[4] & bit})
        return {"sm_mhz": statistics.median(x[1] for x in use), "sm_max_mhz": float(use[0][2]),
                "reasons": reasons, "samples_timed": len(timed), "samples_total": len(self.samples),
                "power_w_max": max(x[3] for x in use),
                "how": "NVML every 2 ms; median over the samples inside the timed region "
                       "(all samples, warm-up included, when the region is shorter than one interval)"}


# ---------------------------------------------------------------------------
# CPU baseline: the float64 oracle on a bounded sample of rows
# ---------------------------------------------------------------------------

def oracle_sample(s, q, k, v, rows_per_partition: int, heads):
    """Times the oracle's all-fresh step on a seeded sample of query rows
    (all keys, the given heads).  Returns (seconds, flops)."""
    from oracle import as_oracle as O
    rows = W.sample_rows(s, rows_per_partition).numpy()
    qn = q[:, heads][:, :, rows].float().cpu().double().numpy()
    kn = k[:, heads].float().cpu().double().numpy()
    vn = v[:, heads].float().cpu().double().numpy()
    cache = O.StateCache(s.P)
    plan = np.ones((s.P, s.P), np.uint8)
    # the oracle's step takes full-length Q and selects `rows`; pad Q
    qfull = np.zeros((s.B, len(heads), s.S, s.d))
    qfull[:, :, rows] = qn
    t0 = time.perf_counter()
    O.step(cache, qfull, kn, vn, plan, 0, s.scale, rows=rows)
    dt = time.perf_counter() - t0
    flops = 4.0 * s.B * len(heads) * len(rows) * s.S * s.d
    return dt, flops


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 0) for i in threadpool_info()), default=0)
        if n:
            return n
    except Exception:  # noqa: BLE001
        pass
    return os.cpu_count()


# ---------------------------------------------------------------------------
# the timed legs
# ---------------------------------------------------------------------------

def run_own(args, rank, world, device):
    from attention_state_reuse_partition_b200 import api
    s = W.spec(WORKLOAD)
    q, k, v = W.flux_qkv(s, device=device)
    plan = W.all_fresh_plan(s.P).numpy()
    cache = api.AsCache(s.B, s.H, s.S, s.d, s.P, device=device)
    out = torch.empty((s.B, s.H, s.S, s.d), device=device, dtype=torch.float32)
    lse = torch.empty((s.B, s.H, s.S), device=device, dtype=torch.float32)
    flush = torch.empty(L2_FLUSH_BYTES // 4, device=device, dtype=torch.float32)
    stream = torch.cuda.current_stream()

    def step():
        api.as_step(cache, q, k, v, plan, 0, out=out, lse=lse)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        t_end = time.perf_counter() + args.warm_seconds   # warm the clocks up
        done = 0
        while done < args.warmup or time.perf_counter() < t_end:
            flush.fill_(1.0)
            step()
            done += 1
            if done % 16 == 0:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        clk.mark_timed(True)
        for i in range(args.steps):
            flush.fill_(float(i))           # L2 flush, keeps the GPU busy across the launch gap
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        clk.mark_timed(False)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    times = [a.elapsed_time(b) for a, b in ev]
    ms = sum(times) / len(times)
    api.as_device_status()
    ms_max = max_over_ranks(ms, device)
    flops = attn_flops(s)
    value = weak_scaling_value(flops, world, ms_max) / 1e12

    result = {"ms": ms, "ms_max": ms_max, "value": value, "flops": flops, "clocks": clk.summary(),
              "gpu_launches": args.steps, "step_ms": times, "e2e": None}
    if args.kernel_only:
        return result, (q, k, v, s)

    # end to end through the public API with pinned host buffers.  Steps are
    # independent, so they are pipelined over three streams with two buffer
    # sets: the host->device copy of step i+1 and the device->host copy of
    # step i-1 overlap the attention of step i (PCIe is full duplex).  Every
    # step still copies its inputs in and its result out inside the timed
    # region.
    hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    NB = 2
    hout = [torch.empty(out.shape, dtype=torch.float32).pin_memory() for _ in range(NB)]
    hlse = [torch.empty(lse.shape, dtype=torch.float32).pin_memory() for _ in range(NB)]
    din = [tuple(torch.empty_like(x) for x in (q, k, v)) for _ in range(NB)]
    dout = [(torch.empty_like(out), torch.empty_like(lse)) for _ in range(NB)]
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(NB)]
    ev_cmp = [torch.cuda.Event() for _ in range(NB)]
    ev_out = [torch.cuda.Event() for _ in range(NB)]
    for b in range(NB):  # nothing in flight yet
        ev_cmp[b].record(s_cmp)
        ev_out[b].record(s_out)

    def e2e_step(i):
        b = i % NB
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_cmp[b])             # the step that last read din[b] is done
            for dst, src in zip(din[b], (hq, hk, hv)):
                dst.copy_(src, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[b])
            s_cmp.wait_event(ev_out[b])            # dout[b] has been copied out
            api.as_step(cache, *din[b], plan, 0, out=dout[b][0], lse=dout[b][1], stream=s_cmp)
            ev_cmp[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[b])
            hout[b].copy_(dout[b][0], non_blocking=True)
            hlse[b].copy_(dout[b][1], non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(max(3, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(args.steps):
        e2e_step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_cmp)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, device)
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
    d2h = hout[0].numel() * 4 + hlse[0].numel() * 4
    for b in range(NB):
        assert torch.allclose(hout[b].to(device), out), "e2e output differs from the device-resident run"

    result["e2e"] = {"value": weak_scaling_value(flops, world, e2e_ms) / 1e12, "unit": "TFLOP/s",
                     "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                     "pipeline": "3 streams, 2 buffer sets: copy-in, attention and copy-out of consecutive "
                                 "steps overlap"}
    del cache, flush
    torch.cuda.empty_cache()
    return result, (q, k, v, s)


def ncu_compose_rows() -> int:
    """Rows of the compose case the committed ncu capture ran (196608)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if os.path.exists(path):
        with open(path) as f:
            e = json.load(f).get("compose_strided_kernel<128>")
        if e:
            return int(e.get("rows", 196608))
    return 196608


def run_compose(args, device):
    """Compose-bound workload: 32 fp32 states per row merged into one."""
    from attention_state_reuse_partition_b200 import api
    s = W.spec("compose_bound")
    outs, lses = W.compose_states(s, device=device, rows=args.compose_rows)
    out = torch.empty(outs.shape[1:], device=device)
    lse = torch.empty(lses.shape[1:], device=device)
    for _ in range(3):
        api.as_compose(outs, lses, out=out, lse=lse)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(5)]
    for a, b in ev:
        a.record()
        api.as_compose(outs, lses, out=out, lse=lse)
        b.record()
    torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    rows = outs.shape[1]
    nbytes = (s.n_states + 1) * rows * (s.d + 1) * 4
    del outs, lses, out, lse
    torch.cuda.empty_cache()
    return {"workload": "compose_bound", "ms": ms, "bytes": nbytes, "GB/s": nbytes / (ms * 1e-3) / 1e9}


def run_reuse(args, device):
    """Two-step video reuse: anchor step then a reuse step (window 2).
    ``--reuse-heads`` runs fewer heads (a smaller case for profiling);
    ``--reuse-groups`` / ``--reuse-cache`` set the cache's group size and
    entry type."""
    from attention_state_reuse_partition_b200 import api
    s = W.spec("video_reuse") if args.reuse_heads is None else W.spec("video_reuse", H=args.reuse_heads)
    g, cdt = args.reuse_groups, args.reuse_cache
    steps = [(q, k, v) for _, q, k, v in W.video_trajectory(s, device=device)]
    plans = [W.grouped_plan_for_step(s, t, g).numpy() for t in range(s.steps)]
    cache = api.AsCache(s.B, s.H, s.S, s.d, s.P, device=device, g=g, cache_dtype=cdt)
    out = torch.empty((s.B, s.H, s.S, s.d), device=device)
    lse = torch.empty((s.B, s.H, s.S), device=device)
    q1, k1, v1 = steps[1]
    n_fresh = int((plans[1] != W.PLAN_REUSE).sum())
    n_reuse = int((plans[1] == W.PLAN_REUSE).sum())
    fresh_flops = 4.0 * s.B * s.H * n_fresh * s.n * s.n * s.d
    times = []
    for rep in range(4):
        c = api.AsCache(s.B, s.H, s.S, s.d, s.P, buffer=cache.buffer, g=g, cache_dtype=cdt)
        api.as_step(c, *steps[0], plans[0], 0, out=out, lse=lse)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        api.as_step(c, q1, k1, v1, plans[1], 1, out=out, lse=lse)
        b.record()
        torch.cuda.synchronize()
        if rep > 0:
            times.append(a.elapsed_time(b))
    ms = statistics.mean(times)
    full_o, _ = api.as_partition_attn(q1, k1, v1, s.P, -1, list(range(s.P)))
    torch.cuda.synchronize()
    mse = torch.mean((out - full_o) ** 2).item()
    entry_bytes = s.B * s.H * s.n * (s.d * (2 if cdt == "bf16" else 4) + 4)  # one (i, G) entry
    NG = (s.P + g - 1) // g
    reused_entries = sum(bool((plans[1][i, G * g:(G + 1) * g] == W.PLAN_REUSE).any())
                         for i in range(s.P) for G in range(NG))
    reuse_bytes = reused_entries * entry_bytes
    del cache, steps, full_o
    torch.cuda.empty_cache()
    name = "video_reuse step t" + ("" if (g, cdt, s.H) == (1, "f32", 24) else f" (H={s.H}, g={g}, {cdt} entries)")
    return {"workload": name, "ms": ms, "fresh_pairs": n_fresh, "reused_pairs": n_reuse,
            "reused_entries": reused_entries,
            "fresh_tflops_whole_step": fresh_flops / (ms * 1e-3) / 1e12, "reuse_bytes": reuse_bytes,
            "reuse_mse_vs_full": mse}


def run_video_long(args, device, g=1, cache_dtype="f32"):
    """Long video trajectory: an anchor step, then three reuse steps (window 4,
    a seeded 10% of reused pairs forced fresh and stored each step).  With
    g > 1 the cache keeps one composed entry per (query partition, group of g
    KV partitions) and a forced pair refreshes its whole group."""
    from attention_state_reuse_partition_b200 import api
    heads = getattr(args, "video_heads", None)
    s = W.spec("video_long") if heads is None else W.spec("video_long", H=heads)
    cache = api.AsCache(s.B, s.H, s.S, s.d, s.P, device=device, g=g, cache_dtype=cache_dtype)
    NG = (s.P + g - 1) // g
    entry_bytes = s.B * s.H * s.n * (s.d * (2 if cache_dtype == "bf16" else 4) + 4)  # one (i, G) entry
    out = torch.empty((s.B, s.H, s.S, s.d), device=device)
    lse = torch.empty((s.B, s.H, s.S), device=device)
    per_step = []
    last = None
    for t, q, k, v in W.video_trajectory(s, device=device):
        plan = W.grouped_plan_for_step(s, t, g).numpy()
        reused_entries = sum(bool((plan[i, G * g:(G + 1) * g] == W.PLAN_REUSE).any())
                             for i in range(s.P) for G in range(NG))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        api.as_step(cache, q, k, v, plan, t, out=out, lse=lse)
        b.record()
        torch.cuda.synchronize()
        n_fresh = int((plan != W.PLAN_REUSE).sum())
        n_reuse = int((plan == W.PLAN_REUSE).sum())
        n_store = int((plan == W.PLAN_FRESH_STORE).sum())
        ms = a.elapsed_time(b)
        fl = 4.0 * s.B * s.H * n_fresh * s.n * s.n * s.d
        per_step.append({"step": t, "ms": round(ms, 3), "fresh_pairs": n_fresh, "reused_pairs": n_reuse,
                         "stored_pairs": n_store, "reused_entries": reused_entries,
                         "reuse_read_gb": round(reused_entries * entry_bytes / 1e9, 3),
                         "fresh_tflops_whole_step": round(fl / (ms * 1e-3) / 1e12, 1)})
        last = (q, k, v)
    q, k, v = last
    full_o, _ = api.as_partition_attn(q, k, v, s.P, -1, list(range(s.P)))
    torch.cuda.synchronize()
    mse = torch.mean((out - full_o) ** 2).item()
    cache_gb = cache.buffer.numel() / 1e9
    del cache, full_o, out, lse, last, q, k, v
    torch.cuda.empty_cache()
    name = "video_long (4 steps)" if g == 1 and cache_dtype == "f32" else \
        f"video_long (4 steps), cache groups of {g} partitions, {cache_dtype} OUT entries"
    if heads is not None:
        name += f" with {s.H} heads"
    return {"workload": name, "g": g, "cache_dtype": cache_dtype, "cache_gb": round(cache_gb, 2),
            "steps": per_step, "reuse_mse_vs_full_last_step": mse}


def run_planner(args, device, window=2, reuse_ratio=0.7, eps_local=0.5, g=1, cache_dtype="f32"):
    """Long video trajectory with the anchor-guided planner choosing each
    step's plan: local states, drift, selection, the step (which composes the
    local states instead of recomputing the diagonal pairs), and the anchor
    statistics after anchor steps.  With g > 1 the planner decides per cache
    group of g KV partitions."""
    from attention_state_reuse_partition_b200 import api
    heads = getattr(args, "video_heads", None)
    s = W.spec("video_long") if heads is None else W.spec("video_long", H=heads)
    cache = api.AsCache(s.B, s.H, s.S, s.d, s.P, device=device, g=g, cache_dtype=cache_dtype)
    pl = api.AsPlanner(s.P, window, reuse_ratio, eps_local, s.B, s.H, s.S, s.d, device=device, g=g)
    out = torch.empty((s.B, s.H, s.S, s.d), device=device)
    lse = torch.empty((s.B, s.H, s.S), device=device)
    local = torch.empty((s.B, s.H, s.S, s.d), device=device)
    local_lse = torch.empty((s.B, s.H, s.S), device=device)
    per_step = []
    last = None
    for t, q, k, v in W.video_trajectory(s, device=device):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        api.as_local_states(q, k, v, s.P, out=local, lse=local_lse)
        plan, is_anchor, _ = api.as_planner_next(pl, local)          # synchronises
        t1 = time.perf_counter()
        api.as_step_local(cache, q, k, v, plan, t, local, local_lse, out=out, lse=lse)
        torch.cuda.synchronize()
        t2 = time.perf_counter()
        if is_anchor:
            api.as_planner_commit_anchor(pl, cache, lse, plan)
        t3 = time.perf_counter()
        per_step.append({"step": t, "anchor": is_anchor, "planner_ms": round((t1 - t0) * 1e3, 3),
                         "step_ms": round((t2 - t1) * 1e3, 3), "anchor_stats_ms": round((t3 - t2) * 1e3, 3),
                         "reused_pairs": int((plan == W.PLAN_REUSE).sum()),
                         "fresh_pairs": int((plan != W.PLAN_REUSE).sum()),
                         "max_rel_drift": round(float(pl.rel_drift.max()), 5)})
        last = (q, k, v)
    q, k, v = last
    full_o, _ = api.as_partition_attn(q, k, v, s.P, -1, list(range(s.P)))
    torch.cuda.synchronize()
    mse = torch.mean((out - full_o) ** 2).item()
    del cache, pl, full_o, out, lse, local, local_lse, last, q, k, v
    torch.cuda.empty_cache()
    name = "video_long (4 steps) with the planner" if g == 1 else \
        f"video_long (4 steps) with the planner over cache groups of {g} partitions, {cache_dtype} OUT entries"
    return {"workload": name, "g": g, "cache_dtype": cache_dtype, "window": window, "reuse_ratio": reuse_ratio,
            "eps_local": eps_local, "steps": per_step, "reuse_mse_vs_full_last_step": mse,
            "timing": "wall clock around synchronising calls"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["own", "reference"], default="own")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--warm-seconds", type=float, default=1.0,
                    help="minimum duration of the warm-up (clocks settle; the sampler runs throughout)")
    ap.add_argument("--only", choices=["compose", "reuse", "video_long", "video_long_grouped", "planner",
                                       "planner_grouped"], default=None,
                    help="run one secondary workload alone and print its JSON (for profiling)")
    ap.add_argument("--compose-rows", type=int, default=None,
                    help="rows of the compose workload (default: all B*H*S rows)")
    ap.add_argument("--reuse-heads", type=int, default=None, help="heads of the reuse workload (default 24)")
    ap.add_argument("--video-heads", type=int, default=None,
                    help="heads of the video_long workloads (default 40; fewer for a small profiling case)")
    ap.add_argument("--reuse-groups", type=int, default=1, help="cache group size of the reuse workload")
    ap.add_argument("--reuse-cache", choices=["f32", "bf16"], default="f32", help="cache entry type of the reuse workload")
    ap.add_argument("--kernel-only", action="store_true",
                    help="time the device-resident step only (no e2e, CPU baseline or secondary workloads)")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, rank, world)

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if args.only is not None:
        fn = {"compose": run_compose, "reuse": run_reuse, "video_long": run_video_long,
              "video_long_grouped": lambda a, dev: run_video_long(a, dev, g=4, cache_dtype="bf16"),
              "planner": run_planner,
              "planner_grouped": lambda a, dev: run_planner(a, dev, g=4, cache_dtype="bf16")}[args.only]
        print(json.dumps({"only": args.only, **fn(args, device)}))
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    peaks = load_peaks()
    res, (q, k, v, s) = run_own(args, rank, world, device)
    secondary = {}
    if not args.no_secondary and not args.kernel_only and world == 1:
        comp = run_compose(args, device)
        comp["frac_of_hbm"] = comp["GB/s"] / peaks["hbm_gbs"]
        rows_full = W.spec("compose_bound").B * W.spec("compose_bound").H * W.spec("compose_bound").S
        comp["traffic"] = measured_traffic("compose_strided_kernel<128>", rows_full / ncu_compose_rows())
        secondary["compose"] = comp
        secondary["reuse"] = run_reuse(args, device)
        secondary["video_long"] = run_video_long(args, device)
        secondary["video_long_grouped"] = run_video_long(args, device, g=4, cache_dtype="bf16")
        secondary["planner"] = run_planner(args, device)
        secondary["planner_grouped"] = run_planner(args, device, g=4, cache_dtype="bf16")

    cpu = None
    if rank == 0 and world == 1 and not args.kernel_only:
        heads = list(range(s.H))
        dt, fl = oracle_sample(s, q, k, v, s.n, heads)
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
               "sample": f"the whole {WORKLOAD} step (all {s.S} query rows x {s.H} heads, all {s.S} keys), "
                         f"float64, one pass ({dt:.1f} s)"}

    ms = res["ms_max"]
    achieved = res["flops"] / (res["ms"] * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    line = {
        "metric": METRIC, "value": round(res["value"], 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT, "global_batch": world, "seq_len": s.S,
                   "parallelism": f"replicas{world}" if world > 1 else "single", "l2": "flushed (256 MiB write) "
                   "before every timed step"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": measured_traffic("attn_tc_kernel<128>"),
                     "kernel": "attn_tc_kernel<128>", "peak_source": f"{peaks['source']} bf16 burst",
                     # the kernel is timed after a second of full load, at the power-capped clock
                     "peak_sustained": peaks["bf16_tflops_sustained"],
                     "frac_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4)},
        "e2e": res["e2e"], "clocks": res["clocks"], "gpu_launches": res["gpu_launches"],
    }
    if line["e2e"] is None:
        del line["e2e"]
    if cpu:
        line["cpu_baseline"] = cpu
    if secondary:
        line["secondary"] = secondary
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))


def run_reference(args, rank, world):
    """The float64 oracle on the host cores, each step a bounded sample of the
    workload's query rows (all keys, three heads)."""
    if rank != 0:
        return
    s = W.spec(WORKLOAD)
    q, k, v = W.flux_qkv(s)
    heads = [0, 11, 23]
    rows = s.n
    for _ in range(args.warmup):
        oracle_sample(s, q, k, v, rows, heads)
    tot_t, tot_f = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl = oracle_sample(s, q, k, v, rows, heads)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    sample = f"per step: all {s.S} query rows x {len(heads)} of {s.H} heads of {WORKLOAD}, all {s.S} keys, float64"
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": WORKLOAD_TEXT, "global_batch": 1, "seq_len": s.S,
                   "parallelism": "host cores (float64 oracle)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


if __name__ == "__main__":
    main()
