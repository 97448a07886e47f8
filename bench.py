"""Benchmark: fresh-partition attention TFLOP/s (and state-compose GB/s) on B200.

One step = one ``as_step`` over the FLUX-like image-DiT attention workload
(B=1, H=24, S=4608 = 4096 image + 512 text tokens, d=128, bf16 in / fp32
states, P=8 partitions of 576, every pair fresh and composed): plan
resolution, the partition states of all eight KV partitions and their
composition, on the tensor cores.  FLOPs counted: 4*B*H*S*S*d per step (QK^T
and PV, fresh pairs only).  Inputs are resident in HBM; the L2 is flushed
(a 256 MiB write) before every timed step, outside the timed events.

Also reported on the same line (same run), in fields of the contract:
* ``e2e``: the same step through the public API from pinned HOST buffers,
  with the host->device copy of Q, K, V and the device->host copy of OUT and
  LSE inside the timed region;
* ``roofline``: the attention kernel against the measured dense bf16 peak;
  ``roofline.compose`` the state-compose kernel on the compose-bound workload
  against the measured HBM copy bandwidth; ``roofline.steps`` every reuse
  workload's step time against its step-level roofline (tensor time of the
  fresh pairs and HBM time of the bytes the step must move, summed and
  overlapped), with the reuse MSE against full attention;
  ``roofline.partition_boundary`` the flux_image step with one state emitted
  per KV partition (ragged 576-token partitions inside the timed region);
  ``roofline.locality`` the MSE of dropping a near against a far partition;
  ``roofline.residual_codec`` the residual codec of the context-parallel
  exchange against the measured HBM copy bandwidth;
* ``cpu_baseline``: the float64 oracle on the host cores -- the whole
  flux_image step, and in ``cpu_baseline.legs`` the compose-bound workload and
  the video workloads on bounded samples of rows and heads (full-step times
  extrapolated from the sample, labelled as such).

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


class OracleTrajectory:
    """The float64 oracle stepped beside a GPU trajectory on a bounded sample:
    a few heads and a seeded sample of query rows in every query partition,
    against all keys, under the same plans and cache history.  Each step is
    timed; its full-workload time is extrapolated by the ratio of rows and
    heads (labelled as extrapolated).  The GPU's states on the sampled rows
    are compared with the oracle's (max-abs error, reported)."""

    def __init__(self, s, heads, rows_per_partition: int, g: int = 1, cache_dtype: str = "f32"):
        from oracle import as_oracle as O
        self.O, self.s, self.heads = O, s, list(heads)
        self.rows = W.sample_rows(s, rows_per_partition).numpy()
        self.cache = O.StateCache(s.P, g, cache_dtype)
        self.records = []

    def step(self, t, q, k, v, plan, out_gpu=None):
        s, O = self.s, self.O
        f = lambda x: x[:, self.heads].float().cpu().double().numpy()  # noqa: E731
        qn, kn, vn = f(q), f(k), f(v)
        t0 = time.perf_counter()
        out, lse, _, _ = O.step(self.cache, qn, kn, vn, plan, t, s.scale, rows=self.rows)
        dt = time.perf_counter() - t0
        r = self.rows.size // s.P
        fresh = int((plan != W.PLAN_REUSE).sum())
        flop = 4.0 * s.B * len(self.heads) * r * s.n * s.d * fresh
        factor = (s.S / self.rows.size) * (s.H / len(self.heads))
        rec = {"step": t, "seconds": round(dt, 3), "tflops": flop / dt / 1e12,
               "extrapolated_full_step_s": round(dt * factor, 1)}
        if out_gpu is not None:
            g = out_gpu[:, self.heads][:, :, torch.from_numpy(self.rows).to(out_gpu.device)]
            rec["gpu_max_abs_err"] = float(np.max(np.abs(g.double().cpu().numpy() - out)))
        self.records.append(rec)
        return rec

    def summary(self, name):
        s = self.s
        return {"workload": name, "kind": "oracle", "unit": "TFLOP/s",
                "value": statistics.mean(x["tflops"] for x in self.records[1:] or self.records),
                "sample": f"{self.rows.size // s.P} query rows in each of the {s.P} query partitions x "
                          f"{len(self.heads)} of {s.H} heads, all {s.S} keys, every step of the trajectory; "
                          f"value = fresh FLOPs of the sample / oracle time, averaged over the non-anchor steps; "
                          f"extrapolated_full_step_s scales the time by rows and heads (extrapolated, not run)",
                "steps": self.records}


def oracle_compose_sample(outs, lses, rows: int):
    """The oracle's one-pass compose on the first ``rows`` rows of the
    compose-bound states; returns (seconds, algorithmic bytes of the sample)."""
    from oracle import as_oracle as O
    o = outs[:, :rows].double().cpu().numpy()
    l = lses[:, :rows].double().cpu().numpy()
    t0 = time.perf_counter()
    O.compose([(o[k], l[k]) for k in range(o.shape[0])])
    dt = time.perf_counter() - t0
    return dt, (o.shape[0] + 1) * rows * (o.shape[2] + 1) * 4


def step_roofline(ms: float, fresh_flop: float, hbm_bytes: float, peaks) -> dict:
    """A step's time against its roofline: the tensor time of its fresh pairs
    at the measured bf16 peak and the HBM time of the bytes it must move at
    the measured copy bandwidth, both serialised (sum) and overlapped (max)."""
    t_tensor = fresh_flop / (peaks["bf16_tflops"] * 1e12) * 1e3
    t_hbm = hbm_bytes / (peaks["hbm_gbs"] * 1e9) * 1e3
    return {"ms": round(ms, 3), "fresh_flop": fresh_flop, "hbm_bytes": hbm_bytes,
            "t_tensor_ms": round(t_tensor, 3), "t_hbm_ms": round(t_hbm, 3),
            "bound_serial_ms": round(t_tensor + t_hbm, 3), "bound_overlap_ms": round(max(t_tensor, t_hbm), 3),
            "frac_of_serial_bound": round((t_tensor + t_hbm) / ms, 4),
            "frac_of_overlap_bound": round(max(t_tensor, t_hbm) / ms, 4),
            "fresh_tflops_whole_step": round(fresh_flop / (ms * 1e-3) / 1e12, 1)}


def step_hbm_bytes(s, plan, g: int, cache_dtype: str) -> int:
    """Bytes a step must move at least: Q, K, V once (bf16), the final OUT and
    LSE once (fp32), every reused cache entry read once and every stored entry
    written once (entries of the cache's type, LSE fp32)."""
    P, NG = s.P, (s.P + g - 1) // g
    entry = s.B * s.H * s.n * (s.d * (2 if cache_dtype == "bf16" else 4) + 4)
    reused = sum(bool((plan[i, G * g:(G + 1) * g] == W.PLAN_REUSE).any()) for i in range(P) for G in range(NG))
    stored = sum(bool((plan[i, G * g:(G + 1) * g] == W.PLAN_FRESH_STORE).any()) for i in range(P) for G in range(NG))
    io = 3 * s.B * s.H * s.S * s.d * 2 + s.B * s.H * s.S * (s.d + 1) * 4
    return io + (reused + stored) * entry


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


def run_compose(args, device, peaks, with_oracle=False):
    """Compose-bound workload: 32 fp32 states per row merged into one, against
    the measured HBM copy bandwidth; optionally the oracle on a row sample."""
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
    gbs = nbytes / (ms * 1e-3) / 1e9
    rows_full = s.B * s.H * s.S
    res = {"bound": "hbm", "kernel": "compose_strided_kernel<128>",
           "workload": f"compose_bound: {rows} rows (B=2 H=24 S=16384) x {s.n_states} fp32 states, d=128",
           "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
           "frac": round(gbs / peaks["hbm_gbs"], 4), "ms": round(ms, 4), "bytes": nbytes,
           "traffic": measured_traffic("compose_strided_kernel<128>", rows / ncu_compose_rows()),
           "peak_source": f"{peaks['source']} HBM copy"}
    cpu = None
    if with_oracle:
        n = min(rows, args.oracle_compose_rows)
        dt, ob = oracle_compose_sample(outs, lses, n)
        cpu = {"workload": "compose_bound", "kind": "oracle", "unit": "GB/s", "value": ob / dt / 1e9,
               "sample": f"the first {n} of {rows_full} rows, all {s.n_states} states, float64 one-pass compose; "
                         f"bytes counted as the GPU's (fp32 states read once, output written once)",
               "seconds": round(dt, 3), "extrapolated_full_s": round(dt * rows_full / n, 1)}
    del outs, lses, out, lse
    torch.cuda.empty_cache()
    return res, cpu


def run_reuse(args, device, peaks=None, with_oracle=False):
    """Two-step video reuse: anchor step then a reuse step (window 2).
    ``--reuse-heads`` runs fewer heads (a smaller case for profiling);
    ``--reuse-groups`` / ``--reuse-cache`` set the cache's group size and
    entry type.  With the oracle: both steps on a sample of rows and heads."""
    from attention_state_reuse_partition_b200 import api
    peaks = peaks or load_peaks()
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
    NG = (s.P + g - 1) // g
    reused_entries = sum(bool((plans[1][i, G * g:(G + 1) * g] == W.PLAN_REUSE).any())
                         for i in range(s.P) for G in range(NG))
    res = step_roofline(ms, fresh_flops, step_hbm_bytes(s, plans[1], g, cdt), peaks)
    res.update({"workload": f"video_reuse step 1 (B=1 H={s.H} S={s.S} P={s.P}, window {s.window}), cache groups "
                            f"of {g}, {cdt} entries",
                "fresh_pairs": n_fresh, "reused_pairs": n_reuse, "reused_entries": reused_entries,
                "reuse_mse_vs_full": mse})
    cpu = None
    if with_oracle:
        orc = OracleTrajectory(s, heads=args.oracle_heads[:min(len(args.oracle_heads), s.H)],
                               rows_per_partition=args.oracle_rows, g=g, cache_dtype=cdt)
        c = api.AsCache(s.B, s.H, s.S, s.d, s.P, buffer=cache.buffer, g=g, cache_dtype=cdt)
        for t in range(s.steps):
            api.as_step(c, *steps[t], plans[t], t, out=out, lse=lse)
            torch.cuda.synchronize()
            orc.step(t, *steps[t], plans[t], out_gpu=out)
        cpu = orc.summary(res["workload"])
    del cache, steps, full_o
    torch.cuda.empty_cache()
    return res, cpu


def run_locality(args, device):
    """Locality of the video_reuse inputs (the trend DiTango's review page
    reports in its Core claim: dropping the nearest KV partition costs far
    more than dropping a distant one).  For every query partition i, the MSE
    against full attention of the state that leaves out KV partition i+1 (or
    i-1 at the end) and of the one that leaves out i+8 (or i-8)."""
    from attention_state_reuse_partition_b200 import api
    s = W.spec("video_reuse")
    _, q, k, v = next(iter(W.video_trajectory(s, device=device)))
    full_o, _ = api.as_partition_attn(q, k, v, s.P, -1, list(range(s.P)))
    n = s.n
    near, far = [], []
    for i in range(s.P):
        ref = full_o[:, :, i * n:(i + 1) * n]
        for dist, acc in ((1, near), (8, far)):
            j = i + dist if i + dist < s.P else i - dist
            o, _ = api.as_partition_attn(q, k, v, s.P, i, [x for x in range(s.P) if x != j])
            acc.append(torch.mean((o - ref) ** 2).item())
    torch.cuda.synchronize()
    del q, k, v, full_o
    torch.cuda.empty_cache()
    m_near, m_far = statistics.mean(near), statistics.mean(far)
    return {"workload": "video_reuse step 0", "mse_drop_neighbour": m_near, "mse_drop_distance_8": m_far,
            "ratio": m_near / m_far if m_far > 0 else None,
            "what": "mean over query partitions of the MSE against full attention when KV partition i+-1, "
                    "or i+-8, is left out"}


def run_boundary(args, device, merged_tflops: float):
    """flux_image with one state emitted per KV partition, so that the ragged
    576-token partitions (4.5 key tiles each) are inside the timed region:
    (a) the attention kernel alone emitting all eight partition states
    (as_partition_attn, compose=0); (b) an as_step whose plan stores every
    pair (the same emission, then the step compose of the eight entries).
    TFLOP/s count the unmasked work only (4*B*H*S*S*d)."""
    from attention_state_reuse_partition_b200 import api
    s = W.spec(WORKLOAD)
    q, k, v = W.flux_qkv(s, device=device)
    flops = attn_flops(s)
    planes = torch.empty((s.P, s.B, s.H, s.S, s.d), device=device)
    plse = torch.empty((s.P, s.B, s.H, s.S), device=device)
    cache = api.AsCache(s.B, s.H, s.S, s.d, s.P, device=device)
    plan = np.full((s.P, s.P), W.PLAN_FRESH_STORE, np.uint8)
    out = torch.empty((s.B, s.H, s.S, s.d), device=device)
    lse = torch.empty((s.B, s.H, s.S), device=device)
    flush = torch.empty(L2_FLUSH_BYTES // 4, device=device, dtype=torch.float32)

    def timed(fn, reps=10):
        for _ in range(3):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for i, (a, b) in enumerate(ev):
            flush.fill_(float(i))
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in ev)

    ms_emit = timed(lambda: api.as_partition_attn(q, k, v, s.P, -1, list(range(s.P)), compose=False,
                                                  out=planes, lse=plse))
    ms_step = timed(lambda: api.as_step(cache, q, k, v, plan, 0, out=out, lse=lse))
    tiles_real = s.P * math.ceil(s.n / 128)
    tiles_merged = math.ceil(s.S / 128)
    del q, k, v, planes, plse, cache, out, lse, flush
    torch.cuda.empty_cache()
    emit_tf = flops / (ms_emit * 1e-3) / 1e12
    return {"workload": f"{WORKLOAD}, one state per KV partition (P={s.P} partitions of {s.n} keys)",
            "attn_emit_ms": round(ms_emit, 4), "attn_emit_tflops": round(emit_tf, 1),
            "step_store_all_ms": round(ms_step, 4),
            "step_store_all_tflops": round(flops / (ms_step * 1e-3) / 1e12, 1),
            "merged_range_tflops": round(merged_tflops, 1),
            "emit_vs_merged": round(emit_tf / merged_tflops, 4),
            "key_tiles_per_query_tile": {"per_partition": tiles_real, "merged": tiles_merged},
            "masked_tile_fraction": round(1 - tiles_merged / tiles_real, 4),
            "extra_bytes_written": (s.P - 1) * s.B * s.H * s.S * (s.d + 1) * 4}


def run_residual(args, device, peaks):
    """The residual codec of the context-parallel exchange on what one rank
    of video_long sends a neighbour per step at 2 ranks (4 partitions of
    K and V: 8 x 81,920 rows of d = 128), against the measured HBM copy
    bandwidth.  Algorithmic bytes per row: encode reads x and base and
    writes codes, scale and base (7 d + 4); decode reads codes, scale and
    base and writes base (5 d + 4).  Link bytes per row: d + 4 coded
    against 2 d raw."""
    from attention_state_reuse_partition_b200 import api
    s = W.spec("video_long")
    rows = 8 * s.B * s.H * s.n
    g = torch.Generator(device=device).manual_seed(91)
    x = torch.randn((rows, s.d), generator=g, device=device).to(torch.bfloat16)
    base = (x.float() + 0.05 * torch.randn((rows, s.d), generator=g, device=device)).to(torch.bfloat16)
    recv = base.clone()
    codes = torch.empty((rows, s.d), dtype=torch.int8, device=device)
    scales = torch.empty((rows,), dtype=torch.float32, device=device)
    enc_base = base.clone()

    def timed(fn, reps=10):
        for _ in range(3):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in ev:
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in ev)

    # the kernels' work does not depend on the values (the base moves
    # towards x from one repetition to the next)
    ms_enc = timed(lambda: api.as_residual_encode(x, enc_base, codes, scales))
    ms_dec = timed(lambda: api.as_residual_decode(codes, scales, recv))
    d = s.d
    enc_b, dec_b = rows * (7 * d + 4), rows * (5 * d + 4)
    del x, base, recv, codes, scales, enc_base
    torch.cuda.empty_cache()
    return {"bound": "hbm", "workload": f"{rows} rows of d = {d} (4 video_long partitions of K and V)",
            "encode_ms": round(ms_enc, 4), "encode_gbs": round(enc_b / (ms_enc * 1e-3) / 1e9, 1),
            "encode_frac": round(enc_b / (ms_enc * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "decode_ms": round(ms_dec, 4), "decode_gbs": round(dec_b / (ms_dec * 1e-3) / 1e9, 1),
            "decode_frac": round(dec_b / (ms_dec * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "peak": peaks["hbm_gbs"], "link_bytes_per_row": {"coded": d + 4, "raw": 2 * d},
            "link_ratio": round((d + 4) / (2 * d), 4)}


def run_video_long(args, device, g=1, cache_dtype="f32", peaks=None, with_oracle=False):
    """Long video trajectory: an anchor step, then three reuse steps (window 4,
    a seeded 10% of reused pairs forced fresh and stored each step).  With
    g > 1 the cache keeps one composed entry per (query partition, group of g
    KV partitions) and a forced pair refreshes its whole group."""
    from attention_state_reuse_partition_b200 import api
    peaks = peaks or load_peaks()
    heads = getattr(args, "video_heads", None)
    s = W.spec("video_long") if heads is None else W.spec("video_long", H=heads)
    cache = api.AsCache(s.B, s.H, s.S, s.d, s.P, device=device, g=g, cache_dtype=cache_dtype)
    NG = (s.P + g - 1) // g
    out = torch.empty((s.B, s.H, s.S, s.d), device=device)
    lse = torch.empty((s.B, s.H, s.S), device=device)
    orc = OracleTrajectory(s, heads=args.oracle_heads[:2], rows_per_partition=args.oracle_rows // 2, g=g,
                           cache_dtype=cache_dtype) if with_oracle else None
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
        fl = 4.0 * s.B * s.H * n_fresh * s.n * s.n * s.d
        rec = step_roofline(a.elapsed_time(b), fl, step_hbm_bytes(s, plan, g, cache_dtype), peaks)
        rec.update({"step": t, "fresh_pairs": n_fresh, "reused_pairs": int((plan == W.PLAN_REUSE).sum()),
                    "stored_pairs": int((plan == W.PLAN_FRESH_STORE).sum()), "reused_entries": reused_entries})
        per_step.append(rec)
        if orc is not None:
            orc.step(t, q, k, v, plan, out_gpu=out)
        last = (q, k, v)
    q, k, v = last
    full_o, _ = api.as_partition_attn(q, k, v, s.P, -1, list(range(s.P)))
    torch.cuda.synchronize()
    mse = torch.mean((out - full_o) ** 2).item()
    cache_gb = cache.buffer.numel() / 1e9
    del cache, full_o, out, lse, last, q, k, v
    torch.cuda.empty_cache()
    name = f"video_long (B=1 H={s.H} S={s.S} P={s.P}, window {s.window}, 4 steps), cache groups of {g}, " \
           f"{cache_dtype} entries"
    res = {"workload": name, "cache_gb": round(cache_gb, 2), "steps": per_step,
           "reuse_mse_vs_full_last_step": mse}
    return res, (orc.summary(name) if orc is not None else None)


def run_cp(args, device, world=None):
    """One rank after another of a context-parallel split of the long video
    trajectory (DiTango review page, Referee Report "Summary": group-wise KV
    transfer; each rank owns a run of query partitions, its cache entries and
    the K/V rows it must compute fresh), on this one GPU: each rank's
    as_step_cp over its Q rows and the compact K/V buffer the exchange would
    give it (gathered here outside the timed region), timed with CUDA events.
    The exchange itself needs several GPUs; its bytes come from the plan
    (per-pair entries: reused pairs move nothing) and, with residual
    compression, from the codec's 132 bytes per 256-byte row."""
    from attention_state_reuse_partition_b200 import api, cp
    world = world or getattr(args, "cp_world", 4)
    heads = getattr(args, "video_heads", None)
    s = W.spec("video_long") if heads is None else W.spec("video_long", H=heads)
    n = s.n
    layout = cp.CpLayout(s.P, world)
    # one untimed small rank step first, so that no rank pays the process's
    # first launches
    sw = W.spec("video_long", H=2, rows=8, cols=16, S=16 * 8 * 16)
    lw = cp.CpLayout(sw.P, world)
    _, qw, kw, vw = next(iter(W.video_trajectory(sw, device=device)))
    pw = W.grouped_plan_for_step(sw, 0, 1).numpy()
    cw = api.AsCache(sw.B, sw.H, sw.S, sw.d, sw.P, device=device, q_first=0, q_count=len(lw.parts(0)))
    kb, vb, sl = cp.gather_kv_local(kw, vw, cp.needed_kv(pw, lw.parts(0)), sw.n)
    api.as_step_cp(cw, qw[:, :, :len(lw.parts(0)) * sw.n].contiguous(), kb, vb, sl, pw, 0)
    torch.cuda.synchronize()
    del cw, kb, vb, qw, kw, vw
    caches = [api.AsCache(s.B, s.H, s.S, s.d, s.P, device=device, q_first=layout.parts(r).start,
                          q_count=len(layout.parts(r))) for r in range(world)]
    per_step = []
    for t, q, k, v in W.video_trajectory(s, device=device):
        plan = W.grouped_plan_for_step(s, t, 1).numpy()
        ms = []
        for r in range(world):
            mine = layout.parts(r)
            rows = slice(mine.start * n, mine.stop * n)
            k_buf, v_buf, slots = cp.gather_kv_local(k, v, cp.needed_kv(plan, mine), n)
            q_r = q[:, :, rows].contiguous()
            out = torch.empty((s.B, s.H, len(mine) * n, s.d), device=device)
            lse = torch.empty((s.B, s.H, len(mine) * n), device=device)
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            api.as_step_cp(caches[r], q_r, k_buf, v_buf, slots, plan, t, out=out, lse=lse)
            b.record()
            torch.cuda.synchronize()
            ms.append(round(a.elapsed_time(b), 3))
            del k_buf, v_buf, q_r, out, lse
        xb = cp.exchange_bytes(plan, layout, s.B, s.H, n, s.d, 2)
        per_step.append({"step": t, "rank_ms": ms, "max_rank_ms": max(ms), "sum_rank_ms": round(sum(ms), 3),
                         "balance": round(sum(ms) / (world * max(ms)), 4),
                         "exchange_bytes": xb["moved"], "all_gather_bytes": xb["all_gather"],
                         "exchange_bytes_residual_coded": int(xb["moved"] * 132 / 256)})
    del caches
    torch.cuda.empty_cache()
    return {"workload": f"video_long (B=1 H={s.H} S={s.S} P={s.P}, window {s.window}, 4 steps), fp32 pair "
                        f"entries, split over {world} ranks of {s.P // world} query partitions",
            "timing": "each rank's as_step_cp alone on this GPU (CUDA events); the exchange is not run",
            "steps": per_step}


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
                                       "planner_grouped", "boundary", "locality", "residual", "cp"], default=None,
                    help="run one secondary workload alone and print its JSON (for profiling)")
    ap.add_argument("--cp-world", type=int, default=4, help="ranks of the context-parallel leg (default 4)")
    ap.add_argument("--compose-rows", type=int, default=None,
                    help="rows of the compose workload (default: all B*H*S rows)")
    ap.add_argument("--reuse-heads", type=int, default=None, help="heads of the reuse workload (default 24)")
    ap.add_argument("--video-heads", type=int, default=None,
                    help="heads of the video_long workloads (default 40; fewer for a small profiling case)")
    ap.add_argument("--reuse-groups", type=int, default=1, help="cache group size of the reuse workload")
    ap.add_argument("--reuse-cache", choices=["f32", "bf16"], default="f32", help="cache entry type of the reuse workload")
    ap.add_argument("--kernel-only", action="store_true",
                    help="time the device-resident step only (no e2e, CPU baseline or secondary workloads)")
    ap.add_argument("--no-oracle", action="store_true", help="skip every oracle (CPU baseline) leg")
    ap.add_argument("--oracle-rows", type=int, default=64,
                    help="query rows per partition of the oracle's video samples (video_long uses half)")
    ap.add_argument("--oracle-heads", type=int, nargs="+", default=[0, 13, 23],
                    help="heads of the oracle's video samples (video_long uses the first two)")
    ap.add_argument("--oracle-compose-rows", type=int, default=8192,
                    help="rows of the oracle's compose-bound sample")
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
        peaks = load_peaks()
        fn = {"compose": lambda a, dev: run_compose(a, dev, peaks)[0],
              "reuse": lambda a, dev: run_reuse(a, dev, peaks)[0],
              "video_long": lambda a, dev: run_video_long(a, dev, peaks=peaks)[0],
              "video_long_grouped": lambda a, dev: run_video_long(a, dev, g=4, cache_dtype="bf16", peaks=peaks)[0],
              "planner": run_planner,
              "planner_grouped": lambda a, dev: run_planner(a, dev, g=4, cache_dtype="bf16"),
              "boundary": lambda a, dev: run_boundary(a, dev, float("nan")),
              "residual": lambda a, dev: run_residual(a, dev, peaks),
              "locality": run_locality,
              "cp": run_cp}[args.only]
        print(json.dumps({"only": args.only, **fn(args, device)}))
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    peaks = load_peaks()
    res, (q, k, v, s) = run_own(args, rank, world, device)
    ms = res["ms_max"]
    achieved = res["flops"] / (res["ms"] * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    roofline = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": measured_traffic("attn_tc_kernel<128>"),
                "kernel": "attn_tc_kernel<128>", "peak_source": f"{peaks['source']} bf16 burst",
                # the kernel is timed after a second of full load, at the power-capped clock
                "peak_sustained": peaks["bf16_tflops_sustained"],
                "frac_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4)}
    cpu = None
    legs = {}
    full = not args.no_secondary and not args.kernel_only and world == 1
    oracle_on = rank == 0 and world == 1 and not args.kernel_only and not args.no_oracle
    if oracle_on:
        heads = list(range(s.H))
        dt, fl = oracle_sample(s, q, k, v, s.n, heads)
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
               "sample": f"the whole {WORKLOAD} step (all {s.S} query rows x {s.H} heads, all {s.S} keys), "
                         f"float64, one pass ({dt:.1f} s)"}
    del q, k, v
    torch.cuda.empty_cache()
    if full:
        roofline["compose"], legs["compose_bound"] = run_compose(args, device, peaks, with_oracle=oracle_on)
        steps = {}
        steps["video_reuse"], legs["video_reuse"] = run_reuse(args, device, peaks, with_oracle=oracle_on)
        a2 = argparse.Namespace(**{**vars(args), "reuse_groups": 4, "reuse_cache": "bf16"})
        steps["video_reuse_g4_bf16"], _ = run_reuse(a2, device, peaks)
        steps["video_long"], legs["video_long"] = run_video_long(args, device, peaks=peaks, with_oracle=oracle_on)
        steps["video_long_g4_bf16"], _ = run_video_long(args, device, g=4, cache_dtype="bf16", peaks=peaks)
        steps["planner"] = run_planner(args, device)
        steps["planner_g4_bf16"] = run_planner(args, device, g=4, cache_dtype="bf16")
        roofline["steps"] = steps
        roofline["partition_boundary"] = run_boundary(args, device, achieved)
        roofline["residual_codec"] = run_residual(args, device, peaks)
        roofline["locality"] = run_locality(args, device)
        roofline["context_parallel"] = run_cp(args, device)
    if cpu is not None and legs:
        cpu["legs"] = {k: v for k, v in legs.items() if v is not None}

    line = {
        "metric": METRIC, "value": round(res["value"], 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT, "global_batch": world, "seq_len": s.S,
                   "parallelism": f"replicas{world}" if world > 1 else "single", "l2": "flushed (256 MiB write) "
                   "before every timed step"},
        "roofline": roofline,
        "e2e": res["e2e"], "clocks": res["clocks"], "gpu_launches": res["gpu_launches"],
    }
    if line["e2e"] is None:
        del line["e2e"]
    if cpu:
        line["cpu_baseline"] = cpu
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
