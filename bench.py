"""Benchmark: streaming block-causal sink + sliding-window attention at 720p on B200.

One step = one steady-state chunk of the 720p stream: two denoise-step forwards (attention of
the chunk's 3180 queries over condition + sink + window + current keys) and the commit of the
chunk into the ring cache (append/evict copy + visibility-table rebuild).  The metric is the
attention TFLOP/s over the timed steps (algorithmic FLOPs: 4 * B * H * T * N_vis * d per
forward, visible keys only), with ms per chunk and the fraction of the measured dense bf16 peak.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference] [--config 720p]

Under torchrun (N > 1) every rank runs an independent replica (the path has no exchange step);
the time is the max over ranks and the value sums all ranks' FLOPs.
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

import torch  # noqa: E402

from block_causal_attention_sliding_b200 import synth  # noqa: E402
from block_causal_attention_sliding_b200.configs import WORKLOADS  # noqa: E402

METRIC = "attention TFLOP/s and ms/chunk at 720p, % of B200 dense BF16 peak"
UNIT = "TFLOP/s"
L2_BYTES = 126 * 2 ** 20


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"bf16_tflops": float(d["bf16_tflops"]), "bf16_tflops_sustained": float(d["bf16_tflops_sustained"]),
                "hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    except Exception:
        return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


# DRAM traffic of one attention launch from an ncu capture of the 720p steady-state forward
# (dram__bytes_read.sum + dram__bytes_write.sum).  It is reported only while the kernel's
# sources hash to what was captured; any change to them makes the figure stale (null).
PROFILED_TRAFFIC = {
    ("720p", "persistent"): {"bytes": 231_243_520 + 16_276_480,
                             "sources_sha256": "cfb4ae54ebd3c2e1fcf495ccef98bb143511a58ffa0a2a13b7285f0bdb6a6355"},
}
KERNEL_SOURCES = ("attn_persistent.cu", "persist_sched.cuh", "attn_common.cuh", "ptx.cuh", "swattn_internal.h")


def _profiled_traffic(workload: str, schedule: str):
    import hashlib
    rec = PROFILED_TRAFFIC.get((workload, schedule))
    if rec is None:
        return None
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        try:
            with open(os.path.join(ROOT, "block_causal_attention_sliding_b200", "csrc", name), "rb") as f:
                h.update(f.read())
        except OSError:
            return None
    return rec["bytes"] if h.hexdigest() == rec["sources_sha256"] else None


# ---------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            uuid = None
        self.target = uuid

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.target:
            cmd += ["-i", self.target]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self._t.join(timeout=2)
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power)}


# ---------------------------------------------------------------------------- distributed plumbing

def _dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _init_dist(world, backend="nccl", timeout_s=120):
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def reduce_max_time(dist, seconds: float, device) -> float:
    """Max over ranks of a device-timed interval (seconds)."""
    if dist is None:
        return seconds
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(dist, elapsed_s: float, flops_per_rank: float, device):
    """Whole-job throughput of independent replicas: every rank's FLOPs over the slowest rank's
    device time.  Returns (t_max seconds, TFLOP/s)."""
    world = 1 if dist is None else dist.get_world_size()
    t_max = reduce_max_time(dist, elapsed_s, device)
    return t_max, flops_per_rank * world / t_max / 1e12


def barrier(dist, device):
    if dist is not None:
        dist.barrier(device_ids=[device.index] if device.type == "cuda" else None)


# ---------------------------------------------------------------------------- CPU baseline (oracle)

def host_cpu() -> dict:
    """The host's CPU model string and logical core count."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count()}


def oracle_inputs(wl, k: int) -> dict:
    """The inputs of one forward of active chunk k (condition K/V, the visible history, Q and
    the current K/V), drawn once and held as float32 host arrays (bf16 values, exact), the form
    the oracle takes without copying."""
    import oracle

    def f32(t):
        return t.float().numpy()

    Kc, Vc = synth.cond_inputs(wl)
    hist_K = [None] * k
    hist_V = [None] * k
    for c in range(k):
        if oracle.visible(k, wl.W, wl.sink, c):
            _, K, V = synth.chunk_inputs(wl, c, wl.steps - 1)
            hist_K[c], hist_V[c] = f32(K), f32(V)
    Q, K, V = synth.chunk_inputs(wl, k, 0)
    return {"Kc": f32(Kc), "Vc": f32(Vc), "hist_K": hist_K, "hist_V": hist_V, "Q": f32(Q), "K_cur": f32(K),
            "V_cur": f32(V)}


def cpu_baseline(wl, k: int, rows: int | None, repeats: int = 1, inputs: dict | None = None):
    """Time the FP64 oracle on one forward of active chunk k: `rows` query rows (None: all T
    rows, i.e. the full forward) for every head, over all visible keys (inputs drawn here unless
    given by oracle_inputs).  Returns (TFLOP/s, seconds, flops, threads)."""
    import numpy as np

    import oracle
    oracle.build()
    x = inputs if inputs is not None else oracle_inputs(wl, k)
    sel = None if rows is None else np.linspace(0, wl.T - 1, rows).astype(np.int32)
    n_rows = wl.T if rows is None else rows
    nvis = wl.n_vis(k)
    flops = 4.0 * wl.B * wl.H * n_rows * nvis * wl.d
    best = None
    for _ in range(repeats):
        t0 = time.perf_counter()
        oracle.attention(H=wl.H, d=wl.d, T=wl.T, n_cond=wl.n_cond, W=wl.W, sink=wl.sink, k=k, rows=sel, **x)
        dt = time.perf_counter() - t0
        best = dt if best is None else min(best, dt)
    return flops / best / 1e12, best, flops, oracle.num_threads()


def cpu_stream_ms(wl) -> float:
    """Time the FP64 oracle over a whole stream of a small workload, every chunk (each chunk's
    forwards with all rows, then its commit to the history): ms per chunk."""
    import oracle
    oracle.build()
    Kc, Vc = synth.cond_inputs(wl)
    hist_K, hist_V = [], []
    t0 = time.perf_counter()
    for k in range(wl.chunks):
        for step in range(wl.steps):
            Q, K, V = synth.chunk_inputs(wl, k, step)
            oracle.attention(H=wl.H, d=wl.d, T=wl.T, n_cond=wl.n_cond, W=wl.W, sink=wl.sink, k=k, Kc=Kc, Vc=Vc,
                             hist_K=hist_K, hist_V=hist_V, Q=Q, K_cur=K, V_cur=V)
        hist_K.append(K)
        hist_V.append(V)
    return (time.perf_counter() - t0) * 1e3 / wl.chunks


def cpu_baseline_record(wl, k: int) -> dict:
    """The oracle as it stands on this host's cores, on full rows: one whole steady-state forward
    of the benchmarked workload (the line's value), plus every chunk of the tiny workload and one
    whole 480p forward for context."""
    v, secs, fl, thr = cpu_baseline(wl, k, rows=None)
    rec = {"value": v, "unit": UNIT, "cores": thr, "kind": "oracle",
           "sample": f"full rows: one whole steady-state {wl.name} forward (k={k}), all {wl.T} query rows x "
                     f"{wl.B * wl.H} heads over all {wl.n_vis(k)} visible keys, FP64 "
                     f"({fl / 1e9:.1f} GFLOP in {secs:.1f} s, {thr} OpenMP threads)",
           "ms_per_forward": round(secs * 1e3, 1), "ms_per_chunk": round(secs * 1e3 * wl.steps, 1)}
    rec.update(host_cpu())
    other = {}
    try:
        other["tiny_ms_per_chunk_all_chunks"] = round(cpu_stream_ms(WORKLOADS["tiny"]), 3)
        w4 = WORKLOADS["480p"]
        v4, s4, f4, _ = cpu_baseline(w4, w4.steady_k(), rows=None)
        other["480p_ms_per_forward_full_rows"] = round(s4 * 1e3, 1)
        other["480p_TFLOP/s"] = v4
    except Exception as e:   # context only; never blocks the line
        other["error"] = str(e)
    rec["other_workloads"] = other
    return rec


# ---------------------------------------------------------------------------- the workload

def bench_config(wl, pool: int, world: int) -> dict:
    """The `config` object of the JSON line: the workload and the timing protocol, the same for
    both arms."""
    k = wl.steady_k()
    set_mib = 3 * wl.B * wl.T * wl.H * wl.d * 2 * wl.steps / 2 ** 20
    return {"workload": wl.name, "B": wl.B, "H": wl.H, "d": wl.d, "T": wl.T, "n_cond": wl.n_cond,
            "W": wl.W, "sink": wl.sink, "N_vis": wl.n_vis(k),
            "step": "one steady-state chunk: 2 forwards + append/evict + table",
            "gflop_per_forward": round(wl.flops_forward(k) / 1e9, 2),
            "l2": f"inputs larger than L2: {pool} resident input sets of {set_mib:.0f} MiB plus the cache, "
                  f"cycled per step",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


# ---------------------------------------------------------------------------- the CUDA arm

def run_cuda(args, wl, world, rank, local):
    from block_causal_attention_sliding_b200.api import SlidingWindowAttention

    dist = _init_dist(world)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peaks = _peaks()

    h = SlidingWindowAttention(B=wl.B, H=wl.H, d=wl.d, T=wl.T, W=wl.W, n_cond=wl.n_cond, sink=wl.sink,
                               out_dtype=torch.bfloat16, schedule=args.schedule, device=dev)
    Kc, Vc = synth.cond_inputs(wl, seed=rank, device=dev)
    h.set_cond(Kc, Vc)
    # a pool of distinct input sets, resident in HBM; together with the 160 MB cache the
    # working set of every step is far larger than the 126 MB L2
    pool = []
    for i in range(args.pool):
        per_step = [synth.chunk_inputs(wl, 1000 + i, s, seed=rank, device=dev) for s in range(wl.steps)]
        pool.append(per_step)
    outs = [torch.empty((wl.B, wl.T, wl.H, wl.d), dtype=torch.bfloat16, device=dev) for _ in range(wl.steps)]

    def step(i, ev=None):
        inputs = pool[i % len(pool)]
        for s, (Q, K, V) in enumerate(inputs):
            if ev is not None:
                ev[2 * s].record(stream)
            h.forward(Q, K, V, out=outs[s])
            if ev is not None:
                ev[2 * s + 1].record(stream)
        Q, K, V = inputs[-1]
        h.append_chunk(K, V)

    # reach the steady state (sink + full window visible), untimed
    for i in range(wl.steady_k()):
        step(i)
    k_start = wl.steady_k()
    torch.cuda.synchronize(dev)
    assert h.status() == 0
    # The clock sampler starts before the warm-up, so the warm-up runs straight into the timed
    # region: no idle gap before it (work started after an idle gap runs several per cent faster
    # for its first tens of milliseconds on this part, which would flatter a short run).  The
    # warm-up is the W steps asked for, extended to at least 0.2 s of device work.
    clocks = ClockSampler(local)
    clocks.start()
    t_warm = time.perf_counter()
    i = 0
    while i < args.warmup or time.perf_counter() - t_warm < 0.2:
        step(i)
        i += 1
        if i % 16 == 0:
            torch.cuda.synchronize(dev)   # keep the host's clock in step with the device's
    warm_steps = i

    # timed region: K steps, per-forward events for the attention kernel's own time
    fwd_events = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * wl.steps)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist, dev)
    torch.cuda.synchronize(dev)
    assert h.status() == 0
    start.record(stream)
    for i in range(args.steps):
        step(i, fwd_events[i])
    end.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    barrier(dist, dev)
    elapsed = start.elapsed_time(end) / 1e3
    fwd_ms = [fwd_events[i][2 * s].elapsed_time(fwd_events[i][2 * s + 1])
              for i in range(args.steps) for s in range(wl.steps)]
    # per chunk: from one step's first forward to the next step's (the last one to `end`)
    chunk_ms = [fwd_events[i][0].elapsed_time(fwd_events[i + 1][0]) for i in range(args.steps - 1)]
    chunk_ms.append(fwd_events[-1][0].elapsed_time(end))
    status = h.status()

    flops_fwd = wl.flops_forward(k_start)
    flops_step = wl.steps * flops_fwd
    t_max, value = aggregate(dist, elapsed, flops_step * args.steps, dev)
    fwd_avg = sum(fwd_ms) / len(fwd_ms) / 1e3
    achieved = flops_fwd / fwd_avg / 1e12

    # ---- e2e: the same steps through the public API with host buffers (pinned), copies timed.
    # Pipelined as on the pages (host copies overlapped with device compute on other streams):
    # step i's inputs go up on one copy stream while step i-1 computes, and step i-1's outputs
    # come down on another; two sets of device buffers alternate, ordered by events.
    host_in = [[t.cpu().pin_memory() for t in per_step] for per_step in pool[0]]
    host_out = [[torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs] for _ in range(2)]
    dev_in = [[[torch.empty_like(t) for t in per_step] for per_step in pool[0]] for _ in range(2)]
    dev_out = [[torch.empty_like(o) for o in outs] for _ in range(2)]
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    up_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    down_done = [torch.cuda.Event() for _ in range(2)]
    e2e_steps = max(3, min(args.steps, 50))

    def e2e_step(i):
        b = i % 2
        up.wait_event(comp_done[b])                  # buffer set b no longer read by step i - 2
        with torch.cuda.stream(up):
            for s in range(wl.steps):
                for dst, src in zip(dev_in[b][s], host_in[s]):
                    dst.copy_(src, non_blocking=True)
        up_done[b].record(up)
        stream.wait_event(up_done[b])
        stream.wait_event(down_done[b])              # step i - 2's outputs have come down
        for s in range(wl.steps):
            Q, K, V = dev_in[b][s]
            h.forward(Q, K, V, out=dev_out[b][s], stream=stream)
        h.append_chunk(dev_in[b][-1][1], dev_in[b][-1][2], stream=stream)
        comp_done[b].record(stream)
        down.wait_event(comp_done[b])
        with torch.cuda.stream(down):
            for s in range(wl.steps):
                host_out[b][s].copy_(dev_out[b][s], non_blocking=True)
        down_done[b].record(down)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_stream(stream)
    down.wait_stream(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_stream(up)
    stream.wait_stream(down)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_t, e2e_value = aggregate(dist, e0.elapsed_time(e1) / 1e3, flops_step * e2e_steps, dev)
    bi = sum(t.numel() * t.element_size() for per_step in host_in for t in per_step)
    bo = sum(t.numel() * t.element_size() for t in host_out[0])
    link = host_link_peaks(host_in, dev_in[0], host_out[0], dev_out[0], up, down, dev)
    e2e_ms = e2e_t / e2e_steps * 1e3
    bound_ms = max(bi / link["h2d_gbs"], bo / link["d2h_gbs"]) / 1e6
    link.update({"bound_ms_per_step": round(bound_ms, 4), "frac": round(bound_ms / e2e_ms, 4),
                 "note": "the step's copies alone at the measured pinned-host link rates (both directions "
                         "run at once); frac = that time / e2e ms per step"})

    # ---- side measurements (untimed for the metric): append/evict and the split-K path
    paths = {}
    ws_bytes = h.workspace_bytes()
    sched = h.schedule_for()   # the schedule the timed forwards ran with
    if rank == 0:
        paths = side_paths(h, wl, pool, dev, stream, peaks)
        paths["chunk_ms"] = {"median": round(statistics.median(chunk_ms), 4),
                             "p95": round(sorted(chunk_ms)[min(len(chunk_ms) - 1, int(0.95 * len(chunk_ms)))], 4),
                             "chunks": len(chunk_ms)}
        if not args.no_extra and world == 1:   # side measurements at N = 1 only: all N GPUs are held
            h.close()
            h = None
            paths["long_horizon"] = long_horizon(args, dev, stream, pool)
            paths["commit"] = commit_path(args, dev, stream, pool)
            paths["layers"] = layers_path(args, dev, stream, peaks=peaks)
            paths["fp8"] = fp8_path(args, dev, stream, peaks)
            paths["workloads"] = other_workloads(args, dev, stream, peaks)

    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:   # the CPU baseline is an N = 1 figure
            try:
                cpu = cpu_baseline_record(wl, k_start)
            except Exception as e:   # the baseline never blocks the GPU line
                cpu = {"value": None, "unit": UNIT, "cores": None, "kind": "oracle", "sample": f"failed: {e}"}
        peak = peaks["bf16_tflops"]
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(t_max / args.steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": bench_config(wl, args.pool, world),
            "warmup_steps_run": warm_steps,
            "schedule": sched,
            "workspace_bytes": ws_bytes,
            "pct_of_peak": round(100.0 * value / world / peak, 2),
            "roofline": {"bound": "tensor",
                         "kernel": {"persistent": "attn_persistent_kernel<128, false, false, false>", "tri": "attn_tri_kernel<128, false, false>",
                                    "grid": "attn_fwd_kernel<128,2>", "pair": "attn_pair_kernel"}[sched],
                         "achieved": round(achieved, 2),
                         # the launches are timed inside a continuous, power-capped stream of chunk
                         # steps (no idle gap before the timed region), so the sustained GEMM figure
                         # is the applicable peak; the burst one is given beside it
                         "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                         "frac": round(achieved / peaks["bf16_tflops_sustained"], 4),
                         "traffic": _profiled_traffic(wl.name, sched),
                         "peak_source": f"{peaks['source']} bf16_tflops_sustained",
                         "frac_of_burst": round(achieved / peak, 4), "burst_peak": peak,
                         "launch_ms_avg": round(fwd_avg * 1e3, 4)},
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
                    "steps": e2e_steps, "ms_per_step": round(e2e_t / e2e_steps * 1e3, 4),
                    "pipelining": "uploads, compute and downloads on three streams, two buffer sets",
                    "link_roofline": link},
            "gpu_launches": args.steps * (wl.steps + 1),   # per step: the forwards and one commit launch
            "clocks": clk,
            "device_status": status,
            "paths": paths,
        }
        print(json.dumps(line), flush=True)
    if h is not None:
        h.close()
    if dist is not None:
        dist.destroy_process_group()


def long_horizon(args, dev, stream, pool):
    """The 225-chunk 720p stream.
    (1) Drift: on a fresh handle, the per-chunk device time (2 forwards + append) of the whole
    stream, with the host only enqueueing; drift = mean time of chunks 200-224 over chunks 5-29,
    minus 1.  The stream is enqueued right behind a few seconds of the same chunk step on another
    handle, so that the device never idles: after an idle gap the part runs its first ~60 ms
    measurably faster (its power controller allows a short burst, which NVML's sampled SM clock
    does not show), and that would put the early window, not the stream length, in the ratio.
    The same ratio after an idle gap ("cold start") is given beside it.
    (2) On another fresh handle, the device memory in use (allocator and driver view) after every
    chunk, which must not change.
    (3) A same-work control: one handle advanced to chunk 5 and one to chunk 200 run their chunks
    alternately; from chunk W + 1 on the visible keys are the same, so this shows that nothing
    else in the handle slows down with stream length."""
    from block_causal_attention_sliding_b200.api import SlidingWindowAttention
    wl = WORKLOADS["long720p"]

    def handle():
        hx = SlidingWindowAttention(B=wl.B, H=wl.H, d=wl.d, T=wl.T, W=wl.W, n_cond=wl.n_cond, sink=wl.sink,
                                    out_dtype=torch.bfloat16, schedule=args.schedule, device=dev)
        hx.set_cond(Kc, Vc)
        return hx

    Kc, Vc = synth.cond_inputs(wl, seed=7, device=dev)
    outs = [torch.empty((wl.B, wl.T, wl.H, wl.d), dtype=torch.bfloat16, device=dev) for _ in range(wl.steps)]

    def chunk(hx, c):
        inputs = pool[c % len(pool)]
        for s, (Q, K, V) in enumerate(inputs):
            hx.forward(Q, K, V, out=outs[s])
        hx.append_chunk(inputs[-1][1], inputs[-1][2])

    def timed_stream(hx):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(wl.chunks + 1)]
        for c in range(wl.chunks):
            ev[c].record(stream)
            chunk(hx, c)
        ev[wl.chunks].record(stream)
        torch.cuda.synchronize(dev)
        return [ev[c].elapsed_time(ev[c + 1]) for c in range(wl.chunks)]

    def drift_of(ms):
        return (sum(ms[200:225]) / 25) / (sum(ms[5:30]) / 25) - 1.0

    # (1a) cold start: a fresh stream after the device has idled for two seconds
    torch.cuda.synchronize(dev)
    hc = handle()
    time.sleep(2.0)
    cms = timed_stream(hc)
    hc.close()
    # (1b) the device kept busy: warm-up chunk steps, at most ~100 queued at a time, and the timed
    # stream enqueued right behind them
    hw, h = handle(), handle()
    torch.cuda.synchronize(dev)
    marks = []
    t_end = time.perf_counter() + args.warm_seconds
    while time.perf_counter() < t_end:
        for c in range(50):
            chunk(hw, c)
        marks.append(torch.cuda.Event())
        marks[-1].record(stream)
        if len(marks) >= 2:
            marks[-2].synchronize()
    ms = timed_stream(h)
    hw.close()
    status = h.status()
    h.close()
    steady = ms[wl.W + 1:]
    # (2) memory pass on a fresh handle: allocator and driver view after every chunk
    h = handle()
    alloc, free = [], []
    for c in range(wl.chunks):
        chunk(h, c)
        alloc.append(torch.cuda.memory_allocated(dev))
        free.append(torch.cuda.mem_get_info(dev)[0])
    torch.cuda.synchronize(dev)
    res = {"chunks": wl.chunks, "drift": round(drift_of(ms), 4), "target": "<= 0.02",
           "protocol": f"sequential 225-chunk stream on a fresh handle, enqueued behind {args.warm_seconds:.0f} s "
                       "of the same chunk step on another handle (no idle gap)",
           "ms_chunks_5_29": round(sum(ms[5:30]) / 25, 4), "ms_chunks_200_224": round(sum(ms[200:225]) / 25, 4),
           "ms_median": round(statistics.median(steady), 4),
           "ms_p95": round(sorted(steady)[int(0.95 * (len(steady) - 1))], 4),
           "drift_cold_start": round(drift_of(cms), 4),
           "cold_start_ms_per_25_chunks": [round(sum(cms[i:i + 25]) / 25, 4) for i in range(0, wl.chunks, 25)],
           "allocated_bytes_constant": len(set(alloc)) == 1, "driver_free_bytes_constant": len(set(free)) == 1,
           "workspace_bytes": h.workspace_bytes(), "status": status | h.status()}
    h.close()
    # (3) same-work control: chunks 5-29 and 200-224 interleaved on two handles
    hs = []
    for start in (5, 200):
        hx = handle()
        for _ in range(start):
            hx.append_chunk(pool[0][-1][1], pool[0][-1][2])
        hs.append(hx)
    t_ms = [[], []]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    for c in range(25):
        for which, hx in enumerate(hs):
            e0.record(stream)
            chunk(hx, c)
            e1.record(stream)
            e1.synchronize()
            t_ms[which].append(e0.elapsed_time(e1))
    ctrl = (sum(t_ms[1]) / 25) / (sum(t_ms[0]) / 25) - 1.0
    res["same_work_control"] = {"ratio_minus_1": round(ctrl, 4), "ms_chunks_5_29": round(sum(t_ms[0]) / 25, 4),
                                "ms_chunks_200_224": round(sum(t_ms[1]) / 25, 4),
                                "status": max(hx.status() for hx in hs)}
    for hx in hs:
        hx.close()
    return res


def commit_path(args, dev, stream, pool):
    """The steady-state 720p chunk step with the clean pass committing its own K/V
    (forward, forward_commit) against forward, forward, append_chunk, on one handle created with
    commit_in_forward (the append path writes the same slots).  Chunks alternate between the two
    forms so both see the same clock."""
    from block_causal_attention_sliding_b200.api import SlidingWindowAttention
    wl = WORKLOADS["720p"]
    h = SlidingWindowAttention(B=wl.B, H=wl.H, d=wl.d, T=wl.T, W=wl.W, n_cond=wl.n_cond, sink=wl.sink,
                               out_dtype=torch.bfloat16, schedule=args.schedule, commit_in_forward=True,
                               device=dev)
    Kc, Vc = synth.cond_inputs(wl, seed=9, device=dev)
    h.set_cond(Kc, Vc)
    outs = [torch.empty((wl.B, wl.T, wl.H, wl.d), dtype=torch.bfloat16, device=dev) for _ in range(wl.steps)]
    for c in range(wl.W + 2):
        (Q0, K0, V0), (Q1, K1, V1) = pool[c % len(pool)]
        h.forward(Q0, K0, V0, out=outs[0])
        h.forward_commit(Q1, K1, V1, out=outs[1])
    reps = 30
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4 * reps)]
    torch.cuda.synchronize(dev)
    for r in range(reps):
        (Q0, K0, V0), (Q1, K1, V1) = pool[r % len(pool)]
        ev[4 * r].record(stream)
        h.forward(Q0, K0, V0, out=outs[0])
        h.forward_commit(Q1, K1, V1, out=outs[1])
        ev[4 * r + 1].record(stream)
        ev[4 * r + 2].record(stream)
        h.forward(Q0, K0, V0, out=outs[0])
        h.forward(Q1, K1, V1, out=outs[1])
        h.append_chunk(K1, V1)
        ev[4 * r + 3].record(stream)
    torch.cuda.synchronize(dev)
    fused = statistics.median(ev[4 * r].elapsed_time(ev[4 * r + 1]) for r in range(reps))
    plain = statistics.median(ev[4 * r + 2].elapsed_time(ev[4 * r + 3]) for r in range(reps))
    res = {"chunk_ms_fused_commit": round(fused, 4), "chunk_ms_forward_append": round(plain, 4),
           "saved_us": round((plain - fused) * 1e3, 1), "chunks_each": reps, "status": h.status(),
           "schedule": h.schedule_for()}
    h.close()
    return res


def fp8_path(args, dev, stream, peaks):
    """The steady-state forward with e4m3 queries and keys (S on kind::f8f6f4, e4m3 K cache) and
    bf16 V, and with e4m3 V as well (e4m3 V cache, P in e4m3, PV on kind::f8f6f4), against the
    bf16 forward of the same draws, each timed alone: at 720p (the persistent kernel) with the
    split-K path beside it, and at 480p (the three-buffer kernel)."""
    from block_causal_attention_sliding_b200.api import SlidingWindowAttention
    sc = synth.FP8_SCALE
    res = {}
    # read (not written) to flush L2: a written buffer would leave dirty lines whose write-backs
    # land inside the timed launch
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)   # 256 MiB, twice the L2
    for wname in ("720p", "480p"):
        wl = WORKLOADS[wname]
        res_w = {}
        for name, fp8, v8 in (("bf16", False, False), ("e4m3_qk", True, False), ("e4m3_qkv", True, True)):
            h = SlidingWindowAttention(B=wl.B, H=wl.H, d=wl.d, T=wl.T, W=wl.W, n_cond=wl.n_cond, sink=wl.sink,
                                       out_dtype=torch.bfloat16, qk_fp8=fp8, q_scale=sc, k_scale=sc,
                                       pv_fp8=v8, v_scale=sc, device=dev)
            if fp8:
                Kc, Vc = synth.cond_inputs_fp8(wl, seed=11, device=dev, v8=v8)
                Q, K, V = synth.chunk_inputs_fp8(wl, 0, 0, seed=11, device=dev, v8=v8)
            else:
                Kc, Vc = synth.cond_inputs(wl, seed=11, device=dev)
                Q, K, V = synth.chunk_inputs(wl, 0, 0, seed=11, device=dev)
            h.set_cond(Kc, Vc)
            for _ in range(wl.steady_k()):
                h.append_chunk(K, V)
            out = torch.empty((wl.B, wl.T, wl.H, wl.d), dtype=torch.bfloat16, device=dev)
            for _ in range(3):
                h.forward(Q, K, V, out=out)
            torch.cuda.synchronize(dev)
            reps = 50
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(torch.cuda.current_stream())
            for _ in range(reps):
                h.forward(Q, K, V, out=out)
            e1.record(torch.cuda.current_stream())
            torch.cuda.synchronize(dev)
            t = e0.elapsed_time(e1) / 1e3 / reps
            tf = wl.flops_forward(wl.steady_k()) / t / 1e12
            kc, vc = h.cache_views()
            rec = {"ms_per_forward": round(t * 1e3, 4), "TFLOP/s": round(tf, 2), "schedule": h.schedule_for(),
                   "workspace_bytes": h.workspace_bytes(),
                   "cache_bytes": kc.numel() * kc.element_size() + vc.numel() * vc.element_size()}
            if wname == "720p":
                # split-K with 128 queries: HBM-bound, so the e4m3 cache shows up as time.  The e4m3
                # key set fits in L2, so L2 is flushed before every launch and each launch timed alone.
                q = Q[:, :128].contiguous()
                o = torch.empty((wl.B, 128, wl.H, wl.d), dtype=torch.bfloat16, device=dev)
                for _ in range(3):
                    h.forward(q, K, V, out=o)
                ts = []
                for _ in range(20):
                    flush.amax()
                    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a0.record(torch.cuda.current_stream())
                    h.forward(q, K, V, out=o)
                    a1.record(torch.cuda.current_stream())
                    torch.cuda.synchronize(dev)
                    ts.append(a0.elapsed_time(a1) / 1e3)
                tq = statistics.median(ts)
                kv_bytes = wl.B * wl.H * wl.n_vis(wl.steady_k()) * wl.d * (K.element_size() + V.element_size())
                rec["split_k_128"] = {"us": round(tq * 1e6, 2), "GB/s": round(kv_bytes / tq / 1e9, 1),
                                      "frac_hbm": round(kv_bytes / tq / 1e9 / peaks["hbm_gbs"], 3), "bytes": kv_bytes,
                                      "timing": "L2 flushed by a 256 MiB read before each launch, median of 20"}
            rec["status"] = h.status()
            res_w[name] = rec
            h.close()
        res[wname] = res_w
    res["note"] = ("e4m3 inputs with per-tensor scale 2^-4; e4m3_qk: bf16 V and P; e4m3_qkv: e4m3 V and P; "
                   "FLOPs counted as for bf16")
    return res


def layers_path(args, dev, stream, n_layers=8, peaks=None):
    """A chunk step of an n-layer model at 480p: each layer (one handle, its own cache) runs its
    two forwards, then every layer commits the chunk.  Timed with per-layer appends, with one
    batched append for all layers, and with the whole step replayed from a CUDA graph; and the
    batched commit alone (HBM-bound: every layer's K/V read once and written once)."""
    from block_causal_attention_sliding_b200.api import SlidingWindowAttention, append_chunk_batched
    wl = WORKLOADS["480p"]
    hs, ins, outs = [], [], []
    for l in range(n_layers):
        h = SlidingWindowAttention(B=wl.B, H=wl.H, d=wl.d, T=wl.T, W=wl.W, n_cond=wl.n_cond, sink=wl.sink,
                                   out_dtype=torch.bfloat16, schedule=args.schedule, device=dev)
        Kc, Vc = synth.cond_inputs(wl, seed=20 + l, device=dev)
        h.set_cond(Kc, Vc)
        hs.append(h)
        ins.append([synth.chunk_inputs(wl, 3, s, seed=20 + l, device=dev) for s in range(wl.steps)])
        outs.append([torch.empty((wl.B, wl.T, wl.H, wl.d), dtype=torch.bfloat16, device=dev) for _ in range(wl.steps)])

    def forwards():
        for l in range(n_layers):
            for s in range(wl.steps):
                hs[l].forward(*ins[l][s], out=outs[l][s])

    def step_each():
        forwards()
        for l in range(n_layers):
            hs[l].append_chunk(ins[l][-1][1], ins[l][-1][2])

    def step_batched():
        forwards()
        append_chunk_batched(hs, [x[-1][1] for x in ins], [x[-1][2] for x in ins])

    for _ in range(wl.steady_k()):
        step_batched()
    reps = 20

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(torch.cuda.current_stream())
        for _ in range(reps):
            fn()
        e1.record(torch.cuda.current_stream())
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / reps

    t_each = timed(step_each)
    t_batched = timed(step_batched)
    # the batched commit alone, alternating each layer's two (K, V) sets: 2 x 8 x 11.5 MB of
    # sources, more than L2 holds, so the copies read from HBM
    flip = [0]

    def commit_only():
        s = flip[0] % wl.steps
        flip[0] += 1
        append_chunk_batched(hs, [x[s][1] for x in ins], [x[s][2] for x in ins])

    t_commit = timed(commit_only)
    commit_bytes = 2 * 2 * n_layers * ins[0][0][1].numel() * ins[0][0][1].element_size()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            step_batched()
    torch.cuda.current_stream().wait_stream(side)
    t_graph = timed(graph.replay)
    status = max(h.status() for h in hs)
    del graph
    for h in hs:
        h.close()
    commit = {"us": round(t_commit * 1e3, 2), "GB/s": round(commit_bytes / t_commit / 1e6, 1), "bytes": commit_bytes}
    if peaks:
        commit["frac_hbm"] = round(commit_bytes / t_commit / 1e6 / peaks["hbm_gbs"], 3)
    return {"workload": wl.name, "layers": n_layers, "ms_per_chunk_appends_each": round(t_each, 4),
            "ms_per_chunk_batched_append": round(t_batched, 4), "ms_per_chunk_graph": round(t_graph, 4),
            "batched_commit_alone": commit, "status": status}


def other_workloads(args, dev, stream, peaks):
    """Steady-state forward throughput of the other attention workloads (480p, stress): the
    stream is advanced to the steady state (sink and full window visible), then forwards are
    timed with CUDA events."""
    from block_causal_attention_sliding_b200.api import SlidingWindowAttention
    res = {}
    for name in ("480p", "stress"):
        wl = WORKLOADS[name]
        h = SlidingWindowAttention(B=wl.B, H=wl.H, d=wl.d, T=wl.T, W=wl.W, n_cond=wl.n_cond, sink=wl.sink,
                                   out_dtype=torch.bfloat16, schedule=args.schedule, device=dev)
        Kc, Vc = synth.cond_inputs(wl, seed=3, device=dev)
        h.set_cond(Kc, Vc)
        Q, K, V = synth.chunk_inputs(wl, 0, 0, seed=3, device=dev)
        for _ in range(wl.steady_k()):
            h.append_chunk(K, V)
        out = torch.empty_like(Q)
        for _ in range(3):
            h.forward(Q, K, V, out=out)
        torch.cuda.synchronize(dev)
        reps = 20
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            h.forward(Q, K, V, out=out)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        t = e0.elapsed_time(e1) / 1e3 / reps
        k = wl.steady_k()
        tf = wl.flops_forward(k) / t / 1e12
        res[name] = {"schedule": h.schedule_for(), "ms_per_forward": round(t * 1e3, 4), "TFLOP/s": round(tf, 2),
                     "frac_of_peak": round(tf / peaks["bf16_tflops"], 4), "N_vis": wl.n_vis(k),
                     "status": h.status()}
        h.close()
        del Q, K, V, out, Kc, Vc
    return res


def host_link_peaks(host_in, dev_in, host_out, dev_out, up, down, dev, reps: int = 5) -> dict:
    """Pinned host <-> device copy rates on this machine: the step's H2D copies alone on the upload
    stream, its D2H copies alone on the download stream, best of `reps` (GB/s)."""
    def timed(st, fn):
        best = None
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            a.record(st)
            with torch.cuda.stream(st):
                n = fn()
            b.record(st)
            torch.cuda.synchronize(dev)
            t = a.elapsed_time(b) / 1e3
            best = t if best is None else min(best, t)
        return n / best / 1e9

    def h2d():
        n = 0
        for dst_s, src_s in zip(dev_in, host_in):
            for dst, src in zip(dst_s, src_s):
                dst.copy_(src, non_blocking=True)
                n += src.numel() * src.element_size()
        return n

    def d2h():
        n = 0
        for dst, src in zip(host_out, dev_out):
            dst.copy_(src, non_blocking=True)
            n += src.numel() * src.element_size()
        return n

    return {"h2d_gbs": round(timed(up, h2d), 2), "d2h_gbs": round(timed(down, d2h), 2)}


def side_paths(h, wl, pool, dev, stream, peaks):
    """Append/evict (HBM-bound copy), the split-K short-query path and the joint forward with
    condition-stream queries, timed alone."""
    out = {}
    reps = 50
    # every resident (K, V) input in turn, more bytes than L2 holds: the copy reads from HBM
    kv = [(K, V) for steps in pool for (_, K, V) in steps]
    Q, K, V = pool[0][-1]
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(reps):
        h.append_chunk(*kv[i % len(kv)])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    t = e0.elapsed_time(e1) / 1e3 / reps
    nbytes = 2 * 2 * K.numel() * K.element_size()          # K and V, read + write
    out["append"] = {"us": round(t * 1e6, 2), "GB/s": round(nbytes / t / 1e9, 1),
                     "frac_hbm": round(nbytes / t / 1e9 / peaks["hbm_gbs"], 3), "bytes": nbytes,
                     "sources": f"{len(kv)} (K, V) inputs cycled, {len(kv) * 2 * K.numel() * K.element_size() >> 20} MiB",
                     "note": f"one launch ({h.commit_kind()} commit): the copy, then the counter and table advance"}
    k = wl.steady_k()
    nvis = wl.n_vis(k)
    dec = {}
    for nq in (16, 64, 128):
        q = Q[:, :nq].contiguous()
        o = torch.empty((wl.B, nq, wl.H, wl.d), dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            h.forward(q, K, V, out=o)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(reps):
            h.forward(q, K, V, out=o)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        t = e0.elapsed_time(e1) / 1e3 / reps
        kv_bytes = 2 * wl.B * wl.H * nvis * wl.d * 2
        dec[str(nq)] = {"us": round(t * 1e6, 2), "GB/s": round(kv_bytes / t / 1e9, 1),
                        "frac_hbm": round(kv_bytes / t / 1e9 / peaks["hbm_gbs"], 3)}
    out["split_k"] = dec
    # the joint forward: the chunk's T queries and the n_cond condition-stream queries in one
    # launch, against the two as separate forwards
    Qc = synth.cond_queries(wl, 0, 0, seed=5, device=dev)
    o = torch.empty((wl.B, wl.T, wl.H, wl.d), dtype=torch.bfloat16, device=dev)
    oc = torch.empty((wl.B, wl.n_cond, wl.H, wl.d), dtype=torch.bfloat16, device=dev)

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / 1e3 / reps

    t_joint = timed(lambda: h.forward_joint(Q, Qc, K, V, out=o, out_cond=oc))
    t_sep = timed(lambda: (h.forward(Q, K, V, out=o), h.forward(Qc, K, V, out=oc)))
    fl = wl.flops_forward(k, wl.T + wl.n_cond)
    out["joint"] = {"queries": f"{wl.T} chunk + {wl.n_cond} condition", "ms": round(t_joint * 1e3, 4),
                    "TFLOP/s": round(fl / t_joint / 1e12, 2), "frac_of_peak": round(fl / t_joint / 1e12 / peaks["bf16_tflops"], 4),
                    "separate_forwards_ms": round(t_sep * 1e3, 4)}
    return out


# ---------------------------------------------------------------------------- the reference arm

def run_reference(args, wl, world, rank):
    """The oracle, as it stands, on the host cores: each step is a bounded sample of the same
    workload (ref_rows query rows of one steady-state forward, all heads, all visible keys).
    ms_per_step is the measured time of the work a step actually does; the time a whole chunk
    would take is given separately, extrapolated from the measured throughput."""
    if rank != 0:
        return
    # rank 0 runs alone: every host core it may run on, whatever thread count a multi-process
    # launcher set for the job's processes
    import oracle
    oracle.set_num_threads(len(os.sched_getaffinity(0)))
    k = wl.steady_k()
    x = oracle_inputs(wl, k)   # the workload's inputs, resident on the host like the GPU arm's
    per_row = None
    for _ in range(max(1, args.warmup)):
        _, secs, _, _ = cpu_baseline(wl, k, rows=2, inputs=x)
        per_row = secs / 2
    # rows per step: as given, else sized so that all K steps take about 90 s of host time
    rows = args.ref_rows if args.ref_rows else max(1, min(48, int(90.0 / max(1, args.steps) / per_row)))
    t_total, fl_total, thr = 0.0, 0.0, 1
    for _ in range(args.steps):
        v, secs, fl, thr = cpu_baseline(wl, k, rows=rows, inputs=x)
        t_total += secs
        fl_total += fl
    value = fl_total / t_total / 1e12
    full_step = wl.steps * wl.flops_forward(k)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_total / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(wl, args.pool, world),
        "step_sample": f"{rows} query rows x {wl.B * wl.H} heads of one steady-state forward over "
                       f"all {wl.n_vis(k)} visible keys ({fl_total / args.steps / 1e9:.2f} GFLOP per step)",
        "ms_per_chunk_extrapolated": full_step / (fl_total / t_total) * 1e3,
        "cpu_baseline": dict({"kind": "oracle", "cores": thr, "value": value, "unit": UNIT,
                              "sample": f"per step {rows} query rows x {wl.B * wl.H} heads of one "
                                        f"steady-state forward over {wl.n_vis(k)} keys"}, **host_cpu()),
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--config", default="720p", choices=sorted(WORKLOADS))
    ap.add_argument("--pool", type=int, default=3)
    ap.add_argument("--ref-rows", type=int, default=0,
                    help="query rows per reference step (0: sized so the K steps take about 90 s)")
    ap.add_argument("--warm-seconds", type=float, default=4.0,
                    help="seconds of chunk steps before the timed long-horizon stream")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--schedule", choices=["auto", "persistent", "grid", "tri", "pair"], default="auto")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the long-horizon and other-workload side measurements")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = WORKLOADS[args.config]
    world, rank, local = _dist_env()
    if args.impl == "reference":
        run_reference(args, wl, world, rank)
        return
    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}))
        sys.exit(1)
    run_cuda(args, wl, world, rank, local)


if __name__ == "__main__":
    main()
