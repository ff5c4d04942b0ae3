"""Benchmark: fused causal attention on B200, prefill TFLOP/s and decode KV-read GB/s.

One step = one pass of the whole hot path over the five synthetic workloads, each once: the tiny
causal prefill (B1 H2 S64 D32), the causal prefill of an 8B-shaped layer (B1 Hq32 Hkv8 S4096 D128),
the GQA decode over a 16 x 4096-token KV cache, the chunked prefill (B8, 256 new tokens over a
768-token cache) and the long-context prefill (B1 Hq32 Hkv8 S32768 D128, 1% of the keys x8). Inputs
are resident in HBM before timing; L2 is flushed before every launch (a 256 MiB write, then a
256 MiB read so that the written lines are cleaned before the kernel starts), outside the kernel
events. Each launch is timed with CUDA events on the launching stream.

The line's ``value`` is the prefill TFLOP/s of the largest single-GPU workload (the 32K prefill);
``configs`` holds every workload's own throughput, roofline fraction, DRAM traffic and oracle
baseline, and ``decode`` repeats the GQA decode's. After the timed steps come the end-to-end leg
(``e2e``: the 32K prefill from pinned host buffers through ``attn_fwd_host``), the e4m3 decode,
the event-timing floor of an empty launch (``launch_floor_us``), the paged chunked prefill, the
e4m3 chunked prefill and the backward pass of the 8B layer, each timed the same way.

``python bench.py --gpus N --steps K --warmup W`` prints one JSON line (rank 0). For N > 1 it is
launched with torchrun, one rank per GPU; every rank processes its own copy of the workloads (the
(batch, head) problems are independent, so there is no data-path collective) and the time is the
max over ranks. ``--impl reference`` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from causal_attention_attn_b200 import inputs  # noqa: E402

METRIC = "prefill attn TFLOP/s & decode KV-read GB/s, as fraction of B200 roofline"
PREFILL = inputs.PREFILL_8B
DECODE = inputs.DECODE_GQA
HEADLINE = inputs.LONG_PREFILL  # the largest workload that fits one GPU: the line's value
STEP_WORKLOADS = (inputs.TINY_PREFILL, inputs.PREFILL_8B, inputs.DECODE_GQA, inputs.CHUNKED_PREFILL,
                  inputs.LONG_PREFILL)
SHORT = {w.name: n for n, w in inputs.SHORT_NAMES.items()}
L2_FLUSH_BYTES = 256 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET_BF16_TFLOPS = 2250.0  # B200 dense bf16, nominal


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class Ranks:
    """Host-side plumbing of the replicas: a barrier and a max over ranks of device-timed values.

    The ranks exchange only timings (no data-path collective: every rank runs the whole workload on
    its own GPU). NCCL on GPU tensors when the process group uses it, gloo on CPU tensors otherwise;
    with one process both are no-ops.
    """

    def __init__(self, world: int, device):
        self.world = world
        self.device = device

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist

            dist.barrier()

    def max(self, values):
        """Element-wise maximum of `values` (a list of floats) over all ranks."""
        if self.world == 1:
            return list(values)
        import torch.distributed as dist

        t = torch.tensor(list(values), dtype=torch.float64, device=self.device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return t.tolist()


def whole_job_rate(world: int, units_per_rank: float, seconds: float) -> float:
    """Units all ranks processed per second: every rank did `units_per_rank`; `seconds` is the
    slowest rank's device time."""
    return world * units_per_rank / seconds


class ClockSampler:
    """nvidia-smi clock / power / throttle-reason samples taken every 20 ms while the timed region
    runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    LOAD_WATTS = 300.0  # a sample drawing at least this much is taken while a kernel runs

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.out = open(os.devnull, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.device_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=self.out, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        if self.out:
            self.out.close()

    def summary(self):
        return summarise_clock_lines(getattr(self, "lines", []), self.LOAD_WATTS)


def summarise_clock_lines(lines, load_watts):
    """Median SM clock over every sample and over the samples drawing >= load_watts (under load),
    the highest max clock seen, and the throttle reasons active in any sample."""
    sm, sm_load, smax, reasons = [], [], 0.0, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for ln in lines:
        parts = [p.strip() for p in ln.split(",")]
        if len(parts) < 9:
            continue
        try:
            mhz = float(parts[1])
            smax = max(smax, float(parts[2]))
        except ValueError:
            continue
        sm.append(mhz)
        try:
            if float(parts[3]) >= load_watts:
                sm_load.append(mhz)
        except ValueError:
            pass
        for name, val in zip(names, parts[5:9]):
            if val.lower() == "active":
                reasons.add(name)
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax or None,
            "reasons": sorted(reasons), "samples": len(sm),
            "sm_mhz_under_load": statistics.median(sm_load) if sm_load else None,
            "samples_under_load": len(sm_load)}


def prefill_sample_flops(w, rows):
    i = rows % w.Sq
    visible = (i + w.offset + 1) if w.causal else torch.full_like(i, w.Skv)
    return int(4 * w.D * int(visible.sum()))


def cpu_baseline(w, every: int, offset: int = 0, threads=None, data=None):
    """Time the oracle on every `every`-th row of workload `w` (rows offset, offset+every, ...).
    Returns (TFLOP/s, seconds, cores, rows)."""
    import oracle  # the CPU baseline is the oracle as it stands

    q, k, v = data if data is not None else inputs.generate(w)
    total = w.B * w.Hq * w.Sq
    rows = torch.arange(offset % every, total, every, dtype=torch.int64)
    cores = len(os.sched_getaffinity(0))
    t0 = time.perf_counter()
    oracle.attention(q, k, v, w.scale, w.causal, rows=rows.numpy() if every > 1 else None,
                     threads=threads or cores)
    dt = time.perf_counter() - t0
    flops = prefill_sample_flops(w, rows)
    return flops / dt / 1e12, dt, cores, rows.numel()


# Rows of each workload the oracle baseline times in the bench: every row, except the long
# prefill's every 64th (its full 8.8 TFLOP would take minutes of fp64).
BASELINE_EVERY = {inputs.LONG_PREFILL.name: 64}


def workload_baseline(w, data=None):
    every = BASELINE_EVERY.get(w.name, 1)
    tf, dt, cores, n = cpu_baseline(w, every, data=data)
    d = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "seconds": dt,
         "sample": (f"every query row ({n} rows, {dt:.2f} s); fp64 three-pass oracle" if every == 1 else
                    f"every {every}th query row ({n} rows, {dt:.2f} s), rate extrapolated to the whole "
                    f"workload; fp64 three-pass oracle")}
    if w.Sq == 1:  # the decode's own unit: K/V bytes per second
        d["value_gbs"] = w.io_bytes() / (dt * (w.B * w.Hq * w.Sq) / n) / 1e9
    return d


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    w = HEADLINE
    every = 1024
    data = inputs.generate(w)
    times, flops = [], []
    for s in range(args.warmup + args.steps):
        tf, dt, cores, n = cpu_baseline(w, every, offset=97 * s, data=data)
        if s >= args.warmup:
            times.append(dt)
            flops.append(tf * dt * 1e12)
    value = sum(flops) / sum(times) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16 inputs)", "config": HEADLINE.config(),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"one query row in {every} of the workload per step (rows offset by 97 x the "
                                   f"step index), {n} rows; fp64 three-pass oracle"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# A timed region at least this long runs the step's kernels back to back under the power cap: the
# prefills are then "timed inside a long step" and their roofline peak is the measured sustained
# bf16 figure (a seconds-long loop of cuBLAS under the same cap); shorter runs use the burst one.
SUSTAINED_REGION_MS = 1000.0


def config_entry(w, launch_s, world, peaks, peak_kind, baseline=None, sustained_regime=False):
    """The JSON object of one workload: throughput, roofline of its kernel, oracle baseline."""
    tensor_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    kernel = "decode_tc_kernel" if w.Sq == 1 else "prefill_kernel"
    if w.Sq == 1:
        achieved = w.io_bytes() / launch_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
                "peak_kind": f"{peak_kind} HBM copy", "bytes_per_launch": w.io_bytes()}
        value, unit = whole_job_rate(world, w.io_bytes(), launch_s) / 1e9, "GB/s"
    else:
        achieved = w.flops() / launch_s / 1e12
        sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        peak = sustained if sustained_regime else tensor_peak
        kind = ("sustained: the timed region ran the step back to back for at least "
                f"{SUSTAINED_REGION_MS / 1000:.0f} s under the power cap") if sustained_regime else "burst"
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_kind": f"{peak_kind} bf16 dense ({kind})",
                "frac_of_burst": achieved / tensor_peak,  # the measured peak of a short run
                "frac_of_sustained": achieved / sustained,  # the measured peak under the power cap
                "frac_of_datasheet": achieved / DATASHEET_BF16_TFLOPS,  # nominal dense bf16
                "flops_per_launch": w.flops()}
        value, unit = whole_job_rate(world, w.flops(), launch_s) / 1e12, "TFLOP/s"
    roof["traffic"] = read_traffic(kernel, w.name)
    roof["kernel"] = f"{kernel}<{w.D}>" if w.Sq > 1 else "decode_tc_kernel<4>"
    e = {"workload": w.name, "value": value, "unit": unit, "us_per_launch": launch_s * 1e6, "roofline": roof,
         "config": w.config()}
    if w.name == inputs.TINY_PREFILL.name:
        e["note"] = "launch-latency bound (0.5 MFLOP); the roofline fraction is reported but is not the measure"
    if baseline is not None:
        e["cpu_baseline"] = baseline
        if unit == "TFLOP/s":
            e["vs_oracle"] = value / baseline["value"]
    return e


def run_ours(args):
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    ranks = Ranks(world, dev)
    from causal_attention_attn_b200 import attn

    attn.load_library()
    peaks, peak_kind = load_peaks()

    host = {w.name: inputs.generate(w) for w in STEP_WORKLOADS}
    bufs = {}
    for w in STEP_WORKLOADS:
        q, k, v = (t.to(dev) for t in host[w.name])
        bufs[w.name] = (q, k, v, torch.empty_like(q), torch.empty(q.shape[:3], dtype=torch.float32, device=dev))
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_clean = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_sum = torch.empty((), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def clear_l2():
        # Write 256 MiB (evicts every input from the 126 MB L2), then read another 256 MiB so that
        # the dirty lines of that write are written back now and not during the next kernel.
        flush.zero_()
        torch.sum(flush_clean, dim=0, out=flush_sum)

    def launch(w):
        q, k, v, o, lse = bufs[w.name]
        attn.attn_fwd(q, k, v, scale=w.scale, causal=w.causal, out=o, lse=lse, stream=stream)

    def step(evs=None):
        for i, w in enumerate(STEP_WORKLOADS):
            clear_l2()
            if evs:
                evs[i][0].record(stream)
            launch(w)
            if evs:
                evs[i][1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    n_w = len(STEP_WORKLOADS)
    events = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n_w)]
              for _ in range(args.steps)]
    t_all0 = torch.cuda.Event(enable_timing=True)
    t_all1 = torch.cuda.Event(enable_timing=True)
    ranks.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        t_all0.record(stream)
        for s in range(args.steps):
            step(events[s])
        t_all1.record(stream)
        torch.cuda.synchronize(dev)
    ranks.barrier()
    per_w_ms = [sum(events[s][i][0].elapsed_time(events[s][i][1]) for s in range(args.steps)) for i in range(n_w)]
    region_ms = t_all0.elapsed_time(t_all1)
    timed = ranks.max(per_w_ms + [region_ms])
    per_w_ms, region_ms = timed[:n_w], timed[n_w]
    launch_s = {w.name: per_w_ms[i] * 1e-3 / args.steps for i, w in enumerate(STEP_WORKLOADS)}
    status = attn.device_status(stream)

    head_s = launch_s[HEADLINE.name]
    head_tflops = whole_job_rate(world, args.steps * HEADLINE.flops(), head_s * args.steps) / 1e12
    tensor_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))

    # End to end through the public call on HOST buffers (attn_fwd_host: the H2D copies of q, k, v,
    # the attention and the D2H copies of o and lse, pipelined slice by slice), headline workload.
    hq, hk, hv = (t.pin_memory() for t in host[HEADLINE.name])
    ho = torch.empty(hq.shape, dtype=torch.bfloat16, pin_memory=True)
    hl = torch.empty(hq.shape[:3], dtype=torch.float32, pin_memory=True)
    head_bufs = bufs[HEADLINE.name]
    for _ in range(2):
        attn.attn_fwd_host(hq, hk, hv, scale=HEADLINE.scale, causal=True, stream=stream, out_host=ho, lse_host=hl,
                           dev_bufs=head_bufs)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(3, min(args.steps, 10))
    ranks.barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(e2e_steps):
        attn.attn_fwd_host(hq, hk, hv, scale=HEADLINE.scale, causal=True, stream=stream, out_host=ho, lse_host=hl,
                           dev_bufs=head_bufs)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = ranks.max([e2e_ms])[0]
    ranks.barrier()
    e2e_tflops = whole_job_rate(world, e2e_steps * HEADLINE.flops(), e2e_ms * 1e-3) / 1e12
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()
    del hq, hk, hv, ho, hl

    # The same decode over an e4m3 cache (per-channel coefficients), timed on its own: inputs
    # resident, L2 flushed before every launch, CUDA events around each launch.
    fq, fk8, fv8, fks, fvs = (t.to(dev) for t in inputs.generate_fp8(DECODE))
    fo = torch.empty_like(fq)
    fl = torch.empty(fq.shape[:3], dtype=torch.float32, device=dev)
    fp8_bytes = fp8_decode_bytes(DECODE)
    for _ in range(args.warmup):
        clear_l2()
        attn.attn_decode_fp8(fq, fk8, fv8, fks, fvs, scale=DECODE.scale, out=fo, lse=fl, stream=stream)
    fp8_steps = max(3, min(args.steps, 500))
    fev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(fp8_steps)]
    ranks.barrier()
    torch.cuda.synchronize(dev)
    for s in range(fp8_steps):
        clear_l2()
        fev[s][0].record(stream)
        attn.attn_decode_fp8(fq, fk8, fv8, fks, fvs, scale=DECODE.scale, out=fo, lse=fl, stream=stream)
        fev[s][1].record(stream)
    torch.cuda.synchronize(dev)
    fp8_ms = ranks.max([sum(a.elapsed_time(b) for a, b in fev)])[0]
    fp8_launch_s = fp8_ms * 1e-3 / fp8_steps

    # The floor of this timing method: an empty kernel (torch.cuda._sleep(0), one block) launched
    # and event-timed exactly like the kernels above. A launch's event-timed duration is its body
    # plus about this much; short kernels (the decodes) feel it most.
    floor_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(25)]
    for a, b in floor_ev:
        clear_l2()
        a.record(stream)
        torch.cuda._sleep(0)
        b.record(stream)
    torch.cuda.synchronize(dev)
    launch_floor_us = statistics.median(a.elapsed_time(b) * 1e3 for a, b in floor_ev[5:])

    # Chunked prefill over a paged cache with per-sequence lengths (attn_prefill_paged), timed the
    # same way: inputs resident, L2 flushed before every launch.
    try:
        paged = paged_prefill_leg(attn, args, ranks, dev, stream, clear_l2, world, peaks, peak_kind)
    except Exception as e:  # an extra leg that fails is reported in its object, not allowed to drop the line
        paged = {"metric": "paged chunked prefill TFLOP/s", "error": f"{type(e).__name__}: {e}"}

    # The chunked prefill over an e4m3 cache of the same shape (attn_prefill_fp8), timed the same way.
    try:
        prefill_fp8 = prefill_fp8_leg(attn, args, ranks, dev, stream, clear_l2, world, peaks, peak_kind)
    except Exception as e:
        prefill_fp8 = {"metric": "chunked prefill TFLOP/s, e4m3 K/V cache", "error": f"{type(e).__name__}: {e}"}

    # The backward pass of the 8B prefill workload (dq, dk, dv from dout and the forward's o, lse),
    # timed the same way. Reported beside the step, not part of it.
    try:
        pq, pk, pv, po, pl = bufs[PREFILL.name]
        backward = backward_leg(attn, args, ranks, dev, stream, clear_l2, pq, pk, pv, po, pl, world)
    except Exception as e:  # an extra leg that fails is reported in its object, not allowed to drop the line
        backward = {"metric": "backward TFLOP/s (dq, dk, dv)", "error": f"{type(e).__name__}: {e}"}

    # The ring's per-rank compute at eight ranks, emulated here (blocks and merges, no exchange).
    try:
        lq, lk, lv, _, _ = bufs[HEADLINE.name]
        ring = ring_compute_leg(attn, args, ranks, dev, stream, clear_l2, lq, lk, lv, launch_s[HEADLINE.name])
    except Exception as e:
        ring = {"metric": "ring attention compute per rank (no exchange), ms", "error": f"{type(e).__name__}: {e}"}

    if rank == 0:
        baselines = {w.name: workload_baseline(w, host[w.name]) for w in STEP_WORKLOADS} if world == 1 else {}
        sustained_regime = region_ms >= SUSTAINED_REGION_MS
        configs = {SHORT[w.name]: config_entry(w, launch_s[w.name], world, peaks, peak_kind, baselines.get(w.name),
                                               sustained_regime)
                   for w in STEP_WORKLOADS}
        head = configs[SHORT[HEADLINE.name]]
        dec = configs[SHORT[DECODE.name]]
        clk = clocks.summary()
        if clk.get("sm_mhz_under_load"):
            clk["headline_kcycles_at_load_clock"] = head_s * 1e6 * clk["sm_mhz_under_load"] / 1e3
        line = {
            "metric": METRIC, "value": head_tflops, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": sum(per_w_ms) / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16 inputs)",
            "config": dict(HEADLINE.config(),
                           step="the five workloads, each launched once (tiny, 8B prefill, GQA decode, chunked, 32K)",
                           l2="flushed before every kernel (256 MiB write, then 256 MiB read)",
                           parallelism=f"replicas x{world}"),
            "roofline": dict(head["roofline"]),
            "configs": configs,
            "decode": {"metric": "decode KV-read GB/s", "value": dec["value"], "unit": "GB/s",
                       "config": DECODE.config(), "roofline": dec["roofline"], "us_per_launch": dec["us_per_launch"],
                       "ctas": attn.decode_ctas(DECODE.B, DECODE.Hq, DECODE.Hkv, DECODE.Skv, DECODE.D),
                       "launch_floor_us": launch_floor_us},
            "decode_fp8": {
                "metric": "decode KV-read GB/s, e4m3 K/V cache", "value": whole_job_rate(world, fp8_bytes, fp8_launch_s) / 1e9,
                "unit": "GB/s", "config": dict(DECODE.config(), kv_dtype="e4m3", scales="fp32 per (kv head, channel)"),
                "steps": fp8_steps,
                "roofline": {"bound": "hbm", "achieved": fp8_bytes / fp8_launch_s / 1e9, "peak": hbm_peak,
                             "unit": "GB/s", "frac": fp8_bytes / fp8_launch_s / 1e9 / hbm_peak,
                             "traffic": read_traffic("decode_tc_kernel_fp8", DECODE.name),
                             "peak_kind": f"{peak_kind} HBM copy", "kernel": "decode_tc_kernel<4, e4m3>"},
                "us_per_launch": fp8_launch_s * 1e6,
                "bytes_per_launch": fp8_bytes,
                "launch_floor_us": launch_floor_us,
            },
            "launch_floor_us": launch_floor_us,
            "launch_floor_what": "median event-timed duration of an empty kernel (torch.cuda._sleep(0)) launched like the timed kernels, L2 flushed before each; every us_per_launch includes about this much besides the kernel's body",
            "backward": backward,
            "ring_compute": ring,
            "paged_prefill": paged,
            "prefill_fp8": prefill_fp8,
            "timed_region_ms": region_ms,
            "e2e": {"value": e2e_tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps,
                    "what": "32K prefill through attn_fwd_host on pinned host buffers: copies in and out pipelined against the attention in eight slices, all inside the timed region"},
            "gpu_launches": n_w * args.steps,
            "device_status": status,
            "clocks": clk,
        }
        if baselines:
            b = baselines[HEADLINE.name]
            line["cpu_baseline"] = {k: b[k] for k in ("value", "unit", "cores", "kind", "sample")}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


KERNEL_SOURCES = {
    "prefill_kernel": ["prefill_sm100.cu", "sm100_ptx.cuh"],
    "prefill_kernel_paged": ["prefill_sm100.cu", "sm100_ptx.cuh"],
    "bwd_kernel": ["bwd_sm100.cu", "sm100_ptx.cuh"],
    "decode_tc_kernel": ["decode_tc_sm100.cu", "sm100_ptx.cuh"],
    "decode_tc_kernel_fp8": ["decode_tc_sm100.cu", "sm100_ptx.cuh"],
    "prefill_fp8_kernel": ["prefill_fp8_sm100.cu", "sm100_ptx.cuh"],
}


def kernel_source_hash(kernel: str) -> str:
    """Hash of the kernel's source files with comments and whitespace removed: a capture stays
    valid across comment edits and goes stale with any change to the code itself."""
    import hashlib
    import re

    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "causal_attention_attn_b200", "csrc", name), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update("".join(text.split()).encode())
    return h.hexdigest()[:16]


def read_traffic(kernel: str, workload: str):
    """DRAM bytes per launch for `kernel` on `workload` from the committed ncu summaries
    (profiles/traffic.json: kernel -> workload -> entry), or None when there is no capture for it
    or the kernel's source changed since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        with open(path) as f:
            entry = json.load(f).get(kernel, {}).get(workload, {})
        if entry.get("source_hash") != kernel_source_hash(kernel):
            return None
        return entry.get("dram_bytes_per_launch")
    except (OSError, ValueError, AttributeError):
        return None


def ring_compute_leg(attn, args, ranks, dev, stream, clear_l2, q, k, v, head_launch_s, world_ring=8):
    """The compute of ring attention on the 32K workload at world_ring ranks, emulated on this GPU
    with no exchange: every virtual rank runs its zigzag schedule's blocks (attn_fwd) and LSE merges
    (attn_lse_merge) over K/V shards already resident, L2 flushed before each rank. The slowest
    rank's time is compared with a world_ring-th of the single 32K launch: the cost of cutting the
    sequence into blocks (more launches, each with its ramp and tail) and merging them. The
    exchange over NVLink is not part of it (it needs several GPUs)."""
    from causal_attention_attn_b200.ring import DIAG, ring_schedule, zigzag_shard

    w = HEADLINE
    S = w.Sq // world_ring  # tokens per rank: two chunks
    c = S // 2

    def halves(x):
        return x[:, :, :c].contiguous(), x[:, :, c:].contiguous()

    shards = [(halves(zigzag_shard(q, r, world_ring)), halves(zigzag_shard(k, r, world_ring)),
               halves(zigzag_shard(v, r, world_ring))) for r in range(world_ring)]

    def run_rank(rank):
        qs = shards[rank][0]
        o_acc = [torch.zeros(x.shape, dtype=torch.float32, device=dev) for x in qs]
        lse_acc = [torch.full(x.shape[:-1], float("-inf"), dtype=torch.float32, device=dev) for x in qs]
        out = [torch.empty(x.shape, dtype=torch.bfloat16, device=dev) for x in qs]
        sched = ring_schedule(rank, world_ring, True)
        last = {qh: (t, b) for t, _, blocks in sched for b, (qh, _, _) in enumerate(blocks)}
        launches = 0
        clear_l2()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for t, j, blocks in sched:
            ks, vs = shards[j][1], shards[j][2]
            for b, (qh, kh, mode) in enumerate(blocks):
                o_p, l_p = attn.attn_fwd(qs[qh], ks[kh], vs[kh], scale=w.scale, causal=(mode == DIAG), stream=stream)
                attn.attn_lse_merge(o_acc[qh], lse_acc[qh], o_p, l_p, out=out[qh] if last[qh] == (t, b) else None,
                                    stream=stream)
                launches += 2
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1), launches

    for r in range(world_ring):  # warm-up
        run_rank(r)
    reps = 3
    per_rank = [min(run_rank(r)[0] for _ in range(reps)) for r in range(world_ring)]
    launches = run_rank(0)[1]
    slowest = ranks.max([max(per_rank)])[0]
    share = head_launch_s * 1e3 / world_ring
    return {"metric": "ring attention compute per rank (no exchange), ms", "world": world_ring,
            "config": dict(w.config(), tokens_per_rank=S, chunk=c, order="zigzag"),
            "slowest_rank_ms": slowest, "fastest_rank_ms": min(per_rank),
            "single_launch_share_ms": share, "overhead_vs_share": slowest / share,
            "launches_per_rank": launches,
            "what": "every virtual rank's blocks and LSE merges on K/V shards already in HBM, L2 flushed "
                    "before each rank, best of 3; the exchange between GPUs is not part of it"}


def backward_leg(attn, args, ranks, dev, stream, clear_l2, q, k, v, o, lse, world):
    """Time attn_bwd on the prefill workload: inputs resident, L2 flushed before every launch, CUDA
    events around each launch, max over ranks. FLOPs: five products of 2*D per visible pair (S, dP,
    dV, dK, dQ), 2.5x the forward's. Returns the JSON object of the leg."""
    peaks, peak_kind = load_peaks()
    tensor_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    flops = 5 * PREFILL.flops() // 2
    g = torch.Generator().manual_seed(7)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16).to(dev)
    attn.attn_fwd(q, k, v, scale=PREFILL.scale, causal=True, out=o, lse=lse, stream=stream)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    for _ in range(args.warmup):
        clear_l2()
        attn.attn_bwd(q, k, v, o, lse, dout, scale=PREFILL.scale, causal=True, dq=dq, dk=dk, dv=dv, stream=stream)
    steps = max(3, min(args.steps, 20))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    ranks.barrier()
    torch.cuda.synchronize(dev)
    for s in range(steps):
        clear_l2()
        ev[s][0].record(stream)
        attn.attn_bwd(q, k, v, o, lse, dout, scale=PREFILL.scale, causal=True, dq=dq, dk=dk, dv=dv, stream=stream)
        ev[s][1].record(stream)
    torch.cuda.synchronize(dev)
    ms = ranks.max([sum(a.elapsed_time(b) for a, b in ev)])[0]
    launch_s = ms * 1e-3 / steps
    achieved = flops / launch_s / 1e12
    return {"metric": "backward TFLOP/s (dq, dk, dv)", "value": whole_job_rate(world, flops, launch_s) / 1e12,
            "unit": "TFLOP/s", "config": PREFILL.config(), "steps": steps,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": tensor_peak, "unit": "TFLOP/s",
                         "frac": achieved / tensor_peak, "traffic": read_traffic("bwd_kernel", PREFILL.name),
                         "peak_kind": f"{peak_kind} bf16 dense (burst)", "kernel": "bwd_kernel"},
            "us_per_launch": launch_s * 1e6, "flops_per_launch": flops,
            "device_status": attn.device_status(stream)}


def paged_prefill_inputs(dev):
    w = inputs.PAGED_CHUNKED
    lens = inputs.paged_chunked_lengths()
    q, k, v = inputs.generate(w)
    kp, vp, table = inputs.paged_cache(k, v, lens, inputs.PAGED_CHUNKED_PAGE, seed=w.seed)
    seq = torch.tensor(lens, dtype=torch.int32)
    return w, lens, [t.to(dev) for t in (q, kp, vp, table, seq)]


def paged_prefill_leg(attn, args, ranks, dev, stream, clear_l2, world, peaks, peak_kind):
    """Time attn_prefill_paged on the paged chunked-prefill workload (per-sequence cache lengths):
    L2 flushed before every launch, CUDA events around each, max over ranks."""
    w, lens, (q, kp, vp, table, seq) = paged_prefill_inputs(dev)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    flops = 4 * w.D * w.Hq * inputs.paged_visible_pairs(w.Sq, lens)
    call = lambda: attn.attn_prefill_paged(q, kp, vp, table, seq, max(lens), scale=w.scale, causal=True, out=o,
                                           lse=lse, stream=stream)
    for _ in range(args.warmup):
        clear_l2()
        call()
    steps = max(3, min(args.steps, 100))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    ranks.barrier()
    torch.cuda.synchronize(dev)
    for s in range(steps):
        clear_l2()
        ev[s][0].record(stream)
        call()
        ev[s][1].record(stream)
    torch.cuda.synchronize(dev)
    ms = ranks.max([sum(a.elapsed_time(b) for a, b in ev)])[0]
    launch_s = ms * 1e-3 / steps
    tensor_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = flops / launch_s / 1e12
    return {"metric": "paged chunked prefill TFLOP/s", "value": whole_job_rate(world, flops, launch_s) / 1e12,
            "unit": "TFLOP/s", "config": dict(w.config(), seq_lens=lens, page_size=inputs.PAGED_CHUNKED_PAGE),
            "steps": steps,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": tensor_peak, "unit": "TFLOP/s",
                         "frac": achieved / tensor_peak, "traffic": read_traffic("prefill_kernel_paged", w.name),
                         "peak_kind": f"{peak_kind} bf16 dense (burst)", "kernel": "prefill_kernel<128, paged>"},
            "us_per_launch": launch_s * 1e6, "flops_per_launch": flops}


def prefill_fp8_leg(attn, args, ranks, dev, stream, clear_l2, world, peaks, peak_kind):
    """Time attn_prefill_fp8 on the chunked-prefill workload over its e4m3 cache: L2 flushed
    before every launch, CUDA events around each, max over ranks. The roofline's peak is the e4m3
    dense rate (twice the measured bf16 one, the nominal ratio); the kernel issues every product
    three times (three e4m3 parts of q * k_scale and of the weights), which the algorithmic FLOPs do
    not count."""
    w = inputs.CHUNKED_PREFILL
    q, k8, v8, ks, vs = (t.to(dev) for t in inputs.generate_fp8(w))
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    call = lambda: attn.attn_prefill_fp8(q, k8, v8, ks, vs, scale=w.scale, causal=True, out=o, lse=lse, stream=stream)
    for _ in range(args.warmup):
        clear_l2()
        call()
    steps = max(3, min(args.steps, 100))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    ranks.barrier()
    torch.cuda.synchronize(dev)
    for s in range(steps):
        clear_l2()
        ev[s][0].record(stream)
        call()
        ev[s][1].record(stream)
    torch.cuda.synchronize(dev)
    ms = ranks.max([sum(a.elapsed_time(b) for a, b in ev)])[0]
    launch_s = ms * 1e-3 / steps
    e4m3_peak = 2.0 * float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = w.flops() / launch_s / 1e12
    return {"metric": "chunked prefill TFLOP/s, e4m3 K/V cache", "value": whole_job_rate(world, w.flops(), launch_s) / 1e12,
            "unit": "TFLOP/s", "config": dict(w.config(), kv_dtype="e4m3", scales="fp32 per (kv head, channel)"),
            "steps": steps,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": e4m3_peak, "unit": "TFLOP/s",
                         "frac": achieved / e4m3_peak, "traffic": read_traffic("prefill_fp8_kernel", w.name),
                         "peak_kind": f"{peak_kind} bf16 dense (burst) x 2 (e4m3 nominal ratio)",
                         "kernel": "prefill_fp8_kernel", "products_issued_per_algorithmic": 3},
            "us_per_launch": launch_s * 1e6, "flops_per_launch": w.flops()}


def fp8_decode_bytes(w) -> int:
    """Bytes the e4m3 decode must move once: K and V codes, q, o, lse and both coefficient tables."""
    kv = 2 * w.B * w.Hkv * w.Skv * w.D
    return kv + 2 * w.B * w.Hq * w.D * 2 + w.B * w.Hq * 4 + 2 * w.Hkv * w.D * 4


def run_case(args):
    """Run one named workload `--repeat` times through attn_fwd (no L2 flush, no JSON line): the
    command the committed ncu summaries were captured with."""
    from causal_attention_attn_b200 import attn

    if args.case == "backward":
        w = inputs.PREFILL_8B
        q, k, v = (t.cuda() for t in inputs.generate(w))
        o, lse = attn.attn_fwd(q, k, v, scale=w.scale, causal=True)
        dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16).cuda()
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record()
        for _ in range(args.repeat):
            attn.attn_bwd(q, k, v, o, lse, dout, scale=w.scale, causal=True, dq=dq, dk=dk, dv=dv)
        ev[1].record()
        torch.cuda.synchronize()
        ms = ev[0].elapsed_time(ev[1]) / args.repeat
        print(json.dumps({"case": w.name + "_backward", "repeat": args.repeat, "us_per_launch": ms * 1e3,
                          "tflops": 5 * w.flops() / 2 / (ms * 1e-3) / 1e12,
                          "device_status": attn.device_status()}), flush=True)
        return 0
    if args.case == "chunked_paged":
        w, lens, (q, kp, vp, table, seq) = paged_prefill_inputs(torch.device("cuda"))
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record()
        for _ in range(args.repeat):
            attn.attn_prefill_paged(q, kp, vp, table, seq, max(lens), scale=w.scale, causal=True)
        ev[1].record()
        torch.cuda.synchronize()
        ms = ev[0].elapsed_time(ev[1]) / args.repeat
        flops = 4 * w.D * w.Hq * inputs.paged_visible_pairs(w.Sq, lens)
        print(json.dumps({"case": w.name, "repeat": args.repeat, "us_per_launch": ms * 1e3,
                          "tflops": flops / (ms * 1e-3) / 1e12, "device_status": attn.device_status()}), flush=True)
        return 0
    if args.case == "prefill_fp8":
        w = inputs.CHUNKED_PREFILL
        q, k8, v8, ks, vs = (t.cuda() for t in inputs.generate_fp8(w))
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record()
        for _ in range(args.repeat):
            attn.attn_prefill_fp8(q, k8, v8, ks, vs, scale=w.scale, causal=True)
        ev[1].record()
        torch.cuda.synchronize()
        ms = ev[0].elapsed_time(ev[1]) / args.repeat
        print(json.dumps({"case": w.name + "_e4m3", "repeat": args.repeat, "us_per_launch": ms * 1e3,
                          "tflops": w.flops() / (ms * 1e-3) / 1e12, "device_status": attn.device_status()}),
              flush=True)
        return 0
    if args.case == "decode_fp8":
        w = inputs.DECODE_GQA
        q, k8, v8, ks, vs = (t.cuda() for t in inputs.generate_fp8(w))
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record()
        for _ in range(args.repeat):
            attn.attn_decode_fp8(q, k8, v8, ks, vs, scale=w.scale, out=o, lse=lse)
        ev[1].record()
        torch.cuda.synchronize()
        ms = ev[0].elapsed_time(ev[1]) / args.repeat
        print(json.dumps({"case": w.name + "_e4m3", "repeat": args.repeat, "us_per_launch": ms * 1e3,
                          "io_gbs": fp8_decode_bytes(w) / (ms * 1e-3) / 1e9,
                          "device_status": attn.device_status()}), flush=True)
        return 0
    w = inputs.SHORT_NAMES[args.case]
    q, k, v = (t.cuda() for t in inputs.generate(w))
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for _ in range(args.repeat):
        attn.attn_fwd(q, k, v, scale=w.scale, causal=w.causal, out=o, lse=lse)
    ev[1].record()
    torch.cuda.synchronize()
    ms = ev[0].elapsed_time(ev[1]) / args.repeat
    print(json.dumps({"case": w.name, "repeat": args.repeat, "us_per_launch": ms * 1e3,
                      "tflops": w.flops() / (ms * 1e-3) / 1e12, "io_gbs": w.io_bytes() / (ms * 1e-3) / 1e9,
                      "device_status": attn.device_status()}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--case", choices=sorted(inputs.SHORT_NAMES) + ["decode_fp8", "backward", "chunked_paged", "prefill_fp8"],
                    default=None,
                    help="only run this workload --repeat times (for profiling); prints no bench line")
    ap.add_argument("--repeat", type=int, default=3)
    args = ap.parse_args()
    if args.case:
        return run_case(args)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
