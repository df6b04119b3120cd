#!/usr/bin/env python
"""Benchmark of the GDLA forward core (libgdla.so) on B200.

Headline: packed prefill, batch 1, T = 4096, 64 signal + 16 noise query heads
over 16 KV heads (dqk 192, dv 128), full causal, in TFLOP/s of algorithmic
work (80 heads x (2*192 + 2*128) flops per visible query/key pair). The same
JSON line carries the sliding-window-128 prefill and the varlen decode
workloads (tokens/s and HBM GB/s) under "extra".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl gdla|reference]

N > 1 runs under torch.distributed.run, one rank per GPU: every rank runs the
same workload on its own GPU (independent problems, no collective on the data
path), timing is the max over ranks and "value" counts the work of all ranks.
``--impl reference`` times the fp64 CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import gdla_inputs as gi  # noqa: E402

METRIC = "GDLA fwd TFLOP/s (full causal) & tokens/s (SWA-128, decode) vs B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Datasheet figures, reported beside the measured-peak fractions. The measured HBM
# figure is a copy (read + write) rate, not a ceiling for a kernel that only reads.
NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}
L2_BYTES = 126 << 20
EXTRA_STEPS_MIN = 20  # timed steps of each extra workload (the median is reported)
L2_FLUSH_BYTES = 512 << 20
FLOPS_PER_PAIR_HEAD = 2 * 192 + 2 * 128
PREFILL_KERNEL = "gdla_prefill_kernel"


# ------------------------------------------------------------------ workloads
def prefill_flops(w: gi.PrefillWorkload) -> float:
    return float(w.visible_pairs()) * 5 * w.num_kv_heads * FLOPS_PER_PAIR_HEAD


def prefill_bytes(w: gi.PrefillWorkload) -> float:
    hkv, hs = w.num_kv_heads, 4 * w.num_kv_heads
    per_token = 2 * (hs * 192 + hkv * 192 + hkv * 192 + hkv * 128 + hs * 128 + hs * 128) + 4 * hs
    return float(w.tokens) * per_token


# Backward: per visible (query, key) pair and head the recomputed forward (S 2*192,
# H = PV 2*128: the forward keeps no residuals, and the gate / lambda gradients
# need H) and the gradient products dP (2*128), dQ (2*192), dK (2*192), dV (2*128).
BWD_FLOPS_FACTOR = 3.0


def prefill_bwd_bytes(w: gi.PrefillWorkload) -> float:
    """Inputs (q_sig, q_noise, k, v, lambda, gate, dout) read once, gradients written once."""
    hkv, hs = w.num_kv_heads, 4 * w.num_kv_heads
    per_token = 2 * 2 * (hs * 192 + hkv * 192 + hkv * 192 + hkv * 128 + hs * 128) + 2 * hs * 128 + 2 * 4 * hs
    return float(w.tokens) * per_token


def decode_bytes(lengths, hkv, window) -> float:
    hs = 4 * hkv
    keys = sum(min(int(l), window) if window > 0 else int(l) for l in lengths)
    per_query = 2 * (hs * 192 + hkv * 192 + hs * 128 + hs * 128) + 4 * hs
    return float(keys) * hkv * (192 + 128) * 2 + len(lengths) * per_query


def latent_bytes(lengths, hkv, window) -> float:
    """Decode over the latent cache: 1,152 B per visible key (one 576-wide bf16
    row shared by every head), the absorbed queries, lambda, gate and output of
    each sequence, and W^UV once."""
    hs = 4 * hkv
    keys = sum(min(int(l), window) if window > 0 else int(l) for l in lengths)
    per_query = 2 * (5 * hkv * 576 + hs * 128 + hs * 128) + 4 * hs
    return float(keys) * 576 * 2 + len(lengths) * per_query + hkv * 128 * 512 * 2


def latent_flops(lengths, hkv, window) -> float:
    keys = sum(min(int(l), window) if window > 0 else int(l) for l in lengths)
    return float(keys) * 5 * hkv * (576 + 512) * 2 + len(lengths) * 5 * hkv * 128 * 512 * 2


def decode_flops(lengths, hkv, window) -> float:
    keys = sum(min(int(l), window) if window > 0 else int(l) for l in lengths)
    return float(keys) * 5 * hkv * FLOPS_PER_PAIR_HEAD


# ------------------------------------------------------------------ plumbing
def dist_info():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_max(x: float, world: int, device) -> float:
    """Max of a float over ranks (identity for one rank)."""
    if world == 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(work_per_step: float, steps: int, world: int, max_total_ms: float) -> float:
    """Work of every rank over the slowest rank's device time (units per second)."""
    return work_per_step * steps * world / (max_total_ms * 1e-3)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"]))}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = {
    "gdla_prefill_kernel": ("gdla_prefill.cu", "gdla_ptx.cuh", "gdla_internal.h"),
    "gdla_decode_split_kernel": ("gdla_decode.cu", "gdla_ptx.cuh", "gdla_internal.h"),
    "gdla_decode_latent_split_kernel": ("gdla_decode_latent.cu", "gdla_ptx.cuh", "gdla_internal.h"),
    "gdla_decode_latent_combine_kernel": ("gdla_decode_latent.cu", "gdla_ptx.cuh", "gdla_internal.h"),
    "gdla_bwd_dq_kernel": ("gdla_prefill_bwd.cu", "gdla_ptx.cuh", "gdla_internal.h"),
    "gdla_bwd_dkv_kernel": ("gdla_prefill_bwd.cu", "gdla_ptx.cuh", "gdla_internal.h"),
    "gdla_proj_kernel": ("gdla_prologue.cu", "gdla_prologue.h", "gdla_pair.cuh", "gdla_ptx.cuh", "gdla_internal.h"),
}


def _code_only(text: str) -> str:
    """C/C++/CUDA source text without comments, trailing spaces or blank lines: an
    edit to comments does not change the kernel a profile was taken of."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_source_hash(kernel: str) -> str:
    """Hash of the code a kernel is compiled from (its .cu file and the shared headers, comments excluded)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "differential_latent_attention_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name)) as f:
            h.update(name.encode() + b"\0" + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch recorded in profiles/ by an ncu capture, or None if
    there is none or the kernel sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", f"{kernel}__{workload}.txt")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_t = re.search(r"^traffic_bytes_per_launch:\s*([0-9.eE+]+)", text, re.M)
    m_h = re.search(r"^kernel_sources_sha256_16:\s*([0-9a-f]+)", text, re.M)
    if not m_t or not m_h or m_h.group(1) != kernel_source_hash(kernel):
        return None
    return float(m_t.group(1))


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML while running."""

    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            pass
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._ok:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._ok:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0, "source": "nvml" if self._ok else "unavailable"}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


def time_steps(fn, steps, warmup, flush, world):
    """Per-step device time (ms) of ``fn`` with CUDA events on the current stream;
    L2 is flushed before every step, outside the events."""
    for _ in range(warmup):
        flush()
        fn()
    torch.cuda.synchronize()
    barrier(world)
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for s, e in ev:
        flush()
        s.record(stream)
        fn()
        e.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return [s.elapsed_time(e) for s, e in ev]


# Device-side spin before each rotating step, outside its events (~50 us at 1.9 GHz):
# a call of a few tens of microseconds would otherwise be timed from its start event
# to its end event while the host was still enqueueing its launches.
HOST_LEAD_CYCLES = 100_000


def time_rotating(fns, steps, warmup, world):
    """Per-step device time (ms) with CUDA events, step i running fns[i % len(fns)]
    and no L2 flush: the sets' inputs together exceed twice the L2, so each step's
    inputs have been evicted since their previous use and no dirty flush lines are
    written back inside the timed region. A short device-side spin (touching no
    memory) precedes each step's start event, so the host has enqueued the step's
    launches before the step's timing starts."""
    for i in range(warmup):
        fns[i % len(fns)]()
    torch.cuda.synchronize()
    barrier(world)
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i, (s, e) in enumerate(ev):
        torch.cuda._sleep(HOST_LEAD_CYCLES)
        s.record(stream)
        fns[(warmup + i) % len(fns)]()
        e.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return [s.elapsed_time(e) for s, e in ev]


def hbm_roofline(nbytes, ms, peak):
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s", "frac": round(gbs / peak, 4),
            "frac_nominal": round(gbs / NOMINAL_PEAKS["hbm_gbs"], 4)}


def decode_rotation_sets(wd, lengths, n_sets, shift, dev, rank):
    """``n_sets`` decode problems sharing one packed cache: set r places every
    sequence ``r * shift`` rows further along it (so with ``shift`` >= the window
    the sets read disjoint cache rows) and has its own queries, lambda, gate and
    output."""
    lengths = np.asarray(lengths, dtype=np.int64)
    ext = lengths.copy()
    ext[-1] += (n_sets - 1) * shift
    base = gi.make_decode_inputs(ext, wd.num_kv_heads, wd.seed + 1000 * rank, device=dev)
    cu0 = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    sets = []
    for r in range(n_sets):
        small = gi.make_decode_inputs(np.ones(len(lengths), dtype=np.int64), wd.num_kv_heads,
                                      wd.seed + 1000 * rank + 7919 * (r + 1), device=dev)
        sets.append({"q_sig": small["q_sig"], "q_noise": small["q_noise"], "lam": small["lam"],
                     "gate": small["gate"], "k_cache": base["k_cache"], "v_cache": base["v_cache"],
                     "cu_seqlens_k": torch.as_tensor((cu0 + r * shift).astype(np.int32), device=dev),
                     "out": torch.empty((len(lengths), 4 * wd.num_kv_heads, 128), dtype=torch.bfloat16,
                                        device=dev)})
    return sets


def e2e_pipelined(gdla, w, host, bufs, outs, out_h, steps, world):
    """Mean ms per step of copy-in -> attn_fwd -> read-back with consecutive steps
    overlapped: step i uses device set i % 2; its inputs are copied on one stream
    (after step i-2 finished reading that set), computed on the current stream
    (after step i-2's output in that set was read back) and read back on a third.
    Timed with CUDA events from before the first copy to after the last read-back."""
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_back = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_comp[b])
                for k in host:
                    bufs[b][k].copy_(host[k], non_blocking=True)
                ev_in[b].record(s_in)
            comp.wait_event(ev_in[b])
            if i >= 2:
                comp.wait_event(ev_back[b])
            x = bufs[b]
            gdla.attn_fwd(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"], w.seqlens, w.window,
                          out=outs[b], stream=comp)
            ev_comp[b].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b])
                out_h[b].copy_(outs[b], non_blocking=True)
                ev_back[b].record(s_out)
        comp.wait_stream(s_in)
        comp.wait_stream(s_out)

    run(2)  # warm-up
    torch.cuda.synchronize()
    barrier(world)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(comp)
    s_in.wait_stream(comp)
    s_out.wait_stream(comp)
    run(steps)
    end.record(comp)
    torch.cuda.synchronize()
    barrier(world)
    return start.elapsed_time(end) / steps


# ------------------------------------------------------------------ GPU arm
def run_gdla(args):
    import differential_latent_attention_b200 as gdla
    rank, world, local = dist_info()
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    gdla.library()
    peaks, peak_src = load_peaks()
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush = flush_buf.zero_

    # ---------------- headline: full-causal prefill, T = 4096 ----------------
    w = gi.PREFILL_FULL
    t = gi.make_prefill_inputs(w.seqlens, w.num_kv_heads, w.seed + 1000 * rank, device=dev)
    out = torch.empty((w.tokens, 4 * w.num_kv_heads, 128), dtype=torch.bfloat16, device=dev)

    def step():
        gdla.attn_fwd(t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], t["gate"], w.seqlens, w.window, out=out)

    with ClockSampler(local) as clocks:
        per_step = time_steps(step, args.steps, args.warmup, flush, world)
    total_ms = reduce_max(sum(per_step), world, dev)
    assert gdla.device_error() == 0, "a kernel recorded a device-side failure"
    flops = prefill_flops(w)
    value = whole_job_rate(flops, args.steps, world, total_ms) / 1e12
    launch_ms = statistics.mean(per_step)
    achieved = flops / (launch_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]

    # ---------------- end to end through the public API, host buffers ----------------
    # Every step copies its inputs from pinned host memory to the device and reads
    # its output back. Pipelined (the number reported): two device buffer sets and
    # three streams, so step i+1's host->device copy and step i-1's read-back run
    # while step i computes (PCIe is full duplex). The serial form (copy in,
    # compute, copy out, one after the other) is reported beside it.
    host = {k: v.cpu().pin_memory() for k, v in t.items()}
    out_h = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_h[0].numel() * out_h[0].element_size()

    def e2e_step():
        for k in t:
            t[k].copy_(host[k], non_blocking=True)
        step()
        out_h[0].copy_(out, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 10))
    serial_ms = reduce_max(sum(time_steps(e2e_step, e2e_steps, 2, flush, world)), world, dev) / e2e_steps
    bufs = [t, {k: torch.empty_like(v) for k, v in t.items()}]
    outs = [out, torch.empty_like(out)]
    e2e_ms = reduce_max(e2e_pipelined(gdla, w, host, bufs, outs, out_h, e2e_steps, world), world, dev)
    e2e_value = flops * world / (e2e_ms * 1e-3) / 1e12

    # ---------------- CPU oracle baseline (rank 0, one GPU only) ----------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(t, w)
    del host, out_h

    extra = [] if args.headline_only else extra_workloads(gdla, dev, flush, args, world, rank, peaks)

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": headline_config(w, world),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 3), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "peak_source": f"bf16_tflops (burst) of {peak_src}",
                     "frac_nominal": round(achieved / NOMINAL_PEAKS["bf16_tflops"], 4),
                     "kernel": PREFILL_KERNEL, "traffic": profiled_traffic(PREFILL_KERNEL, w.name)},
        "e2e": {"value": round(e2e_value, 4), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
                "mode": "pipelined: next step's copy-in and previous step's read-back overlap the compute",
                "serial_ms_per_step": round(serial_ms, 4)},
        "gpu_launches": args.steps,  # one gdla_prefill_kernel launch per step for this workload
        "clocks": clocks.summary(),
        "extra": extra,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def headline_config(w, world):
    """The headline workload's config object, the same in both arms' JSON lines."""
    return {"workload": w.name, "batch": len(w.seqlens), "seq_len": w.seqlens[0], "q_heads": 80,
            "signal_heads": 64, "noise_heads": 16, "kv_heads": 16, "dqk": 192, "dv": 128,
            "window": "full causal", "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "flushed (512 MiB write) before every timed step, outside the events",
            "algorithmic_flops_per_step": prefill_flops(w)}


def extra_workloads(gdla, dev, flush, args, world, rank, peaks):
    """The other workloads: SWA-128 prefill, the hybrid 1 full + 3 window-128
    schedule at T = 65536, and varlen decode (full context and window 128). Each
    is timed over at least EXTRA_STEPS_MIN steps and reported as the median.
    On one GPU (rank 0) each also gets the fp64 oracle timed on the same inputs
    (all rows, or a labelled sample for the T = 65536 full-causal layer)."""
    cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    res = []
    steps = max(EXTRA_STEPS_MIN, args.steps)
    hbm = peaks["hbm_gbs"]
    # tiny: T = 256, one KV group (a parity case; launch-latency bound, 1.2 MB fits in L2)
    w = gi.TINY
    t = gi.make_prefill_inputs(w.seqlens, w.num_kv_heads, w.seed + 1000 * rank, device=dev)
    out = torch.empty((w.tokens, 4 * w.num_kv_heads, 128), dtype=torch.bfloat16, device=dev)
    per = time_steps(lambda: gdla.attn_fwd(t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], t["gate"],
                                           w.seqlens, w.window, out=out), steps, 3, lambda: None, world)
    ms = reduce_max(statistics.median(per), world, dev)
    res.append({"workload": w.name, "metric": "tokens/s", "value": w.tokens * world / (ms * 1e-3),
                "ms": round(ms, 5), "steps": steps, "stat": "median",
                "l2": "not flushed (inputs resident; the call is launch-latency bound)",
                "tflops": prefill_flops(w) / (ms * 1e-3) / 1e12})
    if cpu:
        res[-1]["cpu_baseline"] = oracle_prefill_rows(t, w, None, "tokens/s")
    del t, out
    # sliding window 128 prefill, B = 2 x 32768
    w = gi.SWA
    t = gi.make_prefill_inputs(w.seqlens, w.num_kv_heads, w.seed + 1000 * rank, device=dev)
    out = torch.empty((w.tokens, 64, 128), dtype=torch.bfloat16, device=dev)
    per = time_steps(lambda: gdla.attn_fwd(t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], t["gate"],
                                           w.seqlens, w.window, out=out), steps, 3, flush, world)
    ms = reduce_max(statistics.median(per), world, dev)
    res.append({"workload": w.name, "metric": "tokens/s", "value": w.tokens * world / (ms * 1e-3),
                "ms": round(ms, 5), "steps": steps, "stat": "median",
                "roofline": hbm_roofline(prefill_bytes(w), ms, hbm),
                "tflops": prefill_flops(w) / (ms * 1e-3) / 1e12})
    if cpu:
        res[-1]["cpu_baseline"] = oracle_prefill_rows(t, w, None, "tokens/s")
    del t, out
    # the pages' hybrid schedule: one full-causal layer then three window-128 layers, T = 65536
    layer_ms = []
    hyb_flops, hyb_bytes = 0.0, 0.0
    hyb_cpu = {}
    for li, wl in enumerate(gi.HYBRID_LAYERS):
        t = gi.make_prefill_inputs(wl.seqlens, wl.num_kv_heads, wl.seed + 1000 * rank, device=dev)
        out = torch.empty((wl.tokens, 64, 128), dtype=torch.bfloat16, device=dev)
        per = time_steps(lambda: gdla.attn_fwd(t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], t["gate"],
                                               wl.seqlens, wl.window, out=out), steps, 3, flush, world)
        layer_ms.append(reduce_max(statistics.median(per), world, dev))
        hyb_flops += prefill_flops(wl)
        hyb_bytes += prefill_bytes(wl) if wl.window > 0 else 0.0
        if cpu and li == 0:
            rows = gi.sample_rows(wl.seqlens, 512, seed=40, must_include=(0, 1, 127, 128, 65535))
            hyb_cpu["full_layer"] = oracle_prefill_rows(t, wl, rows, "rows/s")
        elif cpu and li == 1:
            hyb_cpu["window_layer"] = oracle_prefill_rows(t, wl, None, "tokens/s")
        del t, out
    hyb_ms = sum(layer_ms)
    full_tflops = prefill_flops(gi.HYBRID_LAYERS[0]) / (layer_ms[0] * 1e-3) / 1e12
    swa_gbs = hyb_bytes / (sum(layer_ms[1:]) * 1e-3) / 1e9
    res.append({"workload": "hybrid_T65536_H16_1full_3w128", "metric": "tokens/s (4 layers)",
                "value": gi.HYBRID_LAYERS[0].tokens * 4 * world / (hyb_ms * 1e-3), "ms": round(hyb_ms, 4),
                "steps": steps, "stat": "median per layer", "layer_ms": [round(x, 4) for x in layer_ms],
                "full_layer_tflops": round(full_tflops, 2),
                "full_layer_frac": round(full_tflops / peaks["bf16_tflops"], 4),
                "swa_layers_gbs": round(swa_gbs, 1), "swa_layers_frac": round(swa_gbs / hbm, 4)})
    if hyb_cpu:
        full_s = hyb_cpu["full_layer"]["extrapolated_full_s"]
        win_s = hyb_cpu["window_layer"]["seconds"]
        hyb_cpu.update({"value": round(gi.HYBRID_LAYERS[0].tokens * 4 / (full_s + 3 * win_s), 3),
                        "unit": "tokens/s (4 layers)", "cores": hyb_cpu["window_layer"]["cores"], "kind": "oracle",
                        "sample": "full-causal layer: 512 sampled rows, extrapolated to all 65,536 rows by flops; "
                                  "window-128 layer: all rows (layers 2 and 3 have the same shape)",
                        "extrapolated": True})
        res[-1]["cpu_baseline"] = hyb_cpu
    # varlen decode, 64 sequences: full context (L2 flushed; 11 GB of cache), and
    # window 128 (88 MB, under L2: 4 rotating input sets, flushed figure beside it)
    for wd in (gi.DECODE_FULL, gi.DECODE_W128):
        lengths = wd.kv_lengths()
        ws_bytes = gdla.decode_workspace_bytes(wd.batch, wd.num_kv_heads, 32768, wd.window)
        ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
        nbytes = decode_bytes(lengths, wd.num_kv_heads, wd.window)

        def call(d):
            gdla.attn_decode(d["q_sig"], d["q_noise"], d["k_cache"], d["v_cache"], d["cu_seqlens_k"], 32768,
                             d["lam"], d["gate"], wd.window, out=d["out"], workspace=ws)

        n_sets = 1 if wd.window <= 0 else max(3, int(math.ceil(2 * L2_BYTES / nbytes)) + 1)
        sets = decode_rotation_sets(wd, lengths, n_sets, max(wd.window, 0), dev, rank)
        flushed = time_steps(lambda: call(sets[0]), steps, 3, flush, world)
        ms_flushed = reduce_max(statistics.median(flushed), world, dev)
        entry = {"workload": wd.name, "metric": "query tokens/s", "steps": steps, "stat": "median"}
        if n_sets > 1:
            rot = time_rotating([lambda d=d: call(d) for d in sets], steps, 3 * n_sets, world)
            ms = reduce_max(statistics.median(rot), world, dev)
            entry["l2"] = (f"{n_sets} rotating input sets ({n_sets * nbytes / 1e6:.0f} MB of visible K/V and "
                           f"per-query tensors, > 2x L2), no flush")
            entry["flushed"] = {"ms": round(ms_flushed, 5), "roofline": hbm_roofline(nbytes, ms_flushed, hbm),
                                "l2": "flushed (512 MiB write) before every timed step"}
        else:
            ms = ms_flushed
            entry["l2"] = "flushed (512 MiB write) before every timed step"
        entry.update({"value": wd.batch * world / (ms * 1e-3), "ms": round(ms, 5),
                      "roofline": hbm_roofline(nbytes, ms, hbm)})
        if cpu:
            entry["cpu_baseline"] = oracle_decode_all(sets[0], wd)
        res.append(entry)
        del sets, ws
    res.extend(latent_workloads(gdla, dev, flush, steps, world, rank, peaks, cpu))
    res.extend(backward_workloads(gdla, dev, flush, steps, world, rank, peaks, cpu))
    res.extend(prologue_workloads(gdla, dev, flush, steps, world, rank, peaks, cpu))
    return res


PROLOGUE_WEIGHTS = ("w_qa", "w_kva", "gamma_q", "gamma_kv", "w_qb", "w_uk", "w_uv", "w_lambda", "w_gate")


def prologue_flops(n_tokens, hkv) -> float:
    """2 flop per multiply-add of the projections: x [4096] -> c^Q (1024), [c^KV; k^R] (576),
    lambda (4H), gate logits (4H x 128); c^Q -> 5H query heads x 192; c^KV -> H x (128 + 128)."""
    per_token = 4096 * (1024 + 576 + 4 * hkv + 4 * hkv * 128) + 1024 * 5 * hkv * 192 + 512 * hkv * 256
    return 2.0 * n_tokens * per_token


def prologue_workloads(gdla, dev, flush, steps, world, rank, peaks, cpu):
    """The prologue (gdla_prologue: the attention inputs from the hidden state) on the
    headline shape (4096 tokens, 16 KV groups), L2 flushed before every timed step."""
    w = gi.PREFILL_FULL
    t = gi.make_prologue_inputs(w.seqlens, w.num_kv_heads, w.seed + 1000 * rank, device=dev)
    ws = torch.empty(gdla.prologue_workspace_bytes(w.tokens), dtype=torch.uint8, device=dev)
    outs = gdla.prologue(t["x"], *[t[k] for k in PROLOGUE_WEIGHTS], w.seqlens, workspace=ws)
    per = time_steps(lambda: gdla.prologue(t["x"], *[t[k] for k in PROLOGUE_WEIGHTS], w.seqlens, outs=outs,
                                           workspace=ws), steps, 3, flush, world)
    ms = reduce_max(statistics.median(per), world, dev)
    flops = prologue_flops(w.tokens, w.num_kv_heads)
    tflops = flops / (ms * 1e-3) / 1e12
    entry = {"workload": f"prologue_T{w.tokens}_H{w.num_kv_heads}", "metric": "TFLOP/s",
             "value": round(tflops * world, 3), "ms": round(ms, 5), "steps": steps, "stat": "median",
             "l2": "flushed (512 MiB write) before every timed step", "flops_per_step": flops,
             "roofline": {"bound": "tensor", "achieved": round(tflops, 3), "peak": peaks["bf16_tflops"],
                          "unit": "TFLOP/s", "frac": round(tflops / peaks["bf16_tflops"], 4)}}
    if cpu:
        import oracle
        host = lambda x: gi.bf16_bits(x) if x.dtype == torch.bfloat16 else x.cpu().numpy()
        sample = 256
        t0 = time.perf_counter()
        oracle.prologue(host(t["x"][:sample]), *[host(t[k]) for k in PROLOGUE_WEIGHTS], (sample,))
        dt = time.perf_counter() - t0
        entry["cpu_baseline"] = {"value": round(prologue_flops(sample, w.num_kv_heads) / dt / 1e12, 6),
                                 "unit": "TFLOP/s", "cores": oracle.default_threads(), "kind": "oracle",
                                 "sample": f"first {sample} tokens of the prologue workload (numpy fp64)",
                                 "seconds": round(dt, 2)}
    del t, ws, outs
    return [entry]


def backward_workloads(gdla, dev, flush, steps, world, rank, peaks, cpu):
    """The prefill backward (gdla_attn_bwd: forward recompute, dQ, dK/dV) on the
    headline shape (T = 4096, full causal) and the SWA-128 shape (B = 2 x 32768),
    L2 flushed before every timed step."""
    res = []
    for w in (gi.PREFILL_FULL, gi.SWA):
        t = gi.make_prefill_inputs(w.seqlens, w.num_kv_heads, w.seed + 1000 * rank, device=dev)
        dout = gi.make_prefill_grad(w.seqlens, w.num_kv_heads, w.seed + 1000 * rank, device=dev)
        hkv, hs, n = w.num_kv_heads, 4 * w.num_kv_heads, w.tokens
        grads = {"dq_sig": torch.empty((n, hs, 192), dtype=torch.bfloat16, device=dev),
                 "dq_noise": torch.empty((n, hkv, 192), dtype=torch.bfloat16, device=dev),
                 "dk": torch.empty((n, hkv, 192), dtype=torch.bfloat16, device=dev),
                 "dv": torch.empty((n, hkv, 128), dtype=torch.bfloat16, device=dev),
                 "dlambda": torch.empty((n, hs), dtype=torch.float32, device=dev),
                 "dgate": torch.empty((n, hs, 128), dtype=torch.bfloat16, device=dev)}
        ws = torch.empty(gdla.attn_bwd_workspace_bytes(n, hkv), dtype=torch.uint8, device=dev)
        per = time_steps(lambda: gdla.attn_bwd(t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], t["gate"], dout,
                                               w.seqlens, w.window, grads=grads, workspace=ws), steps, 3, flush, world)
        ms = reduce_max(statistics.median(per), world, dev)
        flops = BWD_FLOPS_FACTOR * prefill_flops(w)
        tflops = flops / (ms * 1e-3) / 1e12
        entry = {"workload": w.name + "_backward", "metric": "TFLOP/s", "value": round(tflops * world, 3),
                 "ms": round(ms, 5), "steps": steps, "stat": "median",
                 "l2": "flushed (512 MiB write) before every timed step",
                 "flops_per_step": flops, "flops_note": "3x the forward's: recomputed S and PV, then dP, dQ, dK, dV",
                 "roofline": {"bound": "tensor", "achieved": round(tflops, 3), "peak": peaks["bf16_tflops"],
                              "unit": "TFLOP/s", "frac": round(tflops / peaks["bf16_tflops"], 4)},
                 "hbm": hbm_roofline(prefill_bwd_bytes(w), ms, peaks["hbm_gbs"])}
        if cpu and w.window <= 0:
            entry["cpu_baseline"] = oracle_bwd_sample(t, dout, w)
        res.append(entry)
        del t, dout, grads, ws
    return res


def oracle_bwd_sample(t, dout, w, sample_tokens=1024):
    """The fp64 backward oracle, as it stands, on the first sample_tokens tokens of
    the (single-sequence, full-causal) workload, all KV groups; value in TFLOP/s by
    the same flop count."""
    import oracle
    s = slice(0, sample_tokens)
    host = [gi.bf16_bits(t[k][s]) for k in ("q_sig", "q_noise", "k", "v")]
    cores = oracle.default_threads()
    t0 = time.perf_counter()
    oracle.prefill_bwd(*host, t["lam"][s].cpu().numpy(), gi.bf16_bits(t["gate"][s]), gi.bf16_bits(dout[s]),
                       (sample_tokens,), 0, num_threads=cores)
    dt = time.perf_counter() - t0
    pairs = sample_tokens * (sample_tokens + 1) / 2
    flops = BWD_FLOPS_FACTOR * pairs * 5 * w.num_kv_heads * FLOPS_PER_PAIR_HEAD
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"first {sample_tokens} tokens (all {w.num_kv_heads} groups) of {w.name}",
            "seconds": round(dt, 2)}


def latent_rotation_sets(wd, lengths, n_sets, shift, dev, rank):
    """Like decode_rotation_sets, for the latent-cache decode."""
    lengths = np.asarray(lengths, dtype=np.int64)
    ext = lengths.copy()
    ext[-1] += (n_sets - 1) * shift
    base = gi.make_latent_decode_inputs(ext, wd.num_kv_heads, wd.seed + 1000 * rank, device=dev)
    cu0 = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    sets = []
    for r in range(n_sets):
        small = gi.make_latent_decode_inputs(np.ones(len(lengths), dtype=np.int64), wd.num_kv_heads,
                                             wd.seed + 1000 * rank + 7919 * (r + 1), device=dev)
        sets.append({"q_abs_sig": small["q_abs_sig"], "q_abs_noise": small["q_abs_noise"], "lam": small["lam"],
                     "gate": small["gate"], "w_uv": base["w_uv"], "ckv": base["ckv"],
                     "cu_seqlens_k": torch.as_tensor((cu0 + r * shift).astype(np.int32), device=dev),
                     "out": torch.empty((len(lengths), 4 * wd.num_kv_heads, 128), dtype=torch.bfloat16,
                                        device=dev)})
    return sets


def latent_workloads(gdla, dev, flush, steps, world, rank, peaks, cpu):
    """The 64-sequence decode batch over the compressed latent cache (1,152 B per
    key instead of 10,240), full context (L2 flushed) and window 128 (rotating
    input sets, flushed figure beside it)."""
    res = []
    hbm = peaks["hbm_gbs"]
    for wd in (gi.LATENT_FULL, gi.LATENT_W128):
        lengths = wd.kv_lengths()
        ws = torch.empty(max(gdla.decode_latent_workspace_bytes(wd.batch, wd.num_kv_heads, 32768, wd.window), 1),
                         dtype=torch.uint8, device=dev)
        nbytes = latent_bytes(lengths, wd.num_kv_heads, wd.window)
        flops = latent_flops(lengths, wd.num_kv_heads, wd.window)

        def call(d):
            gdla.attn_decode_latent(d["q_abs_sig"], d["q_abs_noise"], d["ckv"], d["cu_seqlens_k"], 32768,
                                    d["w_uv"], d["lam"], d["gate"], wd.window, out=d["out"], workspace=ws)

        n_sets = 1 if wd.window <= 0 else max(3, int(math.ceil(2 * L2_BYTES / nbytes)) + 1)
        sets = latent_rotation_sets(wd, lengths, n_sets, max(wd.window, 0), dev, rank)
        flushed = time_steps(lambda: call(sets[0]), steps, 3, flush, world)
        ms_flushed = reduce_max(statistics.median(flushed), world, dev)
        entry = {"workload": wd.name, "metric": "query tokens/s", "steps": steps, "stat": "median"}
        if n_sets > 1:
            rot = time_rotating([lambda d=d: call(d) for d in sets], steps, 3 * n_sets, world)
            ms = reduce_max(statistics.median(rot), world, dev)
            entry["l2"] = (f"{n_sets} rotating input sets ({n_sets * nbytes / 1e6:.0f} MB of visible cache rows "
                           f"and per-query tensors, > 2x L2), no flush")
            entry["flushed"] = {"ms": round(ms_flushed, 5), "roofline": hbm_roofline(nbytes, ms_flushed, hbm),
                                "l2": "flushed (512 MiB write) before every timed step"}
        else:
            ms = ms_flushed
            entry["l2"] = "flushed (512 MiB write) before every timed step"
        entry.update({"value": wd.batch * world / (ms * 1e-3), "ms": round(ms, 5),
                      "roofline": hbm_roofline(nbytes, ms, hbm),
                      "tflops": round(flops / (ms * 1e-3) / 1e12, 2),
                      "tensor_frac": round(flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4)})
        if cpu:
            entry["cpu_baseline"] = oracle_latent_all(sets[0], wd)
        res.append(entry)
        del sets, ws
    return res


def oracle_latent_all(d, wd):
    """The fp64 latent-cache decode oracle on every sequence (same inputs)."""
    import oracle
    args = [gi.bf16_bits(d["q_abs_sig"]), gi.bf16_bits(d["q_abs_noise"]), gi.bf16_bits(d["ckv"]),
            d["cu_seqlens_k"].cpu().numpy().astype(np.int64), gi.bf16_bits(d["w_uv"]), d["lam"].cpu().numpy(),
            gi.bf16_bits(d["gate"])]
    cores = oracle.default_threads()
    t0 = time.perf_counter()
    oracle.decode_latent(*args, wd.window, num_threads=cores)
    dt = time.perf_counter() - t0
    return {"value": round(wd.batch / dt, 3), "unit": "query tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"all {wd.batch} sequences of {wd.name}", "seconds": round(dt, 3)}


def oracle_prefill_rows(t, w, rows, unit):
    """The fp64 oracle, as it stands, on the same prefill inputs: all rows (rows is
    None; value in tokens/s) or the given rows (value in rows/s, with the
    full-workload time extrapolated by flops and labelled as such)."""
    import oracle
    host = [gi.bf16_bits(t["q_sig"]), gi.bf16_bits(t["q_noise"]), gi.bf16_bits(t["k"]), gi.bf16_bits(t["v"]),
            t["lam"].cpu().numpy(), gi.bf16_bits(t["gate"])]
    cores = oracle.default_threads()
    t0 = time.perf_counter()
    oracle.prefill(*host, w.seqlens, w.window, rows=rows, num_threads=cores)
    dt = time.perf_counter() - t0
    if rows is None:
        return {"value": round(w.tokens / dt, 3), "unit": unit, "cores": cores, "kind": "oracle",
                "sample": f"all {w.tokens} query rows (all heads) of {w.name}", "seconds": round(dt, 2)}
    # visible keys of the sampled rows (one sequence: row r sees min(r + 1, window) keys)
    rows = np.asarray(rows, dtype=np.int64)
    keys = np.minimum(rows + 1, w.window) if w.window > 0 else rows + 1
    sample_flops = float(keys.sum()) * 5 * w.num_kv_heads * FLOPS_PER_PAIR_HEAD
    full_s = prefill_flops(w) / (sample_flops / dt)
    return {"value": round(len(rows) / dt, 3), "unit": unit, "cores": cores, "kind": "oracle",
            "sample": f"{len(rows)} sampled query rows (all heads) of {w.name}", "seconds": round(dt, 2),
            "extrapolated_full_s": round(full_s, 1), "extrapolated": True}


def oracle_decode_all(d, wd):
    """The fp64 oracle on every sequence of a decode workload (same inputs)."""
    import oracle
    args = [gi.bf16_bits(d["q_sig"]), gi.bf16_bits(d["q_noise"]), gi.bf16_bits(d["k_cache"]),
            gi.bf16_bits(d["v_cache"]), d["cu_seqlens_k"].cpu().numpy().astype(np.int64), d["lam"].cpu().numpy(),
            gi.bf16_bits(d["gate"])]
    cores = oracle.default_threads()
    t0 = time.perf_counter()
    oracle.decode(*args, wd.window, num_threads=cores)
    dt = time.perf_counter() - t0
    return {"value": round(wd.batch / dt, 3), "unit": "query tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"all {wd.batch} sequences of {wd.name}", "seconds": round(dt, 3)}


def cpu_baseline(t, w, target_s: float = 12.0):
    """The fp64 oracle, as it stands, on a bounded row sample of the same workload."""
    import oracle
    host = [gi.bf16_bits(t["q_sig"]), gi.bf16_bits(t["q_noise"]), gi.bf16_bits(t["k"]), gi.bf16_bits(t["v"]),
            t["lam"].cpu().numpy(), gi.bf16_bits(t["gate"])]
    cores = oracle.default_threads()
    # rows evenly spaced over the sequence; grow the sample until ~target_s of CPU work
    n_rows = 64
    while True:
        rows = np.linspace(0, w.tokens - 1, n_rows).astype(np.int64)
        t0 = time.perf_counter()
        oracle.prefill(*host, w.seqlens, w.window, rows=rows, num_threads=cores)
        dt = time.perf_counter() - t0
        if dt >= target_s / 4 or n_rows >= w.tokens:
            break
        n_rows = min(w.tokens, n_rows * 4)
    flops = float((rows + 1).sum()) * 5 * w.num_kv_heads * FLOPS_PER_PAIR_HEAD
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{len(rows)} evenly spaced query rows (all 80 heads) of {w.name}, {dt:.1f} s"}


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    """The fp64 CPU oracle as the reference arm: rank 0 only, bounded row samples."""
    rank, world, _ = dist_info()
    if rank != 0:
        return
    import oracle
    w = gi.PREFILL_FULL
    t = gi.make_prefill_inputs(w.seqlens, w.num_kv_heads, w.seed, device="cpu")
    host = [gi.bf16_bits(t["q_sig"]), gi.bf16_bits(t["q_noise"]), gi.bf16_bits(t["k"]), gi.bf16_bits(t["v"]),
            t["lam"].numpy(), gi.bf16_bits(t["gate"])]
    cores = oracle.default_threads()
    rng = np.random.default_rng(0)
    rows_per_step = 16
    flops = 0.0
    for _ in range(args.warmup):
        oracle.prefill(*host, w.seqlens, w.window, rows=rng.integers(0, w.tokens, 2), num_threads=cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        rows = rng.integers(0, w.tokens, rows_per_step)
        oracle.prefill(*host, w.seqlens, w.window, rows=rows, num_threads=cores)
        flops += float((rows + 1).sum()) * 5 * w.num_kv_heads * FLOPS_PER_PAIR_HEAD
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    sample = f"{rows_per_step} random query rows (all 80 heads) of {w.name} per step"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": headline_config(w, world),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


PROFILE_CASES = ("prefill_T4096_full", "prefill_T4096_full_backward", "prologue_T4096", "swa128_B2_T8192", "decode_B64_L1024_4096", "decode_B64_L1024_4096_w128",
                 "latent_decode_B64_L1024_4096", "latent_decode_B64_L1024_4096_w128")


def run_profile_case(args):
    """A few launches of one workload, small enough for a full ncu capture
    (ncu --clock-control none -k <kernel> -s <skip> -c <count> python bench.py --profile-case NAME;
    never omit --clock-control none: without it ncu locks the GPU clocks)."""
    import differential_latent_attention_b200 as gdla
    dev = torch.device("cuda", 0)
    name = args.profile_case
    if name.startswith("latent"):
        wd = gi.DecodeWorkload(name, 64, 16, 128 if name.endswith("w128") else 0, 4, 1024, 4096)
        lengths = wd.kv_lengths()
        d = gi.make_latent_decode_inputs(lengths, 16, wd.seed, device=dev)
        fn = lambda: gdla.attn_decode_latent(d["q_abs_sig"], d["q_abs_noise"], d["ckv"], d["cu_seqlens_k"], 4096,
                                             d["w_uv"], d["lam"], d["gate"], wd.window)
    elif name.startswith("decode"):
        wd = gi.DecodeWorkload(name, 64, 16, 128 if name.endswith("w128") else 0, 4, 1024, 4096)
        lengths = wd.kv_lengths()
        d = gi.make_decode_inputs(lengths, 16, wd.seed, device=dev)
        fn = lambda: gdla.attn_decode(d["q_sig"], d["q_noise"], d["k_cache"], d["v_cache"], d["cu_seqlens_k"],
                                      4096, d["lam"], d["gate"], wd.window)
    elif name.startswith("prologue"):
        w = gi.PREFILL_FULL
        t = gi.make_prologue_inputs(w.seqlens, w.num_kv_heads, w.seed, device=dev)
        fn = lambda: gdla.prologue(t["x"], *[t[k] for k in PROLOGUE_WEIGHTS], w.seqlens)
    elif name.endswith("backward"):
        w = gi.PREFILL_FULL
        t = gi.make_prefill_inputs(w.seqlens, w.num_kv_heads, w.seed, device=dev)
        dout = gi.make_prefill_grad(w.seqlens, w.num_kv_heads, w.seed, device=dev)
        fn = lambda: gdla.attn_bwd(t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], t["gate"], dout, w.seqlens,
                                   w.window)
    else:
        w = gi.PREFILL_FULL if name.startswith("prefill") else gi.PrefillWorkload(name, (8192, 8192), 16, 128, 2)
        t = gi.make_prefill_inputs(w.seqlens, w.num_kv_heads, w.seed, device=dev)
        fn = lambda: gdla.attn_fwd(t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], t["gate"], w.seqlens,
                                   w.window)
    for _ in range(args.steps):
        fn()
    torch.cuda.synchronize()
    assert gdla.device_error() == 0
    print(f"profile case {name}: {args.steps} launches done", flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("gdla", "reference"), default="gdla")
    ap.add_argument("--headline-only", action="store_true", help="skip the SWA and decode workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    ap.add_argument("--profile-case", choices=PROFILE_CASES, help="only launch this small workload --steps times "
                    "(a driver for ncu captures; prints no JSON line)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    _, world, _ = dist_info()
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}; launch N>1 with torch.distributed.run")
    if args.profile_case:
        run_profile_case(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gdla(args)


if __name__ == "__main__":
    main()
