#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200.

One step = forward + recompute backward of causal multi-head attention at the
GPT-2-medium attention shape (B=64, H=16, N=1024, d=64, bf16), the workload the
headline metric is quoted on.  The value is algorithmic TFLOP/s of the whole job:
(4 + 10) * B * H * d * (causal pairs) per step, summed over ranks, divided by the
slowest rank's device time; the K steps are timed back to back with an event after
each step (median / p10 / p90 of the step times under "step_time").  The other
workloads (long prefill, variable-length prefill, decode, long training
sequence) are timed launch by launch, each launch between its own pair of events
with L2 flushed before it, and reported under "extra".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With --gpus N > 1 it runs under torchrun, one process per GPU; every rank
processes its own full workload (weak scaling, no data exchange), and only the
timing is reduced (max over ranks).  ``--impl reference`` times the fp64 CPU
oracle on a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd/bwd TFLOPS (% of BF16 tensor peak); decode KV GB/s (% of HBM)"
WORKLOAD = dict(B=64, H=16, N=1024, d=64, causal=True)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 2 ** 20


# ----------------------------------------------------------------------------- work counts

def causal_pairs(Nq: int, Nk: int, causal: bool) -> int:
    if not causal:
        return Nq * Nk
    return sum(max(0, min(Nk, i + 1 + Nk - Nq)) for i in range(Nq))


def fwd_flops(B, H, Nq, Nk, d, causal):
    return 4 * B * H * d * causal_pairs(Nq, Nk, causal)


def bwd_flops(B, H, Nq, Nk, d, causal):
    return 10 * B * H * d * causal_pairs(Nq, Nk, causal)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons sampled through NVML every
    5 ms while active (the data nvidia-smi's clocks query shows)."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self._stop = None
        self._thread = None

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML unavailable: no clock record
            return
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
                    self.samples.append((sm, rs, pw))
                except Exception:
                    pass
                time.sleep(0.005)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is None:
            return None
        self._stop.set()
        self._thread.join(timeout=2)
        if not self.samples:
            return None
        sm = [x[0] for x in self.samples]
        reasons = sorted({n for _, rs, _ in self.samples for n, bit in self.REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "power_w_max": round(max(x[2] for x in self.samples), 1), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- timing helpers

def device_time_ms(fn, iters, stream=None):
    """Mean device time of `iters` back-to-back calls, one event pair around the loop."""
    stream = stream or torch.cuda.current_stream()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record(stream)
    for i in range(iters):
        fn(i)
    e.record(stream)
    torch.cuda.synchronize()
    return s.elapsed_time(e) / iters


class L2Flush:
    """Reads a buffer of twice the L2 size, so that the next launch finds none of its
    inputs in L2.  It reads rather than writes: a write would leave L2 full of dirty
    lines, and the timed launch would pay for writing them back to HBM.  The read
    also keeps the GPU busy while the host enqueues the launch that follows, so a
    launch's start event is not taken while the GPU waits for the host."""

    def __init__(self, device):
        self.buf = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
        self.sink = torch.zeros((), dtype=torch.float32, device=device)
        torch.cuda.synchronize(device)

    def __call__(self):
        torch.sum(self.buf, dim=0, out=self.sink)


def quantiles(ms):
    xs = sorted(ms)
    n = len(xs)
    return {"median_ms": round(statistics.median(xs), 5), "p10_ms": round(xs[n // 10], 5),
            "p90_ms": round(xs[min(n - 1, (9 * n) // 10)], 5), "mean_ms": round(sum(xs) / n, 5), "launches": n}


def per_launch_ms(fn, n, flush=None, stream=None):
    """Device time of each of `n` calls, each bracketed by its own pair of events on the
    launching stream; with `flush`, L2 is flushed before every call (outside the
    events).  Returns the times in ms, in call order."""
    stream = stream or torch.cuda.current_stream()
    evs = []
    for i in range(n):
        if flush is not None:
            flush()
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(stream)
        fn(i)
        e.record(stream)
        evs.append((s, e))
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in evs]


def timed_steps(fn, k, stream=None):
    """K back-to-back steps with an event before the first and after every step: the
    total (first to last event) and the K per-step times."""
    stream = stream or torch.cuda.current_stream()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(k + 1)]
    evs[0].record(stream)
    for i in range(k):
        fn(i)
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    return evs[0].elapsed_time(evs[k]), [evs[i].elapsed_time(evs[i + 1]) for i in range(k)]


def profile_kernels(fa):
    """Per-kernel launches and device time recorded by the library's launch profiler."""
    import ctypes
    lib = fa.load()
    lib.fa_profile_get.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_int),
                                   ctypes.POINTER(ctypes.c_double)]
    out = {}
    for i in range(lib.fa_profile_count()):
        name = ctypes.c_char_p()
        n = ctypes.c_int()
        ms = ctypes.c_double()
        if lib.fa_profile_get(i, ctypes.byref(name), ctypes.byref(n), ctypes.byref(ms)) == 0 and n.value:
            out[name.value.decode()] = {"launches": n.value, "total_ms": ms.value}
    return out


def source_sha(fname):
    with open(os.path.join(ROOT, "exact_io_aware_54_b200", "csrc", fname), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def committed_traffic(kernel):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source is unchanged."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)[kernel]
        if t["source_sha256_16"] != source_sha(t["source_file"]):
            return None
        return float(t["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


# ----------------------------------------------------------------------------- ranks

def shard_seed(seed: int, rank: int) -> int:
    """Each rank draws its own shard of independent problems (weak scaling)."""
    return seed + 1000 * rank


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time; every rank takes this collective, in the same order."""
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_rank_step: float, ms_max: float, scale: float = 1e12) -> float:
    """Units all ranks processed per second (divided by `scale`), timed by the slowest rank."""
    return world * units_per_rank_step / (ms_max * 1e-3) / scale


# ----------------------------------------------------------------------------- our arm

def end_to_end(fa, q, k, v, do, o, lse, dq, dk, dv, causal, n_steps, world, dev, step_flops):
    """The step through the public calls with its data on the host: every step copies
    Q, K, V and dO in from pinned host memory and dQ, dK, dV back out.  Three streams,
    double-buffered on the device: the inputs of step i + 1 travel in while step i
    computes and the results of step i - 1 travel out (PCIe carries both directions
    at once).  Timed from an event before the first copy to one after the last, on
    the device; the per-step figure includes the pipeline's fill and drain."""
    hin = [x.cpu().pin_memory() for x in (q, k, v, do)]
    din = [[torch.empty_like(x) for x in (q, k, v, do)] for _ in range(2)]
    dout = [[torch.empty_like(x) for x in (dq, dk, dv)] for _ in range(2)]
    hout = [[torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in (dq, dk, dv)] for _ in range(2)]
    s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def run(n):
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        start.record(s_in)
        s_comp.wait_event(start)
        s_out.wait_event(start)
        in_done, comp_done, out_done = {}, {}, {}
        for i in range(n + 2):  # stage i: copy in step i, compute step i - 1, copy out step i - 2
            if i < n:
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(comp_done[i - 2])  # that step has read this input slot
                    for dst, src in zip(din[i % 2], hin):
                        dst.copy_(src, non_blocking=True)
                    in_done[i] = torch.cuda.Event()
                    in_done[i].record(s_in)
            c = i - 1
            if 0 <= c < n:
                with torch.cuda.stream(s_comp):
                    s_comp.wait_event(in_done[c])
                    if c >= 2:
                        s_comp.wait_event(out_done[c - 2])  # that step's results have left this slot
                    qq, kk, vv, dd = din[c % 2]
                    gq, gk, gv = dout[c % 2]
                    fa.fa_fwd(qq, kk, vv, causal=causal, out=o, lse=lse)
                    fa.fa_bwd(qq, kk, vv, o, dd, lse, causal=causal, dq=gq, dk=gk, dv=gv)
                    comp_done[c] = torch.cuda.Event()
                    comp_done[c].record(s_comp)
            d = i - 2
            if 0 <= d < n:
                with torch.cuda.stream(s_out):
                    s_out.wait_event(comp_done[d])
                    for dst, src in zip(hout[d % 2], dout[d % 2]):
                        dst.copy_(src, non_blocking=True)
                    out_done[d] = torch.cuda.Event()
                    out_done[d].record(s_out)
        end.record(s_out)  # after the last copy out, which waits for everything before it
        torch.cuda.synchronize(dev)
        return start.elapsed_time(end) / n

    run(2)  # warm-up
    e_max = max_over_ranks(run(n_steps), world, dev)
    h2d = sum(x.numel() * x.element_size() for x in hin)
    d2h = sum(x.numel() * x.element_size() for x in hout[0])
    del hin, din, dout, hout
    return {"value": round(whole_job_rate(world, step_flops, e_max), 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e_max, 4),
            "steps": n_steps,
            "overlap": "inputs of step i+1 in, step i computed, results of step i-1 out, on three streams"}


def run_ours(args, rank, world, local_rank):
    import exact_io_aware_54_b200 as fa
    from exact_io_aware_54_b200 import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    B, H, N, d, causal = (WORKLOAD[k] for k in ("B", "H", "N", "d", "causal"))
    B = args.batch or B
    q, k, v, do = synth.prefill_inputs(shard_seed(synth.SEEDS["gpt2m"], rank), B, N, N, H, d, with_dout=True,
                                       device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def step(_i=0):
        fa.fa_fwd(q, k, v, causal=causal, out=o, lse=lse)
        fa.fa_bwd(q, k, v, o, do, lse, causal=causal, dq=dq, dk=dk, dv=dv)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert fa.fa_check(fa.workspace(256, dev, "fwd")) == 0 and fa.fa_check(fa.workspace(256, dev, "bwd")) == 0

    sampler = ClockSampler(local_rank)
    sampler.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    fa.load().fa_profile_start()
    total_ms, step_ms = timed_steps(step, args.steps)
    fa.load().fa_profile_stop()
    ms = total_ms / args.steps
    if world > 1:
        torch.distributed.barrier()
    timed_samples = len(sampler.samples)
    # The same step keeps running (untimed) until at least one second has passed
    # since the timed region began, so that the clock record holds enough samples
    # of this workload even when the timed region itself is short.
    soak = 0
    while not args.profile and time.perf_counter() - t_wall0 < 1.0:
        for _ in range(20):
            step()
        soak += 20
        torch.cuda.synchronize()
    clocks = sampler.stop()
    if clocks is not None:
        clocks.update({"timed_region_samples": timed_samples, "soak_steps_after_timed_region": soak,
                       "window_s": round(time.perf_counter() - t_wall0, 3)})
    kernels = profile_kernels(fa)

    ms_max = max_over_ranks(ms, world, dev)
    step_flops = fwd_flops(B, H, N, N, d, causal) + bwd_flops(B, H, N, N, d, causal)
    value = whole_job_rate(world, step_flops, ms_max)

    pk, pk_src = peaks()
    # roofline of the dominant kernel (largest device time in the timed region)
    work = {"fa_fwd_kernel": ("tensor", fwd_flops(B, H, N, N, d, causal)),
            "fa_bwd_main_kernel": ("tensor", bwd_flops(B, H, N, N, d, causal)),
            "fa_bwd_preprocess_kernel": ("hbm", B * N * H * d * (2 + 2 + 4) + B * H * N * 4),
            "fa_bwd_convert_kernel": ("hbm", B * N * H * d * (4 + 2))}
    per_kernel = {}
    for name, kv in kernels.items():
        avg = kv["total_ms"] / kv["launches"]
        bound, units = work.get(name, ("hbm", 0))
        ach = units / (avg * 1e-3) / (1e12 if bound == "tensor" else 1e9)
        peak = pk["bf16_tflops"] if bound == "tensor" else pk["hbm_gbs"]
        per_kernel[name] = {"launches": kv["launches"], "avg_ms": round(avg, 5), "bound": bound,
                            "achieved": round(ach, 1), "unit": "TFLOP/s" if bound == "tensor" else "GB/s",
                            "frac": round(ach / peak, 4)}
    dom = max(kernels, key=lambda n: kernels[n]["total_ms"]) if kernels else None
    roofline = None
    if dom:
        pkk = per_kernel[dom]
        src = {"fa_fwd_kernel": "fwd_sm100.cu"}.get(dom, "bwd_sm100.cu")
        roofline = {"kernel": dom, "bound": pkk["bound"], "achieved": pkk["achieved"],
                    "peak": pk["bf16_tflops"] if pkk["bound"] == "tensor" else pk["hbm_gbs"],
                    "peak_source": pk_src + (" burst bf16 (cuBLAS)" if pkk["bound"] == "tensor" else " copy"),
                    "unit": pkk["unit"], "frac": pkk["frac"], "traffic": committed_traffic(dom),
                    "algorithmic_units_per_launch": work[dom][1], "source": src}

    launches = sum(kv["launches"] for kv in kernels.values())

    # end to end through the public API: pinned host inputs in, gradients out, every step
    e2e = None
    if not args.profile:
        e2e = end_to_end(fa, q, k, v, do, o, lse, dq, dk, dv, causal, max(3, min(args.steps, 20)), world, dev,
                         step_flops)

    extra = run_extra(args, fa, synth, dev, pk) if (rank == 0 and not args.no_extra and not args.profile) else None
    del q, k, v, do, o, lse, dq, dk, dv
    torch.cuda.empty_cache()

    cpu_base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.profile:
        cpu_base = cpu_baseline(args.cpu_seconds)

    if rank != 0:
        return None
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16)",
        "config": {"workload": "gpt2-medium-shaped attention training step: fwd + recompute bwd, causal",
                   "B": B, "H": H, "N": N, "d": d, "causal": causal, "flops_per_step": step_flops,
                   "frac_of_peak": round(value / world / pk["bf16_tflops"], 4),
                   "l2": "no flush: the inputs of one step (Q, K, V, O, dO: 640 MiB) exceed the 126 MB L2",
                   "parallelism": f"replicas x{world} (independent shards, no collective)"},
        "step_time": quantiles(step_ms),
        "roofline": roofline, "kernels": per_kernel, "cpu_baseline": cpu_base, "e2e": e2e,
        "gpu_launches": launches, "clocks": clocks, "extra": extra,
    }
    return line


EXTRA_WORKLOADS = ("prefill8k", "prefill_varlen", "decode_single", "decode_batched", "decode_paged", "long16k",
                   "dropout_gpt2m", "blocksparse16k")


def run_extra(args, fa, synth, dev, pk, only=None):
    """The other workloads, each timed launch by launch: L2 flushed before every
    launch (outside its events), at least `--extra-launches` launches after warm-up,
    median / p10 / p90 reported; rates use the median."""
    out = {}
    n = max(50, args.extra_launches)
    flush = L2Flush(dev)
    want = (lambda name: only is None or only == name)
    if only is None:
        # The HBM-bound decode workloads go first, after a second of idle: right after
        # the tensor-bound workloads (the GPU at its 1000 W cap) the same single-request
        # launch measured 33.8 us instead of 30.8 us.
        time.sleep(1.0)
        out["order"] = "decode workloads first, after 1 s idle; then the tensor-bound ones"
    if want("decode_single"):
        _extra_decode_single(out, n, flush, fa, synth, dev, pk)
    if want("decode_batched"):
        _extra_decode_batched(out, n, flush, fa, synth, dev, pk, args.decode_seqs)
    if want("decode_paged"):
        _extra_decode_paged(out, n, flush, fa, synth, dev, pk, args.decode_seqs)
    if want("prefill8k"):
        _extra_prefill(out, n, flush, fa, synth, dev, pk)
    if want("prefill_varlen"):
        _extra_prefill_varlen(out, n, flush, fa, synth, dev, pk)
    if want("long16k"):
        _extra_long16k(out, n, flush, fa, synth, dev, pk)
    if want("dropout_gpt2m"):
        _extra_dropout_gpt2m(out, n, flush, fa, synth, dev, pk)
    if want("blocksparse16k"):
        _extra_blocksparse16k(out, n, flush, fa, synth, dev, pk)
    del flush
    torch.cuda.empty_cache()
    return out


def _timed(fn, n, flush, warm=3):
    for i in range(warm):
        fn(i)
    return quantiles(per_launch_ms(fn, n, flush))


def _tensor_entry(q, flops, pk, extra=None):
    tf = flops / (q["median_ms"] * 1e-3) / 1e12
    e = {**q, "TFLOP/s": round(tf, 1), "frac_of_peak": round(tf / pk["bf16_tflops"], 4),
         "l2": "flushed before every launch"}
    e.update(extra or {})
    return e


def _hbm_entry(q, nbytes, pk, extra=None):
    gbs = nbytes / (q["median_ms"] * 1e-3) / 1e9
    e = {**q, "GB/s": round(gbs, 1), "frac_of_hbm": round(gbs / pk["hbm_gbs"], 4), "kv_bytes": nbytes,
         "l2": "flushed before every launch"}
    e.update(extra or {})
    return e


def _extra_dropout_gpt2m(out, n, flush, fa, synth, dev, pk):
    # the headline training step (B=64 H=16 N=1024 d=64 causal) with dropout 0.1 and
    # no key mask: what the regenerated Philox mask costs
    B, H, N, d = 64, 16, 1024, 64
    q, k, v, do = synth.prefill_inputs(synth.SEEDS["gpt2m"], B, N, N, H, d, with_dout=True, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def h(i):
        fa.fa_fwd_masked(q, k, v, None, dropout_p=0.1, seed=1234 + i, causal=True, out=o, lse=lse)
        fa.fa_bwd_masked(q, k, v, o, do, lse, None, dropout_p=0.1, seed=1234 + i, causal=True, dq=dq, dk=dk, dv=dv)
    fl = fwd_flops(B, H, N, N, d, True) + bwd_flops(B, H, N, N, d, True)
    out["dropout_gpt2m_fwd_bwd"] = _tensor_entry(_timed(h, n, None), fl, pk, {
        "dropout_p": 0.1, "l2": "no flush: the inputs of one step (640 MiB) exceed the L2"})
    del q, k, v, do, o, lse, dq, dk, dv


def _extra_blocksparse16k(out, n, flush, fa, synth, dev, pk):
    # block-sparse training step, B=1 H=16 N=16384 d=64 causal, local pattern (each
    # query tile keeps its own and the previous key tile): algorithmic work counts the
    # kept blocks' pairs only
    N, H, d = 16384, 16, 64
    q, k, v, do = synth.prefill_inputs(synth.SEEDS["long16k"], 1, N, N, H, d, with_dout=True, device=dev)
    bm = synth.block_mask_inputs(0, H, N, N, pattern="local").to(dev)
    o = torch.empty_like(q)
    lse = torch.empty(1, H, N, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def h(_i):
        fa.fa_fwd_blocksparse(q, k, v, bm, causal=True, out=o, lse=lse)
        fa.fa_bwd_blocksparse(q, k, v, o, do, lse, bm, causal=True, dq=dq, dk=dk, dv=dv)
    # pairs per head: the diagonal block (causal triangle, 128 * 129 / 2) for every
    # query tile and a full previous block for all but the first
    nt = N // 128
    pairs = nt * 128 * 129 // 2 + (nt - 1) * 128 * 128
    fl = (4 + 10) * H * d * pairs
    out["blocksparse16k_fwd_bwd"] = _tensor_entry(_timed(h, n, flush), fl, pk, {
        "kept_fraction_of_causal_blocks": round((2 * nt - 1) / (nt * (nt + 1) / 2), 4)})
    del q, k, v, do, o, lse, dq, dk, dv, bm


def _extra_prefill(out, n, flush, fa, synth, dev, pk):
    # long prefill forward, B=1 H=32 N=8192 d=128 (causal and not)
    q, k, v = synth.prefill_inputs(synth.SEEDS["prefill8k"], 1, 8192, 8192, 32, 128, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(1, 32, 8192, dtype=torch.float32, device=dev)
    for causal in (True, False):
        def f(_i, causal=causal):
            fa.fa_fwd(q, k, v, causal=causal, out=o, lse=lse)
        out["prefill8k_fwd_causal" if causal else "prefill8k_fwd_noncausal"] = _tensor_entry(
            _timed(f, n, flush), fwd_flops(1, 32, 8192, 8192, 128, causal), pk)
    del q, k, v, o, lse


def _extra_prefill_varlen(out, n, flush, fa, synth, dev, pk):
    # packed variable-length prefill: 16 causal sequences, lengths U[256, 4096], H=32, d=128
    lengths = synth.ragged_lengths(synth.SEEDS["prefill8k"], 16, 256, 4096)
    total = int(lengths.sum())
    q, k, v = synth.prefill_inputs(synth.SEEDS["prefill8k"], 1, total, total, 32, 128, device=dev)
    q, k, v = (t.reshape(total, 32, 128) for t in (q, k, v))
    cu = synth.cu_seqlens_of(lengths).to(dev)
    maxL = int(lengths.max())
    o = torch.empty_like(q)
    lse = torch.empty(32, total, dtype=torch.float32, device=dev)

    def f(_i):
        fa.fa_fwd_varlen(q, k, v, cu, cu, maxL, maxL, causal=True, out=o, lse=lse)
    flops = sum(fwd_flops(1, 32, int(L), int(L), 128, True) for L in lengths)
    out["prefill_varlen_causal"] = _tensor_entry(_timed(f, n, flush), flops, pk,
                                                 {"sequences": 16, "total_tokens": total, "max_seqlen": maxL})
    # the backward of the same packed batch (O and lse from the forward above)
    do = synth.prefill_inputs(synth.SEEDS["prefill8k"] + 1, 1, total, total, 32, 128,
                              device=dev)[0].reshape(total, 32, 128)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def g(_i):
        fa.fa_bwd_varlen(q, k, v, o, do, lse, cu, cu, maxL, maxL, causal=True, dq=dq, dk=dk, dv=dv)
    flops_b = sum(bwd_flops(1, 32, int(L), int(L), 128, True) for L in lengths)
    out["prefill_varlen_causal_bwd"] = _tensor_entry(_timed(g, n, flush), flops_b, pk,
                                                     {"kernels": "preprocess + main + dQ convert"})
    del q, k, v, o, lse, cu, do, dq, dk, dv


def _extra_decode_single(out, n, flush, fa, synth, dev, pk):
    # decode: single request, L=8192, H=32, d=128
    L = 8192
    q, k, v, cu = synth.decode_inputs(synth.SEEDS["decode"], [L], 32, 128, device=dev)
    cu = cu.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty(1, 32, dtype=torch.float32, device=dev)

    def g(_i):
        fa.fa_decode_splitkv(q, k, v, cu, L, out=o, lse=lse)
    out["decode_single_8k"] = _hbm_entry(_timed(g, n, flush), 2 * 2 * 32 * 128 * L, pk,
                                         {"splits": fa.fa_decode_num_splits(1, 32, L, 128, 0)})
    del q, k, v, cu, o, lse


def _extra_decode_batched(out, n, flush, fa, synth, dev, pk, n_seqs=64):
    # decode: 64 ragged sequences, lengths U[512, 16384]
    lengths = synth.ragged_lengths(synth.SEEDS["decode"], 64, 512, 16384)[:n_seqs]
    q, k, v, cu = synth.decode_inputs(synth.SEEDS["decode"], lengths, 32, 128, device=dev)
    cu = cu.to(dev)
    maxL = int(lengths.max())
    o = torch.empty_like(q)
    lse = torch.empty(len(lengths), 32, dtype=torch.float32, device=dev)

    def g2(_i):
        fa.fa_decode_splitkv(q, k, v, cu, maxL, out=o, lse=lse)
    out["decode_batched_ragged"] = _hbm_entry(_timed(g2, n, flush), 2 * 2 * 32 * 128 * int(lengths.sum()), pk,
                                              {"splits": fa.fa_decode_num_splits(len(lengths), 32, maxL, 128, 0),
                                               "sequences": len(lengths)})
    del q, k, v, cu, o, lse


def _extra_decode_paged(out, n, flush, fa, synth, dev, pk, n_seqs=64):
    # the same 64 ragged sequences in a paged cache: pages of 64 keys in seeded random order
    lengths = synth.ragged_lengths(synth.SEEDS["decode"], 64, 512, 16384)[:n_seqs]
    q, kp, vp, table, lens = synth.paged_decode_inputs(synth.SEEDS["decode"], lengths, 32, 128, 64, device=dev)
    table, lens = table.to(dev), lens.to(dev)
    maxL = int(lengths.max())
    o = torch.empty_like(q)
    lse = torch.empty(len(lengths), 32, dtype=torch.float32, device=dev)

    def g3(_i):
        fa.fa_decode_paged(q, kp, vp, table, lens, maxL, out=o, lse=lse)
    out["decode_paged_batched"] = _hbm_entry(_timed(g3, n, flush), 2 * 2 * 32 * 128 * int(lengths.sum()), pk,
                                             {"page_size": 64, "num_pages": int(kp.shape[0])})
    del q, kp, vp, table, lens, o, lse


def _extra_long16k(out, n, flush, fa, synth, dev, pk):
    # long training sequence, B=1 H=16 N=16384 d=64 causal: fwd + bwd and peak memory
    q, k, v, do = synth.prefill_inputs(synth.SEEDS["long16k"], 1, 16384, 16384, 16, 64, with_dout=True, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(1, 16, 16384, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_f = fa.workspace(fa.fa_fwd_workspace_size(1, 16, 16384, 16384, 64), dev, "long16k_fwd")
    ws_b = fa.workspace(fa.fa_bwd_workspace_size(1, 16, 16384, 16384, 64), dev, "long16k_bwd")
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    free0, _ = torch.cuda.mem_get_info(dev)

    def h(_i):
        fa.fa_fwd(q, k, v, causal=True, out=o, lse=lse, ws=ws_f)
        fa.fa_bwd(q, k, v, o, do, lse, causal=True, dq=dq, dk=dk, dv=dv, ws=ws_b)
    qs = _timed(h, n, None, warm=2)  # no flush: the flush buffer would count as extra memory here
    free1, _ = torch.cuda.mem_get_info(dev)
    peak_extra = torch.cuda.max_memory_allocated(dev) - base
    fl = fwd_flops(1, 16, 16384, 16384, 64, True) + bwd_flops(1, 16, 16384, 16384, 64, True)
    e = _tensor_entry(qs, fl, pk)
    e.update({"l2": "no flush: Q, K, V, O, dO and the gradients (256 MiB) exceed the L2",
              "peak_alloc_increase_bytes_during_calls": int(peak_extra),
              "device_free_bytes_change": int(free0 - free1),
              "workspace_bytes": int(ws_f.numel() + ws_b.numel()),
              "one_NxN_bf16_matrix_bytes": 16384 * 16384 * 2,
              "o_n_memory_ok": bool(peak_extra < 16384 * 16384 * 2 and
                                    (ws_f.numel() + ws_b.numel()) < 16384 * 16384 * 2)})
    out["long16k_fwd_bwd"] = e
    del q, k, v, do, o, lse, dq, dk, dv


# ----------------------------------------------------------------------------- CPU oracle

def _oracle_sample(seconds, step_idx=0, heads=16):
    """Time the fp64 oracle (fwd + bwd) on `heads` heads of one batch element of the
    bench workload, repeated until `seconds` of oracle time have passed (at least
    once); input generation is not timed.  Returns (algorithmic flops, seconds, heads)."""
    import oracle
    from exact_io_aware_54_b200 import synth
    B, H, N, d, causal = (WORKLOAD[k] for k in ("B", "H", "N", "d", "causal"))
    scale = 1.0 / math.sqrt(d)
    flops, el, calls = 0, 0.0, 0
    while True:
        b = (step_idx * 7 + calls) % B
        q, k, v, do = synth.prefill_inputs(synth.SEEDS["gpt2m"] + 17 * b, 1, N, N, H, d, with_dout=True)
        arrs = [x[:, :, :heads].double().numpy() for x in (q, k, v, do)]
        ts = time.perf_counter()
        oracle.attn_fwd(arrs[0], arrs[1], arrs[2], causal, scale)
        oracle.attn_bwd(*arrs, causal, scale)
        el += time.perf_counter() - ts
        calls += 1
        flops += fwd_flops(1, heads, N, N, d, causal) + bwd_flops(1, heads, N, N, d, causal)
        if el >= seconds:
            return flops, el, calls * heads


def cpu_baseline(seconds):
    import oracle
    flops, el, heads = _oracle_sample(seconds)
    return {"value": round(flops / el / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{heads} whole heads (16 per call) of the B=64 H=16 N=1024 d=64 causal step, "
                      f"fp64 fwd + bwd, {el:.1f} s of oracle time"}


def run_reference(args, rank, world=1):
    """The oracle as it stands, one bounded sample of the workload per step, on rank
    0's host cores; the other ranks of a multi-GPU launch return without work."""
    if rank != 0:
        return None
    import oracle
    n = args.steps + args.warmup
    heads = 16 if n <= 60 else (4 if n <= 300 else 1)
    for i in range(args.warmup):
        _oracle_sample(0.0, i, heads)
    t_flops, t_el, done = 0, 0.0, 0
    for i in range(args.steps):
        f, el, hd = _oracle_sample(0.0, i, heads)
        t_flops += f
        t_el += el
        done += hd
    value = t_flops / t_el / 1e12
    sample = f"{heads} whole head(s) of one batch element per step ({done} heads in total), fp64 fwd + bwd"
    cpu = {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
           "sample": sample}
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * t_el / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) bf16, widened to fp64)",
            "config": {"workload": "gpt2-medium-shaped attention training step: fwd + recompute bwd, causal",
                       **{k: WORKLOAD[k] for k in ("B", "H", "N", "d", "causal")}, "sample": sample},
            "cpu_baseline": cpu, "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                                         "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=EXTRA_WORKLOADS, default=None,
                    help="time only this one of the other workloads and print its figures (profiling aid)")
    ap.add_argument("--batch", type=int, default=0,
                    help="override B of the step (small cases for profiler captures; 0 = the workload's B=64)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--profile", action="store_true",
                    help="time only the K steps (no clock soak, end-to-end leg, other workloads or CPU baseline): "
                         "the command profiler captures run")
    ap.add_argument("--decode-seqs", type=int, default=64,
                    help="sequences of the batched decode workloads (the first ones of the 64 seeded lengths; "
                         "fewer for profiler captures)")
    ap.add_argument("--extra-launches", type=int, default=50,
                    help="timed launches per other workload (at least 50)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.only:
        # one of the other workloads alone (used for profiler captures); no contract line
        import exact_io_aware_54_b200 as fa
        from exact_io_aware_54_b200 import synth
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        print(json.dumps(run_extra(args, fa, synth, dev, peaks()[0], only=args.only)), flush=True)
        return

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
