"""Benchmark of causal kernelized linear attention (phi(x) = x x^T) on B200.

Headline (``value``): prefill tokens/s on the prefill workload B=4, H=8,
T=2048, d=32, bf16, chunk 64 -- one step is one output-only kata_prefill call
over that batch. For this size kata_prefill takes the quadratic form (one
tcgen05 kernel, (Q K^T)^2 [V | 1]); the same call in the chunked form (state
accumulation and carry, then the readout) is timed beside it under
``chunked_form``. The same JSON line carries the decode step (B=64, H=16,
d=64 from a 4096-token prefix), the long prefill (B=2, H=16, T=16384, d=64)
and the LoLA schedule (B=2, H=8, T=8192, d=64) as sub-results, the roofline
of the dominant kernel, the fp64 oracle timed on the host cores, and an
end-to-end number through the C ABI with host buffers.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kata|reference]

With N > 1 it runs under torchrun, one rank per GPU; every rank runs the same
per-GPU workload (weak scaling, no collective on the data path) and the
slowest rank's device time sets the aggregate.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from pathlib import Path

import numpy as np
import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

from kernelized_linear_attention_chunked_b200.inputs import (  # noqa: E402
    WORKLOADS, candidate_inputs, decode_inputs, prefill_inputs, recall_inputs)

METRIC = "prefill tokens/s & TFLOP/s (% bf16 peak); decode tokens/s (% HBM BW), 1×B200"
HEADLINE = "prefill_b4_h8_t2048_d32"
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def prefill_flops(w) -> float:
    """Algorithmic flops of one prefill over the workload: per head-token
    4 D (d+1) for the inter-chunk readout and state update, and
    (C+1)(2d+1) for the causal intra-chunk part (half of the square)."""
    D = w.d * (w.d + 1) // 2
    per = 4 * D * (w.d + 1) + (w.chunk + 1) * (2 * w.d + 1)
    return float(per) * w.B * w.H * w.T


def quadratic_flops(w) -> float:
    """Algorithmic flops of the quadratic form: per causal pair (j <= i) 2d for
    q.k, 2d for the weighted v and 2 for the denominator."""
    return float(w.T * (w.T + 1) // 2 * (4 * w.d + 2)) * w.B * w.H


def prefill_update_flops(w) -> float:
    """The state-update half of the inter-chunk flops: 2 D (d+1) per head-token."""
    D = w.d * (w.d + 1) // 2
    return float(2 * D * (w.d + 1)) * w.B * w.H * w.T


def prefill_bytes(w) -> float:
    """Compulsory HBM bytes: q, k, v in, o (fp32) out."""
    es = 2 if w.dtype == "bf16" else 4
    return float(w.B * w.H * w.T * w.d * (3 * es + 4))


def decode_bytes(w) -> float:
    """Per step: the fp32 state read and written once, q, k, v in, o out."""
    D = w.d * (w.d + 1) // 2
    return float(w.B * w.H * (2 * D * (w.d + 1) * 4 + 3 * w.d * 2 + w.d * 4))


def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        return json.loads(p.read_text()), "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[str] = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [x for x in sm if mx and x > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def traffic_record(kernel: str, workload: str):
    """ncu dram bytes per launch recorded under profiles/, if the kernel source
    has not changed since the counters were taken (else None). The figure is
    a recorded ncu measurement, not one taken by this run."""
    p = ROOT / "profiles" / "traffic.json"
    if not p.exists():
        return None
    rec = json.loads(p.read_text()).get(f"{kernel}@{workload}")
    if not rec:
        return None
    src = ROOT / "kernelized_linear_attention_chunked_b200" / "csrc" / rec["source"]
    if not src.exists() or hashlib.sha256(src.read_bytes()).hexdigest()[:16] != rec["sha"]:
        return None
    return rec["bytes_per_launch"]


def traffic_source(kernel: str, workload: str) -> str:
    rec = None
    p = ROOT / "profiles" / "traffic.json"
    if p.exists():
        rec = json.loads(p.read_text()).get(f"{kernel}@{workload}")
    if traffic_record(kernel, workload) is None:
        return "none: no ncu record for the current kernel source"
    return (f"recorded: ncu dram__bytes_read.sum + dram__bytes_write.sum per launch, "
            f"{rec.get('case', workload)}, kernel source sha {rec['sha']}")


def attach_traffic(roof: dict, kernels: list[str], workload: str) -> dict:
    """Add the recorded ncu DRAM bytes per call (the sum over the call's
    kernels, one launch each) to a roofline object, or None when any record is
    missing or stale."""
    recs = {k: traffic_record(k, workload) for k in kernels}
    roof["traffic"] = sum(recs.values()) if all(v is not None for v in recs.values()) else None
    roof["traffic_source"] = "; ".join(f"{k}: {traffic_source(k, workload)}" for k in kernels)
    if len(kernels) > 1:
        roof["traffic_per_kernel"] = recs
    return roof


def roofline(seconds: float, flops: float | None, nbytes: float | None, peaks,
             tensor_key: str = "bf16_tflops") -> dict:
    """Roofline of one launch or call that does `flops` algorithmic flops and
    moves `nbytes` algorithmic bytes in `seconds`. The bound is the resource
    whose floor time (work / measured peak) is the larger; both fractions are
    given, each against its measured peak."""
    out = {}
    floors = {}
    if flops:
        pk = peaks[tensor_key]
        out["tensor"] = {"achieved": flops / seconds / 1e12, "peak": pk, "unit": "TFLOP/s",
                         "frac": flops / seconds / 1e12 / pk, "peak_key": tensor_key}
        floors["tensor"] = flops / (pk * 1e12)
    if nbytes:
        pk = peaks["hbm_gbs"]
        out["hbm"] = {"achieved": nbytes / seconds / 1e9, "peak": pk, "unit": "GB/s",
                      "frac": nbytes / seconds / 1e9 / pk, "peak_key": "hbm_gbs"}
        floors["hbm"] = nbytes / (pk * 1e9)
    bound = max(floors, key=floors.get)
    main = out[bound]
    return {"bound": bound, "achieved": main["achieved"], "peak": main["peak"],
            "unit": main["unit"], "frac": main["frac"], "seconds": seconds,
            "floor_seconds": floors[bound], "algorithmic_flops": flops,
            "algorithmic_bytes": nbytes, **out}


# ---------------------------------------------------------------- oracle ----

def cpu_model() -> str:
    try:
        for line in Path("/proc/cpuinfo").read_text().splitlines():
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(w, max_heads: int | None = None, min_seconds: float = 0.0,
                 threads: int | None = None):
    """The fp64 oracle (recurrent form, the fastest exact CPU form) on a
    bounded sample of the workload, scaled to tokens/s. The sample is
    `max_heads` heads of the workload (all by default), repeated until
    `min_seconds` of CPU time have passed, on `threads` OpenMP threads (the
    host's default when None; the heads are the parallel loop)."""
    import oracle
    q, k, v = prefill_inputs(w.B, w.H, w.T, w.d, dtype=w.dtype, seed=w.seed, recipe=w.recipe)
    nh = w.B * w.H if max_heads is None else min(max_heads, w.B * w.H)
    qf, kf, vf = (x.reshape(w.B * w.H, w.T, w.d)[:nh] for x in (q, k, v))
    default = oracle.threads()
    if threads is not None:
        oracle.set_threads(threads)
    used = min(oracle.threads(), nh)  # one head per thread at a time
    try:
        reps, dt = 0, 0.0
        t0 = time.perf_counter()
        while reps == 0 or dt < min_seconds:
            oracle.recurrent(qf, kf, vf, w.eps)
            reps += 1
            dt = time.perf_counter() - t0
    finally:
        oracle.set_threads(default)
    tokens = reps * w.T * nh / w.H  # a token is one position of one sequence (all heads)
    return {"value": tokens / dt, "unit": "tokens/s", "cores": used, "kind": "oracle",
            "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
            "sample": f"recurrent fp64 form, {nh} of {w.B * w.H} heads x {w.T} tokens, "
                      f"{reps} repetition(s), {dt:.1f} s, {used} thread(s)",
            "seconds": dt / reps}


def run_reference(args, rank: int):
    if rank != 0:
        return
    import oracle  # noqa: F401
    w = WORKLOADS[HEADLINE]
    # every step is the whole workload: all 32 heads x 2048 tokens (about 0.1 s
    # on 16 host cores; the heads are the parallel loop)
    for _ in range(args.warmup):
        cpu_baseline(w)
    times, vals = [], []
    for _ in range(args.steps):
        r = cpu_baseline(w)
        times.append(r["seconds"])
        vals.append(r["value"])
    value = float(np.mean(vals))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * float(np.mean(times)), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": HEADLINE, "global_batch": w.B, "seq_len": w.T, "heads": w.H,
                       "head_dim": w.d, "chunk": w.chunk, "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "kind": "oracle",
                             "cores": r["cores"], "cpu_model": r["cpu_model"],
                             "sample": r["sample"]},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- GPU ----

def time_events(fn, iters: int, stream) -> float:
    """Device milliseconds for `iters` calls of fn, CUDA events on `stream`."""
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(iters):
        fn(i)
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end)


def per_launch_ms(fn, iters: int, stream) -> float:
    """Mean device time of one call: CUDA events on `stream` around `iters`
    back-to-back calls, divided by `iters`. (A call bracketed alone would also
    count the host's launch preparation, during which the GPU idles.)"""
    torch.cuda.synchronize()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for i in range(iters):
        fn(i)
    e.record(stream)
    e.synchronize()
    return s.elapsed_time(e) / iters


def _sync_device():
    if torch.cuda.is_available() and torch.cuda.is_initialized():
        torch.cuda.synchronize()


def barrier(dist_on):
    """Every rank's queued GPU work done, then a process-group barrier."""
    _sync_device()
    if dist_on:
        torch.distributed.barrier()
    _sync_device()


def max_over_ranks(x: float, dist_on) -> float:
    """The largest of the ranks' values (the slowest rank's time). The tensor
    lives where the process group's backend reduces: the GPU for NCCL, the host
    for gloo."""
    if not dist_on:
        return x
    nccl = torch.distributed.get_backend() == "nccl"
    t = torch.tensor([x], device="cuda" if nccl else "cpu", dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(world: int, units_per_step: float, steps: int, ms: float) -> float:
    """Whole-job throughput under weak scaling: every rank processes the same
    per-GPU work, and the slowest rank's time (ms, max over ranks) bounds it."""
    return world * units_per_step * steps / (ms / 1e3)


def dist_env():
    """(rank, world, local rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def run_kata(args, rank: int, world: int, dist_on: bool):
    import kernelized_linear_attention_chunked_b200 as kata
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    peaks, peak_kind = load_peaks()
    if args.only:
        fn = {"decode": lambda: bench_decode(kata, args, dev, stream, peaks, dist_on, world),
              "long_prefill": lambda: bench_long_prefill(kata, args, dev, stream, peaks,
                                                         dist_on, world),
              "lola": lambda: bench_lola(kata, args, dev, stream, peaks, dist_on, world),
              "sre_stress": lambda: bench_sre_stress(kata, args, dev, stream, peaks, dist_on,
                                                     world)}[args.only]
        res = fn()
        if rank == 0:
            print(json.dumps({"only": args.only, args.only: res}), flush=True)
        return
    with ClockSampler(torch.cuda.current_device()) as clocks:
        line = run_all(kata, args, rank, world, dist_on, dev, stream, peaks, peak_kind)
    line["clocks"] = clocks.summary()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(WORKLOADS[HEADLINE], min_seconds=10.0)
        cpu.pop("seconds")
        # the same form on one thread: 2 heads (one thread walks the heads in turn)
        one = cpu_baseline(WORKLOADS[HEADLINE], max_heads=2, min_seconds=3.0, threads=1)
        cpu["one_thread"] = {"value": one["value"], "unit": "tokens/s", "sample": one["sample"]}
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_all(kata, args, rank, world, dist_on, dev, stream, peaks, peak_kind):
    w = WORKLOADS[HEADLINE]

    # Headline: prefill over resident inputs. The batch's inputs and outputs
    # are 21 MB, so R copies rotate (R x 21 MB > L2) and no step finds its
    # inputs in L2.
    q, k, v = prefill_inputs(w.B, w.H, w.T, w.d, dtype=w.dtype, seed=w.seed, recipe=w.recipe)
    R = int(np.ceil(2 * L2_BYTES / prefill_bytes(w)))
    sets = [tuple(x.to(dev) for x in (q, k, v)) for _ in range(R)]
    outs = [torch.empty(w.B, w.H, w.T, w.d, device=dev) for _ in range(R)]
    ws = torch.empty(max(kata.prefill_workspace_bytes(w.B, w.H, w.T, w.d, w.chunk,
                                                      torch.bfloat16), 1),
                     dtype=torch.uint8, device=dev)

    def step(i):
        qq, kk, vv = sets[i % R]
        kata.prefill(qq, kk, vv, chunk=w.chunk, eps=w.eps, state=False, o=outs[i % R],
                     workspace=ws)

    for i in range(args.warmup):
        step(i)
    kata.sync_status()
    barrier(dist_on)
    n0 = kata.launch_count()
    t0 = time.perf_counter()
    ms = time_events(step, args.steps, stream)
    barrier(dist_on)
    wall = time.perf_counter() - t0
    launches = kata.launch_count() - n0
    kata.sync_status()
    ms = max_over_ranks(ms, dist_on)
    tokens_per_step = w.B * w.T
    value = aggregate_rate(world, tokens_per_step, args.steps, ms)
    ms_step = ms / args.steps
    # the form kata_prefill takes for this output-only call, and its flops
    form = kata.prefill_auto_form(w.B, w.H, w.T, w.d, w.chunk, torch.bfloat16)
    path = "tc" if kata.prefill_uses_tensor_cores(w.B, w.H, w.T, w.d, w.chunk, torch.bfloat16) \
        else "simt"
    # the method's algorithmic flops (the chunked form's count, whichever form
    # runs: the T^2 pair work the quadratic form does instead is not counted)
    flops = prefill_flops(w)
    tflops = flops / (ms_step / 1e3) / 1e12
    lat = per_launch_ms(step, max(args.steps, 10), stream)
    kernel = {"quadratic": "quad_kernel"}.get(form, "state_kernel+readout_kernel"
                                               if path == "tc" else "prefill_simt_kernel")
    # one launch per call for the quadratic form (the call time is that
    # kernel's launch time); the chunked form's two launches are one call
    roof = roofline(lat / 1e3, flops, prefill_bytes(w), peaks)
    roof["peak_source"] = f"{peak_kind} (MEASURED_PEAKS.json, burst)" \
        if peak_kind == "measured" else "fallback"
    roof["kernel"] = kernel
    roof["launch_ms"] = lat
    roof["traffic"] = traffic_record(kernel, HEADLINE)
    roof["traffic_source"] = traffic_source(kernel, HEADLINE)
    roof["counting"] = ("algorithmic flops per head-token 4D(d+1) + (C+1)(2d+1) "
                        "(the chunked form's count); bytes q, k, v in + fp32 o out")
    if form == "quadratic":
        roof["executed_flops_quadratic_form"] = quadratic_flops(w)
    chunked = bench_chunked_form(kata, w, sets, R, ws, args, stream, dev, peaks) \
        if form == "quadratic" else None
    with_state = bench_with_state(kata, w, sets, R, ws, args, stream, dev, peaks)

    # end to end: host q, k, v in, host o out, through the C ABI
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    oh = torch.empty(w.B, w.H, w.T, w.d).pin_memory()
    wsh = torch.empty(kata.prefill_host_workspace_bytes(w.B, w.H, w.T, w.d, w.chunk,
                                                        torch.bfloat16),
                      dtype=torch.uint8, device=dev)

    def e2e_step(i):
        kata.prefill_host(qh, kh, vh, w.chunk, w.eps, oh, wsh)

    for i in range(args.warmup):
        e2e_step(i)
    barrier(dist_on)
    ms_e2e = max_over_ranks(time_events(e2e_step, args.steps, stream), dist_on)
    e2e = {"value": aggregate_rate(world, tokens_per_step, args.steps, ms_e2e), "unit": "tokens/s",
           "h2d_bytes_per_step": 3 * q.numel() * q.element_size(),
           "d2h_bytes_per_step": oh.numel() * 4}
    del sets, outs, qh, kh, vh, oh, wsh

    sub = {}
    if not args.headline_only:
        sub["decode"] = bench_decode(kata, args, dev, stream, peaks, dist_on, world)
        sub["long_prefill"] = bench_long_prefill(kata, args, dev, stream, peaks, dist_on, world)
        sub["lola"] = bench_lola(kata, args, dev, stream, peaks, dist_on, world)
        sub["sre_stress"] = bench_sre_stress(kata, args, dev, stream, peaks, dist_on, world)

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": HEADLINE, "global_batch": w.B * world, "seq_len": w.T,
                       "heads": w.H, "head_dim": w.d, "packed_dim": w.D, "chunk": w.chunk,
                       "parallelism": f"dp{world}", "path": path, "form": form,
                       "l2": f"{R} rotating input sets ({R * prefill_bytes(w) / 2**20:.0f} MB "
                             "> 126 MB L2)"},
            "prefill": {"form": form, "flops_per_step": flops, "tflops": tflops,
                        "frac_bf16_peak": tflops / peaks["bf16_tflops"],
                        "peak_source": peak_kind},
            "chunked_form": chunked,
            "prefill_with_state": with_state,
            "roofline": roof, "cpu_baseline": None, "e2e": e2e, "gpu_launches": launches,
            "wall_s": wall}
    line.update(sub)
    return line


def state_pass(kata, w, sets, R, ws, args, stream, dev):
    """The final-state-only call (a prefill whose outputs are not needed): the
    state kernel without snapshots, its sequence split into segments when the
    feature tiles alone leave SMs idle, then the sums of the partial states."""
    Hs = torch.empty(w.B, w.H, w.D, w.d, device=dev)
    ss = torch.empty(w.B, w.H, w.D, device=dev)

    def state_step(i):
        qq, kk, vv = sets[i % R]
        kata.prefill(qq, kk, vv, chunk=w.chunk, eps=w.eps, output=False, H_out=Hs, s_out=ss,
                     workspace=ws, form="chunked")

    for i in range(3):
        state_step(i)
    n0 = kata.launch_count()
    state_step(0)
    launches = kata.launch_count() - n0
    ms = per_launch_ms(state_step, max(args.steps, 10), stream)
    f_update = prefill_update_flops(w)
    return {"ms": ms, "tflops": f_update / (ms / 1e3) / 1e12, "launches_per_call": launches,
            "traffic_state_kernel": traffic_record("state_kernel", HEADLINE)}


def bench_chunked_form(kata, w, sets, R, ws, args, stream, dev, peaks):
    """The same output-only call in the chunked form (state kernel + readout
    kernel), for comparison with the quadratic form that kata_prefill takes."""
    outs = [torch.empty(w.B, w.H, w.T, w.d, device=dev) for _ in range(R)]

    def step(i):
        qq, kk, vv = sets[i % R]
        kata.prefill(qq, kk, vv, chunk=w.chunk, eps=w.eps, state=False, o=outs[i % R],
                     workspace=ws, form="chunked")

    for i in range(args.warmup):
        step(i)
    ms = time_events(step, args.steps, stream) / args.steps
    lat = per_launch_ms(step, max(args.steps, 10), stream)
    kata.sync_status()
    flops = prefill_flops(w)
    return {"ms_per_step": ms, "tokens_per_s": w.B * w.T / (ms / 1e3),
            "flops_per_step": flops, "call_ms": lat,
            "roofline": roofline(lat / 1e3, flops, prefill_bytes(w), peaks),
            "traffic": {"state_kernel": traffic_record("state_kernel", HEADLINE),
                        "readout_kernel": traffic_record("readout_kernel", HEADLINE)},
            "state_only_call": state_pass(kata, w, sets, R, ws, args, stream, dev)}


def bench_with_state(kata, w, sets, R, ws, args, stream, dev, peaks):
    """The call a prefill that hands its state to decode makes: o and the final
    state (H, s) of the same batch; kata_prefill takes the chunked form."""
    outs = [torch.empty(w.B, w.H, w.T, w.d, device=dev) for _ in range(R)]
    Hs = torch.empty(w.B, w.H, w.D, w.d, device=dev)
    ss = torch.empty(w.B, w.H, w.D, device=dev)

    def step(i):
        qq, kk, vv = sets[i % R]
        kata.prefill(qq, kk, vv, chunk=w.chunk, eps=w.eps, o=outs[i % R], H_out=Hs, s_out=ss,
                     workspace=ws)

    for i in range(args.warmup):
        step(i)
    ms = time_events(step, args.steps, stream) / args.steps
    lat = per_launch_ms(step, max(args.steps, 10), stream)
    kata.sync_status()
    flops = prefill_flops(w)
    # the final state (fp32 H and s) is written once on top of q, k, v, o
    nbytes = prefill_bytes(w) + w.B * w.H * w.D * (w.d + 1) * 4
    return {"form": kata.prefill_auto_form(w.B, w.H, w.T, w.d, w.chunk, torch.bfloat16, True),
            "ms_per_step": ms, "tokens_per_s": w.B * w.T / (ms / 1e3), "call_ms": lat,
            "roofline": roofline(lat / 1e3, flops, nbytes, peaks)}


def bench_decode(kata, args, dev, stream, peaks, dist_on, world):
    w = WORKLOADS["decode_b64_h16_d64"]
    kp, vp, q, k, v = decode_inputs(w.B, w.H, w.d, w.prefix, w.steps, dtype=w.dtype, seed=w.seed)
    D = w.D
    Hst = torch.zeros(w.B, w.H, D, w.d, device=dev)
    s = torch.zeros(w.B, w.H, D, device=dev)
    # the prefix state: the 4096 prefix tokens written in by decode steps
    # (outputs discarded); not timed
    kpd = kp.to(dev).permute(2, 0, 1, 3).contiguous()
    vpd = vp.to(dev).permute(2, 0, 1, 3).contiguous()
    o = torch.empty(w.B, w.H, w.d, device=dev)
    for t in range(w.prefix):
        kata.decode_step(kpd[t], kpd[t], vpd[t], Hst, s, eps=w.eps, o=o)
    del kpd, vpd
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    nsteps = w.steps

    def step(i):
        kata.decode_step(qd[i % nsteps], kd[i % nsteps], vd[i % nsteps], Hst, s, eps=w.eps, o=o)

    for i in range(args.warmup):
        step(i)
    barrier(dist_on)
    n0 = kata.launch_count()
    ms = max_over_ranks(time_events(step, nsteps, stream), dist_on)
    launches = kata.launch_count() - n0
    kata.sync_status()
    ms_step = ms / nsteps
    # per step and head: phi(k) v^T update and phi(q)^T [H | s] readout, 2 flops
    # per multiply-add each, over the D (d+1) state entries
    flops = float(w.B * w.H * 4 * D * (w.d + 1))
    return {"workload": w.name, "tokens_per_s": aggregate_rate(world, w.B, nsteps, ms),
            "us_per_step": 1e3 * ms_step, "steps": nsteps,
            "roofline": attach_traffic(roofline(ms_step / 1e3, flops, decode_bytes(w), peaks),
                                       ["decode_kernel"], w.name),
            "bytes_per_step": decode_bytes(w),
            "gpu_launches": launches, "l2": "state 554 MB > 126 MB L2"}


def bench_sre_stress(kata, args, dev, stream, peaks, dist_on, world):
    """One SRE score + top-k + merge pass over a state larger than L2: B64 H16
    d64 (553.8 MB fp32 state), 192 candidates per head, keep 128, the other 64
    merged in place. The state is seeded normal values (scale 0.01) with a
    positive normaliser; candidates come from the seeded candidate generator.
    Algorithmic bytes per pass: the state read once for scoring, then read and
    written once by the merge (3 x 553.8 MB), plus the candidates."""
    B, H, d, n, keep = 64, 16, 64, 192, 128
    D = d * (d + 1) // 2
    gen = torch.Generator(device=dev).manual_seed(7)
    Hst = torch.randn(B, H, D, d, device=dev, generator=gen) * 0.01
    s = torch.rand(B, H, D, device=dev, generator=gen) + 0.5
    kc, vc, pos = (x.to(dev) for x in candidate_inputs(B, H, n, d, dtype="bf16", seed=5))
    state_bytes = float(B * H * D * (d + 1) * 4)
    nbytes = 3 * state_bytes + float(kc.numel() * 2 * 2 + pos.numel() * 4)

    def step(i):
        kata.sre_score_topk(Hst, s, kc, vc, pos, keep=keep, merge=True)

    for i in range(max(args.warmup, 2)):
        step(i)
    kata.sync_status()
    barrier(dist_on)
    iters = max(args.steps // 2, 3)
    n0 = kata.launch_count()
    ms = max_over_ranks(time_events(step, iters, stream), dist_on) / iters
    launches = (kata.launch_count() - n0) // iters
    kata.sync_status()
    # fp32 work: phi(k)^T [H | s] for every candidate, then a rank-one update
    # of [H | s] for every merged one (2 flops per multiply-add)
    flops = float(B * H * (n + (n - keep)) * D * (d + 1) * 2)
    roof = attach_traffic(roofline(ms / 1e3, None, nbytes, peaks), ["sre_tc_kernel"],
                          "sre_b64_h16_d64_n192_keep128")
    roof["note"] = ("HBM roofline of the algorithmic bytes; the scores run on the tensor "
                    "cores with split bf16 operands at fp32-level accuracy (fp32_tflops is "
                    "the method's fp32 operation count per second, not a roofline)")
    return {"workload": "sre_b64_h16_d64_n192_keep128", "ms_per_pass": ms,
            "roofline": roof, "bytes_per_pass": nbytes,
            "fp32_tflops": flops / (ms / 1e3) / 1e12, "flops_per_pass": flops,
            "gpu_launches_per_pass": launches, "l2": "state 554 MB > 126 MB L2"}


def bench_long_prefill(kata, args, dev, stream, peaks, dist_on, world):
    w = WORKLOADS["long_prefill_b2_h16_t16384_d64"]
    q, k, v = (x.to(dev) for x in prefill_inputs(w.B, w.H, w.T, w.d, dtype=w.dtype,
                                                  seed=w.seed, recipe=w.recipe))
    o = torch.empty(w.B, w.H, w.T, w.d, device=dev)
    ws = torch.empty(max(kata.prefill_workspace_bytes(w.B, w.H, w.T, w.d, w.chunk,
                                                      torch.bfloat16), 1),
                     dtype=torch.uint8, device=dev)

    def step(i):
        kata.prefill(q, k, v, chunk=w.chunk, eps=w.eps, state=False, o=o, workspace=ws)

    step(0)
    barrier(dist_on)
    n = max(2, min(args.steps, 10))
    ms = max_over_ranks(time_events(step, n, stream), dist_on) / n
    kata.sync_status()
    fl = prefill_flops(w)
    return {"workload": w.name, "tokens_per_s": aggregate_rate(world, w.B * w.T, 1, ms), "ms": ms,
            "form": kata.prefill_auto_form(w.B, w.H, w.T, w.d, w.chunk, torch.bfloat16),
            "roofline": attach_traffic(roofline(ms / 1e3, fl, prefill_bytes(w), peaks),
                                       ["state_kernel", "readout_kernel"], w.name),
            "l2": "inputs 335 MB > 126 MB L2"}


def bench_lola(kata, args, dev, stream, peaks, dist_on, world):
    w = WORKLOADS["lola_b2_h8_t8192_d64"]
    q, k, v = (x.to(dev) for x in recall_inputs(w.B, w.H, w.T, w.d, dtype=w.dtype, seed=w.seed))
    D = w.D
    Hst = torch.zeros(w.B, w.H, D, w.d, device=dev)
    s = torch.zeros_like(Hst[..., 0])
    o = torch.empty(w.B, w.H, w.T, w.d, device=dev)
    ws = torch.empty(kata.lola_prefill_workspace_bytes(w.B, w.H, w.T, w.d, w.window, w.cache),
                     dtype=torch.uint8, device=dev)

    def step(i, run="auto"):
        Hst.zero_()
        s.zero_()
        kata.lola_prefill(q, k, v, window=w.window, cache=w.cache, eps=w.eps, Hst=Hst, s=s,
                          o=o, workspace=ws, run=run)

    run = "fused" if kata.lola_fused_applies(torch.bfloat16, w.d, w.window, w.cache) \
        else "segments"
    for i in range(3):
        step(i)
    barrier(dist_on)
    n0 = kata.launch_count()
    n = 10
    ms = max_over_ranks(time_events(step, n, stream), dist_on) / n
    launches = (kata.launch_count() - n0) // n
    kata.sync_status()
    # the same schedule as launches per segment, for comparison
    step(0, "segments")
    ms_seg = time_events(lambda i: step(i, "segments"), 2, stream) / 2
    kata.sync_status()
    # labelled state-streaming model: every update of every head reads and
    # writes that head's fp32 state once (2 x D (d+1) x 4 bytes)
    updates = w.T // w.window - 1
    stream_bytes = float(2 * w.D * (w.d + 1) * 4 * updates * w.B * w.H)
    roof = roofline(ms / 1e3, None, stream_bytes, peaks)
    roof["model"] = ("state-streaming model: each of the 127 updates of each head reads and "
                     "writes its 540,800-byte fp32 state once; the state fits in L2, so this "
                     "is a yardstick, not the bytes HBM moves")
    if run == "fused":
        attach_traffic(roof, ["lola_fused_kernel"], w.name)
    return {"workload": w.name, "tokens_per_s": world * w.B * w.T / (ms / 1e3), "ms": ms,
            "run": run, "updates": updates, "gpu_launches_per_pass": launches, "roofline": roof,
            "segments_run_ms": ms_seg,
            "note": "includes two state zero-fills per pass (torch memset)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["kata", "reference"], default="kata")
    ap.add_argument("--headline-only", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["decode", "long_prefill", "lola", "sre_stress"],
                    default=None,
                    help="run one sub-benchmark alone (for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_env()
    dist_on = world > 1
    if args.impl == "reference":
        run_reference(args, rank)
        return
    torch.cuda.set_device(local)
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    try:
        run_kata(args, rank, world, dist_on)
    finally:
        if dist_on:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
