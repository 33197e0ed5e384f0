#!/usr/bin/env python
"""Benchmark of the ring-ordered attention forward on B200.

One step = one ``ring_attn_fwd`` over the headline workload (causal, B=1,
Hq=Hkv=32, L=131072, d=128, eight ring blocks of 16384 tokens), inputs
already resident in HBM.  The inputs (3 GiB of bf16 Q/K/V) exceed the 126 MB
L2, so no flush is needed between steps.

``python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]``
prints ONE JSON line on rank 0.  Under torchrun every rank runs its own copy
of the workload (independent problems, no collective on the data path:
weak scaling); timing is the max over ranks of the CUDA-event time.

``--impl reference`` times the fp64 CPU oracle (the only reference this
method has) on a bounded sample of query rows of the same workload.
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
sys.path.insert(0, ROOT)

METRIC = "attention fwd TFLOP/s & % of B200 BF16 tensor peak (1 GPU), causal L=128K"
UNIT = "TFLOP/s"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {"bf16_tflops": float(pk["bf16_tflops"]),
                "bf16_tflops_sustained": float(pk["bf16_tflops_sustained"]),
                "hbm_gbs": float(pk["hbm_gbs"]), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0,
                "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms while the
    timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


KERNEL_SOURCES = ["ring_attention_ordered_b200/csrc/ra_fwd.cu",
                  "ring_attention_ordered_b200/csrc/ra_fwd_roles.cuh",
                  "ring_attention_ordered_b200/csrc/ptx_sm100.cuh",
                  "ring_attention_ordered_b200/csrc/ra_api.cu",
                  "ring_attention_ordered_b200/csrc/ra_internal.h",
                  "ring_attention_ordered_b200/csrc/ra_merge_math.cuh",
                  "ring_attention_ordered_b200/csrc/ra_sync.cuh",
                  "ring_attention_ordered_b200/csrc/ra_schedule.cuh"]
FP8_KERNEL_SOURCES = ["ring_attention_ordered_b200/csrc/ra_fwd_fp8.cu",
                      "ring_attention_ordered_b200/csrc/ra_fwd_roles.cuh",
                      "ring_attention_ordered_b200/csrc/ptx_sm100.cuh",
                      "ring_attention_ordered_b200/csrc/ra_api.cu",
                      "ring_attention_ordered_b200/csrc/ra_internal.h",
                      "ring_attention_ordered_b200/csrc/ra_sync.cuh",
                      "ring_attention_ordered_b200/csrc/ra_schedule.cuh"]
# DRAM traffic records of ncu captures (bytes per launch of the named
# workload), keyed by kernel; each carries the SHA-256 of the kernel's sources
# at capture time.  The text summaries in profiles/ describe the captures.
TRAFFIC_RECORDS = "profiles/traffic.json"
KERNEL_FWD = "ra_fwd_kernel<128>"
KERNEL_FP8 = "ra_fwd_fp8_kernel"
SOURCES_OF = {KERNEL_FWD: KERNEL_SOURCES, KERNEL_FP8: FP8_KERNEL_SOURCES}


def sources_digest(sources) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in sources:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic(workload_name: str, kernel: str = KERNEL_FWD):
    """DRAM bytes per launch of ``kernel`` on the workload from the committed
    ncu record, or None when there is no record for that workload or the
    kernel's sources changed since the capture."""
    try:
        with open(os.path.join(ROOT, TRAFFIC_RECORDS)) as f:
            rec = json.load(f).get(kernel)
        if not rec or rec.get("workload") != workload_name:
            return None
        if rec.get("kernel_source_sha256") != sources_digest(SOURCES_OF[kernel]):
            return None
        return int(rec["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError, TypeError):
        return None


def max_over_ranks(ms: float, world: int, device=None) -> float:
    """Largest of the ranks' device-timed milliseconds (every rank calls it,
    in the same order)."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(world: int, steps: int, flops_per_step: float, ms_max: float) -> float:
    """Whole-job TFLOP/s: every rank runs its own copy of the workload (weak
    scaling), so the job does world * steps forward passes in ms_max."""
    return world * steps * flops_per_step / (ms_max / 1e3) / 1e12


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def cpu_oracle_sample(w, budget_s: float, seed: int = 12345):
    """Time the fp64 oracle on uniformly sampled query rows of the workload,
    batches of 64 rows until ``budget_s`` of CPU time is spent.  Returns
    (flops, seconds, rows, threads)."""
    import numpy as np
    import oracle
    from ring_attention_ordered_b200.inputs import sample_rows, workload_inputs

    q, k, v = workload_inputs(w)
    rows = sample_rows(w, 1 << 16, seed=seed)
    done, flops, t_used = 0, 0.0, 0.0
    while t_used < budget_s and done < len(rows):
        batch = rows[done:done + 64]
        t0 = time.perf_counter()
        oracle.attention_rows(q, k, v, w.causal, w.scale, batch)
        t_used += time.perf_counter() - t0
        keys = (batch[:, 2] + 1) if w.causal else np.full(len(batch), w.L)
        flops += float(4.0 * w.d * keys.sum())
        done += len(batch)
    return flops, t_used, done, os.cpu_count()


def run_reference(args, w, world, rank):
    if rank != 0:
        return 0
    os.environ.setdefault("OMP_NUM_THREADS", str(os.cpu_count()))
    per_step = []
    total_flops = total_t = 0.0
    rows = 0
    threads = os.cpu_count()
    budget = getattr(args, "ref_budget", None) or max(2.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup + args.steps):
        fl, t, n, threads = cpu_oracle_sample(w, budget, seed=1000 + i)
        if i >= args.warmup:
            per_step.append(t)
            total_flops += fl
            total_t += t
            rows += n
    value = total_flops / total_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_t / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.describe(), "name": w.name},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{rows} uniformly sampled query rows over {args.steps} steps"
                                   f" (all their allowed keys), fp64 numpy"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def fp8_supported(w) -> bool:
    return w.d == 128 and (w.L // w.n_ring) % 128 == 0


def time_fp8(api, q, k, v, w, stream, steps: int, peaks: dict, world: int = 1, dev=None):
    """The FP8 forward on the workload's inputs: block quantisation of q, k, v
    (timed on its own, HBM-bound: 2 bytes read + 1 byte written per element
    plus the scales) and W = 2 warm-up then ``steps`` timed ring_attn_fwd_fp8
    launches.  Returns a dict for the JSON line."""
    import torch
    q8, sq = api.quantize_fp8(q, stream=stream)
    k8, sk = api.quantize_fp8(k, stream=stream)
    v8, sv = api.quantize_fp8(v, stream=stream)
    out8 = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    lse8 = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=q.device)

    def quant():
        api.quantize_fp8(q, q8, sq, stream=stream)
        api.quantize_fp8(k, k8, sk, stream=stream)
        api.quantize_fp8(v, v8, sv, stream=stream)

    def fwd8():
        api.fwd_fp8(q8, sq, k8, sk, v8, sv, w.n_ring, w.causal, w.scale, out=out8, lse=lse8,
                    stream=stream)

    for _ in range(2):
        quant()
        fwd8()
    api.check_status(stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    qreps = 5
    e0.record(stream)
    for _ in range(qreps):
        quant()
    e1.record(stream)
    torch.cuda.synchronize(q.device)
    q_ms = e0.elapsed_time(e1) / qreps
    e0.record(stream)
    for _ in range(steps):
        fwd8()
    e1.record(stream)
    torch.cuda.synchronize(q.device)
    api.check_status(stream)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / steps
    flops = w.flops()
    achieved = flops / (ms / 1e3) / 1e12
    peak = 2.0 * peaks["bf16_tflops"]
    qbytes = 3 * (q.numel() + k.numel() + v.numel()) + 4 * (sq.numel() + sk.numel() + sv.numel())
    return {
        "ms": ms, "TFLOP/s": world * achieved, "steps": steps, "launches_per_call": 1,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak,
                     "frac_of_sustained": achieved / (2.0 * peaks["bf16_tflops_sustained"]),
                     "traffic": recorded_traffic(w.name, KERNEL_FP8),
                     "kernel": KERNEL_FP8,
                     "peak_kind": "E4M3 dense = 2 x bf16_tflops (burst, "
                                  f"{peaks['source']}), the nominal 4.5 / 2.25 PFLOP/s ratio"},
        "frac_of_bf16_burst": achieved / peaks["bf16_tflops"],
        "quantize": {"ms": q_ms, "GB/s": qbytes / (q_ms / 1e3) / 1e9,
                     "frac_hbm": qbytes / (q_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                     "bytes": qbytes, "launches": 3},
        "ms_with_quantize": ms + q_ms,
        "tolerance": "vs exact attention of the dequantised inputs: per element "
                     "sum_c (2^-4 w_c + 2^-10 / (f_c l_M)) |v_c| + 2^-9 |O| + 1e-3 sum_c w_c |v_c|; "
                     "lse 1e-3",
    }


def run_ours(args, w, world, rank, local):
    import torch
    import torch.distributed as dist

    from ring_attention_ordered_b200 import _lib, api
    from ring_attention_ordered_b200.inputs import workload_inputs

    _lib.load()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=dev)

    peaks = load_peaks()
    q_h, k_h, v_h = workload_inputs(w)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        api.fwd(q, k, v, w.n_ring, w.causal, w.scale, out=out, lse=lse, stream=stream)

    for _ in range(args.warmup):
        step()
    api.check_status(stream)

    sampler = ClockSampler(local) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.start()
        time.sleep(0.3)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    ev[0].record(stream)
    for i in range(args.steps):
        step()
        ev[i + 1].record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop() if sampler else None
    if world > 1:
        dist.barrier()
    api.check_status(stream)
    per_launch = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    elapsed = ev[0].elapsed_time(ev[-1])
    elapsed_max = max_over_ranks(elapsed, world, dev)

    flops = w.flops()
    value = aggregate_throughput(world, args.steps, flops, elapsed_max)

    # End to end through the public API: a stream of independent forward
    # passes whose inputs come from pinned host memory and whose outputs go
    # back to it.  Every step copies its own 3 GiB of inputs in and its
    # outputs out inside the timed region; two device buffer sets let the
    # copies of neighbouring steps run on their own streams while the kernel
    # of the current step computes (a serving pipeline).  The serial latency
    # of one step (copy in, compute, copy out) is reported beside it.
    q_p, k_p, v_p = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
    out_p = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    lse_p = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    e2e_steps = max(4, min(args.steps, 8))
    bufs = [(q, k, v, out, lse),
            (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
             torch.empty_like(out), torch.empty_like(lse))]
    h2d_s = torch.cuda.Stream(dev)
    d2h_s = torch.cuda.Stream(dev)

    def run_e2e(n_steps: int, pipelined: bool):
        h2d_done = [torch.cuda.Event() for _ in range(n_steps)]
        fwd_done = [torch.cuda.Event() for _ in range(n_steps)]
        d2h_done = [torch.cuda.Event() for _ in range(n_steps)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        h2d_s.wait_event(e0)
        d2h_s.wait_event(e0)
        for i in range(n_steps):
            bq, bk, bv, bo, bl = bufs[i % 2] if pipelined else bufs[0]
            with torch.cuda.stream(h2d_s):
                if i >= 2 or (not pipelined and i >= 1):
                    # buffer set reused: its forward must be done
                    h2d_s.wait_event(fwd_done[i - 2 if pipelined else i - 1])
                if not pipelined and i >= 1:
                    h2d_s.wait_event(d2h_done[i - 1])
                bq.copy_(q_p, non_blocking=True)
                bk.copy_(k_p, non_blocking=True)
                bv.copy_(v_p, non_blocking=True)
                h2d_done[i].record(h2d_s)
            stream.wait_event(h2d_done[i])
            if i >= 2 and pipelined:
                stream.wait_event(d2h_done[i - 2])   # outputs of the set read back
            api.fwd(bq, bk, bv, w.n_ring, w.causal, w.scale, out=bo, lse=bl, stream=stream)
            fwd_done[i].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(fwd_done[i])
                out_p.copy_(bo, non_blocking=True)
                lse_p.copy_(bl, non_blocking=True)
                d2h_done[i].record(d2h_s)
        stream.wait_event(d2h_done[n_steps - 1])
        stream.wait_event(h2d_done[n_steps - 1])
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1)

    run_e2e(2, True)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    te_max = max_over_ranks(run_e2e(e2e_steps, True), world, dev)
    e2e_value = aggregate_throughput(world, e2e_steps, flops, te_max)
    serial_ms = max_over_ranks(run_e2e(2, False), world, dev) / 2
    api.check_status(stream)
    del bufs
    h2d = sum(x.numel() * x.element_size() for x in (q_h, k_h, v_h))
    d2h = out.numel() * out.element_size() + lse.numel() * lse.element_size()

    # the merge kernel (the standalone fold of two partials), HBM-bound:
    # 3 * (4d + 4) bytes per row over all rows of the workload
    rows = w.B * w.Hq * w.L
    o_a = torch.randn(rows, w.d, device=dev)
    o_b = torch.randn(rows, w.d, device=dev)
    l_a = torch.randn(rows, device=dev)
    l_b = torch.randn(rows, device=dev)
    o_o, l_o = torch.empty_like(o_a), torch.empty_like(l_a)
    for _ in range(3):
        api.merge(o_a, l_a, o_b, l_b, out=o_o, lse_out=l_o, stream=stream)
    m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 10
    m0.record(stream)
    for _ in range(reps):
        api.merge(o_a, l_a, o_b, l_b, out=o_o, lse_out=l_o, stream=stream)
    m1.record(stream)
    torch.cuda.synchronize(dev)
    merge_ms = m0.elapsed_time(m1) / reps
    merge_bytes = 3 * (4 * w.d + 4) * rows
    del o_a, o_b, l_a, l_b, o_o, l_o

    # the backward pass on the same workload (not part of the timed forward
    # step): dQ kernel + dK/dV kernel per call, seeded synthetic dO
    bwd = None
    if not args.no_bwd:
        from ring_attention_ordered_b200.inputs import make_grad_output
        do = make_grad_output(w.B, w.L, w.Hq, w.d, w.seed).to(dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(max(16, _lib.ring_attn_bwd_workspace_size(w.B, w.Hq, w.L)),
                         dtype=torch.uint8, device=dev)
        api.fwd(q, k, v, w.n_ring, w.causal, w.scale, out=out, lse=lse, stream=stream)

        def bwd_call():
            api.bwd(q, k, v, out, do, lse, w.n_ring, w.causal, w.scale, dq, dk, dv, ws,
                    stream=stream)

        for _ in range(2):
            bwd_call()
        api.check_status(stream)
        bsteps = max(2, min(args.steps, 5))
        if world > 1:
            dist.barrier()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        for _ in range(bsteps):
            bwd_call()
        b1.record(stream)
        torch.cuda.synchronize(dev)
        api.check_status(stream)
        bwd_ms = max_over_ranks(b0.elapsed_time(b1), world, dev) / bsteps
        bflops = 2.5 * flops
        bwd = {"ms": bwd_ms, "TFLOP/s": world * bflops / (bwd_ms / 1e3) / 1e12,
               "frac_of_burst": bflops / (bwd_ms / 1e3) / 1e12 / peaks["bf16_tflops"],
               "steps": bsteps, "launches_per_call": 2,
               "flop_convention": "2.5 x forward (five L^2 d products); the two kernels "
                                  "execute 3.5 x forward (S and dP are recomputed for dQ)"}
        del do, dq, dk, dv, ws

    # the FP8 forward on the same workload (its own line object; the headline
    # value is the bf16 forward above)
    fp8 = None
    if not args.no_fp8 and fp8_supported(w):
        if world > 1:
            dist.barrier()
        fp8 = time_fp8(api, q, k, v, w, stream, max(3, min(args.steps, 10)), peaks, world, dev)

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    avg_launch_ms = sum(per_launch) / len(per_launch)
    achieved = flops / (avg_launch_ms / 1e3) / 1e12
    peak = peaks["bf16_tflops"]
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        fl, tcpu, nrows, threads = cpu_oracle_sample(w, args.cpu_budget)
        cpu = {"value": fl / tcpu / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{nrows} uniformly sampled query rows of the workload with all their "
                         f"allowed keys, fp64 numpy, {tcpu:.1f} s"}
    line = {
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": elapsed_max / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.describe(), "name": w.name, "global_batch": w.B * world,
                   "seq_len": w.L, "parallelism": f"replicas{world}",
                   "l2": "inputs (3 GiB) exceed L2; no flush",
                   "flop_convention": "4*B*Hq*L^2*d / 2 (causal)"},
        "frac_of_peak": {"of_burst": value / world / peaks["bf16_tflops"],
                         "of_sustained": value / world / peaks["bf16_tflops_sustained"],
                         "peaks": peaks["source"]},
        "tokens_per_s": world * args.steps * w.B * w.L / (elapsed_max / 1e3),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak,
                     "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                     "traffic": recorded_traffic(w.name, KERNEL_FWD),
                     "algorithmic_bytes": w.io_bytes(),
                     "kernel": KERNEL_FWD,
                     "peak_kind": f"bf16_tflops, burst ({peaks['source']}): one launch "
                                  "is a ~0.12 s kernel"},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "ms_per_step": te_max / e2e_steps, "serial_latency_ms": serial_ms,
                "mode": "pipelined: step k+1 copies in and step k-1 copies out while step k computes"},
        "gpu_launches": args.steps,
        "clocks": clocks,
        "bwd": bwd,
        "fp8": fp8,
        "merge": {"ms": merge_ms, "GB/s": merge_bytes / (merge_ms / 1e3) / 1e9,
                  "frac_hbm": merge_bytes / (merge_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                  "rows": rows, "d": w.d},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_all_workloads(args):
    """Per-workload forward throughput on one GPU (not the contract line):
    one JSON line per workload with ms, TFLOP/s, tokens/s and the fractions of
    the measured bf16 peaks, plus the SM clock seen during its timed region."""
    import torch

    from ring_attention_ordered_b200 import _lib, api
    from ring_attention_ordered_b200.inputs import WORKLOADS, workload_inputs

    _lib.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    stream = torch.cuda.current_stream(dev)
    for name, w in WORKLOADS.items():
        q_h, k_h, v_h = workload_inputs(w)
        q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
        del q_h, k_h, v_h
        out = torch.empty_like(q)
        lse = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=dev)
        steps = 2 if w.L >= 1 << 20 else (10 if w.L >= 1 << 15 else 50)
        for _ in range(3):
            api.fwd(q, k, v, w.n_ring, w.causal, w.scale, out=out, lse=lse, stream=stream)
        api.check_status(stream)
        sampler = ClockSampler(0)
        sampler.start()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            api.fwd(q, k, v, w.n_ring, w.causal, w.scale, out=out, lse=lse, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        clocks = sampler.stop()
        api.check_status(stream)
        ms = e0.elapsed_time(e1) / steps
        tflops = w.flops() / (ms / 1e3) / 1e12
        print(json.dumps({
            "kind": "workload", "workload": w.describe(), "name": name, "steps": steps,
            "ms": ms, "TFLOP/s": tflops, "tokens_per_s": w.B * w.L / (ms / 1e3),
            "frac_of_burst": tflops / peaks["bf16_tflops"],
            "frac_of_sustained": tflops / peaks["bf16_tflops_sustained"],
            "clocks": clocks}), flush=True)
        from ring_attention_ordered_b200.inputs import make_grad_output
        do = make_grad_output(w.B, w.L, w.Hq, w.d, w.seed).to(dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(max(16, _lib.ring_attn_bwd_workspace_size(w.B, w.Hq, w.L)),
                         dtype=torch.uint8, device=dev)
        bsteps = max(1, steps // 2)
        for _ in range(2):
            api.bwd(q, k, v, out, do, lse, w.n_ring, w.causal, w.scale, dq, dk, dv, ws, stream=stream)
        api.check_status(stream)
        e0.record(stream)
        for _ in range(bsteps):
            api.bwd(q, k, v, out, do, lse, w.n_ring, w.causal, w.scale, dq, dk, dv, ws, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        api.check_status(stream)
        bms = e0.elapsed_time(e1) / bsteps
        btf = 2.5 * w.flops() / (bms / 1e3) / 1e12
        print(json.dumps({
            "kind": "workload_bwd", "workload": w.describe(), "name": name, "steps": bsteps,
            "ms": bms, "TFLOP/s": btf, "frac_of_burst": btf / peaks["bf16_tflops"],
            "flop_convention": "2.5 x forward"}), flush=True)
        del do, dq, dk, dv, ws
        if fp8_supported(w):
            f8 = time_fp8(api, q, k, v, w, stream, max(2, steps // 2), peaks)
            print(json.dumps({"kind": "workload_fp8", "workload": w.describe(), "name": name,
                              **f8}), flush=True)
        del q, k, v, out, lse
        torch.cuda.empty_cache()
    return 0


def run_fwd_only(args, w):
    """The bf16 forward alone on one workload (not the contract line): W
    warm-up and K timed ring_attn_fwd launches; one JSON line.  A small
    command for hardware-counter captures of the forward kernel."""
    import torch

    from ring_attention_ordered_b200 import _lib, api
    from ring_attention_ordered_b200.inputs import workload_inputs

    _lib.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    stream = torch.cuda.current_stream(dev)
    q, k, v = (t.to(dev) for t in workload_inputs(w))
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        api.fwd(q, k, v, w.n_ring, w.causal, w.scale, out=out, lse=lse, stream=stream)
    api.check_status(stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        api.fwd(q, k, v, w.n_ring, w.causal, w.scale, out=out, lse=lse, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    api.check_status(stream)
    ms = e0.elapsed_time(e1) / max(1, args.steps)
    tf = w.flops() / (ms / 1e3) / 1e12
    print(json.dumps({"kind": "fwd", "workload": w.describe(), "name": w.name,
                      "steps": args.steps, "warmup": args.warmup, "ms": ms, "TFLOP/s": tf,
                      "frac_of_burst": tf / peaks["bf16_tflops"]}), flush=True)
    return 0


def run_bwd_only(args, w):
    """The backward pass alone on one workload (not the contract line): one
    forward, W warm-up and K timed ring_attn_bwd calls; one JSON line."""
    import torch

    from ring_attention_ordered_b200 import _lib, api
    from ring_attention_ordered_b200.inputs import make_grad_output, workload_inputs

    _lib.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    stream = torch.cuda.current_stream(dev)
    q, k, v = (t.to(dev) for t in workload_inputs(w))
    do = make_grad_output(w.B, w.L, w.Hq, w.d, w.seed).to(dev)
    out, lse = api.fwd(q, k, v, w.n_ring, w.causal, w.scale, stream=stream)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(16, _lib.ring_attn_bwd_workspace_size(w.B, w.Hq, w.L)),
                     dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        api.bwd(q, k, v, out, do, lse, w.n_ring, w.causal, w.scale, dq, dk, dv, ws, stream=stream)
    api.check_status(stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        api.bwd(q, k, v, out, do, lse, w.n_ring, w.causal, w.scale, dq, dk, dv, ws, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    api.check_status(stream)
    ms = e0.elapsed_time(e1) / max(1, args.steps)
    tf = 2.5 * w.flops() / (ms / 1e3) / 1e12
    print(json.dumps({"kind": "bwd", "workload": w.describe(), "name": w.name,
                      "steps": args.steps, "warmup": args.warmup, "ms": ms, "TFLOP/s": tf,
                      "frac_of_burst": tf / peaks["bf16_tflops"],
                      "flop_convention": "2.5 x forward"}), flush=True)
    return 0


def run_fp8_only(args, w):
    """Only the FP8 leg on one GPU: block quantisation of the workload's q, k,
    v, then W = 2 warm-up and K timed ring_attn_fwd_fp8 launches; one JSON
    line (a small command for profiling the FP8 kernel alone)."""
    import torch

    from ring_attention_ordered_b200 import _lib, api
    from ring_attention_ordered_b200.inputs import workload_inputs

    if not fp8_supported(w):
        print(json.dumps({"kind": "fp8", "name": w.name,
                          "unavailable": "the FP8 forward needs d = 128 and L / n_ring a "
                                         "multiple of 128"}), flush=True)
        return 0
    _lib.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    q, k, v = (t.to(dev) for t in workload_inputs(w))
    stream = torch.cuda.current_stream(dev)
    f8 = time_fp8(api, q, k, v, w, stream, args.steps, peaks)
    print(json.dumps({"kind": "fp8", "workload": w.describe(), "name": w.name, **f8}), flush=True)
    return 0


def run_ring_emulated(args, w):
    """The multi-host ring's compute, host by host, on one GPU (not the
    contract line).  For each layout, every host's visit sequence on the
    workload (its n_ring hosts) is timed alone with CUDA events, as that host
    would run it on its own GPU; the exchange is not part of it.  The ring's
    compute time is the slowest host's; one JSON line per layout gives the
    per-host times, that critical path, the throughput it implies for the
    n_ring-GPU job and its ratio to n_ring times the fused single-GPU kernel."""
    import torch

    from ring_attention_ordered_b200 import _lib, api, ring
    from ring_attention_ordered_b200.inputs import workload_inputs

    _lib.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    stream = torch.cuda.current_stream(dev)
    q_h, k_h, v_h = workload_inputs(w)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    del q_h, k_h, v_h
    N = w.n_ring
    steps = max(1, args.steps)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        api.check_status(stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        api.check_status(stream)
        return e0.elapsed_time(e1) / steps

    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=dev)
    fused_ms = timed(lambda: api.fwd(q, k, v, N, w.causal, w.scale, out=out, lse=lse,
                                     stream=stream))
    if not args.no_bwd:
        from ring_attention_ordered_b200.inputs import make_grad_output
        do_full = make_grad_output(w.B, w.L, w.Hq, w.d, w.seed).to(dev)
        out_full, lse_full = out, lse
        lse_rows = lse_full.permute(0, 2, 1).unsqueeze(-1)
        bwd_fused_ms = timed(lambda: api.bwd(q, k, v, out_full, do_full, lse_full, N, w.causal,
                                             w.scale, stream=stream))
    for layout in ring.LAYOUTS:
        ks = [ring.shard(k, h, N, layout) for h in range(N)]
        vs = [ring.shard(v, h, N, layout) for h in range(N)]
        host_ms, host_launches = [], []
        for host in range(N):
            qh = ring.shard(q, host, N, layout)
            plan = ring.visit_plan(host, N, w.causal, layout)
            host_launches.append(sum(len(vs_) for _, vs_ in plan))
            host_ms.append(timed(lambda: ring._run_host(
                qh, lambda t: ks[plan[t][0]], lambda t: vs[plan[t][0]], plan, w.scale,
                ring.cuda_visit)))
            del qh
        crit = max(host_ms)
        tflops = w.flops() / (crit / 1e3) / 1e12
        # the backward of the same ring, host by host: dQ halves, then dK/dV
        # halves into the held block's accumulators (fresh zeros per step)
        bwd_ms = []
        if not args.no_bwd:
            for host in range(N):
                qh = ring.shard(q, host, N, layout)
                oh = ring.shard(out_full, host, N, layout)
                dh = ring.shard(do_full, host, N, layout)
                lh = ring.shard(lse_rows, host, N, layout)[..., 0].permute(0, 1, 3, 2).contiguous()
                plan = ring.visit_plan(host, N, w.causal, layout)
                last_q = ring._last_visits(plan)
                ws = ring._workspaces(qh)
                dq_acc = torch.zeros(qh.shape, dtype=torch.float32, device=dev)
                dq_out = torch.empty_like(qh)
                acc_k = torch.zeros(ks[0].shape, dtype=torch.float32, device=dev)
                acc_v = torch.zeros(ks[0].shape, dtype=torch.float32, device=dev)

                def host_bwd():
                    for t, (j, visits) in enumerate(plan):
                        for part in (1, 2):
                            ring._bwd_phase(part, t, visits, last_q, qh, oh, dh, lh, ws, ks[j],
                                            vs[j], dq_acc, dq_out, acc_k, acc_v, w.scale,
                                            ring.cuda_bwd_visit)

                bwd_ms.append(timed(host_bwd))
                del qh, oh, dh, lh, ws, dq_acc, dq_out, acc_k, acc_v
        print(json.dumps({
            "kind": "ring_emulated", "workload": w.describe(), "layout": layout, "hosts": N,
            "host_ms": host_ms, "host_launches": host_launches, "critical_ms": crit,
            "sum_ms": sum(host_ms), "job_TFLOP/s_compute_only": tflops,
            "per_gpu_frac_of_burst": tflops / N / peaks["bf16_tflops"],
            "fused_1gpu_ms": fused_ms,
            "frac_of_fused_over_N": fused_ms / (N * crit),
            "bwd_host_ms": bwd_ms,
            "bwd_fused_1gpu_ms": None if args.no_bwd else bwd_fused_ms,
            "bwd_critical_ms": max(bwd_ms) if bwd_ms else None,
            "bwd_job_TFLOP/s_compute_only": (2.5 * w.flops() / (max(bwd_ms) / 1e3) / 1e12
                                             if bwd_ms else None)}), flush=True)
        del ks, vs
        torch.cuda.empty_cache()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-bwd", action="store_true", help="skip the backward-pass leg")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 forward leg")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--all-workloads", action="store_true",
                    help="print one line per named workload instead of the benchmark line")
    ap.add_argument("--fwd-only", action="store_true",
                    help="time only the bf16 forward on the workload")
    ap.add_argument("--bwd-only", action="store_true",
                    help="time only the backward pass on the workload")
    ap.add_argument("--fp8-only", action="store_true",
                    help="time only the FP8 forward (and its quantiser) on the workload")
    ap.add_argument("--ring-emulated", action="store_true",
                    help="time every host of the multi-host ring on this GPU (three layouts)")
    ap.add_argument("--ref-budget", type=float, default=None,
                    help="seconds of oracle time per reference step (default: fits the run in ~2 min)")
    args = ap.parse_args()
    from ring_attention_ordered_b200.inputs import HEADLINE, find_workload
    w = find_workload(args.workload or HEADLINE)
    world, rank, local = dist_setup()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args, w, world, rank)
    if args.all_workloads:
        return run_all_workloads(args)
    if args.ring_emulated:
        return run_ring_emulated(args, w)
    if args.fwd_only:
        return run_fwd_only(args, w)
    if args.bwd_only:
        return run_bwd_only(args, w)
    if args.fp8_only:
        return run_fp8_only(args, w)
    return run_ours(args, w, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
