#!/usr/bin/env python3
"""Throughput benchmark of the exact attention forward (fa_fwd) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one fa_fwd call over the whole workload (every row of the hot path: tile
schedule, TMA loads, QK^T, online softmax, PV, epilogue).  Default workload: the
d=128, N=4096 point of the sequence-length sweep (B=8, H=32), inputs larger than L2.
For N > 1 (launched under torchrun) every rank runs its own replica on its own seeded
batch (weak scaling: no data-path collective exists in the forward pass); the time is
the max over ranks of CUDA-event time.

Prints ONE JSON line (rank 0).  TFLOP/s counts 4*B*Hq*Nq*Nk*d per call (half for causal).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import synth  # noqa: E402

METRIC = "attention fwd TFLOP/s and % of B200 bf16 tensor peak vs seq len (1 GPU)"
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0, "source": "fallback"}
KERNEL_NAME = "fa_fwd_kernel"


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return {"bf16_tflops": float(d["bf16_tflops"]), "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", 0)),
                "hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return dict(FALLBACK_PEAKS)


def fp8_peak():
    """Measured dense E4M3 GEMM throughput (TFLOP/s, burst) from profiles/fp8_gemm_peak.md, or None."""
    f = ROOT / "profiles" / "fp8_gemm_peak.md"
    if not f.exists():
        return None
    m = re.search(r"fp8_tflops_burst:\s*([0-9.]+)", f.read_text())
    return float(m.group(1)) if m else None


def tensor_peak(pk, w):
    """(TFLOP/s, source) of the tensor roofline for a workload's dtype: the measured bf16
    figure (fp16 has the same nominal rate); E4M3 takes the measured E4M3 GEMM figure, else
    the bf16 one x 2 (the nominal dense fp8/bf16 ratio, 4.5 / 2.25 PFLOP/s)."""
    if w.dtype == "e4m3":
        f8 = fp8_peak()
        if f8 is not None:
            return f8, "measured E4M3 GEMM 8192^3 (burst, profiles/fp8_gemm_peak.md)"
        return 2.0 * pk["bf16_tflops"], f"{pk['source']} bf16 dense (burst) x 2 (nominal fp8/bf16 ratio)"
    return pk["bf16_tflops"], f"{pk['source']} bf16 dense (burst)"


FORWARD_SOURCES = ("fa_fwd.cu", "fa_host.h", "fa_kernel.cuh", "sm100.cuh")


def _code_only(text: str) -> str:
    """C/C++ source with comments removed and whitespace collapsed (none of these files
    has a comment marker inside a string literal)."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash() -> str:
    """Hash of the code (comments aside) the forward kernel and its launch are built from;
    the backward's own files are left out, so they can change without invalidating forward
    profiles."""
    h = hashlib.sha256()
    for name in FORWARD_SOURCES:
        h.update(_code_only((ROOT / "exact_attention_146_b200" / "csrc" / name).read_text()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the kernel from the committed ncu summary, if that
    summary was taken on the current kernel source (else None)."""
    f = ROOT / "profiles" / f"{KERNEL_NAME}_{workload}.md"
    if not f.exists():
        return None
    text = f.read_text()
    m_hash = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", text)
    m_bytes = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_hash or not m_bytes or m_hash.group(1) != kernel_source_hash():
        return None
    return float(m_bytes.group(1))


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 50):
        self.rows = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 f"-lms={period_ms}"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                self.rows.append((time.time(), parts))

    def window(self, t0, t1):
        return [r for (t, r) in self.rows if t0 <= t <= t1]

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    @staticmethod
    def summarize(rows):
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus and world > 1:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    return world, rank, local


def rank_workload(w: synth.Workload, rank: int) -> synth.Workload:
    """Each rank's replica: the same shapes on its own seeded data (weak scaling)."""
    return w.with_(seed=w.seed + rank)


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """The max of a per-rank figure (time) over all ranks; the identity without a group."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_tflops(w: synth.Workload, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank processed one workload in (at most) ms_max."""
    return world * w.flops / (ms_max * 1e-3) / 1e12


def oracle_sample_tflops(w: synth.Workload, target_s: float, heads_cap: int | None = None):
    """Time the CPU oracle on a bounded sample of the workload: whole (b, hq) heads of
    batch element 0, as many as fit in ~target_s.  Returns (TFLOP/s, sample text, cores)."""
    import oracle
    orc = oracle.default()
    cores = os.cpu_count() or 1
    one = w.with_(B=1)
    x = synth.make_inputs(one)
    per_head = w.flops / (w.B * w.Hq)
    done_flop, t_used, heads = 0.0, 0.0, 0
    n_rep = w.Hq // w.Hkv
    h = 0
    while t_used < target_s and h < w.Hq and (heads_cap is None or heads < heads_cap):
        g = h // n_rep
        q = np.ascontiguousarray(x["q"][:, :, h:h + 1])
        k = np.ascontiguousarray(x["k"][:, :, g:g + 1])
        v = np.ascontiguousarray(x["v"][:, :, g:g + 1])
        t0 = time.perf_counter()
        orc.forward(q, k, v, w.scale, w.causal, threads=cores, window=w.window, dtype=w.dtype)
        t_used += time.perf_counter() - t0
        done_flop += per_head
        heads += 1
        h += 1
    tf = done_flop / t_used / 1e12
    return tf, f"{heads} of {w.B * w.Hq} (b, head) slices of {w.name} (batch element 0), {t_used:.1f} s", cores, t_used


def run_reference(args, w, world, rank):
    """The CPU fp64 oracle as the reference arm, timed on this host's cores."""
    if rank != 0:
        return 0
    import oracle
    orc = oracle.default()
    cores = os.cpu_count() or 1
    x = synth.make_inputs(w.with_(B=1))
    per_head = w.flops / (w.B * w.Hq)
    times = []
    for step in range(args.warmup + args.steps):
        h = step % w.Hq
        g = h // (w.Hq // w.Hkv)
        q = np.ascontiguousarray(x["q"][:, :, h:h + 1])
        k = np.ascontiguousarray(x["k"][:, :, g:g + 1])
        v = np.ascontiguousarray(x["v"][:, :, g:g + 1])
        t0 = time.perf_counter()
        orc.forward(q, k, v, w.scale, w.causal, threads=cores, window=w.window, dtype=w.dtype)
        dt = time.perf_counter() - t0
        if step >= args.warmup:
            times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = per_head / (ms * 1e-3) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.Nq, "Nk": w.Nk, "d": w.d,
                   "causal": w.causal, "step": "one (b, head) slice of the workload per step"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"one (b, head) slice of {w.name} per step"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def device_inputs(torch, x, w, pin=False):
    """q, k, v of a workload as torch tensors: bf16 / fp16 bits, or E4M3 bytes (uint8)."""
    if w.dtype == "e4m3":
        ts = {n: torch.from_numpy(np.ascontiguousarray(x[n])) for n in ("q", "k", "v")}
    else:
        tdt = torch.float16 if w.dtype == "f16" else torch.bfloat16
        ts = {n: torch.from_numpy(x[n].view(np.int16)).view(tdt) for n in ("q", "k", "v")}
    return {n: (t.pin_memory() if pin else t) for n, t in ts.items()}


def forward_call(fa, w, q, k, v, out, lse, **kw):
    """The entry point a workload runs through (fa_fwd_fp8 for E4M3 inputs)."""
    if w.dtype == "e4m3":
        return fa.fa_fwd_fp8(q, k, v, causal=w.causal, scale=w.scale, out=out, lse=lse, stream=kw.get("stream"))
    return fa.fa_fwd(q, k, v, causal=w.causal, scale=w.scale, out=out, lse=lse, **kw)


def run_ours(args, w, world, rank, local):
    import torch
    import exact_attention_146_b200 as fa

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
        pg = dist
    stream = torch.cuda.current_stream()

    # per-rank replica of the workload on its own seeded data (weak scaling)
    wr = rank_workload(w, rank)
    x = synth.make_inputs(wr)
    host = device_inputs(torch, x, w, pin=True)
    q, k, v = (host[n].to(dev, non_blocking=True) for n in ("q", "k", "v"))
    out = torch.empty(q.shape, dtype=torch.bfloat16 if w.dtype == "e4m3" else q.dtype, device=dev)
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)
    # split-KV workloads: the library's default split count, workspace allocated once here
    splits = (fa.splitkv_default_splits(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d,
                                        torch.cuda.get_device_properties(dev).multi_processor_count)
              if w.splitkv else 1)
    ws = (torch.empty(max(1, fa.splitkv_workspace_bytes(w.B, w.Hq, w.Nq, w.d, splits)), dtype=torch.uint8, device=dev)
          if splits > 1 else None)
    call_kw = dict(window=w.window or None, num_splits=splits if splits > 1 else None, workspace=ws)
    launches_per_step = 2 if splits > 1 else 1      # forward kernel (+ merge kernel)
    torch.cuda.synchronize()

    def step():
        forward_call(fa, w, q, k, v, out, lse, **call_kw)

    for _ in range(args.warmup):
        step()
    st, word = fa.device_status()
    if st != fa.FA_OK:
        raise SystemExit(f"device status after warm-up: {st} ({word:#x})")

    sampler = ClockSampler(local) if not args.no_clocks else None
    if sampler:
        time.sleep(0.3)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if pg:
        pg.barrier()
    ms = e0.elapsed_time(e1) / args.steps
    st, word = fa.device_status()
    if st != fa.FA_OK:
        raise SystemExit(f"device status after timed steps: {st} ({word:#x})")
    clocks = None
    if sampler:
        time.sleep(0.15)
        sampler.stop()
        clocks = ClockSampler.summarize(sampler.window(t_wall0, t_wall1 + 0.1))
    ms_max = max_over_ranks(ms, pg, dev)
    value = weak_scaling_tflops(w, world, ms_max)
    pk = peaks()
    achieved = w.flops / (ms * 1e-3) / 1e12           # per launch on this rank
    gbs = w.io_bytes / (ms * 1e-3) / 1e9
    if w.io_bytes / (pk["hbm_gbs"] * 1e9) > w.flops / (pk["bf16_tflops"] * 1e12):   # bytes bound it (decode)
        roofline = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": gbs / pk["hbm_gbs"], "traffic": profiled_traffic(w.name),
                    "peak_source": f"{pk['source']} HBM copy", "algorithmic_bytes": w.io_bytes,
                    "tflops": achieved}
    else:
        # fp16 takes the bf16 figure: the nominal dense fp16 and bf16 tensor rates are equal
        tp, tsrc = tensor_peak(pk, w)
        roofline = {"bound": "tensor", "achieved": achieved, "peak": tp, "unit": "TFLOP/s",
                    "frac": achieved / tp, "traffic": profiled_traffic(w.name), "peak_source": tsrc,
                    "algorithmic_bytes": w.io_bytes, "hbm_gbs": gbs}

    # End to end through the public API: pinned host inputs in, O and LSE back to host, every
    # step.  The batch is cut into chunks (whole batch elements: contiguous slices of every
    # tensor) that alternate between two streams, so the host->device copy of one chunk, the
    # forward of another and the device->host copy of a third overlap (separate copy engines
    # for each direction, the SMs for the kernel).
    e2e = None
    if not args.no_e2e:
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        lse_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        n_e2e = max(1, min(args.steps, args.e2e_steps))
        n_chunks = max(1, min(args.e2e_chunks, w.B))
        bounds = [round(i * w.B / n_chunks) for i in range(n_chunks + 1)]
        spans = [(bounds[i], bounds[i + 1]) for i in range(n_chunks) if bounds[i + 1] > bounds[i]]
        side = [torch.cuda.Stream(device=dev) for _ in range(2)]
        # split-KV scratch is per stream: chunks in flight on the two streams must not share it
        side_ws = [ws, (torch.empty_like(ws) if ws is not None else None)]

        def e2e_step():
            start = torch.cuda.Event()
            start.record(stream)
            for c, (b0, b1) in enumerate(spans):
                s = side[c % 2]
                s.wait_event(start)
                with torch.cuda.stream(s):
                    for n, t in (("q", q), ("k", k), ("v", v)):
                        t[b0:b1].copy_(host[n][b0:b1], non_blocking=True)
                    forward_call(fa, w, q[b0:b1], k[b0:b1], v[b0:b1], out[b0:b1], lse[b0:b1], stream=s,
                                 **dict(call_kw, workspace=side_ws[c % 2]))
                    out_h[b0:b1].copy_(out[b0:b1], non_blocking=True)
                    lse_h[b0:b1].copy_(lse[b0:b1], non_blocking=True)
            for s in side:
                stream.wait_stream(s)

        e2e_step()
        torch.cuda.synchronize()
        if pg:
            pg.barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        f1.record(stream)
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(f0.elapsed_time(f1) / n_e2e, pg, dev)
        h2d = sum(host[n].numel() * host[n].element_size() for n in ("q", "k", "v"))
        d2h = out.numel() * 2 + lse.numel() * 4
        e2e = {"value": weak_scaling_tflops(w, world, ms_e2e), "unit": "TFLOP/s", "ms_per_step": ms_e2e,
               "steps": n_e2e, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "chunks": len(spans), "streams": 2}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, sample, cores, secs = oracle_sample_tflops(w, args.cpu_seconds)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample}

    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.Nq, "Nk": w.Nk, "d": w.d,
                   "causal": w.causal, "window": w.window, "num_splits": splits,
                   "global_batch": w.B * world, "seq_len": w.Nq,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (no flush)" if w.io_bytes > 3 * 126e6 else "inputs fit L2: warm-L2 number",
                   "pct_of_peak": 100.0 * achieved / pk["bf16_tflops"]},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps * launches_per_step,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


BWD_DEFAULT = ("seq4096_b8_h32_d128,seq1024_b8_h32_d128,gqa_prefill_b4_n4096_hq32_hkv8_d128_causal,"
               "long16k_b1_h32_d128_causal,hdim64_b2_n4096_h16")


def run_bwd_sweep(args):
    """Backward pass (fa_bwd) on workloads of the table, one JSON line each (device time,
    1 GPU).  FLOPs: five matrix products of the forward's size, 2.5x the forward count."""
    import torch
    import exact_attention_146_b200 as fa
    torch.cuda.set_device(0)
    pk = peaks()
    names = (args.sweep_only or BWD_DEFAULT).split(",")
    for name in names:
        w = synth.WORKLOADS[name]
        if w.d not in (32, 64, 80, 96, 128) or w.dtype != "bf16" or w.window or w.splitkv:
            continue
        x = synth.make_inputs(w)
        q, k, v = (torch.from_numpy(x[n].view(np.int16)).view(torch.bfloat16).cuda() for n in ("q", "k", "v"))
        do = torch.from_numpy(synth.make_grad_output(w).view(np.int16)).view(torch.bfloat16).cuda()
        out, lse = fa.fa_fwd(q, k, v, causal=w.causal, scale=w.scale)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(max(1, fa.bwd_workspace_bytes(w.B, w.Hq, w.Nq, w.d)), dtype=torch.uint8, device="cuda")
        flush = torch.empty(int(2 * 126e6) // 4, dtype=torch.float32, device="cuda")

        def call():
            fa.fa_bwd(q, k, v, out, do, lse, causal=w.causal, scale=w.scale, dq=dq, dk=dk, dv=dv, workspace=ws)

        for _ in range(args.warmup):
            call()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            call()
        b.record()
        torch.cuda.synchronize()
        ms_warm = a.elapsed_time(b) / args.steps
        times = []
        for _ in range(min(args.steps, 10)):
            flush.zero_()
            a.record()
            call()
            b.record()
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        ms_cold = sorted(times)[len(times) // 2]
        st, _ = fa.device_status()
        flops = 2.5 * w.flops
        print(json.dumps({"workload": name, "pass": "backward", "ms_warm": ms_warm, "ms_l2_flushed": ms_cold,
                          "tflops": flops / (ms_cold * 1e-3) / 1e12,
                          "pct_peak": 100 * flops / (ms_cold * 1e-3) / 1e12 / pk["bf16_tflops"],
                          "launches_per_call": 3, "status": st}), flush=True)
    return 0


def run_sweep(args):
    """Every workload of the table, one JSON line each (device time only, 1 GPU)."""
    import torch
    import exact_attention_146_b200 as fa
    torch.cuda.set_device(0)
    pk = peaks()
    names = args.sweep_only.split(",") if args.sweep_only else list(synth.WORKLOADS)
    for name in names:
        w = synth.WORKLOADS[name]
        x = synth.make_inputs(w)
        ti = device_inputs(torch, x, w)
        q, k, v = (ti[n].cuda() for n in ("q", "k", "v"))
        out = torch.empty(q.shape, dtype=torch.bfloat16 if w.dtype == "e4m3" else q.dtype, device="cuda")
        lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device="cuda")
        # inputs smaller than L2 are timed both warm and with an L2 flush before each launch
        flush = torch.empty(int(2 * 126e6) // 4, dtype=torch.float32, device="cuda")
        win = w.window or None
        splits = fa.splitkv_default_splits(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, torch.cuda.get_device_properties(0).multi_processor_count) if w.splitkv else None
        ws = torch.empty(max(1, fa.splitkv_workspace_bytes(w.B, w.Hq, w.Nq, w.d, splits)), dtype=torch.uint8, device="cuda") if splits else None
        kw = dict(window=win, num_splits=splits, workspace=ws)
        for _ in range(args.warmup):
            forward_call(fa, w, q, k, v, out, lse, **kw)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            forward_call(fa, w, q, k, v, out, lse, **kw)
        e1.record()
        torch.cuda.synchronize()
        ms_warm = e0.elapsed_time(e1) / args.steps
        cold = []
        for _ in range(min(args.steps, 20)):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            forward_call(fa, w, q, k, v, out, lse, **kw)
            b.record()
            torch.cuda.synchronize()
            cold.append(a.elapsed_time(b))
        ms_cold = statistics.median(cold)
        st, word = fa.device_status()
        roof_ms = max(w.flops / (tensor_peak(pk, w)[0] * 1e12), w.io_bytes / (pk["hbm_gbs"] * 1e9)) * 1e3
        print(json.dumps({
            "workload": name, "ms_warm": ms_warm, "ms_l2_flushed": ms_cold,
            "splits": splits, "tflops": w.flops / (ms_cold * 1e-3) / 1e12, "pct_peak": 100 * w.flops / (ms_cold * 1e-3) / 1e12 / tensor_peak(pk, w)[0],
            "hbm_gbs": w.io_bytes / (ms_cold * 1e-3) / 1e9, "roofline_ms": roof_ms,
            "roofline_frac": roof_ms / ms_cold, "status": st}), flush=True)
        del q, k, v, out, lse, flush
        torch.cuda.empty_cache()
    return 0


def run_fp8_peak(args):
    """Dense E4M3 GEMM throughput (cuBLASLt through torch._scaled_mm, 8192^3, bf16 out): the
    best of 10 calls (burst) and back to back for 3 s (sustained).  One JSON line; the figures
    committed in profiles/fp8_gemm_peak.md come from this mode."""
    import torch
    torch.cuda.set_device(0)
    n = 8192
    a = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn).t()
    one = torch.tensor(1.0, device="cuda")

    def mm():
        return torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)

    for _ in range(3):
        mm()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        mm()
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    calls, t0 = 0, time.time()
    e0.record()
    while time.time() - t0 < 3.0:
        mm()
        calls += 1
    e1.record()
    torch.cuda.synchronize()
    flop = 2.0 * n ** 3
    print(json.dumps({"fp8_tflops_burst": flop / best / 1e9,
                      "fp8_tflops_sustained": flop / (e0.elapsed_time(e1) / calls) / 1e9,
                      "n": n, "sustained_calls": calls}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=synth.HEADLINE, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--e2e-chunks", type=int, default=4, help="batch chunks pipelined over two streams in e2e")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--sweep", action="store_true", help="time every workload of the table (1 GPU)")
    ap.add_argument("--sweep-only", default="", help="comma-separated workload names for --sweep / --bwd-sweep")
    ap.add_argument("--bwd-sweep", action="store_true", help="time the backward pass on workloads of the table")
    ap.add_argument("--fp8-peak", action="store_true", help="measure the dense E4M3 GEMM peak (1 GPU)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.sweep:
        return run_sweep(args)
    if args.bwd_sweep:
        return run_bwd_sweep(args)
    if args.fp8_peak:
        return run_fp8_peak(args)
    w = synth.WORKLOADS[args.workload]
    world, rank, local = dist_setup(args.gpus)
    if args.impl == "reference":
        return run_reference(args, w, world, rank)
    return run_ours(args, w, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
