#!/usr/bin/env python
"""Benchmark: exact attention forward TFLOP/s on B200 (causal bf16, B=4 H=16 N=4096 d=128).

One step = one forward (one launch of the attention kernel) over the whole
workload with inputs resident in HBM.  Prints ONE JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
                    [--workload c3] [--no-cpu-baseline] [--alibi]

``--decode`` times one decoding step (attn_decode, dec1: B=8 H=32 H_kv=8, one
new row against an 8192-position cache, d=128 bf16) and reports GB/s of
algorithmic bytes against the measured HBM bandwidth (an extra line).

``--backward`` times attn_bwd (dQ, dK, dV of the same workload's forward) and
reports TFLOP/s at 10 d flops per kept pair (an extra line).

``--alibi`` times the same workload through attn_fwd_alibi with the pages'
slopes 2^(-8 h / H) (an extra measurement, not the headline line; it has no
host-buffer leg and no CPU-oracle leg).

FLOPs are algorithmic: 4 * d * (kept query-key pairs) per head, summed over
B * H heads (the causal mask keeps N (N + 1) / 2 pairs); masked work is not
counted.  Between timed steps the inputs rotate over two sets of device
buffers whose combined size is several times the 126 MB L2, so no step reads
its inputs from L2 left warm by the step before.
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
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attn fwd TFLOP/s & % of B200 BF16 tensor peak (causal, N=4096, d=128)"
SPEC_BF16_TFLOPS = 2250.0
L2_BYTES = 126 * 2 ** 20
# device code of the forward kernel (its launch geometry is defined there too);
# the committed DRAM traffic figure is used only while these are unchanged
KERNEL_SOURCES = ["exact_tiled_attention_44_b200/csrc/attn_kernel.cuh",
                  "exact_tiled_attention_44_b200/csrc/ptx.cuh"]


# device code of the backward kernel (it builds on the forward's helpers)
BWD_KERNEL_SOURCES = ["exact_tiled_attention_44_b200/csrc/bwd_kernel.cuh"] + KERNEL_SOURCES


def _code_only(text: str) -> str:
    """Source without /* */ blocks, // comments, trailing blanks and empty lines
    (none of the kernel files has // inside a string literal), so that editing a
    comment does not count as a kernel change."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = []
    for line in text.splitlines():
        line = line.split("//", 1)[0].rstrip()
        if line:
            out.append(line)
    return "\n".join(out)


def kernel_source_hash(sources=None) -> str:
    h = hashlib.sha256()
    for f in (sources or KERNEL_SOURCES):
        h.update(_code_only(open(os.path.join(ROOT, f)).read()).encode())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"bf16_tflops": d["bf16_tflops"], "bf16_tflops_sustained": d["bf16_tflops_sustained"],
                "hbm_gbs": d["hbm_gbs"], "source": "measured"}
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0,
            "source": "fallback"}


def load_traffic(workload: str, kind: str = "fwd"):
    """DRAM bytes per launch from the committed ncu summary, if it matches this kernel."""
    path = os.path.join(ROOT, "profiles", f"attn_{kind}_{workload}_traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path))
    srcs = BWD_KERNEL_SOURCES if kind == "bwd" else KERNEL_SOURCES
    if d.get("kernel_src_sha256") != kernel_source_hash(srcs):
        return None
    return d.get("dram_bytes_per_launch")


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""
    FIELDS = ("index,timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, path: str | None = None):
        self.path = path or tempfile.mktemp(prefix="clocks_", suffix=".csv")
        self.gpu_index = gpu_index
        self.proc = None
        self.t_begin = self.t_end = None

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.gpu_index)], stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def mark_begin(self):
        self.t_begin = time.time()

    def mark_end(self):
        self.t_end = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = time.mktime(time.strptime(parts[1].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                frac = float("0." + parts[1].split(".")[1]) if "." in parts[1] else 0.0
                rows.append((ts + frac, float(parts[2]), float(parts[3]), float(parts[4]), parts[5:]))
            except (ValueError, IndexError):
                continue
        window = "timed"
        sel = [r for r in rows if self.t_begin and self.t_begin - 0.05 <= r[0] <= self.t_end + 0.05]
        if not sel:
            sel, window = rows, "whole run (timed region shorter than the sampling interval)"
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in sel:
            for nm, val in zip(names, r[4][1:5]):
                if val.strip().lower() in ("active", "1", "yes"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(r[1] for r in sel), "sm_max_mhz": max(r[2] for r in sel),
                "power_w_max": max(r[3] for r in sel), "samples": len(sel), "window": window,
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------- oracle leg

def _oracle_rows_task(args):
    """Worker: the oracle for query rows [r0, r1) of one head; returns seconds spent."""
    import numpy as np
    import oracle
    Qh, Kh, Vh, scale, causal, window, n_sink, r0, r1 = args
    t0 = time.perf_counter()
    oracle.attention_bh(Qh, Kh, Vh, 0, 0, scale, causal, window, n_sink, rows=np.arange(r0, r1))
    return time.perf_counter() - t0


def _head_arrays(w, q, k, v, b, h):
    from exact_tiled_attention_44_b200.inputs import to_f64
    g = h // (w.H // w.H_kv)
    return (to_f64(q[b:b + 1, h:h + 1]), to_f64(k[b:b + 1, g:g + 1]), to_f64(v[b:b + 1, g:g + 1]))


def _pairs_rows(w, r0, r1):
    """Kept pairs of query rows [r0, r1) (mask rule restated for accounting)."""
    tot = 0
    for i in range(r0, r1):
        if not w.causal:
            tot += w.N
        elif w.window <= 0 or w.window >= w.N:
            tot += i + 1
        else:
            tot += min(i + 1, w.window) + max(0, min(w.n_sink, i - w.window + 1))
    return tot


def cpu_oracle_throughput(name: str, q, k, v, budget_s: float = 20.0):
    """The float64 oracle, as it stands, on a bounded sample of the workload.

    Chunks of complete query rows of distinct heads are spread over all host
    cores (one BLAS thread per worker process, spawn start method; the parent
    sends each worker only the head it needs).  New chunks are submitted until
    ``budget_s`` seconds have passed; the throughput counts the chunks that
    finished.  Returns the cpu_baseline object in TFLOP/s.
    """
    import concurrent.futures as cf
    import multiprocessing as mp
    from exact_tiled_attention_44_b200.inputs import WORKLOADS
    w = WORKLOADS[name]
    cores = len(os.sched_getaffinity(0))
    rows_per_task = 256
    n_chunks = (w.N + rows_per_task - 1) // rows_per_task
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    arrays = {}

    def task(i):
        b, h = heads[i % len(heads)]
        if (b, h) not in arrays:
            arrays[(b, h)] = _head_arrays(w, q, k, v, b, h)
        r0 = ((i // len(heads)) * 7 % n_chunks) * rows_per_task
        return arrays[(b, h)] + (w.scale, w.causal, w.window, w.n_sink, r0,
                                 min(w.N, r0 + rows_per_task))

    saved = {kk: os.environ.get(kk) for kk in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    for kk in saved:
        os.environ[kk] = "1"
    done_rows = []
    try:
        ctx = mp.get_context("spawn")
        with cf.ProcessPoolExecutor(max_workers=cores, mp_context=ctx) as ex:
            list(ex.map(_oracle_rows_task, [task(0)] * cores))      # start the workers
            t0 = time.perf_counter()
            nxt = 0
            pending = {}
            for _ in range(2 * cores):
                args = task(nxt)
                pending[ex.submit(_oracle_rows_task, args)] = args
                nxt += 1
            while pending:
                finished, _ = cf.wait(pending, return_when=cf.FIRST_COMPLETED)
                for f in finished:
                    args = pending.pop(f)
                    f.result()
                    done_rows.append((args[7], args[8]))
                    if time.perf_counter() - t0 < budget_s:
                        a2 = task(nxt)
                        pending[ex.submit(_oracle_rows_task, a2)] = a2
                        nxt += 1
            wall = time.perf_counter() - t0
    finally:
        for kk, val in saved.items():
            if val is None:
                os.environ.pop(kk, None)
            else:
                os.environ[kk] = val
    flops = sum(4.0 * w.d * _pairs_rows(w, r0, r1) for r0, r1 in done_rows)
    return {"value": flops / wall / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{len(done_rows)} chunks of {rows_per_task} complete query rows from the "
                      f"{w.B * w.H} heads of {name} (submitted for {budget_s:.0f} s); float64 full "
                      f"score rows; {wall:.1f} s wall on {cores} worker processes"}


def _blas_threads() -> int:
    """Threads numpy's BLAS uses in this process (the reference arm's core count)."""
    for kk in ("OPENBLAS_NUM_THREADS", "OMP_NUM_THREADS", "MKL_NUM_THREADS"):
        if os.environ.get(kk, "").isdigit():
            return int(os.environ[kk])
    return len(os.sched_getaffinity(0))


def reference_arm(args):
    """--impl reference: the oracle on this machine's host cores, same metric and workload."""
    from exact_tiled_attention_44_b200.inputs import WORKLOADS
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from exact_tiled_attention_44_b200.inputs import make_inputs
    w = WORKLOADS[args.workload]
    q, k, v = make_inputs(w)
    heads = {}

    def head(b, h):
        if (b, h) not in heads:
            heads[(b, h)] = _head_arrays(w, q, k, v, b, h)
        return heads[(b, h)]

    # bounded sample per step: whole query rows of one head, sized so the run ends in minutes
    t_cal = _oracle_rows_task(head(0, 0) + (w.scale, w.causal, w.window, w.n_sink, w.N - 64, w.N))
    per_row = max(t_cal / 64, 1e-5)
    budget = 150.0 / max(1, args.steps + args.warmup)
    rows = int(max(8, min(w.N, budget / per_row)))
    step_rows = []
    for s_ in range(args.warmup + args.steps):
        b, h = divmod(s_ % (w.B * w.H), w.H)
        r0 = (s_ * rows) % max(1, w.N - rows + 1)
        step_rows.append((b, h, r0, r0 + rows))
    for b, h, r0, r1 in step_rows[:args.warmup]:
        _oracle_rows_task(head(b, h) + (w.scale, w.causal, w.window, w.n_sink, r0, r1))
    t0 = time.perf_counter()
    for b, h, r0, r1 in step_rows[args.warmup:]:
        _oracle_rows_task(head(b, h) + (w.scale, w.causal, w.window, w.n_sink, r0, r1))
    wall = time.perf_counter() - t0
    flops = sum(4.0 * w.d * _pairs_rows(w, r0, r1) for _, _, r0, r1 in step_rows[args.warmup:])
    value = flops / wall / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": wall / max(1, args.steps) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{w.name}: B={w.B} H={w.H} H_kv={w.H_kv} N={w.N} d={w.d} "
                                   f"{w.dtype} causal={int(w.causal)} window={w.window} "
                                   f"n_sink={w.n_sink}",
                       "step": f"{rows} complete query rows of one head per step (bounded sample)"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _blas_threads(), "kind": "oracle",
                             "sample": f"{rows} query rows per step, one head per step, "
                                       f"float64 numpy, one process"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- ranks

def max_over_ranks(x: float, dist_mod, device) -> float:
    """Maximum of a per-rank float over all ranks (identity without a process group)."""
    if dist_mod is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_step: float, steps: int, ms: float) -> float:
    """Weak scaling: every rank runs the same-size workload; the job rate counts all ranks."""
    return world * flops_per_step * steps / (ms / 1e3) / 1e12


# ----------------------------------------------------------------- GPU arm

def decode_bench(args):
    """--decode: one decoding step per timed step, inputs resident in HBM and
    rotating over two sets (each larger than L2)."""
    import torch
    import exact_tiled_attention_44_b200 as A
    from exact_tiled_attention_44_b200.inputs import DECODE_WORKLOADS, make_decode_inputs

    w = DECODE_WORKLOADS["dec1"]
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    B, H, H_kv, N_q, N_kv, d = w["B"], w["H"], w["H_kv"], w["N_q"], w["N_kv"], w["d"]
    q, k, v = make_decode_inputs(B, H, H_kv, N_q, N_kv, d)
    sets = []
    for i in range(2):
        qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
        sets.append((qd, kd, vd, torch.empty_like(qd), torch.empty(q.shape[:3], device=dev),
                     torch.empty(A.decode_workspace_bytes(B, H, H_kv, N_q, N_kv, d),
                                 dtype=torch.uint8, device=dev)))
    alg_bytes = 2 * (q.numel() * 2) + 2 * k.numel() * 2 + B * H * N_q * 4   # q, o, k, v, lse
    stream = torch.cuda.current_stream(dev)

    def step(i):
        qd, kd, vd, od, ld, ws = sets[i % 2]
        A.decode(qd, kd, vd, causal=w["causal"], out=od, lse=ld, workspace=ws)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(dev.index if dev.index is not None else 0, args.clocks_csv)
    sampler.start()
    K = args.steps
    # Steps run back to back, as in a decoding loop: no event between them
    # (an event between two launches would also stop the next step's set-up
    # from overlapping the end of the previous one).  The two input sets
    # together exceed L2, so every step reads its cache from HBM.
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    n0 = A.launch_count()
    sampler.mark_begin()
    t0.record(stream)
    for i in range(K):
        step(i)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    sampler.mark_end()
    launches = A.launch_count() - n0
    clocks = sampler.stop()
    total_ms = t0.elapsed_time(t1)
    kern_ms = total_ms / K
    peaks = load_peaks()
    achieved = alg_bytes / (kern_ms / 1e3) / 1e9
    line = {
        "metric": "attn decode GB/s & % of measured HBM bandwidth (split-KV, one step)",
        "value": alg_bytes * K / (total_ms / 1e3) / 1e9, "unit": "GB/s", "n_gpus": 1, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w["dtype"], "data": "synthetic",
        "config": {"workload": f"dec1: B={B} H={H} H_kv={H_kv} N_q={N_q} N_kv={N_kv} d={d} "
                               f"{w['dtype']} causal={int(w['causal'])}",
                   "l2": "inputs larger than L2: 2 rotating sets of "
                         f"{(q.numel() + 2 * k.numel()) * 2 / 2**20:.0f} MiB (L2 126 MiB)",
                   "alg_bytes_per_step": alg_bytes,
                   "splits": A.decode_workspace_bytes(B, H, H_kv, N_q, N_kv, d) > 0},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                     "peak_source": f"{peaks['source']} HBM copy (MEASURED_PEAKS.json)",
                     "kernel_ms": kern_ms,
                     "kernel_ms_scope": "one decoding step (split kernel and, when groups are "
                                        "split, the merge kernel), averaged over the timed steps"},
        "gpu_launches": launches,
        "clocks": clocks,
        "device_status": A.get_status(),
    }
    print(json.dumps(line), flush=True)
    return 0


def backward_bench(args):
    """--backward: one attn_bwd call (D, the tiled backward, dQ conversion) per
    timed step on the c3 workload, inputs resident in HBM and rotating over two
    sets larger than L2.  FLOPs are algorithmic: the five products of the
    backward (S recomputed, dP, dV, dK, dQ) at 2 d flops per kept pair each,
    10 d per pair, 2.5 times the forward's count."""
    import numpy as np
    import torch
    import exact_tiled_attention_44_b200 as A
    import oracle
    from exact_tiled_attention_44_b200.inputs import WORKLOADS, make_grad_output, make_inputs, to_f64

    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    q, k, v = make_inputs(w)
    do = make_grad_output(w.B, w.H, w.N, w.d, dtype=q.dtype, seed=0)
    sets = []
    for i in range(2):
        qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
        od, ld = A.attention(qd, kd, vd, causal=w.causal, window=w.window, n_sink=w.n_sink,
                             scale=w.scale)
        grads = (torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd))
        ws = torch.empty(A.bwd_workspace_bytes(w.B, w.H, w.N, w.d, A._dtype_code(q)),
                         dtype=torch.uint8, device=dev)
        sets.append((qd, kd, vd, od, dod, ld, grads, ws))
    set_bytes = sum(t.numel() * t.element_size() for t in sets[0][:6])
    pairs = A.unmasked_pairs(w.N, w.causal, w.window, w.n_sink)
    flops = 10.0 * w.B * w.H * w.d * pairs
    stream = torch.cuda.current_stream(dev)

    def step(i):
        qd, kd, vd, od, dod, ld, grads, ws = sets[i % 2]
        A.attention_backward(qd, kd, vd, od, dod, ld, causal=w.causal, window=w.window,
                             n_sink=w.n_sink, scale=w.scale, workspace=ws, grads=grads)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(dev.index if dev.index is not None else 0, args.clocks_csv)
    sampler.start()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    n0 = A.launch_count()
    sampler.mark_begin()
    t0.record(stream)
    for i in range(K):
        ev[i][0].record(stream)
        step(i)
        ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    sampler.mark_end()
    launches = A.launch_count() - n0
    clocks = sampler.stop()
    total_ms = t0.elapsed_time(t1)
    step_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)

    # end to end through the Python API from pinned host buffers: inputs in,
    # gradients out, every step
    hq, hk, hv, hdo = (t.pin_memory() for t in (q, k, v, do))
    ho = sets[0][3].cpu().pin_memory()
    hl = sets[0][5].cpu().pin_memory()
    hgrads = tuple(torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in sets[0][6])
    qd, kd, vd, od, dod, ld, grads, ws = sets[0]

    def e2e_step():
        for dst, src in ((qd, hq), (kd, hk), (vd, hv), (od, ho), (dod, hdo), (ld, hl)):
            dst.copy_(src, non_blocking=True)
        A.attention_backward(qd, kd, vd, od, dod, ld, causal=w.causal, window=w.window,
                             n_sink=w.n_sink, scale=w.scale, workspace=ws, grads=grads)
        for dst, src in zip(hgrads, grads):
            dst.copy_(src, non_blocking=True)

    e2e_steps = max(3, min(K, 20))
    e2e_step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, ho, hdo, hl))
    d2h = sum(t.numel() * t.element_size() for t in hgrads)

    # the oracle, as it stands, on a bounded sample: whole heads' gradients
    cpu = None
    if not args.no_cpu_baseline:
        t_s, n_heads = 0.0, 0
        while t_s < 10.0 and n_heads < w.B * w.H:
            b, h = divmod(n_heads, w.H)
            g = h // (w.H // w.H_kv)
            args_h = (to_f64(q[b, h]), to_f64(k[b, g]), to_f64(v[b, g]), to_f64(do[b, h]))
            c0 = time.perf_counter()
            oracle.backward_head(*args_h, w.scale, w.causal, w.window, w.n_sink)
            t_s += time.perf_counter() - c0
            n_heads += 1
        cpu = {"value": 10.0 * w.d * pairs * n_heads / t_s / 1e12, "unit": "TFLOP/s",
               "cores": _blas_threads(), "kind": "oracle",
               "sample": f"{n_heads} whole heads of {w.name} through oracle.backward_head "
                         f"(float64, full N x N matrices), {t_s:.1f} s"}

    peaks = load_peaks()
    achieved = flops / (step_ms / 1e3) / 1e12
    line = {
        "metric": "attn bwd TFLOP/s (dQ, dK, dV; 10 d flops per kept pair) & % of measured BF16 peak",
        "value": flops * K / (total_ms / 1e3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": f"{w.name} backward: B={w.B} H={w.H} H_kv={w.H_kv} N={w.N} d={w.d} "
                               f"{w.dtype} causal={int(w.causal)}",
                   "l2": f"inputs larger than L2: 2 rotating sets of {set_bytes / 2**20:.0f} MiB "
                         "(L2 126 MiB)",
                   "flops_per_step": flops, "kept_pairs_per_head": pairs,
                   "outputs": "dq, dk, dv in the input dtype (fp32 dQ accumulator in the workspace)"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                     "traffic": load_traffic(w.name, "bwd"),
                     "traffic_scope": "DRAM bytes of one launch of the tiled backward kernel",
                     "peak_source": f"{peaks['source']} bf16 burst (MEASURED_PEAKS.json)",
                     "kernel_ms": step_ms,
                     "kernel_ms_scope": "one attn_bwd call: D prep, tiled backward and dQ "
                                        "conversion launches together (conservative for the "
                                        "tiled kernel; its share is in the ncu launch list)"},
        "e2e": {"value": flops * e2e_steps / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "path": "pinned host q,k,v,o,dO,lse -> device, attention_backward, dq,dk,dv -> host"},
        "gpu_launches": launches,
        "clocks": clocks,
        "device_status": A.get_status(),
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--workload", default="c3")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer (e2e) leg")
    ap.add_argument("--clocks-csv", default=None, help="keep the raw nvidia-smi samples here")
    ap.add_argument("--decode", action="store_true",
                    help="time attn_decode on the dec1 workload (GB/s against HBM)")
    ap.add_argument("--alibi", action="store_true",
                    help="add the ALiBi bias with the pages' slopes (attn_fwd_alibi)")
    ap.add_argument("--backward", action="store_true",
                    help="time attn_bwd (dQ, dK, dV) on the workload (an extra line)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    if args.impl == "reference":
        return reference_arm(args)
    if args.decode or args.backward:
        # single-GPU extra lines: under torchrun only rank 0 runs them
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        return decode_bench(args) if args.decode else backward_bench(args)

    import torch
    import exact_tiled_attention_44_b200 as A
    from exact_tiled_attention_44_b200.inputs import WORKLOADS, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)

    if args.workload not in WORKLOADS:
        raise SystemExit(f"unknown workload {args.workload!r}; one of {sorted(WORKLOADS)}")
    w = WORKLOADS[args.workload]
    q, k, v = make_inputs(w)           # identical seeded inputs on every rank (replicas)
    sets = []
    per_set_bytes = 0
    n_sets = 2
    for i in range(n_sets):
        qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
        od = torch.empty_like(qd)
        ld = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
        sets.append((qd, kd, vd, od, ld))
        per_set_bytes = sum(t.numel() * t.element_size() for t in (qd, kd, vd, od, ld))
    pairs = A.unmasked_pairs(w.N, w.causal, w.window, w.n_sink)
    flops = 4.0 * w.B * w.H * w.d * pairs
    stream = torch.cuda.current_stream(dev)
    slopes = A.alibi_slopes(w.H, dev) if args.alibi else None

    def step(i):
        qd, kd, vd, od, ld = sets[i % n_sets]
        A.attention(qd, kd, vd, causal=w.causal, window=w.window, n_sink=w.n_sink, scale=w.scale,
                    out=od, lse=ld, alibi_slopes=slopes)

    # Small workloads fit in L2 even with rotating sets: write a buffer twice
    # the L2 size before every timed step (outside the step's events), so that
    # each step reads its inputs from HBM.  The flush also keeps the launch
    # queue ahead of the GPU, so a step's events time the kernel, not the host.
    flush = None
    if n_sets * per_set_bytes < 4 * L2_BYTES:
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for i in range(args.warmup):
        step(i)
    barrier()

    sampler = ClockSampler(dev.index if dev.index is not None else 0,
                           f"{args.clocks_csv}.r{rank}" if args.clocks_csv else None)
    sampler.start()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t_all0, t_all1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    n_launch0 = A.launch_count()
    sampler.mark_begin()
    t_all0.record(stream)
    for i in range(K):
        if flush is not None:
            flush.fill_(float(i))
        ev[i][0].record(stream)
        step(i)
        ev[i][1].record(stream)
    t_all1.record(stream)
    barrier()
    sampler.mark_end()
    launches = A.launch_count() - n_launch0
    clocks = sampler.stop()
    total_ms = t_all0.elapsed_time(t_all1)
    kern_ms = [a.elapsed_time(b) for a, b in ev]
    if flush is not None:
        # the flushes are not part of the workload: the job time is the sum of
        # the steps' own times
        total_ms = sum(kern_ms)
    total_ms = max_over_ranks(total_ms, dist, dev)
    ms_per_step = total_ms / K
    value = whole_job_tflops(world, flops, K, total_ms)
    avg_kernel_ms = statistics.mean(kern_ms)
    achieved = flops / (avg_kernel_ms / 1e3) / 1e12

    # ---- end to end through the public host-buffer entry point
    e2e_steps = args.e2e_steps or max(3, min(K, 30))
    if args.alibi or args.no_e2e:
        e2e_steps = 0
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    lh = torch.empty(q.shape[:3], dtype=torch.float32).pin_memory()
    staging = {"q": sets[0][0], "k": sets[0][1], "v": sets[0][2], "o": sets[0][3], "lse": sets[0][4]}
    e2e_value = None
    if e2e_steps:
        for _ in range(2):
            A.attention_from_host(qh, kh, vh, staging=staging, out=oh, lse=lh, causal=w.causal,
                                  window=w.window, n_sink=w.n_sink, scale=w.scale)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            A.attention_from_host(qh, kh, vh, staging=staging, out=oh, lse=lh, causal=w.causal,
                                  window=w.window, n_sink=w.n_sink, scale=w.scale)
        e1.record(stream)
        barrier()
        e2e_ms = e0.elapsed_time(e1)
        e2e_ms = max_over_ranks(e2e_ms, dist, dev)
        e2e_value = whole_job_tflops(world, flops, e2e_steps, e2e_ms)
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v))
    d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()

    status = A.get_status()

    if rank == 0:
        peaks = load_peaks()
        traffic = None if args.alibi else load_traffic(w.name)
        alg_bytes = per_set_bytes
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                "traffic": traffic,
                "peak_source": f"{peaks['source']} bf16 burst (MEASURED_PEAKS.json)"
                if peaks["source"] == "measured" else "fallback 1.59 PFLOP/s",
                "frac_of_spec_2250": achieved / SPEC_BF16_TFLOPS,
                "kernel_ms": avg_kernel_ms}
        if flush is not None:
            # launch- and memory-latency bound: report HBM GB/s of the
            # algorithmic bytes (q, k, v, o once, lse) against the copy bandwidth
            gbs = alg_bytes / (avg_kernel_ms / 1e3) / 1e9
            roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": gbs / peaks["hbm_gbs"], "traffic": traffic,
                    "peak_source": f"{peaks['source']} HBM copy (MEASURED_PEAKS.json)",
                    "alg_bytes": alg_bytes, "kernel_ms": avg_kernel_ms,
                    "tensor_tflops": achieved, "tensor_frac": achieved / peaks["bf16_tflops"]}
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": f"{w.name}: B={w.B} H={w.H} H_kv={w.H_kv} N={w.N} d={w.d} "
                                   f"{w.dtype} causal={int(w.causal)} window={w.window} "
                                   f"n_sink={w.n_sink}",
                       "global_batch": w.B * world, "seq_len": w.N,
                       "parallelism": f"replicas x{world} (independent problems, no collective)",
                       "l2": (f"inputs larger than L2: {n_sets} rotating device input sets of "
                              f"{per_set_bytes / 2**20:.0f} MiB (L2 126 MiB)") if flush is None else
                             (f"L2 flushed before every step (a {2 * L2_BYTES / 2**20:.0f} MiB write, "
                              f"outside the step's events; value and ms_per_step are the sum of the "
                              f"steps' own times); {n_sets} input sets of "
                              f"{per_set_bytes / 2**20:.1f} MiB"),
                       "flops_per_step": flops, "kept_pairs_per_head": pairs,
                       "alibi": ("slopes 2^(-8 h / H), h = 1..H (attn_fwd_alibi)" if args.alibi
                                 else None)},
            "roofline": roof,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "path": "attn_fwd_host: pinned host q,k,v -> device, forward, o and lse -> host"},
            "gpu_launches": launches,
            "clocks": clocks,
            "device_status": status,
        }
        if args.alibi:
            line["e2e"] = {"value": None, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0,
                           "path": "none: attn_fwd_host has no ALiBi variant"}
        elif not e2e_steps:
            line["e2e"] = {"value": None, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0, "path": "skipped (--no-e2e)"}
        if not args.no_cpu_baseline and not args.alibi:
            line["cpu_baseline"] = cpu_oracle_throughput(w.name, q, k, v)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
