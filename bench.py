"""Benchmark of the fused attention kernels on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fa|reference]
                    [--workload c5|c1|c2|c3|c4|c5a|c5b|sdxl_xattn|bert_large|prefill_cached|d256_long]
                    [--pass fwd|bwd|sp] [--mask tril] [--dropout P] [--deterministic]
                    [--block-n 64|128] [--q-tiles 1|2]
                    [--sp-world W] [--sp-mode ring|allgather|ulysses]
                    [--no-e2e] [--e2e-chunks C] [--no-cpu-baseline] [--cpu-seconds S]

A step is one pass of the whole forward path over one batch of synthetic
input.  The default workload is the long-context configuration
B=1, H=32, S=16384, D=128, bf16, run both without and with the causal mask
(two fa_fwd launches per step).  Inputs (512 MiB) are larger than the 126 MB
L2, so no L2 flush is needed between steps.  Beside the step, the 13B-style
causal layer (B=1, H=40, S=8192, D=128, Q,K x2) is timed alone with the same
protocol and reported under "extra_runs" (not part of the step's value).

The general-shape workloads (sdxl_xattn: 4096 queries over 77 keys;
bert_large: B=32, H=16, S=512, D=64 in the BSHD layout; prefill_cached:
4096 causal queries over 16384 keys; d256_long: head dimension 256) run
through fa_fwd_ex; their inputs are rotated over enough copies that one
rotation touches more than twice the L2.

Throughput is attention TFLOP/s with the causal case counted at half
(4*B*H*S^2*D per non-causal run), over the whole job: with N GPUs (one
process per GPU, torchrun) every rank runs its own independent batch of the
same shape (weak scaling, no data-path collective) and the value is the
total work of all ranks over the slowest rank's device time.

Other passes: ``--pass bwd`` times the backward pass (2.5x the forward's
flops; BSHD workloads through fa_bwd_ex), ``--pass sp`` every rank's
sequence-parallel schedule run in turn on one GPU.  ``--mask tril`` runs the
causal case as an explicit lower-triangular mask, ``--dropout P`` adds
attention dropout (a fresh offset per step).

The end-to-end figure ("e2e") times steps through the same public calls with
pinned host buffers: each step uploads its inputs and downloads O and LSE.
Each step is split into chunks of whole batches (or heads of a single
batch) pipelined over three streams, so that the copies in both directions
overlap the kernels, and consecutive steps overlap on two sets of device
buffers; the downloaded forward results are checked bit for bit against one
launch over all heads.

``--impl reference`` times the fp64 CPU oracle on bounded samples of the
same workload and pass (rank 0 only) and prints the same JSON line with
"impl": "reference".
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from tiled_attention_18_b200.scaling import job_throughput, max_over_ranks, rank_env, rank_seed  # noqa: E402
from tiled_attention_18_b200.workloads import (GENERAL_WORKLOADS, WORKLOADS, sample_rows,  # noqa: E402
                                               workload_inputs)

METRIC = "attention fwd TFLOPS (causal-adjusted) and % of B200 dense fp16/bf16 peak"
UNIT = "TFLOP/s"
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0
FALLBACK_HBM_GBS = 6650.0
DROPOUT_SEED = 0x5EED5EED5EED
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
# committed DRAM captures (one workload each), matched by workload and by the
# hash of the kernel sources they were taken on
TRAFFIC_PATHS = [os.path.join(ROOT, "profiles", name) for name in ("fa_fwd_traffic.json", "fa_fwd_short_traffic.json")]
CSRC = os.path.join(ROOT, "tiled_attention_18_b200", "csrc")
KERNEL_SRC = os.path.join(CSRC, "fa_fwd_sm100.cu")
L2_BYTES = 126 * 1024 * 1024
ALL_WORKLOADS = {**WORKLOADS, **GENERAL_WORKLOADS}


def e2e_chunks(B: int, H: int, n_chunks: int):
    """Split of one end-to-end step into chunks that are contiguous ranges of
    every tensor: whole batches when B > 1, else heads of the single batch.
    Returns ("b" or "h", [(first, count), ...]) covering the axis in order
    with counts differing by at most one."""
    axis, total = ("b", B) if B > 1 else ("h", H)
    n = max(1, min(n_chunks, total))
    edges = [total * c // n for c in range(n + 1)]
    return axis, [(edges[c], edges[c + 1] - edges[c]) for c in range(n)]


def workload_runs(name: str):
    """The fa_fwd runs of one step: (Workload, ...)."""
    if name == "c5":
        return [WORKLOADS["c5a"], WORKLOADS["c5b"]]
    return [ALL_WORKLOADS[name]]


def workload_label(name: str) -> str:
    runs = workload_runs(name)
    w = runs[0]
    causal = "non-causal + causal" if len(runs) == 2 else ("causal" if w.causal else "non-causal")
    extra = f", Q,K x{w.qk_mult:g}" if w.qk_mult != 1.0 else ""
    if w.general:
        lay = f", {w.layout.upper()} layout" if w.layout != "bhsd" else ""
        return f"attention fwd {w.dtype} B={w.B} H={w.H} Sq={w.S} Sk={w.Skv} D={w.D}, {causal}{extra}{lay}"
    return f"attention fwd {w.dtype} B={w.B} H={w.H} S={w.S} D={w.D}, {causal}{extra}"


def power_capped(clocks) -> bool:
    """The timed region ran under the power cap: sw_power_cap sampled and the
    median SM clock below 95 % of the maximum."""
    return bool(clocks) and "sw_power_cap" in clocks.get("reasons", []) and bool(clocks.get("sm_mhz")) and \
        bool(clocks.get("sm_max_mhz")) and clocks["sm_mhz"] < 0.95 * clocks["sm_max_mhz"]


def peak_tflops(clocks=None):
    """(peak, source, burst peak) of dense bf16: the burst figure for a timed
    region at full clock, the sustained one (a long loop under the power cap)
    when the sampled clocks show the region ran power-capped."""
    capped = power_capped(clocks)
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        burst = float(p["bf16_tflops"])
        if capped and "bf16_tflops_sustained" in p:
            return (float(p["bf16_tflops_sustained"]),
                    "measured (MEASURED_PEAKS.json bf16_tflops_sustained: the timed region ran power-capped)", burst)
        return burst, "measured (MEASURED_PEAKS.json bf16_tflops, burst)", burst
    except Exception:
        if capped:
            return (FALLBACK_BF16_TFLOPS_SUSTAINED,
                    "fallback sustained (1.4 PFLOP/s, an earlier cuBLAS bf16 loop under the power cap on B200: "
                    "the timed region ran power-capped)", FALLBACK_BF16_TFLOPS)
        return FALLBACK_BF16_TFLOPS, "fallback (1.59 PFLOP/s, an earlier cuBLAS bf16 measurement on B200)", \
            FALLBACK_BF16_TFLOPS


def kernel_source_hash(kernel_file: str = "fa_fwd_sm100.cu") -> str:
    """Hash of a forward kernel's sources (its file, the shared device helpers
    and the internal header with the launch helpers)."""
    import hashlib
    h = hashlib.sha256()
    for path in (os.path.join(CSRC, kernel_file), os.path.join(CSRC, "sm100_helpers.cuh"),
                 os.path.join(CSRC, "fa_internal.h")):
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_per_launch(workload: str):
    """DRAM bytes per step from a committed ncu summary, if taken on this kernel source and workload."""
    for path in TRAFFIC_PATHS:
        try:
            with open(path) as f:
                t = json.load(f)
            if t.get("workload_key", "c5") != workload:
                continue
            if t.get("kernel_source_sha256_16") != kernel_source_hash(t.get("kernel_file", "fa_fwd_sm100.cu")):
                return None
            return float(t["dram_bytes_per_step"])
        except Exception:
            continue
    return None


class ClockSampler:
    """nvidia-smi clocks/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self._stop = threading.Event()
        self._proc = None
        self._thread = None

    def start(self):
        try:
            self._proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self._proc = None
            return
        self._thread = threading.Thread(target=self._read, daemon=True)
        self._thread.start()

    def _read(self):
        for line in self._proc.stdout:
            if self._stop.is_set():
                break
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append(parts)

    def stop(self):
        self._stop.set()
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except Exception:
                self._proc.kill()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        smax = [float(s[2]) for s in self.samples if s[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for s in self.samples:
            for n, val in zip(names, s[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(self.samples)}


def cpu_baseline(name: str, target_s: float = 12.0, dropout: float = 0.0):
    """Time the oracle on a bounded row sample of the workload; TFLOP/s of the sample."""
    import oracle
    runs = workload_runs(name)
    per_run_s = target_s / len(runs)
    flops_total, t_total, rows_total = 0.0, 0.0, 0
    desc = []
    for w in runs:
        q, k, v = workload_inputs(w)
        # rows of the sample: random rows over all heads; cost per row = 4*D*(keys seen)
        n = 64
        while True:
            bh, rows = sample_rows(w.B, w.H, w.S, n_random=n, edge=0, seed=99)
            t0 = time.perf_counter()
            if dropout > 0.0:
                oracle.attn_rows_dropout(q, k, v, w.scale, w.causal, w.dtype, int(np.floor(dropout * 256 + 0.5)),
                                         DROPOUT_SEED, 0, bh, rows)
            elif w.general:
                oracle.attn_rows_gen(q, k, v, w.scale, w.causal, w.dtype, bh, rows)
            else:
                oracle.attn_rows(q, k, v, w.scale, w.causal, w.dtype, bh, rows)
            dt = time.perf_counter() - t0
            if dt >= per_run_s * 0.5 or n >= (1 << 20):
                break
            n = int(n * min(16.0, max(2.0, per_run_s / max(dt, 1e-3))))
        keys = np.minimum(rows + (w.Skv - w.S) + 1, w.Skv) if w.causal else np.full_like(rows, w.Skv)
        flops = float(4.0 * w.D * keys.sum())
        flops_total += flops
        t_total += dt
        rows_total += len(rows)
        desc.append(f"{len(rows)} random query rows of {w.describe()}")
    return {"value": flops_total / t_total / 1e12, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "; ".join(desc) + f" ({t_total:.1f} s fp64 on the host cores; TFLOP/s of the sample's"
                      " algorithmic flops)"}


def algorithmic_bytes(w) -> float:
    """Bytes one forward launch must move: Q, K, V read and O written in 16 bits, the fp32 LSE written."""
    return float(w.B * w.H * (2 * w.S * w.D * 2 + 2 * w.Skv * w.D * 2 + 4 * w.S))


def time_single_run(fa, w, dev, stream, steps: int, warmup: int, rank: int):
    """Time one forward workload alone (its own inputs, seeded per rank; rotated over
    device copies when smaller than twice the L2), CUDA events around each launch on
    the launching stream.  Returns the run's mean launch time and TFLOP/s."""
    import torch
    wr = dataclasses.replace(w, seed=rank_seed(w.seed, rank))
    q, k, v = workload_inputs(wr)
    set_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))
    copies = 1 if set_bytes >= 2 * L2_BYTES else min(64, -(-2 * L2_BYTES // set_bytes))
    ins = [tuple(t.to(dev) for t in (q, k, v)) for _ in range(copies)]
    o = torch.empty((w.B, w.H, w.S, w.D), dtype=w.torch_dtype, device=dev)
    lse = torch.empty((w.B, w.H, w.S), dtype=torch.float32, device=dev)
    dt = fa.FA_BF16 if w.dtype == "bf16" else fa.FA_FP16
    sid = stream.cuda_stream

    def launch(i):
        qq, kk, vv = ins[i % copies]
        st = fa.fa_fwd(qq.data_ptr(), kk.data_ptr(), vv.data_ptr(), o.data_ptr(), lse.data_ptr(), w.B, w.H, w.S,
                       w.D, w.scale, int(w.causal), dt, sid)
        if st != 0:
            raise fa.FaError(st)

    for i in range(warmup):
        launch(i)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for i, (a, b) in enumerate(ev):
        a.record(stream)
        launch(i)
        b.record(stream)
    torch.cuda.synchronize(dev)
    st = fa.fa_check_status(sid)
    if st != 0:
        raise fa.FaError(st, "timed run")
    mean_ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    return {"run": w.describe(), "launches": steps, "mean_ms": mean_ms,
            "tflops": w.flops / (mean_ms * 1e-3) / 1e12,
            "hbm_gbs": algorithmic_bytes(w) / (mean_ms * 1e-3) / 1e9}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    runs = workload_runs(args.workload)
    bwd = args.pass_ == "bwd"
    # the oracle keeps no state between calls: warm-up steps have nothing to warm
    times, walls = [], []
    for _ in range(args.steps):
        budget = args.cpu_seconds if args.cpu_seconds > 0 else max(2.0, 60.0 / max(args.steps, 1))
        t0 = time.perf_counter()
        cb = (cpu_baseline_bwd(args.workload, target_s=budget, dropout=args.dropout) if bwd else
              cpu_baseline(args.workload, target_s=budget, dropout=args.dropout))
        walls.append(time.perf_counter() - t0)
        times.append(cb)
    value = float(np.median([c["value"] for c in times]))
    cb = dict(times[-1])
    cb["value"] = value
    step_flops = (BWD_FLOP_FACTOR if bwd else 1.0) * sum(w.flops for w in runs)
    label = ("backward of " if bwd else "") + workload_label(args.workload) + (
        f", attention dropout p = {args.dropout:g}" if args.dropout > 0 else "")
    line = {
        "impl": "reference", "metric": BWD_METRIC if bwd else METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * float(np.mean(walls)),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": label,
                   "note": "fp64 CPU oracle; each step is a bounded sample of the workload (ms_per_step is the"
                           " measured wall time of one sampled step; value is the sample's TFLOP/s)",
                   "projected_ms_per_full_step": step_flops / (value * 1e12) * 1e3},
        "cpu_baseline": cb,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


BWD_FLOP_FACTOR = 2.5  # five S x S x D products in the backward pass against two in the forward pass
BWD_METRIC = "attention bwd TFLOPS (2.5x forward flops, causal-adjusted) and % of B200 dense bf16 peak"


def cpu_baseline_bwd(name: str, target_s: float = 12.0, dropout: float = 0.0):
    """The fp64 backward oracle on one head of the workload's first run with the
    sequence cut to a length whose cost fits ``target_s``; TFLOP/s of that sample
    (2.5x the forward's algorithmic flops of the sample)."""
    import dataclasses as dc

    import oracle
    import torch
    w = workload_runs(name)[-1]
    S = 256
    while True:
        ws = dc.replace(w, B=1, H=1, S=min(S, w.S), Sk=(min(S, w.Skv) if w.Sk else 0))
        q, k, v = workload_inputs(ws)
        g = torch.Generator().manual_seed(5)
        dout = torch.randn(q.shape, generator=g).to(q.dtype)
        t0 = time.perf_counter()
        if dropout > 0.0:
            oracle.attn_bwd_dropout(q, k, v, dout, ws.scale, ws.causal, ws.dtype, int(np.floor(dropout * 256 + 0.5)),
                                    DROPOUT_SEED, 0)
        else:
            oracle.attn_bwd(q, k, v, dout, ws.scale, ws.causal, ws.dtype)
        dt = time.perf_counter() - t0
        if dt >= target_s / 8 or S >= w.S:
            break
        S *= 2
    flops = BWD_FLOP_FACTOR * ws.flops
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"fp64 backward oracle on one head of {ws.describe()} ({dt:.1f} s on the host cores)"}


def run_bwd(args) -> int:
    """Time fa_bwd (the backward pass) on the workload; O and LSE come from one
    forward call before the timed region, dO is seeded random."""
    import torch
    import torch.distributed as dist

    import tiled_attention_18_b200 as fa

    rank, world, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    fa.load()
    from tiled_attention_18_b200.workloads import to_layout
    runs = workload_runs(args.workload)
    for w in runs:
        if w.layout != "bhsd" and (args.dropout > 0.0 or args.deterministic):
            raise SystemExit("--dropout and --deterministic take BHSD workloads")
    stream = torch.cuda.current_stream(dev)
    sid = stream.cuda_stream
    bufs = []
    for w in runs:
        wr = dataclasses.replace(w, seed=rank_seed(w.seed, rank))
        # BSHD workloads: every tensor (inputs, O, dO, gradients) in that layout, through fa_bwd_ex
        q, k, v = (to_layout(t.to(dev), w.layout) for t in workload_inputs(wr))
        g = torch.Generator().manual_seed(rank_seed(w.seed, rank) + 7)
        dout = to_layout(torch.randn(q.shape, generator=g).to(q.dtype).to(dev), w.layout)
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
        dt = fa.FA_BF16 if w.dtype == "bf16" else fa.FA_FP16
        if args.dropout > 0.0:
            st = fa.fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), w.B, w.H,
                                   w.S, w.Skv, w.D, w.scale, int(w.causal), args.dropout, DROPOUT_SEED, 0, dt, sid)
        else:
            st = fa.fa_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), w.B, w.H, w.S,
                              w.Skv, w.D, q.stride()[:3], k.stride()[:3], v.stride()[:3], o.stride()[:3], w.scale,
                              int(w.causal), dt, sid)
        if st != 0:
            raise fa.FaError(st)
        nbytes = fa.fa_bwd_workspace_size(w.B, w.H, w.S, w.D)
        if nbytes < 0:
            raise SystemExit(f"the backward pass takes D = 64 or 128 ({fa.fa_status_string(int(nbytes))})")
        bufs.append(dict(q=q, k=k, v=v, o=o, lse=lse, dout=dout, dq=torch.empty_like(q), dk=torch.empty_like(k),
                         dv=torch.empty_like(v), ws=torch.empty(nbytes, dtype=torch.uint8, device=dev),
                         nbytes=nbytes, dt=dt))

    def launch(i):
        w, b = runs[i], bufs[i]
        if args.dropout > 0.0:
            # the forward's decisions (offset 0), regenerated by the backward
            st = fa.fa_bwd_dropout(b["q"].data_ptr(), b["k"].data_ptr(), b["v"].data_ptr(), b["o"].data_ptr(),
                                   b["dout"].data_ptr(), b["lse"].data_ptr(), b["dq"].data_ptr(), b["dk"].data_ptr(),
                                   b["dv"].data_ptr(), b["ws"].data_ptr(), b["nbytes"], w.B, w.H, w.S, w.Skv, w.D,
                                   w.scale, int(w.causal), args.dropout, DROPOUT_SEED, 0, int(args.deterministic),
                                   b["dt"], sid)
            if st != 0:
                raise fa.FaError(st, "fa_bwd_dropout")
            return
        if w.layout != "bhsd":
            names = ("q", "k", "v", "o", "dout", "dq", "dk", "dv")
            st = fa.fa_bwd_ex(*(b[n].data_ptr() for n in names[:5]), b["lse"].data_ptr(),
                              *(b[n].data_ptr() for n in names[5:]), b["ws"].data_ptr(), b["nbytes"], w.B, w.H, w.S,
                              w.Skv, w.D, *(b[n].stride()[:3] for n in names), w.scale, int(w.causal), 0, b["dt"],
                              sid)
            if st != 0:
                raise fa.FaError(st, "fa_bwd_ex")
            return
        st = fa.fa_bwd(b["q"].data_ptr(), b["k"].data_ptr(), b["v"].data_ptr(), b["o"].data_ptr(),
                       b["dout"].data_ptr(), b["lse"].data_ptr(), b["dq"].data_ptr(), b["dk"].data_ptr(),
                       b["dv"].data_ptr(), b["ws"].data_ptr(), b["nbytes"], w.B, w.H, w.S, w.Skv, w.D, w.scale,
                       int(w.causal), int(args.deterministic), b["dt"], sid)
        if st != 0:
            raise fa.FaError(st, "fa_bwd")

    for _ in range(args.warmup):
        for i in range(len(runs)):
            launch(i)
    torch.cuda.synchronize(dev)
    st = fa.fa_check_status(sid)
    if st != 0:
        raise fa.FaError(st, "warm-up")
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in runs]
          for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    start.record(stream)
    for s_ in range(args.steps):
        for i in range(len(runs)):
            ev[s_][i][0].record(stream)
            launch(i)
            ev[s_][i][1].record(stream)
    stop.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    sampler.stop()
    clk = sampler.summary()
    st = fa.fa_check_status(sid)
    if st != 0:
        raise fa.FaError(st, "timed region")
    kern_ms = np.array([[a.elapsed_time(b) for (a, b) in row] for row in ev])
    max_ms = max_over_ranks(start.elapsed_time(stop), device=dev)
    step_flops = BWD_FLOP_FACTOR * sum(w.flops for w in runs)
    value = job_throughput(step_flops, args.steps, world, max_ms)
    peak, peak_src, peak_burst = peak_tflops(clk)
    per_run = [{"run": w.describe(), "mean_ms": float(kern_ms[:, i].mean()),
                "tflops": BWD_FLOP_FACTOR * w.flops / (float(kern_ms[:, i].mean()) * 1e-3) / 1e12}
               for i, w in enumerate(runs)]
    achieved = step_flops / (float(kern_ms.sum(axis=1).mean()) * 1e-3) / 1e12

    e2e = None
    if not args.no_e2e:
        names_in = ("q", "k", "v", "o", "dout", "lse")
        names_out = ("dq", "dk", "dv")
        host = [{n: torch.empty(b[n].shape, dtype=b[n].dtype).pin_memory() for n in names_in + names_out}
                for b in bufs]
        for hb, b in zip(host, bufs):
            for n in names_in:
                hb[n].copy_(b[n])
        h2d = sum(hb[n].numel() * hb[n].element_size() for hb in host for n in names_in)
        d2h = sum(hb[n].numel() * hb[n].element_size() for hb in host for n in names_out)

        # chunks of whole batches (or heads of a single BHSD batch) pipelined
        # over three streams, consecutive steps on two sets of device buffers,
        # as in the forward pass; dropout keeps one chunk (its keep decisions
        # are drawn per absolute head index) and no step overlap
        def chunk_plan(w):
            # the tensors here are [B, H, S, D] views, so the head axis is 1 in
            # either storage layout; a head range of a BSHD batch is not one
            # block of memory, so BSHD with B = 1 keeps one chunk
            if args.dropout > 0.0 or (w.B == 1 and w.layout != "bhsd"):
                return 0, [(0, w.B)]
            axis, rng = e2e_chunks(w.B, w.H, args.e2e_chunks)
            return (0 if axis == "b" else 1), rng

        plans = [chunk_plan(w) for w in runs]
        up_s, dn_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_up = [[torch.cuda.Event() for _ in p[1]] for p in plans]
        ev_k = [[torch.cuda.Event() for _ in p[1]] for p in plans]
        n_chunk_max = max(len(p[1]) for p in plans)
        overlap_steps = n_chunk_max > 1
        # the second set: the step's inputs and gradients (the workspace is
        # used by one launch at a time on the timing stream, so one suffices)
        buf_sets = [bufs]
        if overlap_steps:
            buf_sets.append([dict(b, **{nm: torch.empty_like(b[nm]) for nm in names_in + names_out}) for b in bufs])
        ev_kend = [torch.cuda.Event(), torch.cuda.Event()]
        ev_dnend = [torch.cuda.Event(), torch.cuda.Event()]
        step_count = [0]

        def launch_chunk(i, ax, a, n, ps):
            w, b = runs[i], buf_sets[ps][i]
            if len(plans[i][1]) == 1:
                launch(i)
                return
            names = ("q", "k", "v", "o", "dout", "dq", "dk", "dv")
            t = {nm: b[nm].narrow(ax, a, n) for nm in names + ("lse",)}
            st = fa.fa_bwd_ex(*(t[nm].data_ptr() for nm in names[:5]), t["lse"].data_ptr(),
                              *(t[nm].data_ptr() for nm in names[5:]), b["ws"].data_ptr(), b["nbytes"],
                              t["q"].shape[0], t["q"].shape[1], w.S, w.Skv, w.D,
                              *(t[nm].stride()[:3] for nm in names), w.scale, int(w.causal), int(args.deterministic),
                              b["dt"], sid)
            if st != 0:
                raise fa.FaError(st, "fa_bwd_ex")

        def e2e_step():
            ps = step_count[0] % 2 if overlap_steps else 0
            step_count[0] += 1
            if not overlap_steps:
                start_ev = torch.cuda.Event()
                start_ev.record(stream)
                up_s.wait_event(start_ev)
                dn_s.wait_event(start_ev)
            else:
                up_s.wait_event(ev_kend[ps])      # this set's inputs read by its previous step
                stream.wait_event(ev_dnend[ps])   # this set's gradients downloaded by its previous step
            for c in range(n_chunk_max):
                for i, hb in enumerate(host):
                    b = buf_sets[ps][i]
                    ax, rng = plans[i]
                    if c >= len(rng):
                        continue
                    a, n = rng[c]
                    with torch.cuda.stream(up_s):
                        for nm in names_in:
                            b[nm].narrow(ax, a, n).copy_(hb[nm].narrow(ax, a, n), non_blocking=True)
                    ev_up[i][c].record(up_s)
                    stream.wait_event(ev_up[i][c])
                    launch_chunk(i, ax, a, n, ps)
                    ev_k[i][c].record(stream)
                    dn_s.wait_event(ev_k[i][c])
                    with torch.cuda.stream(dn_s):
                        for nm in names_out:
                            hb[nm].narrow(ax, a, n).copy_(b[nm].narrow(ax, a, n), non_blocking=True)
            ev_kend[ps].record(stream)
            ev_dnend[ps].record(dn_s)
            if not overlap_steps:
                stream.wait_event(ev_dnend[ps])

        def join():
            for s_ in (up_s, dn_s):
                ev = torch.cuda.Event()
                ev.record(s_)
                stream.wait_event(ev)

        for _ in range(2):
            e2e_step()
        join()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        up_s.wait_event(e0)
        dn_s.wait_event(e0)
        for _ in range(args.e2e_steps):
            e2e_step()
        join()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e = {"value": job_throughput(step_flops, args.e2e_steps, world,
                                       max_over_ranks(e0.elapsed_time(e1), device=dev)),
               "unit": UNIT, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "overlap": (f"{n_chunk_max} chunks per step; uploads, launches and downloads on three streams; "
                           "consecutive steps overlap on two sets of device buffers"
                           if overlap_steps else "none")}
        # the chunked gradients against one launch over all heads (fp32 sums
        # of dQ, and of split dK/dV, may add in another order)
        for i in range(len(runs)):
            launch(i)
        torch.cuda.synchronize(dev)
        for i, (hb, b) in enumerate(zip(host, bufs)):
            for nm in names_out:
                ref = b[nm].float().cpu()
                err = float((hb[nm].float() - ref).abs().max())
                if not err <= 0.02 * float(ref.abs().max()) + 1e-6:
                    raise SystemExit(f"end-to-end {nm} of run {i} differs from a whole launch by {err}")
    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline_bwd(args.workload, dropout=args.dropout)
    if rank == 0:
        w0 = runs[0]
        line = {
            "metric": BWD_METRIC,
            "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": max_ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w0.dtype, "data": "synthetic",
            "config": {"workload": ("deterministic " if args.deterministic else "") + "backward of "
                       + workload_label(args.workload)
                       + (f", attention dropout p = {args.dropout:g}" if args.dropout > 0 else ""), "B": w0.B, "H": w0.H,
                       "S": w0.S, "D": w0.D, "runs_per_step": len(runs),
                       "l2": "inputs larger than L2 (no flush)" if sum(
                           t.numel() * t.element_size() for t in (bufs[0]["q"], bufs[0]["k"], bufs[0]["v"],
                                                                  bufs[0]["dout"])) > L2_BYTES
                       else "inputs smaller than L2 (warm)",
                       "parallelism": f"independent batch per GPU x{world}"},
            "pct_of_peak": 100.0 * value / (peak * world),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                         "frac": achieved / peak, "traffic": None, "peak_source": peak_src,
                         "peak_burst": peak_burst, "frac_burst": achieved / peak_burst, "per_run": per_run},
            "clocks": clk,
            "e2e": e2e,
            "gpu_launches": 3 * len(runs) * args.steps,
            "cpu_baseline": cb,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def hbm_peak():
    try:
        with open(PEAKS_PATH) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s, an earlier copy-bandwidth measurement on B200)"


def run_sp(args) -> int:
    """Sequence-parallel forward: the ring (or all-gather) schedule of
    sequence_parallel.py for --sp-world ranks, run one rank after another on
    this GPU with the K/V blocks handed over in memory -- every partial
    attention, merge and finalize launch of all ranks, no communication.  The
    value is the attention throughput of the split computation (whole-sequence
    flops over the summed device time), to set beside the single-kernel
    forward; the merge kernel's HBM roofline is reported beside it."""
    import torch

    import tiled_attention_18_b200 as fa
    from tiled_attention_18_b200.sequence_parallel import CudaOps, allgather_attention_forward, ring_attention_forward

    rank, world, local = rank_env()
    if world > 1:
        raise SystemExit("--pass sp runs every rank's schedule in one process on one GPU; launch it without torchrun")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    fa.load()
    W = args.sp_world
    runs = workload_runs(args.workload)
    for w in runs:
        if w.layout != "bhsd" or w.S != w.Skv or w.S % W:
            raise SystemExit("--pass sp needs a self-attention BHSD workload whose S divides into --sp-world chunks")
    stream = torch.cuda.current_stream(dev)
    sid = stream.cuda_stream
    data = []
    for w in runs:
        q, k, v = (t.to(dev) for t in workload_inputs(w))
        c = w.S // W
        if args.sp_mode == "ulysses":
            if w.H % W:
                raise SystemExit("--sp-mode ulysses needs H divisible by --sp-world")
            hw = w.H // W
            # each rank's head group over the whole sequence (what the all-to-all delivers)
            heads = [tuple(t[:, r * hw:(r + 1) * hw].contiguous() for t in (q, k, v)) for r in range(W)]
            data.append((w, heads, None, None))
        else:
            qs = [q[:, :, r * c:(r + 1) * c].contiguous() for r in range(W)]
            kv = [torch.stack([k[:, :, r * c:(r + 1) * c], v[:, :, r * c:(r + 1) * c]]).contiguous()
                  for r in range(W)]
            data.append((w, qs, kv, torch.stack(kv) if args.sp_mode == "allgather" else None))
        del q, k, v

    class TimedOps(CudaOps):
        def __init__(self, scale, log):
            super().__init__(scale)
            self.log = log

        def _timed(self, kind, nbytes, fn, *a):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            out = fn(*a)
            e1.record(stream)
            self.log.append((kind, e0, e1, nbytes))
            return out

        def partial(self, q, k, v, causal):
            return self._timed("partial", 0, super().partial, q, k, v, causal)

        def merge(self, state, o_p, lse_p):
            # per row: fp32 O read and written (8 D bytes), the 16-bit partial O (2 D), three fp32 LSE words
            nbytes = (10 * o_p.shape[-1] + 12) * lse_p.numel()
            return self._timed("merge", nbytes, super().merge, state, o_p, lse_p)

        def finalize(self, state):
            return self._timed("finalize", 0, super().finalize, state)

    def step(log):
        for (w, qs, kv, stacked) in data:
            ops = TimedOps(w.scale, log)
            for r in range(W):
                if args.sp_mode == "ulysses":
                    ops.partial(*qs[r], w.causal)
                    continue
                qk = qs[r]
                if args.sp_mode == "ring":
                    ring_attention_forward(qk, kv[r][0], kv[r][1], w.scale, w.causal, ops=ops, rank=r, world=W,
                                           exchange=lambda s, cur, r=r: (None, kv[(r - s - 1) % W]))
                else:
                    allgather_attention_forward(qk, kv[r][0], kv[r][1], w.scale, w.causal, ops=ops, rank=r,
                                                world=W, gather=lambda cur, st=stacked: st)

    for _ in range(args.warmup):
        step([])
    torch.cuda.synchronize(dev)
    st = fa.fa_check_status(sid)
    if st != 0:
        raise fa.FaError(st, "warm-up")
    log = []
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    torch.cuda.synchronize(dev)
    start.record(stream)
    for _ in range(args.steps):
        step(log)
    stop.record(stream)
    torch.cuda.synchronize(dev)
    sampler.stop()
    clk = sampler.summary()
    st = fa.fa_check_status(sid)
    if st != 0:
        raise fa.FaError(st, "timed region")
    total_ms = start.elapsed_time(stop)
    ms = {"partial": 0.0, "merge": 0.0, "finalize": 0.0}
    n = {"partial": 0, "merge": 0, "finalize": 0}
    merge_bytes = 0
    for kind, a, b, nbytes in log:
        ms[kind] += a.elapsed_time(b)
        n[kind] += 1
        merge_bytes += nbytes
    step_flops = sum(w.flops for w in runs)
    value = step_flops * args.steps / (total_ms * 1e-3) / 1e12
    peak, peak_src, peak_burst = peak_tflops(clk)
    achieved = step_flops * args.steps / (ms["partial"] * 1e-3) / 1e12
    hbm, hbm_src = hbm_peak()
    merge_info = None
    if n["merge"]:
        gbs = merge_bytes / (ms["merge"] * 1e-3) / 1e9
        merge_info = {"bytes_per_launch": merge_bytes / n["merge"], "mean_us": 1e3 * ms["merge"] / n["merge"],
                      "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm, "peak_source": hbm_src,
                      "launches_per_step": n["merge"] // args.steps}
    launches = sum(n.values())  # partials, merges, finalizes; the all-gather's K/V copies are torch's
    cb = None if args.no_cpu_baseline else cpu_baseline(args.workload)
    w0 = runs[0]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w0.dtype, "data": "synthetic",
        "config": {"workload": f"sequence-parallel ({args.sp_mode}, {W} ranks run in turn on one GPU, no "
                               f"communication) " + workload_label(args.workload),
                   "B": w0.B, "H": w0.H, "S": w0.S, "D": w0.D, "chunk": w0.S // W,
                   "l2": "inputs larger than L2 (no flush)"},
        "pct_of_peak": 100.0 * value / peak,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
                     "traffic": None, "peak_source": peak_src, "peak_burst": peak_burst,
                     "frac_burst": achieved / peak_burst, "kernel": "fa_fwd_ex partials"},
        "time_split_ms_per_step": {k: v / args.steps for k, v in ms.items()},
        "merge": merge_info,
        "clocks": clk,
        "e2e": None,
        "gpu_launches": launches,
        "cpu_baseline": cb,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["fa", "reference"], default="fa")
    ap.add_argument("--workload", default="c5", choices=["c5"] + list(ALL_WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--e2e-chunks", type=int, default=4,
                    help="chunks (batches, or heads of a single batch) per end-to-end step, pipelined over "
                         "three streams (upload, launches, download)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="do not time the S = 8192 causal layer (c4) beside the default step")
    ap.add_argument("--cpu-seconds", type=float, default=0.0,
                    help="--impl reference: CPU seconds per step (default: about a minute per run)")
    ap.add_argument("--pass", dest="pass_", choices=["fwd", "bwd", "sp"], default="fwd",
                    help="fwd: the forward pass (default); bwd: the backward pass fa_bwd; sp: the "
                         "sequence-parallel schedule of --sp-world ranks run in turn on one GPU")
    ap.add_argument("--sp-world", type=int, default=4, help="with --pass sp: ranks of the schedule")
    ap.add_argument("--sp-mode", choices=["ring", "allgather", "ulysses"], default="ring", help="with --pass sp")
    ap.add_argument("--mask", choices=["none", "tril"], default="none",
                    help="tril: causal runs go through fa_fwd_mask with an explicit lower-triangular mask "
                         "(the catlass page's mode 1) instead of the in-kernel diagonal skip (mode 2)")
    ap.add_argument("--dropout", type=float, default=0.0,
                    help="attention dropout probability (fa_fwd_dropout / fa_bwd_dropout); 0 = none")
    ap.add_argument("--block-n", type=int, default=0, choices=[0, 64, 128],
                    help="forward keys per key tile (0 = automatic, 128); through fa_forward")
    ap.add_argument("--q-tiles", type=int, default=0, choices=[0, 1, 2],
                    help="forward 128-row query tiles per work unit (0 = automatic, 2); through fa_forward")
    ap.add_argument("--graph", action="store_true",
                    help="forward: capture each run's STEPS launches (inputs rotated as usual) in one CUDA graph and "
                         "time its replay, so that the per-launch host cost (argument checks, tensor maps, "
                         "cudaLaunchKernelEx) leaves the device timeline; for kernels shorter than that host cost. "
                         "Per-launch times are the graph's time / STEPS")
    ap.add_argument("--deterministic", action="store_true",
                    help="with --pass bwd: the deterministic dQ mode (key tiles add in order)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.pass_ == "bwd":
        return run_bwd(args)
    if args.pass_ == "sp":
        return run_sp(args)

    import torch
    import torch.distributed as dist

    import tiled_attention_18_b200 as fa

    rank, world, local = rank_env()
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE", file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    fa.load()
    runs = workload_runs(args.workload)
    stream = torch.cuda.current_stream(dev)
    sid = stream.cuda_stream

    # inputs: each rank draws its own independent batch (seed = workload seed + rank).
    # Each tensor is held as "storage" contiguous in the workload's layout
    # (BHSD, or BSHD read through a transposed view); inputs smaller than twice
    # the L2 are rotated over several device copies so that every step reads
    # them from DRAM.
    def storage(w, t):
        return t.contiguous() if w.layout == "bhsd" else t.transpose(1, 2).contiguous()

    def view(w, t):
        return t if w.layout == "bhsd" else t.transpose(1, 2)

    host_in, dev_in, dev_out, n_copies = [], [], [], []
    for i, w in enumerate(runs):
        if i > 0 and not w.general and (w.B, w.H, w.S, w.D, w.dtype, w.qk_mult) == (
                runs[0].B, runs[0].H, runs[0].S, runs[0].D, runs[0].dtype, runs[0].qk_mult):
            host_in.append(host_in[0])
            dev_in.append(dev_in[0])
            n_copies.append(n_copies[0])
        else:
            wr = dataclasses.replace(w, seed=rank_seed(w.seed, rank))
            q, k, v = (storage(w, t) for t in workload_inputs(wr))
            set_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))
            copies = 1 if set_bytes >= 2 * L2_BYTES else min(64, -(-2 * L2_BYTES // set_bytes))
            host_in.append(tuple(t.pin_memory() for t in (q, k, v)))
            dev_in.append([tuple(t.to(dev) for t in (q, k, v)) for _ in range(copies)])
            n_copies.append(copies)
        o = storage(w, torch.empty((w.B, w.H, w.S, w.D), dtype=w.torch_dtype)).to(dev)
        lse = torch.empty((w.B, w.H, w.S), dtype=torch.float32, device=dev)
        dev_out.append((o, lse))

    # --mask tril: one shared [1, 1, Sq, Sk] uint8 lower-triangular mask (rows padded to 16 bytes)
    tril = {}
    if args.mask == "tril":
        for i, w in enumerate(runs):
            if w.causal:
                pad = -(-w.Skv // 16) * 16
                ii = torch.arange(w.S, device=dev)[:, None]
                jj = torch.arange(pad, device=dev)[None, :]
                tril[i] = ((jj <= ii + (w.Skv - w.S)) & (jj < w.Skv)).to(torch.uint8).contiguous()

    def launch(i, step=0, sid=sid):
        w = runs[i]
        q, k, v = (view(w, t) for t in dev_in[i][step % n_copies[i]])
        o, lse = dev_out[i]
        o = view(w, o)
        dt = fa.FA_BF16 if w.dtype == "bf16" else fa.FA_FP16
        if args.dropout > 0.0:
            if w.layout != "bhsd":
                raise SystemExit("--dropout takes BHSD workloads")
            # a fresh offset per step: new keep decisions, as in training
            st = fa.fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), w.B, w.H,
                                   w.S, w.Skv, w.D, w.scale, int(w.causal), args.dropout, DROPOUT_SEED, step, dt, sid)
        elif i in tril:
            if w.layout != "bhsd":
                raise SystemExit("--mask takes BHSD workloads")
            m = tril[i]
            st = fa.fa_fwd_mask(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), w.B, w.H,
                                w.S, w.Skv, w.D, m.data_ptr(), (0, 0, m.stride(0)), w.scale, 0, dt, sid)
        elif args.block_n or args.q_tiles:
            st = fa.fa_forward(sid, q=q.data_ptr(), k=k.data_ptr(), v=v.data_ptr(), o=o.data_ptr(),
                               lse=lse.data_ptr(), B=w.B, H=w.H, Sq=w.S, Sk=w.Skv, D=w.D, q_stride=q.stride()[:3],
                               k_stride=k.stride()[:3], v_stride=v.stride()[:3], o_stride=o.stride()[:3],
                               scale=w.scale, causal=int(w.causal), dtype=dt, block_n=args.block_n,
                               q_tiles=args.q_tiles)
        elif w.general:
            st = fa.fa_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), w.B, w.H, w.S,
                              w.Skv, w.D, q.stride()[:3], k.stride()[:3], v.stride()[:3], o.stride()[:3], w.scale,
                              int(w.causal), dt, sid)
        else:
            st = fa.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), w.B, w.H, w.S,
                           w.D, w.scale, int(w.causal), dt, sid)
        if st != 0:
            raise fa.FaError(st)

    # warm-up
    for s_ in range(args.warmup):
        for i in range(len(runs)):
            launch(i, s_)
    torch.cuda.synchronize(dev)
    st = fa.fa_check_status(sid)
    if st != 0:
        raise fa.FaError(st, "warm-up")

    # --graph: each run's STEPS launches captured in one graph, replayed on the timing stream
    graphs = None
    if args.graph:
        if args.dropout > 0.0:
            raise SystemExit("--graph takes runs without dropout (the offset changes per step)")
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        graphs = []
        for i in range(len(runs)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                for s_ in range(args.steps):
                    launch(i, s_, cap.cuda_stream)
            graphs.append(g)
        stream.wait_stream(cap)
        for g in graphs:
            g.replay()
        torch.cuda.synchronize(dev)

    # timed region: per-launch events on the launching stream
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in runs]
          for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(dev)
    start.record(stream)
    if graphs is not None:
        for i in range(len(runs)):
            ev[0][i][0].record(stream)
            graphs[i].replay()
            ev[0][i][1].record(stream)
    else:
        for s in range(args.steps):
            for i in range(len(runs)):
                ev[s][i][0].record(stream)
                launch(i, s)
                ev[s][i][1].record(stream)
    stop.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    sampler.stop()
    clk = sampler.summary()
    st = fa.fa_check_status(sid)
    if st != 0:
        raise fa.FaError(st, "timed region")
    elapsed_ms = start.elapsed_time(stop)
    if graphs is not None:
        kern_ms = np.array([[a.elapsed_time(b) / args.steps for (a, b) in ev[0]]] * args.steps)
    else:
        kern_ms = np.array([[a.elapsed_time(b) for (a, b) in row] for row in ev])  # [steps, runs]
    max_ms = max_over_ranks(elapsed_ms, device=dev)
    step_flops = sum(w.flops for w in runs)
    value = job_throughput(step_flops, args.steps, world, max_ms)
    peak, peak_src, peak_burst = peak_tflops(clk)
    # roofline of the kernel: algorithmic flops per launch / mean launch duration
    hbm, hbm_src = hbm_peak()
    per_run = []
    for i, w in enumerate(runs):
        mean_ms = float(kern_ms[:, i].mean())
        gbs = algorithmic_bytes(w) / (mean_ms * 1e-3) / 1e9
        per_run.append({"run": w.describe(), "mean_ms": mean_ms, "tflops": w.flops / (mean_ms * 1e-3) / 1e12,
                        "frac": w.flops / (mean_ms * 1e-3) / 1e12 / peak,
                        "hbm_gbs": gbs, "hbm_frac": gbs / hbm})
    achieved = step_flops / (float(kern_ms.sum(axis=1).mean()) * 1e-3) / 1e12
    step_bytes = sum(algorithmic_bytes(w) for w in runs)
    hbm_achieved = step_bytes / (float(kern_ms.sum(axis=1).mean()) * 1e-3) / 1e9
    # fewer work units than SMs: neither the tensor pipe nor HBM can be busy (launch/latency-bound)
    n_units = sum(fa.fa_num_units(w.B, w.H, w.S) for w in runs if not w.general)
    bound = "latency" if (not runs[0].general and n_units < torch.cuda.get_device_properties(dev).multi_processor_count
                          ) else "tensor"
    # short key sets (Sk <= 128, automatic tiling, no mask or dropout) take the
    # short-key kernel: one score tile per query tile, bound by moving Q in and O out
    if (all(w.Skv <= 128 and w.D != 256 for w in runs) and not tril and args.dropout == 0.0
            and not args.block_n and not args.q_tiles):
        bound = "hbm"

    # the 13B-style layer (S = 8192, causal, Q,K x2) timed beside the default step
    extra_runs = []
    if (args.workload == "c5" and args.dropout == 0.0 and not tril and not args.no_extra and not args.block_n
            and not args.q_tiles):
        r = time_single_run(fa, WORKLOADS["c4"], dev, stream, max(args.steps, 10), args.warmup, rank)
        r["frac"] = r["tflops"] / peak
        r["hbm_frac"] = r["hbm_gbs"] / hbm
        extra_runs.append(r)
    # the committed DRAM capture is of the kernels without dropout or an explicit mask
    traffic = (traffic_per_launch(args.workload)
               if (args.dropout == 0.0 and not tril and not args.block_n and not args.q_tiles) else None)

    # end to end through the public call with host buffers
    e2e = None
    if not args.no_e2e:
        host_out = [(torch.empty(o.shape, dtype=o.dtype).pin_memory(), torch.empty(l.shape, dtype=l.dtype).pin_memory())
                    for (o, l) in dev_out]
        h2d = sum(sum(t.numel() * t.element_size() for t in host_in[i]) for i in range(len(runs))
                  if i == 0 or host_in[i] is not host_in[0])
        d2h = sum(o.numel() * o.element_size() + l.numel() * l.element_size() for (o, l) in host_out)

        # The heads are independent problems: each step uploads its inputs in
        # chunks (whole batches, or heads of a single batch: contiguous ranges
        # of every storage tensor) on one stream, runs each chunk's launches on
        # the timing stream once its upload has landed, and downloads each
        # chunk's O and LSE on a third stream once its launches are done, so
        # the copies in both directions overlap the kernels.  Consecutive steps
        # overlap too, as requests do in a serving loop: they alternate between
        # two sets of device buffers, and a step's upload into a set waits only
        # for the launches that read that set two steps before, its launches
        # only for that step's downloads of the set's outputs.
        plain = args.dropout == 0.0 and not tril and not args.block_n and not args.q_tiles
        n_chunks = max(1, args.e2e_chunks) if plain else 1

        def chunk_plan(w):
            # storage tensors: the head axis is 1 in BHSD, 2 in BSHD; LSE is [B, H, S]
            axis, rng = e2e_chunks(w.B, w.H, n_chunks)
            if axis == "b":
                return 0, 0, rng
            return (1 if w.layout == "bhsd" else 2), 1, rng

        plans = [chunk_plan(w) for w in runs]
        n_steps_chunk = max(len(p[2]) for p in plans)
        up_s, dn_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_up = [[torch.cuda.Event() for _ in p[2]] for p in plans]
        ev_k = [[torch.cuda.Event() for _ in p[2]] for p in plans]
        # the second set of device buffers (inputs shared between runs stay shared)
        overlap_steps = n_steps_chunk > 1
        sets_in, sets_out = [[t[0] for t in dev_in]], [list(dev_out)]
        if overlap_steps:
            second_in = []
            for i in range(len(runs)):
                shared = i > 0 and host_in[i] is host_in[0]
                second_in.append(second_in[0] if shared else tuple(torch.empty_like(t) for t in dev_in[i][0]))
            sets_in.append(second_in)
            sets_out.append([(torch.empty_like(o), torch.empty_like(l)) for (o, l) in dev_out])
        ev_kend = [torch.cuda.Event(), torch.cuda.Event()]  # a set's last launch of its latest step
        ev_dnend = [torch.cuda.Event(), torch.cuda.Event()]  # a set's last download of its latest step
        step_count = [0]

        def launch_chunk(i, ax_s, ax_l, a, n, ps):
            w = runs[i]
            if len(plans[i][2]) == 1:
                launch(i)
                return
            q, k, v = (view(w, t.narrow(ax_s, a, n)) for t in sets_in[ps][i])
            o = view(w, sets_out[ps][i][0].narrow(ax_s, a, n))
            lse = sets_out[ps][i][1].narrow(ax_l, a, n)
            dt = fa.FA_BF16 if w.dtype == "bf16" else fa.FA_FP16
            st = fa.fa_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), q.shape[0],
                              q.shape[1], w.S, w.Skv, w.D, q.stride()[:3], k.stride()[:3], v.stride()[:3],
                              o.stride()[:3], w.scale, int(w.causal), dt, sid)
            if st != 0:
                raise fa.FaError(st)

        def e2e_step():
            ps = step_count[0] % 2 if overlap_steps else 0
            step_count[0] += 1
            if not overlap_steps:
                start = torch.cuda.Event()
                start.record(stream)
                up_s.wait_event(start)
                dn_s.wait_event(start)
            else:
                up_s.wait_event(ev_kend[ps])      # this set's inputs read by its previous step
                stream.wait_event(ev_dnend[ps])   # this set's outputs downloaded by its previous step
            for c in range(n_steps_chunk):
                for i in range(len(runs)):
                    ax_s, ax_l, rng = plans[i]
                    if c >= len(rng):
                        continue
                    a, n = rng[c]
                    owner = 0 if (i > 0 and host_in[i] is host_in[0]) else i
                    if owner == i:
                        with torch.cuda.stream(up_s):
                            for hsrc, dsrc in zip(host_in[i], sets_in[ps][i]):
                                dsrc.narrow(ax_s, a, n).copy_(hsrc.narrow(ax_s, a, n), non_blocking=True)
                        ev_up[i][c].record(up_s)
                    stream.wait_event(ev_up[owner][c])
                    launch_chunk(i, ax_s, ax_l, a, n, ps)
                    ev_k[i][c].record(stream)
                    dn_s.wait_event(ev_k[i][c])
                    with torch.cuda.stream(dn_s):
                        o_src, l_src = sets_out[ps][i]
                        host_out[i][0].narrow(ax_s, a, n).copy_(o_src.narrow(ax_s, a, n), non_blocking=True)
                        host_out[i][1].narrow(ax_l, a, n).copy_(l_src.narrow(ax_l, a, n), non_blocking=True)
            ev_kend[ps].record(stream)
            ev_dnend[ps].record(dn_s)
            if not overlap_steps:
                stream.wait_event(ev_dnend[ps])

        def join():
            # the timing stream waits for everything the steps put on the copy streams
            for s_ in (up_s, dn_s):
                ev = torch.cuda.Event()
                ev.record(s_)
                stream.wait_event(ev)

        for _ in range(2):
            e2e_step()
        join()
        torch.cuda.synchronize(dev)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        # the copy streams start no earlier than the timed region
        up_s.wait_event(e0)
        dn_s.wait_event(e0)
        for _ in range(args.e2e_steps):
            e2e_step()
        join()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e2e_val = job_throughput(step_flops, args.e2e_steps, world, max_over_ranks(e0.elapsed_time(e1), device=dev))
        e2e = {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "overlap": (f"{n_steps_chunk} chunks per step; uploads, launches and downloads on three streams; "
                           "consecutive steps overlap on two sets of device buffers"
                           if overlap_steps else "none")}
        # the chunked launches compute each head exactly as one launch over all
        # heads does: the downloaded results equal a whole launch's bit for bit
        for i in range(len(runs)):
            launch(i)
        torch.cuda.synchronize(dev)
        for i in range(len(runs)):
            if not (torch.equal(host_out[i][0], dev_out[i][0].cpu()) and torch.equal(host_out[i][1], dev_out[i][1].cpu())):
                raise SystemExit(f"end-to-end results of run {i} differ from a whole launch")

    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(args.workload, dropout=args.dropout)

    if rank == 0:
        w0 = runs[0]
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w0.dtype, "data": "synthetic",
            "config": {"workload": workload_label(args.workload)
                       + (" (causal as an explicit lower-triangular mask, no tile skipping)" if tril else "")
                       + (f", attention dropout p = {args.dropout:g} (fresh offset per step)" if args.dropout > 0 else "")
                       + (f", tiling block_n={args.block_n or 128} q_tiles={args.q_tiles or 2}"
                          if (args.block_n or args.q_tiles) else ""),
                       "B": w0.B, "H": w0.H, "S": w0.S, "D": w0.D,
                       **({"Sk": w0.Skv, "layout": w0.layout} if w0.general else {}),
                       "runs_per_step": len(runs),
                       "l2": ("inputs larger than L2 (no flush)" if max(n_copies) == 1 else
                              f"inputs rotated over {max(n_copies)} device copies (> 2x L2 per rotation, no flush)"),
                       "parallelism": f"independent batch per GPU x{world}",
                       "timing": ("each run's launches replayed from one CUDA graph (host launch cost off the device "
                                  "timeline; per-launch time = graph time / steps)"
                                  if graphs is not None else "each launch through the C ABI, events around each")},
            "pct_of_peak": 100.0 * value / (peak * world),
            "roofline": ({"bound": bound, "achieved": achieved, "peak": peak, "unit": UNIT,
                          "frac": achieved / peak, "traffic": traffic, "peak_source": peak_src,
                          "peak_burst": peak_burst, "frac_burst": achieved / peak_burst,
                          "per_run": per_run,
                          "hbm": {"algorithmic_bytes_per_step": step_bytes, "achieved": hbm_achieved, "peak": hbm,
                                  "unit": "GB/s", "frac": hbm_achieved / hbm, "peak_source": hbm_src}}
                         if bound != "hbm" else
                         {"bound": "hbm", "achieved": hbm_achieved, "peak": hbm, "unit": "GB/s",
                          "frac": hbm_achieved / hbm, "traffic": traffic, "peak_source": hbm_src,
                          "algorithmic_bytes_per_step": step_bytes, "per_run": per_run,
                          "tensor": {"achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
                                     "peak_source": peak_src}}),
            "extra_runs": extra_runs,
            "clocks": clk,
            "e2e": e2e,
            "gpu_launches": len(runs) * args.steps,
            "cpu_baseline": cb,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
