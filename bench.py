#!/usr/bin/env python
"""Throughput of the BERT-style encoder forward on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload KIND:BATCH[:SEQ]] [--no-graph] [--packed] [--no-cpu-baseline]

A step is one forward over one batch of the workload (every layer, every kernel
of the path; by default one replay of the recorded forward, enc_graph_launch,
else one enc_forward call), inputs already in HBM; the L2 is flushed (256 MiB write)
before every timed step.  value = sequences/s over all ranks (weak scaling:
each rank runs its own batch; no collective on the data path).  e2e = the same
metric through enc_forward_host_async: every step copies its input from pinned
host memory and its output back inside the timed region, consecutive steps
overlapping their copies with the encoder.  The per-kernel breakdown and the
roofline come from CUDA events the library records between its kernels on the
launching stream: during the timed steps with --no-graph, else in as many traced
enc_forward calls right after them (a recorded forward carries no events).  The
events break the overlap between kernels, so those times are upper bounds on the
in-graph ones; the roofline divides by the measured burst tensor peak (kernels of
microseconds inside millisecond steps).  --impl reference times the float64 CPU
oracle on a bounded sample.  Rates use each kernel's in-graph time, estimated as
its share of the traced forward times the graph's step (graph_us).
Default workload: 12-layer BERT-Base shape (12x64, FFN 3072), seq 32, batch 512;
the goal point (BERT-Base, seq 128, batch 256) is timed in the same run and
reported under "secondary" (one GPU; --secondary '' skips it).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import encoder_inputs as EI  # noqa: E402

METRIC = "BERT-Base FP16 encoder fwd sequences/s (seq 32/128); % tensor/HBM roofline"
UNIT = "sequences/s"
DEFAULT_WORKLOAD = "bert-base-s32:512"
# The goal point: BERT-Base, seq 128, batch 256.
SECONDARY_WORKLOAD = "bert-base:256:128"
KERNEL_NAMES = ["qkv_gemm", "attention", "out_proj_gemm", "ln1", "ffn1_gemm", "ffn2_gemm", "ln2"]
# when the output-projection and FFN2 GEMMs write the LayerNorm of their rows
KERNEL_NAMES_FUSED = ["qkv_gemm", "attention", "out_proj_ln_gemm", "ffn1_gemm", "ffn2_ln_gemm"]
KERNEL_NAMES_FFN2_LN = ["qkv_gemm", "attention", "out_proj_gemm", "ln1", "ffn1_gemm", "ffn2_ln_gemm"]
# Six kernels per layer with the output projection fused and FFN2 not: only
# when the options ask for it (ln_fuse_out_proj=2, ln_fuse_ffn2=0).
KERNEL_NAMES_OPROJ_LN = ["qkv_gemm", "attention", "out_proj_ln_gemm", "ffn1_gemm", "ffn2_gemm", "ln2"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_workload(spec: str) -> EI.Workload:
    parts = spec.split(":")
    kind, batch = parts[0], int(parts[1])
    seq = int(parts[2]) if len(parts) > 2 else None
    return EI.named_workload(kind, batch, seq)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# Sources each timed kernel is built from: a DRAM-traffic figure measured by
# ncu holds only while these files are unchanged.
KERNEL_SOURCES = {
    "qkv_gemm": ["gemm_tc.cu", "gelu.cuh", "sm100.cuh", "internal.h"],
    "out_proj_gemm": ["gemm_tc.cu", "gelu.cuh", "sm100.cuh", "internal.h"],
    "ffn1_gemm": ["gemm_tc.cu", "gelu.cuh", "sm100.cuh", "internal.h"],
    "ffn2_gemm": ["gemm_tc.cu", "gelu.cuh", "sm100.cuh", "internal.h"],
    "out_proj_ln_gemm": ["gemm_tc.cu", "gelu.cuh", "sm100.cuh", "internal.h"],
    "ffn2_ln_gemm": ["gemm_tc.cu", "gelu.cuh", "sm100.cuh", "internal.h"],
    "attention": ["attention.cu", "attention_tc.cu", "sm100.cuh", "internal.h"],
    "ln1": ["layernorm.cu", "internal.h"],
    "ln2": ["layernorm.cu", "internal.h"],
    "persistent": ["persistent.cu", "gelu.cuh", "sm100.cuh", "internal.h"],
}


def source_digest(kernel: str) -> str:
    """First 16 hex digits of the SHA-256 of the kernel's source files."""
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, []):
        with open(os.path.join(ROOT, "transformer_encoder_bert_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum) of
    `kernel` on `workload` from profiles/traffic.md, or None when there is no
    capture or the kernel's sources have changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(path) or kernel not in KERNEL_SOURCES:
        return None
    digest = source_digest(kernel)
    with open(path) as f:
        for line in f:
            cells = [c.strip().strip("`") for c in line.strip().strip("|").split("|")]
            if len(cells) >= 4 and cells[0] == kernel and cells[1] == workload and cells[3] == digest:
                try:
                    return float(cells[2].replace(",", ""))
                except ValueError:
                    return None
    return None


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------------ algorithmic work per kernel
def kernel_work(wl: EI.Workload, attn_seq=None, attn_tokens=None):
    """Per launch: (flops, algorithmic HBM bytes) of each kernel of one layer (FP16 storage).
    Attention flops are 4*S*H per token over the padded length (dense mode) or per
    valid token (attn_seq, attn_tokens for the packed mode, an upper bound)."""
    sh = wl.shape
    H, F, M, S = sh.hidden, sh.ffn_dim, wl.tokens, wl.seq
    if attn_seq is not None:
        S = attn_seq
    es = 2 if wl.dtype == "fp16" else 4
    def gemm(n, k, extra_out=0):
        return 2.0 * M * n * k, es * (M * k + k * n + M * n) + extra_out
    L = sh.num_layers
    weight_bytes = es * L * (3 * H * H + H * H + 2 * H * F)
    return {
        # the whole stack in one launch: every GEMM and attention flop; bytes =
        # every weight once plus the input and output rows (the activations in
        # between stay in L2 at these sizes)
        "persistent": (L * (2.0 * M * H * (4 * H + 2 * F) + 4.0 * M * S * H),
                       weight_bytes + es * 2.0 * M * H + 4 * wl.batch),
        "qkv_gemm": gemm(3 * H, H),
        "attention": (4.0 * M * S * H, es * 4.0 * M * H + 4 * wl.batch),
        "out_proj_gemm": gemm(H, H, extra_out=es * M * H),     # epilogue reads the residual
        "ln1": (0.0, es * 2.0 * M * H),                       # z in, normalised row out
        "ffn1_gemm": gemm(F, H),
        "ffn2_gemm": gemm(H, F, extra_out=es * M * H),
        "ln2": (0.0, es * 2.0 * M * H),
        "out_proj_ln_gemm": gemm(H, H, extra_out=es * M * H),  # + residual read, normalised rows written
        "ffn2_ln_gemm": gemm(H, F, extra_out=es * M * H),
    }


# ------------------------------------------------------------------ clocks during the timed region
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        self.index = vis.split(",")[local_rank] if vis else str(local_rank)
        self.proc = None
        # The raw samples go to BENCH_CLOCKS_DIR (default: the temp directory); the
        # JSON line carries their summary.
        out_dir = os.environ.get("BENCH_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"bench_clocks_rank{local_rank}_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.index, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                p = [v.strip() for v in line.split(",")]
                if len(p) < 9:
                    continue
                try:
                    sm.append(float(p[1]))
                    mx.append(float(p[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, p[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------ CPU oracle
def oracle_rate(inp: EI.EncoderInputs, budget_s: float, chunk: int = 4, max_seqs=None, widened=None):
    """Sequences/s of the float64 oracle on sequences 0, 1, ... until budget_s elapses
    (the inputs are widened to float64 before the clock starts)."""
    from oracle import encoder_oracle as O
    wl = inp.workload
    sh = wl.shape
    x64, vl, layers = widened if widened is not None else inp.as_float64()
    done, t0 = 0, time.perf_counter()
    limit = wl.batch if max_seqs is None else min(wl.batch, max_seqs)
    while done < limit:
        idx = list(range(done, min(done + chunk, limit)))
        O.encoder_forward(x64, vl, layers, sh.head_num, sh.size_per_head, seqs=idx)
        done += len(idx)
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return done / dt, done, dt


def run_reference(args, wl: EI.Workload, rank: int, world: int):
    if rank != 0:
        return 0
    inp = EI.make_inputs(wl)
    sample = max(1, args.ref_sample)
    widened = inp.as_float64()
    times = []
    for i in range(args.warmup + args.steps):
        _, n, dt = oracle_rate(inp, budget_s=1e9, chunk=sample, max_seqs=sample, widened=widened)
        if i >= args.warmup:
            times.append(dt)
    step_s = sum(times) / len(times)
    value = sample / step_s
    cores = blas_threads()
    desc = f"float64 numpy oracle, first {sample} sequences of the workload per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, world, l2="n/a (CPU)"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ replicas (N > 1)
def replica_workload(wl: EI.Workload, rank: int) -> EI.Workload:
    """Each rank runs its own batch of the same workload (weak scaling): seed + rank."""
    return wl.with_(seed=wl.seed + rank)


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks of the default process
    group (identity without one).  The job's time is its slowest rank's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_throughput(batch_per_rank: int, world: int, ms_per_step: float) -> float:
    """Sequences per second of the whole job: every rank's batch in the slowest rank's time."""
    return batch_per_rank * world / (ms_per_step * 1e-3)


def workload_config(wl: EI.Workload, world: int, l2: str):
    sh = wl.shape
    return {"workload": wl.name, "batch_per_gpu": wl.batch, "global_batch": wl.batch * world,
            "seq_len": wl.seq, "layers": sh.num_layers, "heads": sh.head_num, "size_per_head": sh.size_per_head,
            "ffn": sh.ffn_dim, "valid_len": f"U[{wl.valid_lo},{wl.valid_hi}]", "storage": wl.dtype,
            "accumulate": "fp32", "parallelism": f"replicas x{world} (batch-sharded, no collective)",
            "l2": l2, "seed": wl.seed}


# ------------------------------------------------------------------ our arm
def kernel_names(nk: int, num_layers: int, packed: bool, ffn2_ln_off: bool = False):
    """Names of the nk kernels of one forward, in launch order (`ffn2_ln_off`:
    the options turned the FFN2 LayerNorm fusion off)."""
    if nk == 1:
        return ["persistent"]                 # the single-launch forward of the whole stack
    per_layer = (nk - (3 if packed else 0)) // num_layers
    six = KERNEL_NAMES_OPROJ_LN if ffn2_ln_off else KERNEL_NAMES_FFN2_LN
    layer_names = {5: KERNEL_NAMES_FUSED, 6: six}.get(per_layer, KERNEL_NAMES)
    if packed:
        return ["offsets", "pack"] + layer_names * num_layers + ["unpack"]
    return layer_names * num_layers


def time_forward(enc, x, vl, out, wl, args, flush, stream, barrier):
    """Device time of args.steps forwards (graph replays by default) after
    args.warmup untimed ones, the L2 flushed before each; then the per-kernel
    breakdown from as many traced enc_forward calls (CUDA events recorded by the
    library between its kernels on the launching stream).  The events break the
    programmatic-dependent-launch overlap between kernels, so each traced kernel
    time is an upper bound on its time inside the timed graph."""
    import torch
    graph = enc.record(x, vl, out) if args.graph else None
    step = (lambda: graph.launch()) if graph is not None else (lambda: enc.forward(x, vl, out))
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    nk = enc.kernels_per_forward(wl.batch, wl.seq)
    ev_sets = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(args.steps)]
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for evs in ev_sets:                                   # create the events before the timed region
        for e in evs:
            e.record()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    launches0 = enc.launch_count()
    for i in range(args.steps):
        flush.zero_()
        if graph is None:
            enc.set_trace_events(ev_sets[i], prepare=False)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    barrier()
    launches = enc.launch_count() - launches0
    if graph is not None:
        for i in range(args.steps):
            flush.zero_()
            enc.set_trace_events(ev_sets[i], prepare=False)
            enc.forward(x, vl, out)
        torch.cuda.synchronize()
        graph.close()
    enc.set_trace_events(None)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ffn2_ln_off = any(o.replace(" ", "") in ("ln_fuse_ffn2=0", "ln_fuse_ffn2=False") for o in args.option)
    names = kernel_names(nk, wl.shape.num_layers, args.packed, ffn2_ln_off)
    per_kernel = {k: [] for k in names}
    traced = []
    for evs in ev_sets:
        for j in range(nk):
            per_kernel[names[j]].append(evs[j].elapsed_time(evs[j + 1]))
        traced.append(evs[0].elapsed_time(evs[nk]))
    return {"ms": sum(step_ms) / len(step_ms), "per_kernel": per_kernel, "launches": launches,
            "traced_ms": sum(traced) / len(traced), "nk": nk, "step_ms": step_ms}


def step_stats(step_ms, device=None):
    """Median, 10th and 90th percentile of the per-step device times (ms), each
    the max over ranks."""
    q = sorted(step_ms)

    def pct(p):
        i = p / 100.0 * (len(q) - 1)
        lo = int(math.floor(i))
        hi = min(lo + 1, len(q) - 1)
        return q[lo] + (q[hi] - q[lo]) * (i - lo)

    med, p10, p90 = max_over_ranks([pct(50), pct(10), pct(90)], device=device)
    return {"median": med, "p10": p10, "p90": p90}


def kernel_table(wl, inp, per_kernel, peaks, packed: bool, graph_ms=None, forwards=None):
    """Per kernel: average traced time, share, TFLOP/s (GEMMs) and algorithmic GB/s,
    each with its fraction of the measured peak (burst tensor peak: the kernels run
    for microseconds inside steps of milliseconds).  With graph_ms (the timed
    graph's step) and the number of traced forwards, the rates come from the
    kernel's in-graph time, estimated as its share of the traced forward times
    graph_ms per launch (graph_us); avg_us, the traced per-launch time, is an
    upper bound (events between kernels break the overlap of programmatic
    dependent launch)."""
    sh = wl.shape
    work = kernel_work(wl)
    if packed:
        # valid tokens only: the algorithmic work of the packed path
        t_valid = int(np.clip(inp.valid_len, 0, wl.seq).sum())
        work = kernel_work(wl.with_(batch=1, seq=t_valid), attn_seq=wl.seq, attn_tokens=t_valid)
        work.update({"offsets": (0.0, 8.0 * wl.batch), "pack": (0.0, 4.0 * t_valid * sh.hidden),
                     "unpack": (0.0, 4.0 * t_valid * sh.hidden)})
    tc_peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    hbm_peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    kernels = {}
    total = sum(sum(v) for v in per_kernel.values())
    for k, vals in per_kernel.items():
        share = sum(vals) / total
        avg_ms = sum(vals) / len(vals)
        entry = {"avg_us": avg_ms * 1e3, "share": share}
        if graph_ms is not None and forwards:
            launches_per_step = len(vals) / forwards
            avg_ms = share * graph_ms / launches_per_step
            entry["graph_us"] = avg_ms * 1e3
        flops, nbytes = work[k]
        if flops and (k.endswith("gemm") or k == "persistent"):
            entry["tflops"] = flops / (avg_ms * 1e-3) / 1e12
            entry["tensor_frac"] = entry["tflops"] / tc_peak
        entry["gbs"] = nbytes / (avg_ms * 1e-3) / 1e9
        if not k.endswith("gemm"):
            entry["hbm_frac"] = entry["gbs"] / hbm_peak
        kernels[k] = entry
    return kernels, work


def roofline_of(kernels, work, dominant, peaks, peak_src, traffic):
    d = kernels[dominant]
    in_graph = "graph_us" in d
    time_source = ("the kernel's share of the traced forward times the timed graph's step, per launch (the traced "
                   "per-launch time, an upper bound, is avg_us)" if in_graph else
                   "traced enc_forward calls (events between kernels): an upper bound on the kernel's time in "
                   "the timed graph, so achieved is a lower bound")
    if dominant == "persistent":
        # small batch: every weight byte is read once per forward, so HBM bounds it
        peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        return {"bound": "hbm", "achieved": d["gbs"], "peak": peak, "unit": "GB/s", "frac": d["gbs"] / peak,
                "traffic": traffic, "kernel": dominant, "per_launch_bytes": work[dominant][1],
                "peak_source": f"{peak_src} HBM copy bandwidth",
                "time_source": "the whole forward is this one launch (CUDA events around it)"}
    if dominant.endswith("gemm"):
        peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        return {"bound": "tensor", "achieved": d["tflops"], "peak": peak, "unit": "TFLOP/s",
                "frac": d["tflops"] / peak, "traffic": traffic,
                "kernel": dominant, "per_launch_flops": work[dominant][0],
                "peak_source": f"{peak_src} burst bf16 matmul (FP16 dense rate = BF16 dense rate); "
                               "the kernel runs for microseconds inside millisecond steps",
                "time_source": time_source}
    peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    return {"bound": "hbm", "achieved": d["gbs"], "peak": peak, "unit": "GB/s", "frac": d["gbs"] / peak,
            "traffic": traffic, "kernel": dominant, "per_launch_bytes": work[dominant][1],
            "peak_source": f"{peak_src} HBM copy bandwidth",
            "time_source": time_source}


def run_ours(args, wl: EI.Workload, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist
    from transformer_encoder_bert_b200 import Encoder

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = replica_workload(wl, rank)             # each replica has its own batch
    inp = EI.make_inputs(wl)
    sh = wl.shape
    enc = Encoder(sh.head_num, sh.size_per_head, sh.ffn_dim, inp.layers, wl.dtype)
    if args.packed:
        enc.set_packing(True)
    options = dict(o.split("=", 1) for o in args.option)
    for name, v in options.items():
        enc.set_option(name, int(v))
    enc.reserve(wl.batch, wl.seq)
    x = torch.from_numpy(inp.x).to(dev)
    vl = torch.from_numpy(inp.valid_len).to(dev)
    out = torch.empty_like(x)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    main_t = time_forward(enc, x, vl, out, wl, args, flush, stream, barrier)
    ms = main_t["ms"]

    # e2e through the pipelined host entry point (enc_forward_host_async): every
    # step copies its input from pinned host memory and its output back to host
    # memory inside the timed region; consecutive steps overlap their copies with
    # the encoder.  Timed over all steps, from before the first input copy to
    # after the last output copy (enc_host_join).
    hx = torch.from_numpy(inp.x).pin_memory()
    hvl = torch.from_numpy(inp.valid_len).pin_memory()
    hout = torch.empty_like(hx).pin_memory()
    for _ in range(2):
        enc.forward_host_ptr(hx.data_ptr(), hvl.data_ptr(), hout.data_ptr(), wl.batch, wl.seq)
    barrier()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for i in range(args.steps):
        flush.zero_()
        enc.forward_host_async_ptr(hx.data_ptr(), hvl.data_ptr(), hout.data_ptr(), wl.batch, wl.seq)
    enc.host_join()
    e.record(stream)
    e.synchronize()
    barrier()
    e2e_step = s.elapsed_time(e) / args.steps
    status = enc.device_status()
    enc.close()

    # The goal point (BERT-Base, seq 128, batch 256) in the same run, device-timed
    # the same way, when it is not already the main workload (one GPU only).
    secondary = None
    sec_wl = parse_workload(args.secondary) if args.secondary else None
    if world == 1 and sec_wl is not None and sec_wl.name != wl.name:
        sec_inp = EI.make_inputs(sec_wl)
        ssh = sec_wl.shape
        enc2 = Encoder(ssh.head_num, ssh.size_per_head, ssh.ffn_dim, sec_inp.layers, sec_wl.dtype)
        if args.packed:
            enc2.set_packing(True)
        for name, v in options.items():
            enc2.set_option(name, int(v))
        enc2.reserve(sec_wl.batch, sec_wl.seq)
        x2 = torch.from_numpy(sec_inp.x).to(dev)
        vl2 = torch.from_numpy(sec_inp.valid_len).to(dev)
        out2 = torch.empty_like(x2)
        sec_t = time_forward(enc2, x2, vl2, out2, sec_wl, args, flush, stream, barrier)
        sec_status = enc2.device_status()
        enc2.close()
        secondary = {"workload": sec_wl.name, "sec_t": sec_t, "inp": sec_inp, "wl": sec_wl, "status": sec_status}
    clk = clocks.stop()

    ms, e2e_step = max_over_ranks([ms, e2e_step], device=dev)
    main_stats = step_stats(main_t["step_ms"], device=dev)
    if rank != 0:
        return 0

    peaks, peak_src = load_peaks()
    kernels, work = kernel_table(wl, inp, main_t["per_kernel"], peaks, args.packed,
                                 graph_ms=ms if args.graph else None, forwards=args.steps)
    dominant = max(kernels, key=lambda k: kernels[k]["share"])
    traffic = args.traffic if args.traffic is not None else measured_traffic(dominant, wl.name)
    roof = roofline_of(kernels, work, dominant, peaks, peak_src, traffic)

    value = job_throughput(wl.batch, world, ms)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "step_ms": main_stats, "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None, "dtype": "fp16" if wl.dtype == "fp16" else "fp32", "data": "synthetic",
        "config": dict(workload_config(wl, world, l2="flushed before every timed step (256 MiB write)"),
                       launch="one recorded CUDA graph per step" if args.graph else "enc_forward per step",
                       padding="removed (valid tokens only; padded outputs zero)" if args.packed
                       else "computed (fixed length)",
                       **({"options": options} if options else {})),
        "roofline": roof,
        "e2e": {"value": job_throughput(wl.batch, world, e2e_step), "unit": UNIT,
                "h2d_bytes_per_step": int(hx.numel() * hx.element_size() + hvl.numel() * 4),
                "d2h_bytes_per_step": int(hout.numel() * hout.element_size())},
        "gpu_launches": int(main_t["launches"]),
        "clocks": clk,
        "traced_ms_per_forward": main_t["traced_ms"],
        "kernels": kernels,
        "device_status": status,
    }
    if secondary is not None:
        sw, st = secondary["wl"], secondary["sec_t"]
        skern, swork = kernel_table(sw, secondary["inp"], st["per_kernel"], peaks, args.packed,
                                    graph_ms=st["ms"] if args.graph else None, forwards=args.steps)
        sdom = max(skern, key=lambda k: skern[k]["share"])
        gemms = [k for k in skern if k.endswith("gemm")]
        g_flops = sum(swork[k][0] * len(st["per_kernel"][k]) for k in gemms) / args.steps
        g_ms = sum(skern[k].get("graph_us", skern[k]["avg_us"]) * 1e-3 * len(st["per_kernel"][k]) for k in gemms) \
            / args.steps
        tc_peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        line["secondary"] = {
            "workload": sw.name, "value": sw.batch / (st["ms"] * 1e-3), "unit": UNIT, "ms_per_step": st["ms"],
            "step_ms": step_stats(st["step_ms"]),
            "traced_ms_per_forward": st["traced_ms"], "gpu_launches": int(st["launches"]),
            "roofline": roofline_of(skern, swork, sdom, peaks, peak_src,
                                    measured_traffic(sdom, sw.name)),
            "gemms_aggregate": {"tflops": g_flops / (g_ms * 1e-3) / 1e12,
                                "tensor_frac": g_flops / (g_ms * 1e-3) / 1e12 / tc_peak},
            "kernels": skern, "device_status": secondary["status"],
        }
    if world == 1 and not args.no_cpu_baseline:
        rate, n, dt = oracle_rate(inp, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                                "sample": f"first {n} of the {wl.batch} sequences of this workload, "
                                          f"float64 numpy oracle, {dt:.1f} s"}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ decoder leg
def decoder_workload(spec: str) -> "EI.DecoderWorkload":
    """decoder-base:B:T:S (BERT-Base structure, 12 layers) or decoder-large:B:T:S
    (BERT-Large structure, 24 layers): target lengths U[T/2, T], memory lengths U[S/2, S]."""
    kind, b, t, sm = spec.split(":")
    shape = {"decoder-base": EI.BERT_BASE, "decoder-large": EI.BERT_LARGE}[kind]
    b, t, sm = int(b), int(t), int(sm)
    return EI.DecoderWorkload(f"{kind}-{shape.num_layers}L-h{shape.hidden}-t{t}-s{sm}-b{b}-fp16", shape, b, t, sm,
                              "fp16", t // 2, t, sm // 2, sm)


def decoder_flops(wl) -> float:
    """GEMM and attention flops of one decoder forward over the padded lengths."""
    sh = wl.shape
    H, F, L = sh.hidden, sh.ffn_dim, sh.num_layers
    mt, ms = wl.batch * wl.tgt_seq, wl.batch * wl.mem_seq
    gemm = 2.0 * mt * H * (3 * H + H + H + H + 2 * F) + 2.0 * ms * H * 2 * H
    attn = 4.0 * mt * wl.tgt_seq * H / 2 + 4.0 * mt * wl.mem_seq * H      # causal half + cross
    return L * (gemm + attn)


def run_decoder(args, rank: int, world: int, local_rank: int):
    """Device time of the decoder stack (enc_decoder_forward per step, L2 flushed
    before each); the roofline is the whole forward's flops at the burst peak."""
    import torch
    from transformer_encoder_bert_b200 import Decoder
    torch.cuda.set_device(local_rank)
    wl = decoder_workload(args.workload).with_(seed=rank)
    inp = EI.make_decoder_inputs(wl)
    sh = wl.shape
    dec = Decoder(sh.head_num, sh.size_per_head, sh.ffn_dim, inp.layers)
    options = dict(o.split("=", 1) for o in args.option)
    for name, v in options.items():
        dec.set_option(name, int(v))
    dev = torch.device("cuda", local_rank)
    y, mem = torch.from_numpy(inp.y).to(dev), torch.from_numpy(inp.mem).to(dev)
    tl, ml = torch.from_numpy(inp.tgt_len).to(dev), torch.from_numpy(inp.mem_len).to(dev)
    out = torch.empty_like(y)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        dec.forward(y, tl, mem, ml, out)
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    ts = []
    launches0 = dec.launch_count()
    for _ in range(args.steps):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        dec.forward(y, tl, mem, ml, out)
        e.record()
        e.synchronize()
        ts.append(s.elapsed_time(e))
    launches = dec.launch_count() - launches0
    # e2e: each step copies its inputs from pinned host memory, runs the
    # decoder and copies the output back to pinned host memory.
    hy, hmem = torch.from_numpy(inp.y).pin_memory(), torch.from_numpy(inp.mem).pin_memory()
    htl, hml = torch.from_numpy(inp.tgt_len).pin_memory(), torch.from_numpy(inp.mem_len).pin_memory()
    hout = torch.empty_like(hy).pin_memory()
    e2e_ts = []
    for _ in range(args.steps):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        y.copy_(hy, non_blocking=True)
        mem.copy_(hmem, non_blocking=True)
        tl.copy_(htl, non_blocking=True)
        ml.copy_(hml, non_blocking=True)
        dec.forward(y, tl, mem, ml, out)
        hout.copy_(out, non_blocking=True)
        e.record()
        e.synchronize()
        e2e_ts.append(s.elapsed_time(e))
    clk = clocks.stop()
    status = dec.device_status()
    ms, e2e_ms = max_over_ranks([sum(ts) / len(ts), sum(e2e_ts) / len(e2e_ts)], device=dev)
    stats = step_stats(ts, device=dev)
    if rank != 0:
        return 0
    h2d = sum(t.numel() * t.element_size() for t in (hy, hmem, htl, hml))
    peaks, peak_src = load_peaks()
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    tf = decoder_flops(wl) / (ms * 1e-3) / 1e12
    line = {"metric": "decoder fwd sequences/s", "value": job_throughput(wl.batch, world, ms), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "step_ms": stats,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp16", "data": "synthetic",
            "config": {"workload": wl.name, "batch_per_gpu": wl.batch, "tgt_seq": wl.tgt_seq, "mem_seq": wl.mem_seq,
                       "layers": sh.num_layers, "l2": "flushed before every timed step (256 MiB write)",
                       "launch": "enc_decoder_forward per step (9 to 12 launches per layer)",
                       **({"options": options} if options else {})},
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                         "traffic": None, "kernel": "whole decoder forward",
                         "peak_source": f"{peak_src} burst bf16 matmul"},
            "e2e": {"value": job_throughput(wl.batch, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": hout.numel() * hout.element_size()},
            "gpu_launches": int(launches), "clocks": clk,
            "device_status": status}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--packed", action="store_true",
                    help="padding removal (enc_set_packing): compute the valid tokens only")
    ap.add_argument("--graph", dest="graph", action="store_true", default=True,
                    help="time replays of a recorded forward (enc_graph_launch); the default")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="time enc_forward calls instead of graph replays")
    ap.add_argument("--secondary", default=SECONDARY_WORKLOAD,
                    help="a second workload device-timed in the same run (one GPU; '' for none)")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-sample", type=int, default=8, help="sequences per reference-arm step")
    ap.add_argument("--option", action="append", default=[], metavar="NAME=VALUE",
                    help="a kernel-path switch of the handle (enc_set_option), e.g. persistent=0")
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu DRAM bytes per launch of the dominant kernel, if captured for the current sources")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE", file=sys.stderr)
    if args.workload.startswith("decoder-"):
        if args.impl == "reference" or world > 1:
            ap.error("the decoder leg runs our implementation on one GPU")
        return run_decoder(args, rank, world, local_rank)
    wl = parse_workload(args.workload)

    if args.impl == "reference":
        return run_reference(args, wl, rank, world)

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_ours(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
