#!/usr/bin/env python
"""Benchmark of the top-k routed MoE FFN forward on B200 (one JSON line on rank 0).

A step is one moe_forward (route -> sort -> gather -> gate_up GEMM -> down GEMM
-> combine) over one batch of T seeded synthetic tokens.  Default workload: the
Mixtral-shaped bf16 prefill layer (T=4096, d=4096, F=14336, E=8, k=2).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl own|reference]

Timing: W warm-up steps, then K steps timed on the device with one CUDA event
pair per step on the launching stream, each step a replay of a CUDA graph of
the moe_forward call (--no-graph: eager calls); the L2 is flushed (a 512 MiB
buffer written, then read back) before every timed step, outside the events.  A second pass of K steps
has the library record an event at every stage boundary (inside the replayed
graph, so without host launch gaps); it gives the per-kernel times behind the
roofline figure.
Under torchrun each rank runs an independent replica (no collective on the data
path); the reported time is the max over ranks and `value` counts the tokens of
all ranks.  `e2e` repeats the measurement through the same C-ABI call with each
step's x and logits copied from pinned host memory and its y copied back inside the
timed region, the copies on two copy streams overlapping the neighbouring steps'
forwards (two device buffer sets); `e2e.serial_value` is the same with copy in,
forward and copy out one after another on one stream.  `--impl reference` times the CPU oracle on the host cores
instead (the only other place this script runs it).
"""
from __future__ import annotations

import argparse
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s; achieved TFLOP/s or HBM GB/s as % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_NOTE = "flushed before every timed step: a 512 MiB buffer written, then read back"


class L2Flush:
    """Evicts the inputs from the 126 MB L2 before a timed step: writes a 512 MiB buffer,
    then reads it back, so that the L2 holds only clean lines of that buffer (a write
    alone would leave ~126 MB of dirty lines, whose write-back the timed step would pay
    for: 13 us of a 82 us decode step)."""

    def __init__(self, torch):
        self.buf = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
        self.acc = torch.empty((), dtype=torch.int64, device="cuda")
        self.torch = torch

    def __call__(self):
        self.buf.zero_()
        self.torch.sum(self.buf.view(self.torch.int64), 0, out=self.acc)


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of a workload's
# dominant GEMM, each from one ncu capture of that kernel, with the kernel's source file and
# the hash of the code of that file and the headers it includes (kernel_sources_hash,
# comments stripped) at capture time.
# A figure whose hash is not the current sources' belongs to an older kernel: reported null.
#   mixtral_bf16 gate_up: full-size capture (2.4584 GB read + 0.2333 GB written; other
#     boxes read up to 2.84 GB: how many repeated weight-tile fetches hit L2 varies).
#   deepseek_bf16 gate_up: captured at E=32 T=1024 (same 256 routed rows per expert and one
#     shared row per token, one eighth of every operand) and scaled by 8: 2.1469 GB read +
#     0.0359 GB written per launch there.
#   gptoss_mxfp4 gate_up: full-size capture, 0.3297 GB read + 0.0375 GB written.
#   decode_T1 / decode_T8: the one launch of both GEMMs, full size (the fourth launch of
#     that kernel): 0.3041 GB + 1.4 MB and 0.9444 GB + 1.2 MB.
NCU_TRAFFIC = {
    ("mixtral_bf16", "gate_up"): (2458378496 + 233282048, "gemm_tcs.cu", "c30a86d32a81"),
    ("deepseek_bf16", "gate_up"): (8 * (2146914048 + 35875072), "gemm_tcs.cu", "c30a86d32a81"),
    ("gptoss_mxfp4", "gate_up"): (329699840 + 37458432, "gemm_fp4.cu", "af0ca3377e18"),
    ("decode_T1", "gate_up"): (304128768 + 1417728, "gemm_tc.cu", "f397cb915a5e"),
    ("decode_T8", "gate_up"): (944408832 + 1224192, "gemm_tc.cu", "f397cb915a5e"),
}


def _code_of(text: bytes) -> bytes:
    """A source file's code without its comments and blank-line differences, so that
    editing a comment leaves the hash of the code unchanged."""
    t = re.sub(rb"/\*.*?\*/", b" ", text, flags=re.S)
    t = re.sub(rb"//[^\n]*", b"", t)
    return b"\n".join(line.rstrip() for line in t.splitlines() if line.strip())


def kernel_sources_hash(kernel_file: str = None) -> str:
    """Short hash of the code (comments stripped) of one kernel source file of the
    library and every local header it includes (transitively, plus include/moe.h);
    without a file, of all of csrc/."""
    import hashlib
    csrc = os.path.join(ROOT, "mixture_experts_ffn_10_b200", "csrc")
    if kernel_file is None:
        files = sorted(f for f in os.listdir(csrc) if f.endswith((".cu", ".cuh")))
    else:
        files, todo = [], [kernel_file]
        while todo:
            f = todo.pop()
            if f in files or not os.path.exists(os.path.join(csrc, f)):
                continue
            files.append(f)
            with open(os.path.join(csrc, f)) as fh:
                todo += re.findall(r'^#include "([^"]+)"', fh.read(), flags=re.M)
        files.sort()
    h = hashlib.sha256()
    for f in [os.path.join(csrc, f) for f in files] + [os.path.join(ROOT, "include", "moe.h")]:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(_code_of(fh.read()))
    return h.hexdigest()[:12]


def ncu_traffic(workload: str, stage: str):
    """ncu DRAM bytes per launch for this workload's stage, or None if not captured for the
    current sources of the kernel that ran it."""
    rec = NCU_TRAFFIC.get((workload, stage))
    if rec is None or rec[2] != kernel_sources_hash(rec[1]):
        return None
    return rec[0]


KERNEL_CHOICE_VARS = ("MOE_B200_PAIR_GEMM", "MOE_B200_SWAP_GEMM", "MOE_B200_FUSED_FFN", "MOE_B200_PAIR_FP4",
                      "MOE_B200_INTERLEAVE", "MOE_B200_GEMV")


def default_kernels() -> bool:
    """True when no environment variable overrides the library's choice of kernels."""
    return not any(os.environ.get(v) for v in KERNEL_CHOICE_VARS)


def traffic_kernel_sources(workload: str, stage: str):
    """(kernel file, current hash) of the kernel a traffic figure belongs to, or None."""
    rec = NCU_TRAFFIC.get((workload, stage))
    return None if rec is None else {"file": rec[1], "hash": kernel_sources_hash(rec[1])}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def max_over_ranks(v: float, dist=None, device="cpu") -> float:
    """The max of a per-rank value over all ranks (identity without a process group)."""
    if dist is None:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_throughput(world: int, tokens_per_rank: int, steps: int, max_ms: float) -> float:
    """Tokens/s of the whole job: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (max_ms / 1e3)


def workload_name(cfg):
    s = f"{cfg.name}: T={cfg.T} d={cfg.d} F={cfg.F} E={cfg.E} k={cfg.k}"
    if cfg.Fs:
        s += f" Fs={cfg.Fs}"
    return s + f" {cfg.act_dtype}/{cfg.w_dtype} {cfg.score}"


def config_dict(cfg, extra=None):
    d = {"workload": workload_name(cfg), "T": cfg.T, "d": cfg.d, "F": cfg.F, "E": cfg.E, "k": cfg.k,
         "Fs": cfg.Fs, "global_batch": cfg.T, "parallelism": "replicas",
         "l2": L2_NOTE}
    if extra:
        d.update(extra)
    return d


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, phys_index):
        self.idx = str(phys_index)
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "50"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        self.p.wait()
        self.f.seek(0)
        rows = [r.split(", ") for r in self.f.read().splitlines() if r.strip()]
        os.unlink(self.f.name)
        rows = [r for r in rows if len(r) >= 9 and r[0].strip() == self.idx]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = max(float(r[2]) for r in rows)
        loaded = [r for r in rows if float(r[3]) > 300.0] or rows  # power draw marks load
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in loaded for n, v in zip(names, r[5:9]) if v.strip() == "Active"})
        sm_loaded = [float(r[1]) for r in loaded]
        return {"sm_mhz": statistics.median(sm_loaded) if sm_loaded else None, "sm_max_mhz": mx,
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded),
                "sm_mhz_min": min(sm) if sm else None}


def physical_gpu_index(local):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",")]
        if local < len(ids) and ids[local].isdigit():
            return int(ids[local])
    return local


# ---------------------------------------------------------------------------- oracle arm
def oracle_sample(cfg, inputs_host, budget_s=15.0, max_tokens=None):
    """Time the oracle on a bounded sample of tokens; returns (tokens/s, n, seconds, threads)."""
    import numpy as np

    import oracle
    oracle.build()
    p = oracle.Problem(cfg, inputs_host)
    threads = oracle.max_threads()
    t0 = time.perf_counter()
    p.forward(np.array([0], dtype=np.int64), nthreads=1)
    t1 = max(time.perf_counter() - t0, 1e-4)
    n = int(max(threads, min(cfg.T, budget_s / t1 * threads)))
    n = min(n, cfg.T if max_tokens is None else max_tokens)
    toks = np.arange(n, dtype=np.int64) % cfg.T
    t0 = time.perf_counter()
    p.forward(toks, nthreads=threads)
    dt = time.perf_counter() - t0
    return n / dt, n, dt, threads


def host_inputs(inputs):
    return {k: (None if v is None else v.detach().cpu()) for k, v in inputs.items()}


def run_reference(args, cfg):
    import torch

    from workloads import make_inputs
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    hin = host_inputs(make_inputs(cfg, dev))
    import numpy as np

    import oracle
    oracle.build()
    p = oracle.Problem(cfg, hin)
    threads = oracle.max_threads()
    # size one step's sample to about a second of the host's cores
    t0 = time.perf_counter()
    p.forward(np.array([0], dtype=np.int64), nthreads=1)
    t1 = max(time.perf_counter() - t0, 1e-4)
    n = int(min(cfg.T, max(threads, 1.0 / t1 * threads)))
    toks = np.arange(n, dtype=np.int64)
    for _ in range(args.warmup):
        p.forward(toks, nthreads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        p.forward(toks, nthreads=threads)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    out = {"metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference",
           "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
           "config": config_dict(cfg, {"sample_tokens_per_step": n}),
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                            "sample": f"{n} of {cfg.T} tokens per step, whole layer per token"},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    return 0


# ---------------------------------------------------------------------------- own arm
def stage_model(cfg, distinct):
    """Algorithmic FLOPs and bytes per launch of each GEMM stage."""
    ab = 2 if cfg.act_dtype == "bf16" else 4
    R = cfg.T * cfg.k
    if cfg.w_dtype == "mxfp4":
        wbytes = lambda n: n / 2 + n / 32  # noqa: E731
    else:
        wbytes = lambda n: n * ab  # noqa: E731
    gu_w = distinct * wbytes(2 * cfg.F * cfg.d) + 2 * cfg.Fs * cfg.d * ab
    dn_w = distinct * wbytes(cfg.d * cfg.F) + cfg.d * cfg.Fs * ab
    return {
        "gate_up": {"flops": 2.0 * (R * cfg.d * 2 * cfg.F + cfg.T * cfg.d * 2 * cfg.Fs),
                    "bytes": gu_w + (R + (cfg.T if cfg.Fs else 0)) * (cfg.d + cfg.F) * ab},
        "down": {"flops": 2.0 * (R * cfg.d * cfg.F + cfg.T * cfg.d * cfg.Fs),
                 "bytes": dn_w + (R + (cfg.T if cfg.Fs else 0)) * (cfg.F + cfg.d) * ab},
    }


def fuse_stages(model):
    """The stage model when gate_up and down are one launch: the gate_up stage (events
    3 .. 4) then spans both GEMMs and the down stage is empty."""
    both = {k: model["gate_up"][k] + model["down"][k] for k in ("flops", "bytes")}
    return {"gate_up": both, "down": {"flops": 0.0, "bytes": 0.0}}


def stage_label(dom, fused):
    """fused: moe_forward_fused_gemms (2: the few-token kernel, 1: both GEMMs in one launch)."""
    if fused == 2:
        return "whole forward, one launch (few-token kernel)"
    return "gate_up + down grouped GEMMs (one launch)" if fused else f"{dom} grouped GEMM"


def measure_workload(cfg, steps, warmup, flush, stream):
    """Device-timed summary of one more workload (rank-local): CUDA-graph replays of
    moe_forward with the L2 flushed before each, then each GEMM stage alone between
    two library events (one graph per stage), and the roofline of the dominant one."""
    import torch

    import mixture_experts_ffn_10_b200 as moe
    from workloads import algorithmic_bytes, flops, make_inputs

    inputs = make_inputs(cfg, "cuda")
    shape, opts = moe.shape_of(cfg), moe.options_of(cfg)
    ws = moe.Workspace(moe.moe_workspace_size(shape, opts))
    y = torch.empty_like(inputs["x"])
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    tens = moe.tensors_of(inputs, y, idx, None)
    # the inputs are generated, and these buffers allocated, on the default stream, whose
    # kernels may still be writing memory the allocator handed out; the forwards run on
    # `stream`: let that work finish first
    torch.cuda.synchronize()
    sptr = stream.cuda_stream
    names = list(moe.STAGES)

    def call(handles=None):
        rc = (moe.moe_forward(shape, opts, tens, ws.ptr, ws.nbytes, sptr) if handles is None else
              moe.moe_forward_events(shape, opts, tens, ws.ptr, ws.nbytes, sptr, handles))
        if rc != 0:
            raise moe.MoeError(rc, moe.moe_last_error())

    def capture(handles=None):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            call(handles)
        torch.cuda.synchronize()
        return g

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            flush()
            call()
    torch.cuda.synchronize()
    graphs = [capture()]
    stage_ev = {}
    for st in ("gate_up", "down"):
        s_i = names.index(st)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        for ev in evs:
            ev.record(stream)
        h = [None] * moe.MOE_STAGE_EVENTS
        h[s_i], h[s_i + 1] = evs[0].cuda_event, evs[1].cuda_event
        stage_ev[st] = evs
        graphs.append(capture(h))
    t0s = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    t1s = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    stage_ms = {"gate_up": 0.0, "down": 0.0}
    with torch.cuda.stream(stream):
        for i in range(steps):
            flush()
            t0s[i].record(stream)
            graphs[0].replay()
            t1s[i].record(stream)
        for gi, st in ((1, "gate_up"), (2, "down")):
            for _ in range(steps):
                flush()
                graphs[gi].replay()
                torch.cuda.synchronize()
                stage_ms[st] += stage_ev[st][0].elapsed_time(stage_ev[st][1]) / steps
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in zip(t0s, t1s)) / steps
    status = moe.moe_debug_status(ws.ptr, sptr)
    if status != 0:
        raise RuntimeError(f"{cfg.name}: device status {moe.STATUS_NAMES.get(status, status)}")
    distinct = int(torch.unique(idx).numel())
    rows = torch.bincount(idx.flatten().long(), minlength=cfg.E)
    pk, pk_src = peaks()
    model = stage_model(cfg, distinct)
    fused = moe.moe_forward_fused_gemms(shape, opts)
    if fused:
        model = fuse_stages(model)
    dom = max(stage_ms, key=stage_ms.get)
    m, t_dom = model[dom], stage_ms[dom] / 1e3
    tensor = m["flops"] / pk["bf16_tflops"] / 1e12 >= m["bytes"] / pk["hbm_gbs"] / 1e9
    achieved = m["flops"] / t_dom / 1e12 if tensor else m["bytes"] / t_dom / 1e9
    peak = pk["bf16_tflops"] if tensor else pk["hbm_gbs"]
    lf, lb = flops(cfg), algorithmic_bytes(cfg, distinct)
    del graphs
    return {"workload": workload_name(cfg), "ms_per_step": ms, "tokens_per_s": cfg.T / (ms / 1e3),
            "stage_ms": stage_ms,
            "roofline": {"kernel": stage_label(dom, fused), "bound": "tensor" if tensor else "hbm",
                         "achieved": achieved, "unit": "TFLOP/s" if tensor else "GB/s", "peak": peak,
                         "frac": achieved / peak, "peak_source": f"{pk_src} (burst)",
                         "traffic": ncu_traffic(cfg.name, dom) if default_kernels() else None},
            "layer": {"tensor_frac": lf / (ms / 1e3) / 1e12 / pk["bf16_tflops"],
                      "hbm_frac": lb / (ms / 1e3) / 1e9 / pk["hbm_gbs"], "distinct_experts": distinct,
                      "rows_per_expert_max": int(rows.max()), "empty_experts": int((rows == 0).sum())},
            "gpu_launches_per_step": moe.moe_forward_kernel_count(shape, opts),
            "timed": f"{steps} CUDA-graph replays after {warmup} warm-up calls, L2 flushed before each"}


def run_own(args, cfg):
    import torch

    import mixture_experts_ffn_10_b200 as moe
    from workloads import algorithmic_bytes, flops, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))

    def barrier():
        if dist is not None:
            dist.barrier()

    stream = torch.cuda.Stream()
    inputs = make_inputs(cfg, "cuda")
    shape, opts = moe.shape_of(cfg), moe.options_of(cfg)
    ws = moe.Workspace(moe.moe_workspace_size(shape, opts))
    y = torch.empty_like(inputs["x"])
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    tens = moe.tensors_of(inputs, y, idx, None)
    flush = L2Flush(torch)
    # the inputs are generated, and these buffers allocated, on the default stream, whose
    # kernels may still be writing memory the allocator handed out (temporaries of the
    # input generation); the forwards run on `stream`: let that work finish first
    torch.cuda.synchronize()
    nev = moe.MOE_STAGE_EVENTS
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(args.steps)]
    for row in events:
        for ev in row:
            ev.record(stream)  # creates the underlying cudaEvent_t
    handles = [[ev.cuda_event for ev in row] for row in events]
    sptr = stream.cuda_stream

    def step(ev=None):
        if ev is None:
            rc = moe.moe_forward(shape, opts, tens, ws.ptr, ws.nbytes, sptr)
        else:
            rc = moe.moe_forward_events(shape, opts, tens, ws.ptr, ws.nbytes, sptr, ev)
        if rc != 0:
            raise moe.MoeError(rc, moe.moe_last_error())

    sampler = ClockSampler(physical_gpu_index(local))
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush()
            step()
    torch.cuda.synchronize()
    status = moe.moe_debug_status(ws.ptr, sptr)
    if status != 0:
        raise RuntimeError(f"device status {moe.STATUS_NAMES.get(status, status)}")

    # ------------------------------------------------------------ device-timed steps
    # Pass 1 (the reported time): one event pair per step around the forward,
    # replayed from a CUDA graph of the C-ABI call unless --no-graph.
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        torch.cuda.synchronize()
    t0s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    t1s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            flush()
            t0s[i].record(stream)
            if graph is not None:
                graph.replay()
            else:
                step()
            t1s[i].record(stream)
    torch.cuda.synchronize()
    barrier()
    total_ms = sum(a.elapsed_time(b) for a, b in zip(t0s, t1s))
    status = moe.moe_debug_status(ws.ptr, sptr)
    if status != 0:
        raise RuntimeError(f"device status {moe.STATUS_NAMES.get(status, status)}")

    # Pass 2 (per-kernel breakdown for the roofline): the library records an event at
    # every stage boundary on the launching stream.  The call with its events is
    # replayed from a CUDA graph as in pass 1 (the events become graph nodes), so the
    # stage times hold no host launch gaps; --no-graph records them on eager calls.
    stage_graph = None
    if graph is not None:
        stage_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(stage_graph, stream=stream):
            step(handles[0])
        torch.cuda.synchronize()
    stage_ms = [0.0] * (nev - 1)
    staged_ms = 0.0

    def add_row(row):
        nonlocal staged_ms
        staged_ms += row[0].elapsed_time(row[-1])
        for s in range(nev - 1):
            stage_ms[s] += row[s].elapsed_time(row[s + 1])

    with torch.cuda.stream(stream):
        for i in range(args.steps):
            flush()
            if stage_graph is not None:
                stage_graph.replay()
                torch.cuda.synchronize()
                add_row(events[0])
            else:
                step(handles[i])
    torch.cuda.synchronize()
    if stage_graph is None:
        for row in events:
            add_row(row)
    stage_ms = [v / args.steps for v in stage_ms]
    stage_launch = "cuda graph" if stage_graph is not None else "eager"

    # Pass 3 (the roofline's kernel time): the same call with only the two events
    # around the dominant GEMM stage (its GEMM launch), so
    # that no other event node adds to that stage's time.
    names = list(moe.STAGES)
    dom = max(("gate_up", "down"), key=lambda n: stage_ms[names.index(n)])
    s_dom = names.index(dom)  # the stage spans events[s_dom] .. events[s_dom + 1]
    dom_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for ev in dom_ev:
        ev.record(stream)
    dom_handles = [None] * nev
    dom_handles[s_dom], dom_handles[s_dom + 1] = dom_ev[0].cuda_event, dom_ev[1].cuda_event
    dom_graph = None
    if graph is not None:
        dom_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(dom_graph, stream=stream):
            step(dom_handles)
        torch.cuda.synchronize()
    dom_ms = 0.0
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            flush()
            if dom_graph is not None:
                dom_graph.replay()
            else:
                step(dom_handles)
            torch.cuda.synchronize()
            dom_ms += dom_ev[0].elapsed_time(dom_ev[1])
    dom_ms /= args.steps
    total_ms = max_over_ranks(total_ms, dist, "cuda")
    ms_per_step = total_ms / args.steps
    value = whole_job_throughput(world, cfg.T, args.steps, total_ms)

    # ------------------------------------------------------------ end to end (host buffers)
    # Every step copies its x and logits from pinned host memory and reads its y back.
    # Serial: copy in, forward, copy out, one stream.  Pipelined (the reported value):
    # two device buffer sets; a step's host-to-device copies run on one copy stream and
    # its read-back on another while the neighbouring steps compute, so that the copies
    # overlap the forwards as they would in a serving loop.
    x_h = inputs["x"].cpu().pin_memory()
    l_h = inputs["logits"].cpu().pin_memory()
    y_hs = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    x_d, l_d = inputs["x"], inputs["logits"]
    e2e_steps = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(e2e_steps):
            x_d.copy_(x_h, non_blocking=True)
            l_d.copy_(l_h, non_blocking=True)
            step()
            y_hs[0].copy_(y, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_serial_ms = max_over_ranks(e0.elapsed_time(e1), dist, "cuda")

    slots = [(x_d, l_d, y, tens)]
    xb, lb, yb = x_d.clone(), l_d.clone(), torch.empty_like(y)
    slots.append((xb, lb, yb, moe.tensors_of(dict(inputs, x=xb, logits=lb), yb, idx, None)))
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    p0.record(h2d)
    for i in range(e2e_steps):
        b = i % 2
        xs, ls, ys, ts = slots[b]
        with torch.cuda.stream(h2d):
            if i >= 2:
                h2d.wait_event(ev_done[b])  # step i-2 finished reading this slot's inputs
            xs.copy_(x_h, non_blocking=True)
            ls.copy_(l_h, non_blocking=True)
            ev_in[b].record(h2d)
        stream.wait_event(ev_in[b])
        if i >= 2:
            stream.wait_event(ev_out[b])  # step i-2's y was read back
        rc = moe.moe_forward(shape, opts, ts, ws.ptr, ws.nbytes, sptr)
        if rc != 0:
            raise moe.MoeError(rc, moe.moe_last_error())
        ev_done[b].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(ev_done[b])
            y_hs[b].copy_(ys, non_blocking=True)
            ev_out[b].record(d2h)
    p1.record(d2h)  # after the last read-back (d2h runs in order)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(p0.elapsed_time(p1), dist, "cuda")
    e2e_value = whole_job_throughput(world, cfg.T, e2e_steps, e2e_ms)
    e2e_serial_value = whole_job_throughput(world, cfg.T, e2e_steps, e2e_serial_ms)
    y_h = y_hs[0]
    clocks = sampler.stop()

    # ------------------------------------------------------------ roofline of the dominant kernel
    distinct = int(torch.unique(idx).numel())
    rows_per_expert = torch.bincount(idx.flatten().long(), minlength=cfg.E)
    pk, pk_src = peaks()
    model = stage_model(cfg, distinct)
    fused = moe.moe_forward_fused_gemms(shape, opts)
    if fused:
        model = fuse_stages(model)
    t_dom = dom_ms / 1e3
    m = model[dom]
    t_tc, t_hbm = m["flops"] / (pk["bf16_tflops"] * 1e12), m["bytes"] / (pk["hbm_gbs"] * 1e9)
    if t_tc >= t_hbm:
        achieved, peak, unit, bound = m["flops"] / t_dom / 1e12, pk["bf16_tflops"], "TFLOP/s", "tensor"
    else:
        achieved, peak, unit, bound = m["bytes"] / t_dom / 1e9, pk["hbm_gbs"], "GB/s", "hbm"
    sustained = pk["bf16_tflops_sustained"] if bound == "tensor" else None
    roofline = {"bound": bound, "kernel": stage_label(dom, fused), "achieved": achieved, "peak": peak,
                "unit": unit, "frac": achieved / peak, "peak_source": f"{pk_src} (burst)",
                "frac_vs_sustained_peak": (achieved / sustained) if sustained else None,
                # the figures belong to the kernels the library picks by itself
                "traffic": ncu_traffic(cfg.name, dom) if default_kernels() else None,
                "kernel_sources": traffic_kernel_sources(cfg.name, dom) or kernel_sources_hash(),
                "algorithmic_per_launch": m["flops"] if bound == "tensor" else m["bytes"],
                "kernel_ms": dom_ms,
                "timed": "CUDA events around this stage only (its GEMM launch), "
                         + ("graph replay" if dom_graph is not None else "eager calls") + ", L2 flushed"}
    layer_flops = flops(cfg)
    layer_bytes = algorithmic_bytes(cfg, distinct)
    t_step = ms_per_step / 1e3
    layer = {"tflops": layer_flops / t_step / 1e12, "tensor_frac": layer_flops / t_step / 1e12 / pk["bf16_tflops"],
             "hbm_gbs": layer_bytes / t_step / 1e9, "hbm_frac": layer_bytes / t_step / 1e9 / pk["hbm_gbs"],
             "tensor_frac_vendor_2250": layer_flops / t_step / 1e12 / 2250.0,
             "hbm_frac_vendor_8000": layer_bytes / t_step / 1e9 / 8000.0,
             "distinct_experts": distinct, "flops": layer_flops, "bytes": layer_bytes,
             "rows_per_expert": {"max": int(rows_per_expert.max()), "mean_touched": cfg.T * cfg.k / distinct,
                                 "empty_experts": int((rows_per_expert == 0).sum())}}

    if graph is not None:
        del graph
    if stage_graph is not None:
        del stage_graph
    if dom_graph is not None:
        del dom_graph
    out = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": cfg.act_dtype if cfg.w_dtype != "mxfp4" else "bf16 (mxfp4 weights)",
           "data": "synthetic (seeded; random-init weights)",
           "config": config_dict(cfg, {"parallelism": f"replicas x{world}",
                                       "launch": "cuda graph of moe_forward" if not args.no_graph else "eager moe_forward"}),
           "roofline": roofline, "layer": layer,
           "stage_ms": dict(zip(names, stage_ms)),
           "stage_timing": {"launch": stage_launch,
                            "ms_per_step_with_stage_events": staged_ms / args.steps},
           "e2e": {"value": e2e_value, "unit": "tokens/s",
                   "h2d_bytes_per_step": x_h.numel() * x_h.element_size() + l_h.numel() * l_h.element_size(),
                   "d2h_bytes_per_step": y_h.numel() * y_h.element_size(),
                   "timing": "copies of each step overlapped with the neighbouring steps' forwards "
                             "(two device buffer sets, separate copy streams); no L2 flush between "
                             "steps, unlike the device-timed value",
                   "serial_value": e2e_serial_value},
           "gpu_launches": moe.moe_forward_kernel_count(shape, opts) * args.steps,
           "clocks": clocks}

    # ------------------------------------------------------------ CPU baseline (rank 0, N=1)
    if world == 1 and not args.no_cpu_baseline:
        hin = host_inputs(inputs)
        v, n, dt, threads = oracle_sample(cfg, hin, budget_s=args.cpu_budget)
        out["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                               "sample": f"{n} of {cfg.T} tokens (whole layer per token), {dt:.1f} s"}
    # ------------------------------------------------------------ the other workloads (N=1)
    # Device-timed summaries of every other workload of the benchmark suite in the same
    # run, so that one default invocation measures them all (the fields above stay the
    # default workload's).
    if world == 1 and args.workloads == "all":
        from workloads import CONFIGS
        del tens, ws, inputs, y, slots, xb, lb, yb
        torch.cuda.empty_cache()
        others = {}
        sampler2 = ClockSampler(physical_gpu_index(local))
        for name, ocfg in CONFIGS.items():
            if name == cfg.name:
                continue
            try:
                others[name] = measure_workload(ocfg, args.other_steps, 3, flush, stream)
            except Exception as exc:  # report it on the line; the default workload's figures stand
                others[name] = {"workload": workload_name(ocfg), "error": f"{type(exc).__name__}: {exc}"}
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
        out["other_workloads"] = others
        out["other_workloads_clocks"] = sampler2.stop()

    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def run_ep(args, cfg):
    """The expert-parallel layer (mixture_experts_ffn_10_b200.ep), timed eagerly: every rank
    holds cfg.T tokens of its own and E / N experts; a step is one forward of the layer --
    routing, permute, the all-to-all of the rows, the rank's experts, the all-to-all back,
    the combine -- with its host copy of the split sizes and its collectives, between CUDA
    events on the rank's stream, L2 flushed before it; max over ranks.  At N = 1 the
    exchange is a copy and the line also times moe_forward on the same tokens."""
    import torch

    import mixture_experts_ffn_10_b200 as moe
    from mixture_experts_ffn_10_b200.ep import ExpertParallelMoE
    from workloads import make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    if cfg.E % world or cfg.Fs:
        raise SystemExit(f"--ep needs E divisible by {world} and no shared expert ({cfg.name})")
    inputs = make_inputs(cfg, "cuda")
    El = cfg.E // world
    keep = ("gate_up", "gate_up_scales", "gate_up_bias", "down", "down_scales", "down_bias", "gate", "gate_scales",
            "gate_bias")
    mine = {k: (v[rank * El:(rank + 1) * El].clone() if v is not None else None) for k, v in inputs.items()
            if k in keep}
    mine["router_bias"], mine["selection_bias"] = inputs.get("router_bias"), inputs.get("selection_bias")
    layer = ExpertParallelMoE(cfg, mine, group=None)
    flush = L2Flush(torch)
    torch.cuda.synchronize()

    def timed(fn, steps):
        ts = []
        for _ in range(steps):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return ts

    def ep_step():
        layer.forward(inputs["x"], inputs["logits"])

    sampler = ClockSampler(physical_gpu_index(local))
    timed(ep_step, args.warmup)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ts = timed(ep_step, args.steps)
    clocks = sampler.stop()
    total = max_over_ranks(sum(ts), dist, "cuda")
    out = {"metric": METRIC, "value": whole_job_throughput(world, cfg.T, args.steps, total), "unit": "tokens/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": cfg.act_dtype if cfg.w_dtype != "mxfp4" else "bf16 (mxfp4 weights)",
           "data": "synthetic (seeded; random-init weights)",
           "config": config_dict(cfg, {"parallelism": f"expert-parallel x{world}", "experts_per_rank": El,
                                       "launch": "eager layer forwards (host split sizes each step)"}),
           "clocks": clocks}
    if world == 1:
        y = torch.empty_like(inputs["x"])

        def fwd_step():
            moe.forward(cfg, inputs, y=y)

        timed(fwd_step, args.warmup)
        out["moe_forward_ms_per_step"] = statistics.median(timed(fwd_step, args.steps))
        out["ep_ms_per_step_median"] = statistics.median(ts)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--config", default="mixtral_bf16")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workloads", default=None, choices=["all", "none"],
                    help="also time every other workload briefly (default: all for the default "
                         "workload at N=1, none otherwise)")
    ap.add_argument("--other-steps", type=int, default=10, help="timed steps per other workload")
    ap.add_argument("--no-graph", action="store_true", help="time eager calls instead of a CUDA graph replay")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle wall time")
    ap.add_argument("--ep", action="store_true",
                    help="time the expert-parallel layer (experts split over the N ranks) instead")
    ap.add_argument("--set", action="append", default=[], metavar="FIELD=VALUE",
                    help="override a workload field (profiling / sweeps), e.g. --set T=1024")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    from workloads import CONFIGS, small
    if args.workloads is None:
        args.workloads = "all" if args.config == "mixtral_bf16" and not args.set else "none"
    cfg = CONFIGS[args.config]
    for kv in args.set:
        k, v = kv.split("=", 1)
        cur = getattr(cfg, k)
        cfg = small(cfg, **{k: type(cur)(v) if not isinstance(cur, bool) else v in ("1", "true", "True")})
    if args.set:
        cfg = small(cfg, name=cfg.name + "[" + ",".join(args.set) + "]")
    if args.impl == "reference":
        return run_reference(args, cfg)
    if args.ep:
        return run_ep(args, cfg)
    return run_own(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
