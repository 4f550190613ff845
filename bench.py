#!/usr/bin/env python
"""Throughput of the masked attention JVP on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload tf|frame_causal|chunk_tf|tf_long]

One step is one call of the whole hot path (mask -> tile work list, the
score / score-tangent contractions, the online softmax and JVP state, the
three PV-type accumulations and the finish) over one synthetic batch of
the 65,520-token teacher-forcing workload (B=1, H=12, d=128; 21 frames of
1560 tokens, clean + noisy). Throughput counts 12*d FLOPs per admitted
(query, key) pair.

Multi-GPU (launched by torch.distributed.run): every rank runs its own,
independently seeded batch (weak scaling, no collective on the data path);
the timed region is bracketed by barriers and the slowest rank's time is
reported. Rank 0 prints one JSON line.

``--impl reference`` times the float64 CPU oracle on this machine's host cores
instead (rank 0 only), on a bounded sample of query rows per step.

``--op cache`` measures the read-only forward of causal rollout instead:
the last chunk of the workload's video (chunk * tokens_per_frame queries)
attends to a key/value cache holding all n_frames frames; one step writes
the chunk's keys (rotated by RoPE) and values into their cache slots and
runs the cache attention; 4*d FLOPs per (query, key) pair.

``--op prologue`` measures the attention layer's tangent prologue on the
workload's tokens: from the fused QKV projections of x and dx ([B, L, 3 H d]
each), QK-norm over all H*d channels with its tangent, RoPE, and the
[B, H, L, d] layout of the JVP kernel; memory-bound, reported as
algorithmic GB/s (inputs read once, outputs written once).

``--op ulysses`` measures the context-parallel JVP (Ulysses, the pages'
sequence-parallel path): every rank holds a token shard [B, H, L/P, d] of
one workload problem; one step is one ulysses_jvp_attn_fused call (the
input exchange, this rank's head group through the JVP kernel, the output
rows stored into their owners' shards by the kernel's epilogue). Strong
scaling: the job computes one problem whatever P is. The line also reports
the bare kernel's time on the same problem at P = 1 and the overhead of
the exchange over it.

``--op bwd`` measures the masked attention backward instead (gradients of
<G, O> for the primal output, jvp_attn_bwd) on the same workload, counting
10*d FLOPs per admitted pair: S recomputed (2d), dP = G V^T (2d), and the
three gradient products (2d each); the two passes execute 14*d.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention-JVP TFLOP/s (12*d per unmasked pair) and % of B200 bf16 tensor peak"
METRIC_CACHE = ("KV-cache chunk attention TFLOP/s (4*d per query-key pair) and % of B200 "
                "bf16 tensor peak")
METRIC_PROLOGUE = ("attention-layer tangent prologue GB/s (QK-norm JVP + RoPE + layout; "
                   "algorithmic bytes) and % of measured HBM bandwidth")
METRIC_BWD = ("masked attention backward TFLOP/s (10*d per unmasked pair) and % of B200 "
              "bf16 tensor peak")
UNIT = "TFLOP/s"
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
_CSRC = "attention_jvp_continuous_b200/csrc/"
# Sources of each op's kernels: a stored DRAM-traffic figure is used only
# while these files are unchanged since its capture.
KERNEL_SOURCES = {
    "jvp": [_CSRC + f for f in ("jvp_attn_sm100.cu", "sm100_pipeline.cuh", "sm100_ptx.cuh",
                                "mask_rows.cuh")],
    "bwd": [_CSRC + f for f in ("jvp_attn_bwd_sm100.cu", "sm100_pipeline.cuh", "sm100_ptx.cuh",
                                "mask_rows.cuh")],
    "cache": [_CSRC + f for f in ("attn_cache_sm100.cu", "sm100_pipeline.cuh", "sm100_ptx.cuh")],
    "prologue": [_CSRC + f for f in ("qkv_prologue.cu", "sm100_ptx.cuh")],
}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


# ------------------------------------------------------------ host logic --

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


_TOKEN = re.compile(r'"(?:\\.|[^"\\\n])*"'       # string literal
                    r"|'(?:\\.|[^'\\\n])*'"       # character literal
                    r"|//[^\n]*"                     # line comment
                    r"|/\*.*?\*/"                    # block comment
                    r"|\s+", re.S)


def code_only(src: str) -> str:
    """C/C++ source without comments, with every run of whitespace as one
    space: what a comment or layout edit leaves unchanged."""
    def keep(m):
        t = m.group(0)
        if t.startswith("//") or t.startswith("/*"):
            return " "
        return " " if t.isspace() else t
    return re.sub(r"\s+", " ", _TOKEN.sub(keep, src)).strip()


def kernel_hash(op: str = "jvp") -> str:
    """Hash of the code (comments and layout aside) of the sources that make
    up one op's kernels: a stored ncu figure is used only while it matches."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[op]:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(code_only(f.read()).encode())
    return h.hexdigest()[:16]


def stored_traffic(key: str, op: str = "jvp", **shape):
    """DRAM bytes per launch (per call, for ops of several kernels) from a
    committed ncu capture, if it was taken on the current kernel source and
    the entry's recorded shape (e.g. H) matches; else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    e = d.get(key)
    if not e or e.get("kernel_hash") != kernel_hash(op):
        return None
    if any(k in e and e[k] != v for k, v in shape.items()):
        return None
    return e.get("dram_bytes_per_launch")


def flops_per_pair(w, op: str = "jvp") -> float:
    return (10.0 if op == "bwd" else 12.0) * w.d


def flops_per_step(w, pairs_per_head: int, op: str = "jvp") -> float:
    return flops_per_pair(w, op) * pairs_per_head * w.B * w.H


def rank_seed(base_seed: int, rank: int) -> int:
    """Independent, reproducible input stream per rank."""
    return base_seed + 1000003 * rank


def max_over_ranks(value: float, world: int) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""
    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = (bus_id or "").lower()
        self.proc = None
        # The raw samples go to BENCH_CLOCK_DIR (default: the system temp
        # directory); the JSON line carries their summary.
        log_dir = os.environ.get("BENCH_CLOCK_DIR") or tempfile.gettempdir()
        self.path = os.path.join(log_dir, f"clocks_{os.getpid()}.csv")

    @staticmethod
    def bus_id_of(props) -> str | None:
        """'dddddddd:bb:dd.0' from torch device properties, if available."""
        try:
            return "%08x:%02x:%02x.0" % (int(props.pci_domain_id), int(props.pci_bus_id),
                                         int(props.pci_device_id))
        except (AttributeError, TypeError, ValueError):
            return None

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        return self.parse(self.path, self.bus_id)

    @classmethod
    def parse(cls, path: str, bus_id: str = ""):
        rows = {}
        with open(path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                rows.setdefault(parts[0].lower(), []).append(parts)
        key = None
        for k in rows:
            if bus_id and k[-7:] == bus_id[-7:]:
                key = k
        if key is None and len(rows) == 1:
            key = next(iter(rows))
        if key is None:
            return {"sm_mhz": None, "sm_max_mhz": None,
                    "reasons": ["could not match the GPU in nvidia-smi output"]}
        sm, mx, reasons = [], [], set()
        for parts in rows[key]:
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(cls.NAMES, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ---------------------------------------------------------------- our arm --

def device_timed(step, steps: int, world: int, local: int, stream, ja):
    """Times ``steps`` calls of ``step`` with CUDA events on ``stream``,
    bracketed by barriers and device synchronisation, with nvidia-smi clock
    samples meanwhile. Returns (per-step ms, max-over-ranks total ms, clocks)."""
    import torch
    import torch.distributed as dist
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    bus = ClockSampler.bus_id_of(torch.cuda.get_device_properties(local))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    with ClockSampler(bus) as clk:
        ev[0].record(stream)
        for i in range(steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ja.check_device_error()
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    total = max_over_ranks(ev[0].elapsed_time(ev[-1]), world)
    return per, total, clk.summary()


def e2e_pipelined(host_in, out_like, compute, steps: int, world: int, ja) -> float:
    """End-to-end throughput of a stream of batches held in pinned host
    memory: every step copies its inputs host->device, runs ``compute``
    (dev_in, dev_out) through the library and copies its outputs back.
    Double-buffered on three streams (copy in, compute, copy out) ordered by
    events, so that step i+1's inputs and step i-1's outputs cross the host
    link while step i computes. Returns the max-over-ranks ms of ``steps``
    steps, from before the first copy in to after the last copy out."""
    import torch
    import torch.distributed as dist
    cs = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    dev_in = [[torch.empty(h.shape, dtype=h.dtype, device="cuda") for h in host_in]
              for _ in range(2)]
    dev_out = [[torch.empty_like(t) for t in out_like] for _ in range(2)]
    host_out = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in out_like]
                for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n, start_ev=None):
        if start_ev is not None:
            s_in.wait_event(start_ev)
        for i in range(n):
            k = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_done[k])  # buffer k's last compute finished
                for d, h in zip(dev_in[k], host_in):
                    d.copy_(h, non_blocking=True)
                ev_in[k].record(s_in)
            cs.wait_event(ev_in[k])
            if i >= 2:
                cs.wait_event(ev_out[k])  # buffer k's last outputs copied out
            compute(dev_in[k], dev_out[k])
            ev_done[k].record(cs)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[k])
                for h, d in zip(host_out[k], dev_out[k]):
                    h.copy_(d, non_blocking=True)
                ev_out[k].record(s_out)
        cs.wait_stream(s_in)
        cs.wait_stream(s_out)

    run(2)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cs)
    run(steps, e0)
    e1.record(cs)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ja.check_device_error()
    return max_over_ranks(e0.elapsed_time(e1), world)


def run_ours(args, w):
    import datetime

    import torch
    import torch.distributed as dist

    import attention_jvp_continuous_b200 as ja
    from attention_jvp_continuous_b200.inputs import make_inputs

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    ja._lib.lib()  # fail loudly if the CUDA library is missing
    mask = ja.Mask(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)
    pairs, n_full, n_part, _ = ja.mask_stats(mask)
    bwd = args.op == "bwd"
    flops = flops_per_step(w, pairs, args.op)

    inputs, _ = make_inputs(w, device="cuda", seed=rank_seed(w.seed, rank))
    q = inputs[0]
    o = torch.empty_like(q)
    d_o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=q.device)
    stream = torch.cuda.current_stream()

    if bwd:
        # Backward inputs: q, k, v, the primal output and LSE of the forward
        # (computed once, outside the timed region) and a seeded N(0, 1)
        # cotangent G; outputs and scratch preallocated.
        gen = torch.Generator(device=q.device).manual_seed(rank_seed(w.seed, rank) + 17)
        g = torch.randn(q.shape, generator=gen, device=q.device).to(q.dtype)
        ja.jvp_attn_fwd(*inputs, o, d_o, lse, mask)
        grads = [torch.empty_like(q) for _ in range(3)]
        scratch = torch.empty((ja.bwd_scratch_len(w.B, w.H, w.L),), dtype=torch.float32,
                              device=q.device)
        step_in = [inputs[0], inputs[1], inputs[2], o, g, lse]

        def step():
            ja.jvp_attn_bwd(*step_in, *grads, scratch, mask)
    else:
        step_in = list(inputs)

        def step():
            ja.jvp_attn_fwd(*inputs, o, d_o, lse, mask)

    for _ in range(args.warmup):
        step()
    ja.check_device_error()

    # ---- device-timed region (inputs resident in HBM) ----
    per, total_ms_max, clocks = device_timed(step, args.steps, world, local, stream, ja)
    value = flops * args.steps * world / (total_ms_max * 1e-3) / 1e12
    launch_ms = sum(per) / len(per)

    # ---- end to end through the C ABI: pinned host in, host out ----
    host_in = [t.cpu().pin_memory() for t in step_in]
    out_like = grads if bwd else [o, d_o, lse]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in out_like)
    e2e_steps = max(2, min(args.steps, 10))

    def compute(dev_in, dev_out):
        if bwd:
            ja.jvp_attn_bwd(*dev_in, *dev_out, scratch, mask)
        else:
            ja.jvp_attn_fwd(*dev_in, *dev_out, mask)

    e2e_ms = e2e_pipelined(host_in, out_like, compute, e2e_steps, world, ja)
    e2e_value = flops * e2e_steps * world / (e2e_ms * 1e-3) / 1e12

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    peaks, peak_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = flops / (launch_ms * 1e-3) / 1e12
    traffic = (stored_traffic(w.name + "_bwd", "bwd", H=w.H) if bwd
               else stored_traffic(w.name, H=w.H))
    kernel = ("bwd_kernel<false> + bwd_kernel<true> (query pass, key/value pass)" if bwd
              else "jvp_attn_sm100_kernel")
    line = {
        "metric": METRIC_BWD if bwd else METRIC, "value": round(value, 2), "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms_max / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": describe_workload(w),
            "B": w.B, "H": w.H, "L": w.L, "d": w.d, "mode": w.mode,
            "tokens_per_frame": w.tokens_per_frame, "n_frames": w.n_frames, "chunk": w.chunk,
            "pairs_per_head": pairs, "flops_per_step": flops,
            "tiles_128x64_per_head": {"full": n_full, "partial": n_part},
            "l2": "inputs larger than L2 (%.2f GB read per step vs 126 MB L2); no flush"
                  % (h2d / 1e9),
            "parallelism": f"dp{world} (independent problems per rank, no data collective)",
        },
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "note": "pinned host batches; copies in, compute and copies out on three "
                        "streams, double-buffered (step i+1's inputs and step i-1's outputs "
                        "move while step i computes)"},
        "gpu_launches": args.steps * (2 if bwd else 1),
        "roofline": {
            "bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": UNIT,
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "peak_source": f"{peak_src} bf16 burst (cuBLAS)",
            "frac_of_sustained": round(achieved / float(peaks.get(
                "bf16_tflops_sustained", peak)), 4),
            "frac_of_nominal_2250": round(achieved / NOMINAL_BF16_TFLOPS, 4),
            "kernel": kernel, "launch_ms": round(launch_ms, 4),
        },
        "clocks": clocks,
    }
    if bwd:
        line["config"]["cotangent"] = "G ~ N(0, 1), bf16, seeded"
        line["config"]["executed_flops_per_pair"] = 14 * w.d
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = (cpu_baseline_bwd(w, step_in, rows_per_head=args.cpu_rows_bwd)
                                if bwd else
                                cpu_baseline(w, inputs, rows_per_head=args.cpu_rows))
    return line


def run_ours_ulysses(args, w):
    import datetime
    import socket

    import torch
    import torch.distributed as dist

    import attention_jvp_continuous_b200 as ja
    from attention_jvp_continuous_b200.inputs import make_inputs
    from attention_jvp_continuous_b200.ulysses import ShardBuffers, ulysses_jvp_attn_fused

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    if "MASTER_ADDR" not in os.environ:  # a single process outside torchrun
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", local))
    ja._lib.lib()
    mask = ja.Mask(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)
    pairs, _, _, _ = ja.mask_stats(mask)
    flops = flops_per_step(w, pairs)
    if w.H % world or w.L % world:
        raise SystemExit(f"{w.H} heads / {w.L} tokens do not split over {world} ranks")
    Ls = w.L // world
    # Every rank draws the same full problem and keeps its token shard.
    full, _ = make_inputs(w, device="cuda")
    shard = [x[:, :, rank * Ls:(rank + 1) * Ls].contiguous() for x in full]
    bufs = ShardBuffers(w.B, w.H, w.L, w.d, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        ulysses_jvp_attn_fused(*shard, mask, bufs)

    for _ in range(args.warmup):
        step()
    ja.check_device_error()
    per, total_ms_max, clocks = device_timed(step, args.steps, world, local, stream, ja)
    value = flops * args.steps / (total_ms_max * 1e-3) / 1e12
    launch_ms = sum(per) / len(per)

    # The bare kernel on the whole problem, one GPU (rank 0), same loop.
    bare_ms = None
    if rank == 0:
        o, d_o = torch.empty_like(full[0]), torch.empty_like(full[0])
        lse = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device="cuda")
        for _ in range(args.warmup):
            ja.jvp_attn_fwd(*full, o, d_o, lse, mask)
        bper, _, _ = device_timed(lambda: ja.jvp_attn_fwd(*full, o, d_o, lse, mask),
                                  args.steps, 1, local, stream, ja)
        bare_ms = sum(bper) / len(bper)
        del o, d_o, lse

    # End to end: pinned host shards in, the call, this rank's shard of the
    # outputs back, every step, on the current stream.
    host_in = [t.cpu().pin_memory() for t in shard]
    host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory()
                for t in (bufs.o, bufs.do, bufs.lse)]
    dev_in = [torch.empty_like(t) for t in shard]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    e2e_steps = max(2, min(args.steps, 10))

    def e2e_step():
        for d_, h_ in zip(dev_in, host_in):
            d_.copy_(h_, non_blocking=True)
        ulysses_jvp_attn_fused(*dev_in, mask, bufs)
        for h_, d_ in zip(host_out, (bufs.o, bufs.do, bufs.lse)):
            h_.copy_(d_, non_blocking=True)

    e2e_step()
    _, e2e_ms, _ = device_timed(e2e_step, e2e_steps, world, local, stream, ja)
    e2e_value = flops * e2e_steps / (e2e_ms * 1e-3) / 1e12
    dist.barrier()
    del bufs
    dist.destroy_process_group()
    if rank != 0:
        return None
    peaks, peak_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = flops / world / (launch_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC + " (context-parallel, Ulysses)", "value": round(value, 2),
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms_max / args.steps, 4), "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": describe_workload(w) + f"; token shards of {Ls} tokens on each of "
                        f"{world} ranks", "B": w.B, "H": w.H, "L": w.L, "d": w.d,
            "pairs_per_head": pairs, "flops_per_step": flops,
            "l2": "inputs larger than L2; no flush",
            "parallelism": f"cp{world} (Ulysses: token shards -> head groups, P2P exchange in, "
                           "the kernel's scatter epilogue out)",
            "bare_kernel_ms_one_gpu": None if bare_ms is None else round(bare_ms, 4),
            "overhead_vs_bare_kernel": (None if bare_ms is None or world != 1
                                        else round(launch_ms / bare_ms - 1.0, 4)),
        },
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "note": "this rank's pinned host shards in and its output shard out, serial "
                        "with the call on one stream"},
        "gpu_launches": args.steps,  # the JVP kernel; the exchange runs NCCL and torch kernels
        "roofline": {
            "bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": UNIT,
            "frac": round(achieved / peak, 4), "traffic": None,
            "peak_source": f"{peak_src} bf16 burst (cuBLAS)",
            "kernel": "jvp_attn_sm100_kernel (scatter epilogue) with the exchange around it",
            "launch_ms": round(launch_ms, 4),
        },
        "clocks": clocks,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, full, rows_per_head=args.cpu_rows)
    return line


def describe_workload(w) -> str:
    """One-line name of a workload: its mask, shape and value recipe."""
    from attention_jvp_continuous_b200.inputs import CHUNK_CAUSAL, FRAME_CAUSAL, TEACHER_FORCING
    head = f"B={w.B} H={w.H} d={w.d}"
    if w.mode == TEACHER_FORCING:
        kind = ("frame-wise teacher-forcing mask" if w.chunk == 1 else
                f"chunk-wise teacher-forcing mask (chunks of {w.chunk} frames)")
        toks = f"{w.n_frames} frames x {w.tokens_per_frame} tokens x {{clean,noisy}}"
    elif w.mode == FRAME_CAUSAL:
        kind, toks = "frame-causal mask", f"{w.n_frames} frames x {w.tokens_per_frame} tokens"
    elif w.mode == CHUNK_CAUSAL:
        kind = f"chunk-causal mask (chunks of {w.chunk} frames)"
        toks = f"{w.n_frames} frames x {w.tokens_per_frame} tokens"
    else:
        kind, toks = "dense (no mask)", f"{w.n_frames} frames x {w.tokens_per_frame} tokens"
    text = f"{w.name}: {kind}, {head}, {toks} = {w.L} tokens, {w.dtype}"
    if w.head_scale is not None:
        lo, hi = w.head_scale
        text += f", Q and K of each head scaled by s_h ~ U({lo:g}, {hi:g})"
    return text


# The oracle evaluates all sampled rows of one admissible key set with one
# BLAS call, so its speed per pair grows with the number of rows sampled per
# head: two samples of one workload give different rates.
SAMPLE_NOTE = ("the oracle batches the sampled rows that share a key set into one BLAS "
               "call, so its rate per pair depends on how many rows are sampled")


def cache_shape(w):
    """(Lq, Lk) of the rollout's last chunk: one chunk of queries against all
    frames of the video (the committed prefix plus the chunk itself)."""
    chunk = max(1, w.chunk)
    return chunk * w.tokens_per_frame, w.n_frames * w.tokens_per_frame


def run_ours_cache(args, w):
    import datetime

    import torch
    import torch.distributed as dist

    import attention_jvp_continuous_b200 as ja
    from attention_jvp_continuous_b200.inputs import rope_table

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    ja._lib.lib()
    Lq, Lk = cache_shape(w)
    B, H, d = w.B, w.H, w.d
    flops = 4.0 * d * Lq * Lk * B * H
    gen = torch.Generator(device="cuda").manual_seed(rank_seed(w.seed, rank))

    def draw(rows):
        return torch.randn((B, H, rows, d), generator=gen, device="cuda").to(torch.bfloat16)

    q, k_cur, v_cur = draw(Lq), draw(Lq), draw(Lq)
    kc, vc = draw(Lk), draw(Lk)  # committed prefix (post-RoPE keys) and values
    cos, sin = rope_table(Lk, d, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Lq), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    pos = Lk - Lq
    attn_ev = []

    def step(record=False):
        ja.rope_copy(k_cur, kc, Lq, 0, pos, cos, sin, rope_row0=pos)
        ja.rope_copy(v_cur, vc, Lq, 0, pos)
        if record:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            ja.cache_attn(q, kc, vc, Lk, o, lse)
            e1.record(stream)
            attn_ev.append((e0, e1))
        else:
            ja.cache_attn(q, kc, vc, Lk, o, lse)

    for _ in range(args.warmup):
        step()
    ja.check_device_error()
    per, total_ms_max, clocks = device_timed(lambda: step(True), args.steps, world, local,
                                             stream, ja)
    value = flops * args.steps * world / (total_ms_max * 1e-3) / 1e12
    attn_ms = sum(a.elapsed_time(b) for a, b in attn_ev) / len(attn_ev)

    # end to end: the chunk's q, k, v from pinned host memory, o and LSE back;
    # the cache is rollout state and stays in HBM
    host_in = [t.cpu().pin_memory() for t in (q, k_cur, v_cur)]

    def compute(dev_in, dev_out):
        ja.rope_copy(dev_in[1], kc, Lq, 0, pos, cos, sin, rope_row0=pos)
        ja.rope_copy(dev_in[2], vc, Lq, 0, pos)
        ja.cache_attn(dev_in[0], kc, vc, Lk, dev_out[0], dev_out[1])

    e2e_steps = max(2, min(args.steps, 10))
    e2e_ms = e2e_pipelined(host_in, [o, lse], compute, e2e_steps, world, ja)
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in (o, lse))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None
    peaks, peak_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = flops / (attn_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC_CACHE, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms_max / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": f"{w.name} rollout, last chunk: {Lq} queries ({max(1, w.chunk)} "
                        f"frame(s) x {w.tokens_per_frame} tokens) over a cache of {Lk} keys "
                        f"({w.n_frames} frames), B={B} H={H} d={d}, post-RoPE keys",
            "B": B, "H": H, "d": d, "Lq": Lq, "Lk": Lk, "flops_per_step": flops,
            "step": "rope_copy(k chunk, rotated) + rope_copy(v chunk) + cache attention",
            "l2": "cache %.0f MB read per step (above the 126 MB L2); no flush"
                  % (2 * B * H * Lk * d * 2 / 1e6),
            "parallelism": f"dp{world} (independent problems per rank, no data collective)",
        },
        "e2e": {"value": round(flops * e2e_steps * world / (e2e_ms * 1e-3) / 1e12, 2),
                "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps,
                "note": "chunk q, k, v in and o, lse out (pipelined as in the jvp op); "
                        "the cache stays resident"},
        "gpu_launches": args.steps * 4,
        "roofline": {
            "bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": UNIT,
            "frac": round(achieved / peak, 4),
            "traffic": stored_traffic(w.name + "_cache", "cache", H=H, Lq=Lq, Lk=Lk),
            "peak_source": f"{peak_src} bf16 burst (cuBLAS)",
            "frac_of_sustained": round(achieved / float(peaks.get(
                "bf16_tflops_sustained", peak)), 4),
            "frac_of_nominal_2250": round(achieved / NOMINAL_BF16_TFLOPS, 4),
            "kernel": "attn_cache_sm100_kernel + attn_cache_combine_kernel (one call)",
            "launch_ms": round(attn_ms, 4),
        },
        "clocks": clocks,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_cache(w, q, kc, vc, rows_per_head=args.cpu_rows_cache)
    return line


def run_ours_prologue(args, w):
    import datetime

    import torch
    import torch.distributed as dist

    import attention_jvp_continuous_b200 as ja
    from attention_jvp_continuous_b200.inputs import rope_table

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    ja._lib.lib()
    B, L, H, d = w.B, w.L, w.H, w.d
    C = H * d
    gen = torch.Generator(device="cuda").manual_seed(rank_seed(w.seed, rank))
    P = torch.randn((B, L, 3 * C), generator=gen, device="cuda").to(torch.bfloat16)
    dP = (torch.randn((B, L, 3 * C), generator=gen, device="cuda") * w.tangent_std).to(
        torch.bfloat16)
    wq = 1.0 + 0.1 * torch.randn((C,), generator=gen, device="cuda")
    wk = 1.0 + 0.1 * torch.randn((C,), generator=gen, device="cuda")
    # teacher forcing: clean token i and noisy token F*T + i share position i
    half = L // 2 if w.mode == 3 else L
    cos, sin = rope_table(half, d, device="cuda")
    if w.mode == 3:
        cos, sin = torch.cat([cos, cos]).contiguous(), torch.cat([sin, sin]).contiguous()
    out = [torch.empty((B, H, L, d), dtype=torch.bfloat16, device="cuda") for _ in range(6)]
    stream = torch.cuda.current_stream()
    nbytes = 2 * P.numel() * 2 + 6 * B * H * L * d * 2

    def step():
        ja.qkv_prologue(P, dP, H, wq, wk, C, 1e-6, cos, sin, out=out)

    for _ in range(args.warmup):
        step()
    ja.check_device_error()
    per, total_ms_max, clocks = device_timed(step, args.steps, world, local, stream, ja)
    value = nbytes * args.steps * world / (total_ms_max * 1e-3) / 1e9
    launch_ms = sum(per) / len(per)
    host_in = [t.cpu().pin_memory() for t in (P, dP)]

    def compute(dev_in, dev_out):
        ja.qkv_prologue(dev_in[0], dev_in[1], H, wq, wk, C, 1e-6, cos, sin, out=dev_out)

    e2e_steps = max(2, min(args.steps, 10))
    e2e_ms = e2e_pipelined(host_in, out, compute, e2e_steps, world, ja)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None
    peaks, peak_src = load_peaks()
    peak = float(peaks["hbm_gbs"])
    achieved = nbytes / (launch_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC_PROLOGUE, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms_max / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": f"{w.name} tokens: B={B} L={L} H={H} d={d}, projections [B, L, 3*{C}] "
                        f"of x and dx, QK-norm over {C} channels, RoPE",
            "B": B, "L": L, "H": H, "d": d, "bytes_per_step": nbytes,
            "l2": "%.2f GB moved per step (above the 126 MB L2); no flush" % (nbytes / 1e9),
            "parallelism": f"dp{world} (independent problems per rank, no data collective)",
        },
        "e2e": {"value": round(nbytes * e2e_steps * world / (e2e_ms * 1e-3) / 1e9, 1),
                "unit": "GB/s", "h2d_bytes_per_step": sum(t.numel() * t.element_size()
                                                          for t in host_in),
                "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in out),
                "steps": e2e_steps, "note": "pipelined as in the jvp op"},
        "gpu_launches": args.steps,
        "roofline": {
            "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": stored_traffic(w.name + "_prologue", "prologue", H=H, L=L),
            "peak_source": f"{peak_src} HBM copy bandwidth",
            "kernel": "qkv_prologue_kernel", "launch_ms": round(launch_ms, 4),
        },
        "clocks": clocks,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_prologue(w, P, dP, wq, wk, cos, sin,
                                                     tokens=args.cpu_tokens_prologue)
    return line


def cpu_baseline_prologue(w, P, dP, wq, wk, cos, sin, tokens: int):
    """The float64 prologue oracle on the first `tokens` tokens of each batch
    row, in algorithmic GB/s of the same bf16 layout."""
    from oracle.layer_prologue import qkv_prologue
    n = min(tokens, w.L)
    Ph, dPh = P[:, :n].cpu(), dP[:, :n].cpu()
    t0 = time.perf_counter()
    qkv_prologue(Ph, dPh, w.H, w.d, wq.cpu(), wk.cpu(), w.H * w.d, 1e-6, cos[:n].cpu(),
                 sin[:n].cpu())
    dt = time.perf_counter() - t0
    nbytes = (2 * Ph.numel() * 2 + 6 * w.B * w.H * n * w.d * 2)
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"first {n} tokens x {w.B} batch rows ({dt:.1f} s, float64 numpy)"}


# ---------------------------------------------------- oracle on the host --

def oracle_sample(w, host_inputs, rows_per_head: int, seed: int = 1234):
    """Times the float64 oracle on ``rows_per_head`` seeded query rows of
    every head; returns (seconds, sampled admitted pairs, threads)."""
    import numpy as np

    from attention_jvp_continuous_b200.inputs import sample_rows
    from oracle import MaskSpec, jvp_attention, key_intervals

    spec = MaskSpec(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)
    rows = sample_rows(w.L, rows_per_head, seed=seed)
    pairs_per_head = sum(b - a for r in rows for a, b in key_intervals(spec, int(r)))
    t0 = time.perf_counter()
    jvp_attention(*host_inputs, spec, rows=rows)
    dt = time.perf_counter() - t0
    return dt, pairs_per_head * w.B * w.H


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def cpu_baseline(w, inputs, rows_per_head: int):
    host = [t.cpu() for t in inputs]
    dt, sp = oracle_sample(w, host, rows_per_head)
    return {"value": round(12.0 * w.d * sp / dt / 1e12, 6), "unit": UNIT,
            "cores": blas_threads(), "kind": "oracle",
            "sample": f"{rows_per_head} seeded query rows per head x {w.B * w.H} heads "
                      f"({sp} admitted pairs, {dt:.1f} s, float64 numpy); {SAMPLE_NOTE}"}


def oracle_sample_bwd(w, host_in, rows_per_head: int, seed: int = 1234):
    """Times the float64 backward oracle restricted to ``rows_per_head``
    seeded query rows of every head (their gradient contributions); returns
    (seconds, admitted pairs of those rows)."""
    from attention_jvp_continuous_b200.inputs import sample_rows
    from oracle import MaskSpec, key_intervals
    from oracle.attention_backward import attention_backward

    spec = MaskSpec(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)
    rows = sample_rows(w.L, rows_per_head, seed=seed)
    pairs_per_head = sum(b - a for r in rows for a, b in key_intervals(spec, int(r)))
    q, k, v, _, g = host_in[:5]
    t0 = time.perf_counter()
    attention_backward(q, k, v, g, spec, rows=[int(r) for r in rows])
    dt = time.perf_counter() - t0
    return dt, pairs_per_head * w.B * w.H


def cpu_baseline_bwd(w, step_in, rows_per_head: int):
    host = [t.cpu() for t in step_in]
    dt, sp = oracle_sample_bwd(w, host, rows_per_head)
    return {"value": round(flops_per_pair(w, "bwd") * sp / dt / 1e12, 6), "unit": UNIT,
            "cores": blas_threads(), "kind": "oracle",
            "sample": f"gradient contributions of {rows_per_head} seeded query rows per "
                      f"head x {w.B * w.H} heads ({sp} admitted pairs, {dt:.1f} s, "
                      f"float64 numpy); {SAMPLE_NOTE}"}


def oracle_sample_cache(w, q, kc, vc, rows_per_head: int, seed: int = 1234):
    """Times the float64 cache-attention oracle on ``rows_per_head`` seeded
    query rows of every head; returns (seconds, query-key pairs)."""
    from attention_jvp_continuous_b200.inputs import sample_rows
    from oracle import cache_attention_head

    Lq, Lk = cache_shape(w)
    rows = sample_rows(Lq, rows_per_head, seed=seed)
    t0 = time.perf_counter()
    for b in range(w.B):
        for h in range(w.H):
            cache_attention_head(q[b, h, rows], kc[b, h], vc[b, h], Lk)
    return time.perf_counter() - t0, len(rows) * Lk * w.B * w.H


def cpu_baseline_cache(w, q, kc, vc, rows_per_head: int):
    q, kc, vc = q.cpu(), kc.cpu(), vc.cpu()
    dt, pairs = oracle_sample_cache(w, q, kc, vc, rows_per_head)
    return {"value": round(4.0 * w.d * pairs / dt / 1e12, 6), "unit": UNIT,
            "cores": blas_threads(), "kind": "oracle",
            "sample": f"{rows_per_head} seeded query rows per head x {w.B * w.H} heads "
                      f"over the full cache ({pairs} pairs, {dt:.1f} s, float64 numpy)"}


def reference_prologue(args, w, world: int):
    """--impl reference --op prologue: the float64 prologue oracle on
    16 * ref_rows tokens per step, in algorithmic GB/s."""
    import torch

    from attention_jvp_continuous_b200.inputs import rope_table
    from oracle.layer_prologue import qkv_prologue
    C, n = w.H * w.d, min(16 * args.ref_rows, w.L)
    gen = torch.Generator().manual_seed(w.seed)
    P = torch.randn((w.B, n, 3 * C), generator=gen).to(torch.bfloat16)
    dP = torch.randn((w.B, n, 3 * C), generator=gen).to(torch.bfloat16)
    wq, wk = torch.ones(C), torch.ones(C)
    cos, sin = rope_table(n, w.d)
    nbytes = 2 * P.numel() * 2 + 6 * w.B * w.H * n * w.d * 2
    for _ in range(args.warmup):
        qkv_prologue(P, dP, w.H, w.d, wq, wk, C, 1e-6, cos, sin)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        qkv_prologue(P, dP, w.H, w.d, wq, wk, C, 1e-6, cos, sin)
    total = time.perf_counter() - t0
    value = nbytes * args.steps / total / 1e9
    sample = f"{n} tokens x {w.B} batch rows per step"
    return {
        "impl": "reference", "metric": METRIC_PROLOGUE, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{w.name} tokens (oracle on a token sample)", "B": w.B,
                   "H": w.H, "L": w.L, "d": w.d, "parallelism": "host cores, rank 0 only"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def run_reference(args, w):
    world, rank, _ = dist_setup()
    if rank != 0:
        return None
    if args.op == "prologue":
        return reference_prologue(args, w, world)
    import torch

    from attention_jvp_continuous_b200.inputs import make_inputs
    inputs, _ = make_inputs(w, device="cpu")
    rows = args.ref_rows
    if args.op == "cache":
        Lq, Lk = cache_shape(w)
        gen = torch.Generator().manual_seed(w.seed)
        qh = torch.randn((w.B, w.H, Lq, w.d), generator=gen).to(torch.bfloat16)
        kh = torch.randn((w.B, w.H, Lk, w.d), generator=gen).to(torch.bfloat16)
        vh = torch.randn((w.B, w.H, Lk, w.d), generator=gen).to(torch.bfloat16)
        run_sample = lambda seed: oracle_sample_cache(w, qh, kh, vh, rows, seed=seed)  # noqa: E731
    elif args.op == "bwd":
        # The oracle's gradient needs no primal output; a seeded cotangent.
        gen = torch.Generator().manual_seed(w.seed + 17)
        g = torch.randn(inputs[0].shape, generator=gen).to(inputs[0].dtype)
        host = [inputs[0], inputs[1], inputs[2], None, g]
        run_sample = lambda seed: oracle_sample_bwd(w, host, rows, seed=seed)  # noqa: E731
    else:
        run_sample = lambda seed: oracle_sample(w, inputs, rows, seed=seed)  # noqa: E731
    for i in range(args.warmup):
        run_sample(100 + i)
    times, pairs = [], 0
    for i in range(args.steps):
        dt, sp = run_sample(1234 + i)
        times.append(dt)
        pairs += sp
    total = sum(times)
    value = (4.0 * w.d if args.op == "cache" else flops_per_pair(w, args.op)) * pairs / total / 1e12
    cores = blas_threads()
    sample = f"{rows} seeded query rows per head x {w.B * w.H} heads per step; {SAMPLE_NOTE}"
    line = {
        "impl": "reference",
        "metric": {"bwd": METRIC_BWD, "cache": METRIC_CACHE,
                   "ulysses": METRIC + " (context-parallel, Ulysses)"}.get(args.op, METRIC),
        "value": round(value, 6), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{w.name} (oracle on sampled rows)", "B": w.B, "H": w.H,
                   "L": w.L, "d": w.d, "mode": w.mode, "chunk": w.chunk,
                   "parallelism": "host cores, rank 0 only"},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    if args.op == "cache":
        Lq, Lk = cache_shape(w)
        line["config"].update({"workload": f"{w.name} rollout, last chunk (oracle on sampled "
                                           f"rows)", "Lq": Lq, "Lk": Lk})
    return line


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="tf",
                    choices=["tf", "frame_causal", "chunk_tf", "tf_long"])
    ap.add_argument("--cpu-rows", type=int, default=3072,
                    help="query rows per head in the cpu_baseline sample")
    ap.add_argument("--ref-rows", type=int, default=256,
                    help="query rows per head per step of --impl reference")
    ap.add_argument("--cpu-rows-bwd", type=int, default=1024,
                    help="query rows per head in the --op bwd cpu_baseline sample")
    ap.add_argument("--cpu-rows-cache", type=int, default=512,
                    help="query rows per head in the --op cache cpu_baseline sample")
    ap.add_argument("--cpu-tokens-prologue", type=int, default=16384,
                    help="tokens in the --op prologue cpu_baseline sample")
    ap.add_argument("--op", choices=["jvp", "bwd", "cache", "prologue", "ulysses"],
                    default="jvp",
                    help="jvp: the attention JVP (default); bwd: the masked backward; "
                         "cache: KV-cache chunk attention of the rollout's last chunk; "
                         "prologue: the layer's tangent prologue; ulysses: the "
                         "context-parallel JVP over the ranks")
    ap.add_argument("--heads", type=int, default=None,
                    help="override the workload's head count (small cases for ncu captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from attention_jvp_continuous_b200.inputs import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.heads is not None:
        if args.heads < 1:
            ap.error("--heads must be >= 1")
        import dataclasses
        w = dataclasses.replace(w, H=args.heads)
    world, rank, _ = dist_setup()
    if world != args.gpus and args.impl == "ours":
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    if args.impl == "reference":
        line = run_reference(args, w)
    elif args.op == "cache":
        line = run_ours_cache(args, w)
    elif args.op == "prologue":
        line = run_ours_prologue(args, w)
    elif args.op == "ulysses":
        line = run_ours_ulysses(args, w)
    else:
        line = run_ours(args, w)
    if line is not None and rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
