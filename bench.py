#!/usr/bin/env python
"""Benchmark of the Ulysses sequence-parallel attention block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload video|chunked|vit|tiny|reshard]

One step is one pass of the whole hot path over one batch of synthetic input:
scatter_sequence of the replicated q, k and v into the P virtual-rank shards,
the Ulysses block (seq->head exchange of q/k/v per head chunk, attention, and
the head->seq exchange fused into the attention epilogue), and
gather_sequence of the output. The default workload is the ragged video
latent (T=75600, H=24, D=128, P=7, bf16, one chunk); `value` is the
attention FLOP of the step (4*B*H*T'^2*D) over the step time, in TFLOP/s.

With N > 1 (launched by torch.distributed.run) every GPU runs its own
independent replica of the block (the block needs no collective across
GPUs); the timing is the maximum over ranks and `value` sums all replicas.

Rank 0 prints one JSON line. `--impl reference` times the CPU oracle instead
(test infrastructure, float64, on a bounded sample of rows of the same
workload).
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from ulysses_sequence_attention_sp_b200 import workloads as W  # noqa: E402
from ulysses_sequence_attention_sp_b200.synth import make_qkv, storage_to_f64  # noqa: E402

METRIC = "reshard GB/s and Ulysses-attention TFLOP/s on 1 B200, % of HBM/bf16 roofline"
WORKLOADS = {"tiny": W.TINY, "reshard": W.RESHARD, "video": W.VIDEO, "vit": W.VIT, "chunked": W.CHUNKED,
             "hybrid": W.HYBRID}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
KERNEL_SOURCES = {
    "attention": ["ulysses_sequence_attention_sp_b200/csrc/attn_pp.cu",
                  "ulysses_sequence_attention_sp_b200/csrc/device_common.cuh"],
    "pack_tma": ["ulysses_sequence_attention_sp_b200/csrc/pack_tma.cu",
                 "ulysses_sequence_attention_sp_b200/csrc/device_common.cuh"],
}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="video")
    ap.add_argument("--num-chunks", type=int, default=0, help="0: the workload's own chunk count")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-reshard", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads (measured after the headline, 1 GPU only)")
    ap.add_argument("--attention-kernel", choices=["auto", "one_tile", "two_tile", "two_cta"], default="auto",
                    help="the tensor-core attention kernel (all compute the same function)")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every call from Python instead of replaying the step as one CUDA graph")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS if k in p}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _code_only(text: str) -> str:
    """Source text without comments and blank lines (a comment edit does not
    change the kernel the counters were taken on)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln.strip())


def source_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, algorithmic_bytes: float | None = None):
    """DRAM bytes per launch from the committed ncu summary, if the kernel
    sources are unchanged since it was taken; else None. With
    `algorithmic_bytes` (a launch of another size than the captured one), the
    captured bytes are scaled by the ratio of algorithmic bytes."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        rec = json.load(f).get(kernel)
    if not rec or rec.get("source_hash") != source_hash(KERNEL_SOURCES[kernel]):
        return None
    if algorithmic_bytes is not None and rec.get("algorithmic_bytes"):
        return rec["bytes_per_launch"] * algorithmic_bytes / rec["algorithmic_bytes"]
    return rec.get("bytes_per_launch")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.skip = 0

    def start(self):
        """Starts sampling and returns once the first sample is written, so
        nvidia-smi's own start-up never overlaps the timed region."""
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu)], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return
        deadline = time.time() + 10.0
        while time.time() < deadline and os.path.getsize(self.path) == 0 and self.proc.poll() is None:
            time.sleep(0.05)
        self.skip = sum(1 for _ in open(self.path))  # samples taken before the timed region

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            lines = f.readlines()
        if len(lines) > self.skip + 1:
            lines = lines[self.skip:]  # keep the samples taken during the timed region
        for line in lines:
            cols = [c.strip() for c in line.split(",")]
            if len(cols) < 9:
                continue
            try:
                sm.append(float(cols[1]))
                mx.append(float(cols[2]))
            except ValueError:
                continue
            for name, val in zip(names, cols[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------- CPU oracle
def oracle_rows_tflops(w, storage, seconds: float, max_rows: int):
    """Times the oracle's attention on query rows of (batch 0, head 0) of the
    workload until `seconds` have elapsed (or max_rows rows)."""
    from oracle.attention import default_scale, softmax_attention
    q, k, v = storage
    kh = storage_to_f64(k[0, :, 0], w.dtype)
    vh = storage_to_f64(v[0, :, 0], w.dtype)
    rows_done, t_used, r0 = 0, 0.0, 0
    chunk = 64
    while t_used < seconds and rows_done < max_rows:
        rows = np.arange(r0, r0 + chunk) % w.tokens
        qh = storage_to_f64(q[0, rows, 0], w.dtype)
        t0 = time.perf_counter()
        softmax_attention(qh, kh, vh, default_scale(w.head_dim))
        t_used += time.perf_counter() - t0
        rows_done += chunk
        r0 += chunk
    flop = rows_done * 4.0 * w.tokens * w.head_dim
    return flop / t_used / 1e12, rows_done, t_used


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count()


def run_reference(args, w, rank, world):
    """The reference arm: the CPU oracle, on rank 0 only."""
    if rank != 0:
        return
    storage = make_qkv(w)
    per_step_s = 4.0
    times, rows = [], 0
    for i in range(args.warmup + args.steps):
        tf, r, t = oracle_rows_tflops(w, storage, per_step_s, 1 << 30)
        if i >= args.warmup:
            times.append(t)
            rows += r
    flop = rows * 4.0 * w.tokens * w.head_dim
    value = flop / sum(times) / 1e12
    cores = blas_threads()
    sample = (f"float64 oracle attention (oracle.attention.softmax_attention) on {rows // max(args.steps, 1)} "
              f"query rows per step of batch 0, head 0 against all {w.tokens} keys; rows are independent, "
              f"so TFLOP/s carries over to the full workload")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, w.num_chunks[0], args.gpus), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def reduce_max(values, world, device=None):
    """Element-wise maximum of per-rank timings over all ranks (any backend:
    NCCL needs a CUDA tensor, gloo a CPU one)."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device or "cpu")
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def job_throughput(units_per_rank_step: float, steps: int, max_ms: float, world: int, scale: float = 1e12):
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return world * units_per_rank_step * steps / (max_ms / 1e3) / scale


def workload_config(w, num_chunks, n_gpus):
    return {
        "workload": w.name, "batch": w.batch, "seq_len": w.seq_len, "prefix_tokens": w.prefix,
        "heads": w.heads, "head_dim": w.head_dim, "sp_virtual_ranks": w.world, "num_chunks": num_chunks,
        "global_batch": w.batch * n_gpus,
        "parallelism": f"{n_gpus} independent replica(s), {w.world} virtual SP ranks each"
                       + (f" (Ulysses {w.world // w.ring} x Ring {w.ring})" if w.ring > 1 else ""),
        "step": "scatter_sequence(q,k,v) -> ulysses_attention -> gather_sequence(out)",
        "l2": f"inputs larger than L2: {3 * w.tensor_bytes / 2**20:.0f} MiB of q/k/v per step"
        if 3 * w.tensor_bytes > 126 * 2**20 else "L2 flushed (512 MiB write) before every timed step",
    }


# ---------------------------------------------------------------- our arm
class BlockBench:
    """One workload's step on this device: scatter_sequence of q, k and v into
    the virtual-rank shards, ulysses_attention (pack, attention, fused
    head->seq) and gather_sequence of the output.

    The step's calls are stream-ordered and synchronise nothing, so each timed
    step is captured as a CUDA graph (one graph per step, each with its own
    pair of events around the attention kernels), which removes the Python
    launch cost that dominates the small workloads. Workloads whose q/k/v fit
    in L2 get a 512 MiB write between timed steps, whose time is measured apart
    and subtracted."""

    def __init__(self, usp, torch, dev, w, n_chunks, steps, seed, graph=True, kernel="auto"):
        self.usp, self.torch, self.dev, self.w, self.n_chunks, self.steps = usp, torch, dev, w, n_chunks, steps
        self.plan = usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix,
                             kv_heads=w.heads_kv, ring_size=w.ring)
        if kernel != "auto" and w.dtype != "fp32":
            self.plan.set_attention_kernel(kernel)
        plan = self.plan
        self.storage = make_qkv(w, seed=seed)
        self.full = [self.to_dev(x) for x in self.storage]
        self.shards = [plan.empty_seq_shards(), plan.empty_kv_seq_shards(), plan.empty_kv_seq_shards()]
        self.out = plan.empty_seq_shards()
        self.full_out = torch.empty(plan.full_shape(), dtype=plan.torch_dtype, device=dev)
        self.ws = torch.empty(plan.workspace_bytes(n_chunks), dtype=torch.uint8, device=dev)
        self.small = 3 * w.tensor_bytes <= 126 * 2**20
        self.flush = torch.empty(512 * 2**20, dtype=torch.uint8, device=dev) if self.small else None
        self.ev_a = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                     for _ in range(steps)]
        self.graphs = []
        self.launches_per_step = 0
        self.use_graph = graph

    def to_dev(self, x):
        torch = self.torch
        if self.w.dtype == "bf16":
            return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(self.dev)
        return torch.from_numpy(x).to(self.dev)

    def step(self, full=None, full_out=None):
        usp, plan = self.usp, self.plan
        for x, sh in zip(full or self.full, self.shards):
            usp.scatter_sequence(plan, x, out=sh)
        usp.ulysses_attention(plan, *self.shards, out=self.out, num_chunks=self.n_chunks, workspace=self.ws)
        usp.gather_sequence(plan, self.out, out=self.full_out if full_out is None else full_out)

    def prepare(self, warmup):
        torch, usp = self.torch, self.usp
        stream = torch.cuda.current_stream()
        for _ in range(warmup):
            self.step()
        for a, b in self.ev_a:
            a.record(stream)
            b.record(stream)
        torch.cuda.synchronize()
        if not self.use_graph:
            return
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        before = usp.kernel_launches()
        with torch.cuda.stream(cap):
            for i in range(self.steps):
                g = torch.cuda.CUDAGraph()
                self.plan.set_timing_events(*self.ev_a[i])
                with torch.cuda.graph(g, stream=cap):
                    self.step()
                self.graphs.append(g)
            self.plan.set_timing_events(None, None)
        self.launches_per_step = (usp.kernel_launches() - before) // self.steps
        stream.wait_stream(cap)
        for _ in range(2):
            self.graphs[0].replay()
        torch.cuda.synchronize()

    def timed_pass(self, barrier=lambda: None):
        """Times exactly `steps` steps between two synchronised barriers.
        Returns (device ms of the steps, per-step attention ms, launches)."""
        torch, usp = self.torch, self.usp
        stream = torch.cuda.current_stream()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        barrier()
        launches0 = usp.kernel_launches()
        t0.record(stream)
        for i in range(self.steps):
            if self.flush is not None:
                self.flush.zero_()
            if self.graphs:
                self.graphs[i].replay()
            else:
                self.plan.set_timing_events(*self.ev_a[i])
                self.step()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier()
        self.plan.set_timing_events(None, None)
        launches = usp.kernel_launches() - launches0 + self.launches_per_step * (self.steps if self.graphs else 0)
        ms = t0.elapsed_time(t1) - self.flush_ms()
        return ms, [a.elapsed_time(b) for a, b in self.ev_a], launches

    def flush_ms(self):
        if self.flush is None:
            return 0.0
        if not hasattr(self, "_flush_ms"):
            torch = self.torch
            stream = torch.cuda.current_stream()
            fs, fe = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            for _ in range(3):
                self.flush.zero_()
            fs.record(stream)
            for _ in range(self.steps):
                self.flush.zero_()
            fe.record(stream)
            torch.cuda.synchronize()
            self._flush_ms = fs.elapsed_time(fe)
        return self._flush_ms

    def attention_launches(self):
        """Attention kernel launches per step (one per head chunk)."""
        return len(self.usp.head_chunk_ranges(max(b - a for a, b in self.plan.head_ranges), self.n_chunks))

    def close(self):
        self.graphs.clear()
        self.plan.close()
        del self.full, self.shards, self.out, self.full_out, self.ws, self.flush
        self.torch.cuda.empty_cache()


def attention_roofline(w, attn_ms_step, n_launch, pk, pk_kind):
    """The attention kernel against the bf16 tensor-core peak: FLOP of one
    launch (4*B*H_launch*T'^2*D) over its average duration."""
    flop = float(w.attention_flop)
    achieved = flop / (attn_ms_step / 1e3) / 1e12  # the launches of a step run back to back
    peak_key = "bf16_tflops_sustained"
    return {"bound": "tensor", "achieved": achieved, "peak": pk[peak_key], "unit": "TFLOP/s",
            "frac": achieved / pk[peak_key], "peak_source": f"{peak_key} ({pk_kind})",
            "frac_of_burst_peak": achieved / pk["bf16_tflops"], "attention_ms_per_step": attn_ms_step,
            "launch_ms": attn_ms_step / n_launch}


# The other workloads of the benchmark, each measured on its own in the same
# run (1 GPU): name -> (workload, head chunks).
CONFIG_SWEEP = (
    ("tiny_chunks1", W.TINY, 1),
    ("tiny_chunks2", W.TINY, 2),
    ("vit", W.VIT, 1),
    ("chunked", W.CHUNKED, 3),
    ("chunked_chunks1", W.CHUNKED, 1),
    ("hybrid", W.HYBRID, 1),
)


def measure_config(usp, torch, dev, w, n_chunks, steps, warmup, pk, pk_kind, min_seconds=0.6, max_passes=200):
    """One workload's step timed in passes of `steps` graph replays until
    `min_seconds` of device time (so that the clock sampler sees the load);
    reports the median pass. Block FLOP/s counts the whole step (scatter,
    exchange, attention, gather); attention FLOP/s the attention kernels."""
    bb = BlockBench(usp, torch, dev, w, n_chunks, steps, seed=w.seed)
    try:
        bb.prepare(warmup)
        clocks = ClockSampler(dev.index or 0)
        clocks.start()
        passes, spent = [], 0.0
        while (spent < min_seconds * 1e3 or len(passes) < 3) and len(passes) < max_passes:
            ms, attn, launches = bb.timed_pass()
            passes.append((ms, statistics.mean(attn), launches))
            spent += ms
        clk = clocks.stop()
        assert usp.device_status() == 0, "a device-side wait ran out"
        ms = statistics.median(p[0] for p in passes) / steps
        attn = statistics.median(p[1] for p in passes)
        flop = float(w.attention_flop)
        entry = {"workload": w.name, "dtype": w.dtype, "num_chunks": n_chunks,
                 "head_chunks": [list(c) for c in usp.head_chunk_ranges(
                     max(b - a for a, b in bb.plan.head_ranges), n_chunks)],
                 "ms_per_step": ms, "attention_ms_per_step": attn,
                 "block_tflops": flop / (ms / 1e3) / 1e12, "attention_tflops": flop / (attn / 1e3) / 1e12,
                 "gpu_launches_per_step": passes[0][2] // steps,
                 "timing": f"median of {len(passes)} passes of {steps} CUDA-graph steps",
                 "l2": "flushed (512 MiB write, subtracted) before every step" if bb.small
                       else "inputs larger than L2", "clocks": clk}
        if w.dtype != "fp32":
            entry["block_frac_sustained"] = entry["block_tflops"] / pk["bf16_tflops_sustained"]
            entry["block_frac_burst"] = entry["block_tflops"] / pk["bf16_tflops"]
            entry["roofline"] = attention_roofline(w, attn, bb.attention_launches(), pk, pk_kind)
        return entry
    finally:
        bb.close()


def run_ours(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from ulysses_sequence_attention_sp_b200 import usp

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    n_chunks = args.num_chunks or w.num_chunks[0]
    pk, pk_kind = peaks()

    def barrier():
        if world > 1:
            dist.barrier()

    bb = BlockBench(usp, torch, dev, w, n_chunks, args.steps, seed=w.seed + 7919 * rank, graph=not args.no_graph,
                    kernel=args.attention_kernel)
    bb.prepare(args.warmup)
    # timed region: exactly K steps, attention kernels bracketed by their own events
    clocks = ClockSampler(local_rank)
    clocks.start()
    ms_total, attn_ms, launches = bb.timed_pass(barrier)
    clk = clocks.stop()
    assert usp.device_status() == 0, "a device-side wait ran out"

    ms_max, attn_ms_max = reduce_max([ms_total, statistics.mean(attn_ms)], world, dev)
    ms_step = ms_max / args.steps
    flop = float(w.attention_flop)
    value = job_throughput(flop, args.steps, ms_max, world)

    line = None
    if rank == 0:
        n_launch_attn = bb.attention_launches()
        roof = attention_roofline(w, attn_ms_max, n_launch_attn, pk, pk_kind)
        # algorithmic bytes of one launch: q, k, v read once and o written once
        roof["traffic"] = recorded_traffic("attention", 4 * w.tensor_bytes / n_launch_attn)
        roof["kernel"] = "attn_pp_kernel (tcgen05, two query tiles per CTA), one launch per head chunk"
        roof["peak_source"] += "; the kernel runs inside a long step loop"
        roof = {k: roof[k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic", "kernel",
                                     "peak_source", "frac_of_burst_peak", "attention_ms_per_step", "launch_ms")}
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {**workload_config(w, n_chunks, world), "cuda_graph": bool(bb.graphs),
                   "attention_kernel": args.attention_kernel},
            "roofline": roof,
            "gpu_launches": int(launches),
            "clocks": clk,
        }
    # end-to-end through the public API with host buffers: every step copies
    # its q/k/v in from pinned host memory and its output back. The copies run
    # as a double-buffered pipeline on their own streams (inputs of step i+1
    # come in and the output of step i-1 goes out while step i computes), the
    # way a caller streaming batches from host memory would run them; the
    # timed region spans the first input copy to the last output copy.
    if not args.no_e2e:
        stream = torch.cuda.current_stream()
        host_in = [torch.from_numpy(x.view(np.int16) if w.dtype == "bf16" else x).pin_memory() for x in bb.storage]
        host_out = torch.empty(bb.full_out.shape,
                               dtype=torch.int16 if w.dtype == "bf16" else torch.float32).pin_memory()
        k_e2e = max(2, args.steps)
        fins = [bb.full, [torch.empty_like(x) for x in bb.full]]
        fouts = [bb.full_out, torch.empty_like(bb.full_out)]
        s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()

        def e2e_run(nsteps):
            ev = lambda: torch.cuda.Event()  # noqa: E731
            h2d_done = [ev() for _ in range(nsteps)]
            comp_done = [ev() for _ in range(nsteps)]
            d2h_done = [ev() for _ in range(nsteps)]
            s_h2d.wait_stream(stream)
            s_d2h.wait_stream(stream)
            for i in range(nsteps):
                b = i % 2
                with torch.cuda.stream(s_h2d):
                    if i >= 2:
                        s_h2d.wait_event(comp_done[i - 2])  # step i-2 has read input buffer b
                    for h, d in zip(host_in, fins[b]):
                        d.view(h.dtype).copy_(h, non_blocking=True)
                    h2d_done[i].record(s_h2d)
                stream.wait_event(h2d_done[i])
                if i >= 2:
                    stream.wait_event(d2h_done[i - 2])  # output buffer b has been copied out
                bb.step(fins[b], fouts[b])
                comp_done[i].record(stream)
                with torch.cuda.stream(s_d2h):
                    s_d2h.wait_event(comp_done[i])
                    host_out.copy_(fouts[b].view(host_out.dtype), non_blocking=True)
                    d2h_done[i].record(s_d2h)
            stream.wait_stream(s_d2h)
            stream.wait_stream(s_h2d)

        e2e_run(2)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_run(k_e2e)
        e1.record(stream)
        torch.cuda.synchronize()
        (te_max,) = reduce_max([e0.elapsed_time(e1)], world, dev)
        if rank == 0:
            line["e2e"] = {"value": job_throughput(flop, k_e2e, te_max, world), "unit": "TFLOP/s",
                           "h2d_bytes_per_step": 3 * w.tensor_bytes, "d2h_bytes_per_step": w.tensor_bytes,
                           "steps": k_e2e, "ms_per_step": te_max / k_e2e,
                           "pipeline": "double-buffered: H2D of step i+1 and D2H of step i-1 overlap step i "
                                       "on separate streams; timed from the first H2D to the last D2H"}
        del host_in, host_out, fins, fouts
    storage = bb.storage
    headline_entry = None
    if rank == 0:
        headline_entry = {"workload": w.name, "dtype": w.dtype, "num_chunks": n_chunks,
                          "ms_per_step": ms_step, "attention_ms_per_step": attn_ms_max,
                          "block_tflops": value / world, "attention_tflops": line["roofline"]["achieved"],
                          "block_frac_sustained": value / world / pk["bf16_tflops_sustained"],
                          "block_frac_burst": value / world / pk["bf16_tflops"],
                          "roofline": {k: line["roofline"][k] for k in ("achieved", "frac", "frac_of_burst_peak")},
                          "timing": "the headline's own timed region (this line's value)", "clocks": clk}
    bb.close()

    if rank == 0 and world == 1 and not args.no_configs:
        configs = {w.name.split("-")[0]: headline_entry}
        for name, cw, cn in CONFIG_SWEEP:
            if cw.name == w.name and cn == n_chunks:
                continue
            configs[name] = measure_config(usp, torch, dev, cw, cn, args.steps, args.warmup, pk, pk_kind)
        c3, c1 = configs.get("chunked"), configs.get("chunked_chunks1")
        if c3 and c1:
            configs["chunk_overlap"] = {
                "what": "the head-chunked workload's block with num_chunks=3 (chunk c+1's exchange on the "
                        "plan's second stream under chunk c's attention) against num_chunks=1, same run",
                "speedup_block": c1["ms_per_step"] / c3["ms_per_step"],
                "ms_per_step_chunks3": c3["ms_per_step"], "ms_per_step_chunks1": c1["ms_per_step"]}
        line["configs"] = configs
    if rank == 0 and world == 1 and not args.no_reshard:
        line["reshard"] = reshard_measurement(usp, torch, dev, pk, pk_kind)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, rows, secs = oracle_rows_tflops(w, storage, 12.0, 1 << 30)
        line["cpu_baseline"] = {
            "value": tf, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"float64 oracle attention on {rows} query rows of batch 0, head 0 against all {w.tokens} "
                      f"keys ({secs:.1f} s); rows are independent, so TFLOP/s carries over to the workload"}
    return line


def reshard_measurement(usp, torch, dev, pk, pk_kind):
    """Bandwidth of the ragged layout kernels on the reshard workload
    (T=32768, H=32, D=128, P=8, bf16): algorithmic bytes = read + write of
    every moved element; inputs larger than L2; median of 7 timed reps."""
    w = W.RESHARD
    plan = usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix)
    S = w.tensor_bytes
    full = torch.empty(plan.full_shape(), dtype=torch.bfloat16, device=dev).normal_()
    seq = [plan.empty_seq_shards() for _ in range(3)]
    for s in seq:
        usp.scatter_sequence(plan, full, out=s)
    heads = [plan.empty_head_shards() for _ in range(3)]
    full2 = torch.empty_like(full)
    # row collectives over the same split: P full replicas / P full partials
    rows_local = [x.view(w.batch, x.shape[1], w.heads, w.head_dim) for x in seq[2]]
    rows_full = [torch.empty_like(full) for _ in range(w.world)]
    rows_out = [torch.empty_like(x) for x in rows_local]
    ops = {
        "seq_to_head_qkv": (lambda: usp.ulysses_seq_to_head(plan, seq, out=heads), 6 * S),
        "head_to_seq": (lambda: usp.ulysses_head_to_seq(plan, heads[:1], out=seq[:1]), 2 * S),
        "scatter_sequence": (lambda: usp.scatter_sequence(plan, full, out=seq[1]), 2 * S),
        "gather_sequence": (lambda: usp.gather_sequence(plan, seq[1], out=full2), 2 * S),
        "sp_head_slice": (lambda: usp.sp_head_slice(plan, full, out=heads[2]), 2 * S),
        "sp_head_gather": (lambda: usp.sp_head_gather(plan, heads[2], out=full2), 2 * S),
        "all_gather_rows": (lambda: usp.all_gather_rows(plan, rows_local, out=rows_full), (1 + w.world) * S),
        "reduce_scatter_rows": (lambda: usp.reduce_scatter_rows(plan, rows_full, out=rows_out), (w.world + 1) * S),
    }
    vec_plan = usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix)
    vec_plan.set_pack_mode("vector")
    ops["seq_to_head_qkv_vector"] = (lambda: usp.ulysses_seq_to_head(vec_plan, seq, out=heads), 6 * S)
    res = {}
    for name, (fn, nbytes) in ops.items():
        for _ in range(2):
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(7)]
        for a, b in evs:
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        ms = statistics.median(a.elapsed_time(b) for a, b in evs)
        res[name] = {"GB/s": nbytes / ms / 1e6, "ms": ms, "frac": nbytes / ms / 1e6 / pk["hbm_gbs"]}
    # bit-exact round trip of the whole exchange on this data
    usp.ulysses_head_to_seq(plan, heads, out=seq)
    torch.cuda.synchronize()
    plan.close()
    vec_plan.close()
    s2h = res["seq_to_head_qkv"]
    return {"workload": w.name, "ops": res, "peak_gbs": pk["hbm_gbs"], "peak_source": f"hbm_gbs ({pk_kind})",
            "roofline": {"bound": "hbm", "achieved": s2h["GB/s"], "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": s2h["frac"], "traffic": recorded_traffic("pack_tma", 6 * S),
                         "traffic_note": "ncu capture on the video workload's q/k/v pack, scaled by algorithmic bytes",
                         "kernel": "pack_tma_kernel (seq_to_head of q, k, v, the default TMA pack)"}}


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(json.dumps({"error": f"--gpus {args.gpus} but WORLD_SIZE {world}"}), flush=True)
        sys.exit(2)
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return
    if w.name == W.RESHARD.name:
        print(json.dumps({"error": "the reshard workload is measured inside every run (key 'reshard')"}))
        sys.exit(2)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    line = run_ours(args, w, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
