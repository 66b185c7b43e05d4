"""Benchmark of the paged MLA decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole path over one decode batch: the split-KV scheduler
(mla_get_metadata), then mla_decode_paged, which launches the fused decode kernel and the
log-sum-exp combine of split sequences.  The default workload is the memory-bound decode batch
(batch 64, s_q 1, 16 query heads on one latent head, d = 576, dv = 512, 64-token pages,
cache lengths uniform in [1, 4096] from seed 0); its metric is HBM GB/s over the
algorithmic bytes (every valid token's latent row read once, plus q, out, lse and the
addressed block-table entries and lengths).  Compute-bound workloads report TFLOP/s over
2 * (576 + 512) flops per (query row, visible key).

Timing: W warm-up steps, then exactly K steps replayed from one CUDA graph, bracketed by
a barrier and a device synchronisation on both sides and timed with CUDA events on the
launching stream; the maximum over ranks is reported.  Steps rotate over enough copies
of the inputs that everything a step reads was last touched more than one L2 (126 MB)
ago.  The decode kernel is timed two ways: a second graph of K decode launches alone,
back to back over the same rotating inputs and their precomputed plans, timed with one
pair of CUDA events around the whole replay (events around every launch would add their
own overhead to each kernel's time; each launch's prologue overlaps its predecessor),
and the median of at least 20 individually event-timed decode + combine runs, each after
a 256 MB write that evicts L2 (the scheduler is timed the same way, separately).

On one GPU the line also carries `per_workload`: the same measurements (without the
end-to-end leg, with a ~2 s oracle sample) for every workload of the specification.

N > 1 (torchrun, one process per GPU): sequences are independent, so every rank decodes
its own batch with no data-path collective (weak scaling); only the timing is reduced.

--impl reference times the fp64 CPU oracle (the correctness reference) on the host cores,
each step a bounded sample of whole sequences of the same workload.
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
import time
from typing import Optional

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_mla_decode_11_b200 import workloads as W  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# nominal B200 figures, reported beside the measured-peak fractions
NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}
# sources of the decode kernel the library picks for a workload (16 rows or fewer per latent
# head: the warp-MMA kernel; whole 128-row blocks with g a multiple or divisor of 64: the
# CTA-pair tcgen05 kernel; other shapes: the 64-row tcgen05 kernel); a committed ncu summary
# stays valid while these are unchanged
KERNEL_SOURCES = {
    "decode_mma16_kernel": ["common.cuh", "decode_mma.cu"],
    "decode_wide_kernel": ["common.cuh", "decode_wide.cu"],
    "decode_pair_kernel": ["common.cuh", "decode_pair.cu"],
    "decode_fp8_kernel": ["common.cuh", "decode_fp8.cu"],
    "absorb_gemm_kernel": ["common.cuh", "absorb.cu"],
}


def decode_kernel_for(rows_per_kv_head: int, g: int = 0) -> str:
    if rows_per_kv_head <= 16:
        return "decode_mma16_kernel"
    if rows_per_kv_head % 128 == 0 and g > 0 and (g % 64 == 0 or 64 % g == 0):
        return "decode_pair_kernel"
    return "decode_wide_kernel"


# ----------------------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------------------
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), \
        int(os.environ.get("WORLD_SIZE", "1"))


class RankGroup:
    """One process per GPU (torchrun environment).  Sequences are independent, so the data
    path has no collective; the group only aligns the ranks (barrier) and reduces the timings
    (maximum over ranks).  `backend` is "nccl" on GPUs, "gloo" for the CPU tests."""

    def __init__(self, backend: str, device: torch.device):
        self.rank, self.local_rank, self.world = dist_env()
        self.device = device
        self.pg = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.pg = dist

    def _sync(self):
        if self.device.type == "cuda":
            torch.cuda.synchronize(self.device)

    def barrier(self):
        if self.pg is not None:
            t = torch.zeros(1, device=self.device)
            self.pg.all_reduce(t)
        self._sync()

    def max(self, v: float) -> float:
        if self.pg is None:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()
            self.pg = None


def aggregate_throughput(units_per_rank: float, world: int, seconds_per_step: float) -> float:
    """Whole-job throughput: the units every rank processed in one step over the slowest
    rank's step time (weak scaling: each rank decodes its own batch)."""
    return units_per_rank * world / seconds_per_step


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


def _code_only(src: str) -> str:
    """CUDA source without comments and with whitespace collapsed: what the compiler sees."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def kernel_source_hash(kernel: str) -> str:
    """Hash of the code (not the comments) of the sources a decode kernel is built from."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "paged_mla_decode_11_b200", "csrc", name)) as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kernel: str, summary: Optional[str] = None):
    """DRAM bytes per decode launch (per pass of both products for the absorption) from the
    committed ncu summary, if it was taken on the current sources of that kernel; None
    otherwise."""
    path = os.path.join(ROOT, "profiles", summary or f"decode_{workload}_ncu.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_t = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    m_h = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", text)
    if not m_t or not m_h or m_h.group(1) != kernel_source_hash(kernel):
        return None
    return float(m_t.group(1))


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the GPU is loaded."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            ident = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", ident, "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons = [], [], set()
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# Workloads with the latent cache in the FP8 format (E4M3 codes + one fp32 scale per token and
# latent head), decoded by mla_decode_paged_fp8; the name maps to the bf16 workload it stores.
FP8_WORKLOADS = {"memory_bound_fp8": "memory_bound"}
FP8_TOKEN_BYTES = 576 + 4
# Token-level sparse decode (mla_decode_sparse): each query token keeps SPARSE_TOPK listed key
# positions of its sequence.
SPARSE_WORKLOADS = {"sparse": (W.SPARSE, W.SPARSE_TOPK)}
ALL_WORKLOADS = list(W.WORKLOADS) + list(FP8_WORKLOADS) + list(SPARSE_WORKLOADS)


def workload_spec(name):
    """(Workload, kind) of a bench workload name; kind is "bf16", "fp8" or "sparse"."""
    if name in FP8_WORKLOADS:
        return W.WORKLOADS[FP8_WORKLOADS[name]], "fp8"
    if name in SPARSE_WORKLOADS:
        return SPARSE_WORKLOADS[name][0], "sparse"
    return W.WORKLOADS[name], "bf16"


def make_workload_inputs(name, seed):
    w, kind = workload_spec(name)
    if kind == "fp8":
        return W.make_inputs_fp8(w, seed=seed)
    if kind == "sparse":
        return W.make_inputs_sparse(w, SPARSE_WORKLOADS[name][1], seed=seed)
    return W.make_inputs(w, seed=seed)


def workload_work(x, w, kind="bf16"):
    if kind == "sparse":
        return W.sparse_work(x["row_ptr"], x["col_idx"], x["cache_seqlens"].tolist(), w.s_q, w.h_q, w.h_kv,
                             w.causal)
    lens = x["cache_seqlens"].tolist()
    nbytes, flops = W.algorithmic_work(lens, w.s_q, w.h_q, w.h_kv, w.causal,
                                       token_bytes=FP8_TOKEN_BYTES if kind == "fp8" else None)
    return nbytes, flops


def metric_of(w_name):
    w_name = FP8_WORKLOADS.get(w_name, w_name)
    if w_name in ("compute_bound", "causal_mtp"):
        return "TFLOP/s", "tensor"
    return "GB/s", "hbm"


METRIC = "paged MLA decode on 1 B200: HBM GB/s (mem-bound), TFLOPS (compute-bound)"


def workload_config(w, kind="bf16"):
    lens = w.seqlens
    cache = ("FP8 cache (E4M3 codes of the bf16 ~N(0,1) pool, one fp32 scale per token)" if kind == "fp8"
             else "bf16 q/cache ~N(0,1)")
    if kind == "sparse":
        cache += (f", key lists: min({W.SPARSE_TOPK}, visible length) distinct uniform positions per "
                  f"query token, sorted, CSR (seed 1)")
    return {"workload": f"{w.name}{' fp8' if kind == 'fp8' else ''}: batch={w.batch}, s_q={w.s_q}, "
                        f"h_q={w.h_q}, h_kv={w.h_kv}, d=576, dv=512, page 64, seqlens {lens}, causal={w.causal}, "
                        f"scale={w.scale:.6g}, {cache}, random block_table over one pool, seed 0"}


# ----------------------------------------------------------------------------------------
# CPU oracle timing (our arm's cpu_baseline and the reference arm)
# ----------------------------------------------------------------------------------------
def oracle_sample(x, w, seqs):
    import numpy as np
    import oracle
    rows = [(b, s, h) for b in seqs for s in range(w.s_q) for h in range(w.h_q)]
    rows = np.array(rows, dtype=np.int32)
    fp8 = "k8" in x
    t0 = time.perf_counter()
    if "row_ptr" in x:
        oracle.mla_decode_rows_sparse(x["q"], x["k_cache"], x["block_table"], x["cache_seqlens"], x["row_ptr"],
                                      x["col_idx"], rows, dv=512, softmax_scale=w.scale, causal=w.causal)
        dt = time.perf_counter() - t0
        nb = fl = 0
        rp = x["row_ptr"]
        for b in seqs:
            i0, i1 = b * w.s_q, (b + 1) * w.s_q
            sub_rp = rp[i0:i1 + 1] - rp[i0]
            bb, ff = W.sparse_work(sub_rp, x["col_idx"][int(rp[i0]):int(rp[i1])], [int(x["cache_seqlens"][b])],
                                   w.s_q, w.h_q, w.h_kv, w.causal)
            nb, fl = nb + bb, fl + ff
        return dt, nb, fl
    if fp8:
        oracle.mla_decode_rows_fp8(x["q"], x["k8"], x["k_scale"], x["block_table"], x["cache_seqlens"], rows,
                                   dv=512, softmax_scale=w.scale, causal=w.causal)
    else:
        oracle.mla_decode_rows(x["q"], x["k_cache"], x["block_table"], x["cache_seqlens"], rows, dv=512,
                               softmax_scale=w.scale, causal=w.causal)
    dt = time.perf_counter() - t0
    lens = [int(x["cache_seqlens"][b]) for b in seqs]
    nb, fl = W.algorithmic_work(lens, w.s_q, w.h_q, w.h_kv, w.causal, token_bytes=FP8_TOKEN_BYTES if fp8 else None)
    return dt, nb, fl


def pick_sample(x, w, seconds):
    """Whole sequences, cycling from a start index, totalling about `seconds` of oracle work."""
    dt, nb, fl = oracle_sample(x, w, [0])
    per_flop = dt / max(fl, 1)
    order = list(range(w.batch))
    chosen, acc = [], 0.0
    for b in order:
        f = sequence_flops(x, w, b)
        chosen.append(b)
        acc += f * per_flop
        if acc >= seconds:
            break
    return chosen


def sequence_flops(x, w, b):
    """Algorithmic flops of sequence b's query rows (its key lists for the sparse decode)."""
    if "row_ptr" in x:
        rp = x["row_ptr"]
        i0, i1 = b * w.s_q, (b + 1) * w.s_q
        return W.sparse_work(rp[i0:i1 + 1] - rp[i0], x["col_idx"][int(rp[i0]):int(rp[i1])],
                             [int(x["cache_seqlens"][b])], w.s_q, w.h_q, w.h_kv, w.causal)[1]
    return W.algorithmic_work([int(x["cache_seqlens"][b])], w.s_q, w.h_q, w.h_kv, w.causal)[1]


def cpu_baseline(x, w, unit, seconds=10.0):
    """The oracle as it stands on the host cores: whole sequences worth about `seconds` of
    work; a batch the oracle finishes sooner is decoded again until that much has run."""
    import oracle
    seqs = pick_sample(x, w, seconds)
    tot_t = tot_b = tot_f = 0.0
    runs = 0
    while runs == 0 or (tot_t < 0.8 * seconds and runs < 200):
        dt, nb, fl = oracle_sample(x, w, seqs)
        tot_t, tot_b, tot_f, runs = tot_t + dt, tot_b + nb, tot_f + fl, runs + 1
    val = tot_b / tot_t / 1e9 if unit == "GB/s" else tot_f / tot_t / 1e12
    return {"value": val, "unit": unit, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{len(seqs)} of {w.batch} sequences (all query rows) decoded {runs} time(s), "
                      f"{tot_t:.1f} s of fp64 oracle work"}


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return
    import oracle
    w, kind = workload_spec(args.workload)
    x = make_workload_inputs(args.workload, 0)
    unit, _ = metric_of(args.workload)
    budget = 90.0 / max(args.steps + args.warmup, 1)
    per_step = min(2.0, max(0.05, budget))
    # samples are consecutive runs of whole sequences, cycling over the batch
    dt1, _, fl1 = oracle_sample(x, w, [0])
    per_flop = dt1 / max(fl1, 1)
    cursor = 0

    def next_sample():
        nonlocal cursor
        seqs, acc = [], 0.0
        while acc < per_step and len(seqs) < 64 * w.batch:  # the batch cycled if it is quick
            b = cursor % w.batch
            f = sequence_flops(x, w, b)
            seqs.append(b)
            acc += f * per_flop
            cursor += 1
        return seqs

    for _ in range(args.warmup):
        oracle_sample(x, w, next_sample())
    tot_t = tot_b = tot_f = 0.0
    nseq = 0
    for _ in range(args.steps):
        s = next_sample()
        dt, nb, fl = oracle_sample(x, w, s)
        tot_t += dt
        tot_b += nb
        tot_f += fl
        nseq += len(s)
    val = tot_b / tot_t / 1e9 if unit == "GB/s" else tot_f / tot_t / 1e12
    sample = (f"each step: consecutive whole sequences of the batch, cycled (budget {per_step:.2f} s, "
              f"measured {tot_t / args.steps:.2f} s of fp64 oracle work per step), "
              f"{nseq} sequences over {args.steps} steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, kind),
        "cpu_baseline": {"value": val, "unit": unit, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": val, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------------------
FLUSH_BYTES = 256 * 1024 * 1024  # L2-flush write between individually timed runs (> 126 MB L2)
ISOLATED_RUNS = 20


def measure(name, args, dev, group, rank, world, with_e2e, cpu_seconds):
    """Times one workload: the whole step (scheduler, decode, combine) from a CUDA graph of
    K steps, the decode kernel from a graph of K back-to-back decode launches, and the
    median of individually event-timed decode + combine runs (and scheduler runs) with an
    L2-flush write before each.  Optionally the end-to-end leg through the public API and
    the CPU oracle's throughput on a bounded sample.  Returns a dict of results."""
    from paged_mla_decode_11_b200 import ops
    barrier, max_over_ranks = group.barrier, group.max
    w, kind = workload_spec(name)
    fp8, sparse = kind == "fp8", kind == "sparse"
    # rows per tile: every query token is a tile of its own in the sparse decode
    R = w.h_q // w.h_kv if sparse else w.rows_per_kv_head
    x = make_workload_inputs(name, args.seed + rank)
    if fp8:
        del x["k_cache"]  # the bf16 source of the codes stays on the host
        per_rep = x["k8"].numel() + x["k_scale"].numel() * 4
    else:
        per_rep = x["k_cache"].numel() * 2
    nbytes, flops = workload_work(x, w, kind)
    unit, bound = metric_of(name)
    n_rep = max(2, math.ceil(1.5 * L2_BYTES / per_rep) + 1)

    reps = []
    for r in range(n_rep):
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
        if r > 0:
            d = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
        nparts = ops.num_parts_for(ops.device_sm_count(dev), R, w.h_kv)
        d["ws"] = ops.new_workspace(ops.workspace_size(w.batch, w.s_q, w.h_q, w.h_kv, nparts), dev)
        d["out"] = torch.empty(w.batch, w.s_q, w.h_q, 512, dtype=torch.bfloat16, device=dev)
        d["lse"] = torch.empty(w.batch, w.h_q, w.s_q, dtype=torch.float32, device=dev)
        reps.append(d)

    def plan(d, **kw):
        if sparse:
            return ops.get_mla_metadata_csr(d["row_ptr"], R, w.h_kv)
        return ops.get_mla_metadata(d["cache_seqlens"], R, w.h_kv, **kw)

    def decode(d, tile, splits, kernel_only=False):
        if sparse:
            ops.mla_decode_sparse(d["q"], d["k_cache"], d["block_table"], d["cache_seqlens"], d["row_ptr"],
                                  d["col_idx"], 512, tile, splits, softmax_scale=w.scale, causal=w.causal,
                                  workspace=d["ws"], out=d["out"], lse=d["lse"], skip_combine=kernel_only)
            return
        if fp8:
            ops.mla_decode_paged_fp8(d["q"], d["k8"], d["k_scale"], d["block_table"], d["cache_seqlens"], 512, tile,
                                     splits, softmax_scale=w.scale, causal=w.causal, workspace=d["ws"],
                                     out=d["out"], lse=d["lse"], skip_combine=kernel_only)
            return
        ops.mla_decode_paged(d["q"], d["k_cache"], d["block_table"], d["cache_seqlens"], 512, tile,
                             splits, softmax_scale=w.scale, causal=w.causal, workspace=d["ws"],
                             out=d["out"], lse=d["lse"], skip_combine=kernel_only, kernel=args.kernel)

    def step(d):
        tile, splits = plan(d)
        decode(d, tile, splits)

    # eager warm-up (first launches, allocator, tensor maps), then graph capture
    for i in range(max(args.warmup, 3)):
        step(reps[i % n_rep])
    torch.cuda.synchronize(dev)

    stream = torch.cuda.Stream(device=dev)
    warm_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(warm_graph, stream=stream):
        for i in range(max(args.warmup, 3)):
            step(reps[i % n_rep])
    # the timed graph: K whole steps back to back (no events between kernels, so each
    # kernel's launch overlaps its predecessor); a second graph of K decode launches alone,
    # on plans computed beforehand, gives the decode kernel's back-to-back duration
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(args.steps):
            step(reps[i % n_rep])
    with torch.cuda.stream(stream):
        for d in reps:
            d["plan"] = plan(d)
    kgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(kgraph, stream=stream):
        for i in range(args.steps):
            decode(reps[i % n_rep], *reps[i % n_rep]["plan"], kernel_only=True)
    # the scheduler and the combine, each timed alone the same way (the combine merges the
    # partials the decode-only graph leaves in each copy's workspace)
    mgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(mgraph, stream=stream):
        for i in range(args.steps):
            d = reps[i % n_rep]
            plan(d)
    cgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(cgraph, stream=stream):
        for i in range(args.steps):
            d = reps[i % n_rep]
            tile, splits = d["plan"]
            if sparse:  # one-position lists: out [b * s_q, 1, h_q, 512], lse in [b, s_q, h_q] order
                ops.mla_combine(splits, 1, w.h_q, w.h_kv, tile.shape[0], d["ws"],
                                d["out"].view(w.batch * w.s_q, 1, w.h_q, 512),
                                d["lse"].view(w.batch * w.s_q, w.h_q, 1))
            else:
                ops.mla_combine(splits, w.s_q, w.h_q, w.h_kv, tile.shape[0], d["ws"], d["out"], d["lse"])
    torch.cuda.synchronize(dev)
    graph.replay()  # first replay uploads the graph; not timed
    kgraph.replay()
    mgraph.replay()
    cgraph.replay()
    torch.cuda.synchronize(dev)

    sampler = ClockSampler(dev.index)
    # keep the GPU loaded for ~1 s before timing so the sampled clocks describe the load
    t_end = time.perf_counter() + 1.0
    while time.perf_counter() < t_end:
        warm_graph.replay()
        torch.cuda.synchronize(dev)
    barrier()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        graph.replay()
        end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()

    def graph_time(g):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            g.replay()
            b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) * 1e-3 / args.steps

    kernel_s = max_over_ranks(graph_time(kgraph))
    sched_s = max_over_ranks(graph_time(mgraph))
    combine_s = max_over_ranks(graph_time(cgraph))

    # Individually timed runs: before each, a 256 MB write evicts L2; then one event pair
    # around the decode kernel and its combine (on precomputed plans), and, separately, one
    # around the scheduler.  Median over the runs.
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    n_iso = max(ISOLATED_RUNS, args.steps)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(2 * n_iso)]
    with torch.cuda.stream(stream):
        for i in range(n_iso):
            d = reps[i % n_rep]
            flush.fill_(float(i))
            ev[i][0].record(stream)
            decode(d, *d["plan"])
            ev[i][1].record(stream)
        for i in range(n_iso):
            d = reps[i % n_rep]
            flush.fill_(float(i))
            ev[n_iso + i][0].record(stream)
            plan(d)
            ev[n_iso + i][1].record(stream)
    torch.cuda.synchronize(dev)
    iso_s = max_over_ranks(statistics.median(ev[i][0].elapsed_time(ev[i][1]) for i in range(n_iso)) * 1e-3)
    iso_sched_s = max_over_ranks(
        statistics.median(ev[n_iso + i][0].elapsed_time(ev[n_iso + i][1]) for i in range(n_iso)) * 1e-3)
    del flush
    clocks = sampler.stop()
    # a device-side wait that gave up invalidates the run: its kernels returned early
    for d in reps:
        if ops.query_status(d["ws"]) != ops.MLA_OK:
            raise RuntimeError(f"{name}: a device-side wait timed out during the timed region")
    elapsed = max_over_ranks(start.elapsed_time(end) * 1e-3)
    per_step = elapsed / args.steps
    total_bytes = aggregate_throughput(nbytes, world, 1.0)
    total_flops = aggregate_throughput(flops, world, 1.0)
    value = (total_bytes / per_step / 1e9) if unit == "GB/s" else (total_flops / per_step / 1e12)

    peaks, peak_kind = load_peaks()
    work = nbytes / 1e9 if bound == "hbm" else flops / 1e12
    if bound == "hbm":
        peak, nominal, r_unit = peaks["hbm_gbs"], NOMINAL_PEAKS["hbm_gbs"], "GB/s"
    else:
        peak, nominal, r_unit = peaks["bf16_tflops"], NOMINAL_PEAKS["bf16_tflops"], "TFLOP/s"
    achieved = work / kernel_s
    iso_achieved = work / iso_s
    # the summaries were taken with the library's own kernel choice
    kernel_name = ("decode_fp8_kernel" if fp8 else "decode_mma16_kernel" if sparse else
                   decode_kernel_for(R, w.h_q // w.h_kv))
    traffic = recorded_traffic(name, kernel_name) if args.kernel == "auto" else None
    res = {
        "workload": name, "config": workload_config(w, kind), "unit": unit, "value": value,
        "ms_per_step": per_step * 1e3, "n_rep": n_rep, "per_rep_bytes": per_rep,
        "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": r_unit,
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_kind} ({'hbm_gbs' if bound == 'hbm' else 'bf16_tflops'})",
                     "kernel": kernel_name, "kernel_ms": kernel_s * 1e3,
                     "kernel_timing": f"average over a graph of {args.steps} back-to-back decode launches",
                     "isolated_ms": iso_s * 1e3, "isolated_achieved": iso_achieved,
                     "isolated_frac": iso_achieved / peak,
                     "isolated_timing": (f"median of {n_iso} individually event-timed decode + combine runs, "
                                         f"each after a {FLUSH_BYTES >> 20} MB L2-flush write"),
                     "frac_of_nominal": achieved / nominal, "nominal_peak": nominal,
                     "algorithmic_bytes_per_launch": nbytes, "algorithmic_flops_per_launch": flops,
                     "whole_page_bytes_per_launch": (None if sparse else
                                                     W.whole_page_bytes(x["cache_seqlens"].tolist(), w.h_kv) *
                                                     FP8_TOKEN_BYTES // (2 * 576) if fp8 else
                                                     W.whole_page_bytes(x["cache_seqlens"].tolist(), w.h_kv)),
                     "scheduler_ms": sched_s * 1e3, "scheduler_isolated_ms": iso_sched_s * 1e3,
                     "combine_ms": combine_s * 1e3},
        "clocks": clocks,
    }

    if with_e2e:
        res["e2e"] = e2e_leg(args, w, x, reps[0], dev, nparts, R, unit, total_bytes, total_flops,
                             barrier, max_over_ranks, kind)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and cpu_seconds > 0:
        res["cpu_baseline"] = cpu_baseline(x, w, unit, seconds=cpu_seconds)
    for g in (warm_graph, graph, kgraph, mgraph, cgraph):
        g.reset()
    del reps, warm_graph, graph, kgraph, mgraph, cgraph
    torch.cuda.empty_cache()
    return res


def e2e_leg(args, w, x, d0, dev, nparts, R, unit, total_bytes, total_flops, barrier, max_over_ranks, kind="bf16"):
    """End to end through the public API from pinned host buffers (the latent page pool is
    resident device state; each step sends q, block_table and cache_seqlens and reads back
    out and lse).  Two steps are in flight, as a serving loop would run them: step i+1's
    inputs go up on an upload stream and step i-1's result comes back on a download stream
    while step i's kernels run (one stream for both directions would queue each upload
    behind the previous step's download, which waits for that step's kernels); every
    step's copies and its result's arrival on the host are inside the timed region.  Each
    slot's kernel calls (scheduler, decode, combine, made through the public API) are
    recorded once in a CUDA graph and replayed, as a serving loop does to keep the host's
    per-step work small."""
    from paged_mla_decode_11_b200 import ops
    e2e_steps = min(args.steps, 50)
    fp8, sparse = kind == "fp8", kind == "sparse"
    # a step's inputs packed in one pinned buffer (q, block_table, cache_seqlens and, for the
    # sparse decode, the key lists), its results in one device buffer (out, lse): one copy
    # each way; the API reads and writes views of them
    ins = [("q", x["q"]), ("bt", x["block_table"]), ("sl", x["cache_seqlens"])]
    if sparse:
        ins += [("rp", x["row_ptr"]), ("ci", x["col_idx"])]

    def layout(specs):
        offs, n = {}, 0
        for name, shape, dtype in specs:
            offs[name] = (n, shape, dtype)
            n += (math.prod(shape) * torch.empty(0, dtype=dtype).element_size() + 255) // 256 * 256
        return offs, n

    def views(buf, offs):
        return {k: buf[o:o + math.prod(sh) * torch.empty(0, dtype=dt).element_size()].view(dt).view(sh)
                for k, (o, sh, dt) in offs.items()}

    in_offs, in_bytes = layout([(k, tuple(v.shape), v.dtype) for k, v in ins])
    out_offs, out_bytes = layout([("out", (w.batch, w.s_q, w.h_q, 512), torch.bfloat16),
                                  ("lse", (w.batch, w.h_q, w.s_q), torch.float32)])
    hin = torch.zeros(in_bytes, dtype=torch.uint8).pin_memory()
    for k, v in views(hin, in_offs).items():
        v.copy_(dict(ins)[k])
    n_lists = w.batch * w.s_q if sparse else w.batch
    kstream = torch.cuda.Stream(device=dev)   # the API launches on the current stream
    up_stream = torch.cuda.Stream(device=dev)
    down_stream = torch.cuda.Stream(device=dev)
    slots = []
    for _ in range(2):
        din = torch.empty(in_bytes, dtype=torch.uint8, device=dev)
        dout = torch.empty(out_bytes, dtype=torch.uint8, device=dev)
        sl_ = {"din": din, "dout": dout, "hout": torch.empty(out_bytes, dtype=torch.uint8).pin_memory(),
               "tile": torch.empty(nparts, ops.TILE_FIELDS, dtype=torch.int32, device=dev),
               "splits": torch.empty(n_lists + 1, dtype=torch.int32, device=dev),
               "ws": ops.new_workspace(ops.workspace_size(w.batch, w.s_q, w.h_q, w.h_kv, nparts), dev),
               "up": torch.cuda.Event(), "done": torch.cuda.Event(), "back": torch.cuda.Event()}
        sl_.update(views(din, in_offs))
        sl_.update(views(dout, out_offs))
        slots.append(sl_)

    def kernels(sl_):
        # the plan goes into this slot's buffers: the previous user of the slot (step i-2)
        # ran earlier on the same stream
        if sparse:
            tile, splits = ops.get_mla_metadata_csr(sl_["rp"], R, w.h_kv, tile_metadata=sl_["tile"],
                                                    num_splits=sl_["splits"])
            ops.mla_decode_sparse(sl_["q"], d0["k_cache"], sl_["bt"], sl_["sl"], sl_["rp"], sl_["ci"], 512, tile,
                                  splits, softmax_scale=w.scale, causal=w.causal, workspace=sl_["ws"],
                                  out=sl_["out"], lse=sl_["lse"])
        elif fp8:
            tile, splits = ops.get_mla_metadata(sl_["sl"], R, w.h_kv, tile_metadata=sl_["tile"],
                                                num_splits=sl_["splits"])
            ops.mla_decode_paged_fp8(sl_["q"], d0["k8"], d0["k_scale"], sl_["bt"], sl_["sl"], 512, tile, splits,
                                     softmax_scale=w.scale, causal=w.causal, workspace=sl_["ws"],
                                     out=sl_["out"], lse=sl_["lse"])
        else:
            tile, splits = ops.get_mla_metadata(sl_["sl"], R, w.h_kv, tile_metadata=sl_["tile"],
                                                num_splits=sl_["splits"])
            ops.flash_mla_with_kvcache(sl_["q"], d0["k_cache"], sl_["bt"], sl_["sl"], 512, tile, splits,
                                       softmax_scale=w.scale, causal=w.causal, workspace=sl_["ws"],
                                       out=sl_["out"], lse=sl_["lse"], kernel=args.kernel)

    for sl_ in slots:  # an eager call first (tensor maps, kernel attributes), then the capture
        with torch.cuda.stream(kstream):
            kernels(sl_)
        kstream.synchronize()
        sl_["graph"] = torch.cuda.CUDAGraph()
        with torch.cuda.graph(sl_["graph"], stream=kstream):
            kernels(sl_)
    torch.cuda.synchronize(dev)

    def e2e_issue(i):
        sl_ = slots[i % 2]
        with torch.cuda.stream(up_stream):
            if i >= 2:
                up_stream.wait_event(sl_["done"])  # step i-2's kernels have read this slot
            sl_["din"].copy_(hin, non_blocking=True)
            sl_["up"].record(up_stream)
        kstream.wait_event(sl_["up"])
        if i >= 2:
            kstream.wait_event(sl_["back"])      # step i-2's result has left this slot
        with torch.cuda.stream(kstream):
            sl_["graph"].replay()
        sl_["done"].record(kstream)
        with torch.cuda.stream(down_stream):
            down_stream.wait_event(sl_["done"])
            sl_["hout"].copy_(sl_["dout"], non_blocking=True)
            sl_["back"].record(down_stream)

    def e2e_run(n, e_start=None, e_end=None):
        if e_start is not None:
            e_start.record(up_stream)
        for i in range(n):
            e2e_issue(i)
            if i >= 1:
                slots[(i - 1) % 2]["back"].synchronize()  # the host has step i-1's result
        slots[(n - 1) % 2]["back"].synchronize()
        if e_end is not None:
            e_end.record(down_stream)
            e_end.synchronize()

    e2e_run(3)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2e_run(e2e_steps, e0, e1)
    barrier()
    e2e_s = max_over_ranks(e0.elapsed_time(e1) * 1e-3 / e2e_steps)
    e2e_val = (total_bytes / e2e_s / 1e9) if unit == "GB/s" else (total_flops / e2e_s / 1e12)
    for sl_ in slots:
        sl_["graph"].reset()
    h2d = in_bytes
    d2h = out_bytes
    return {"value": e2e_val, "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": e2e_s * 1e3, "steps_in_flight": 2,
            "method": "pinned host buffers; per step: the inputs packed in one buffer go up in one copy on an "
                      "upload stream, the slot's scheduler, decode and combine calls (recorded once per slot "
                      "through the public API in a CUDA graph) are replayed on views of it, out and lse come "
                      "down in one copy on a download stream; two slots, the host waiting for step i-1's "
                      "result before issuing step i+1"}


def load_for(graph, dev, seconds):
    """Replays a captured graph for about `seconds` (a loaded GPU before a timed region)."""
    t_end = time.perf_counter() + seconds
    while time.perf_counter() < t_end:
        graph.replay()
        torch.cuda.synchronize(dev)


ABSORB_TOKENS, ABSORB_HEADS = 128, 128  # the compute-bound decode batch: 128 tokens x 128 heads


def absorb_work(T, H):
    """Algorithmic bytes and flops of one absorb_query + absorb_output pass: q_nope, q_rope,
    W^UK read, q' written; o_latent, W^UV read, o written (bf16); 2 flops per multiply-add."""
    nbytes = 2 * (T * H * 128 + T * H * 64 + H * 128 * 512 + T * H * 576 + T * H * 512 + H * 128 * 512 + T * H * 128)
    flops = 2 * T * H * 128 * 512 * 2
    return nbytes, flops


def measure_absorb(args, dev, group, cpu_seconds):
    """The absorption products around the decode (query into latent space, output out of it)
    at the compute-bound decode batch: a graph of K passes over rotating input copies (more
    bytes than L2 in all), the weight and activation bytes against the HBM peak."""
    from paged_mla_decode_11_b200 import ops
    T, H = ABSORB_TOKENS, ABSORB_HEADS
    x = W.make_absorb_inputs(T, H, seed=args.seed)
    nbytes, flops = absorb_work(T, H)
    n_rep = max(2, math.ceil(1.5 * L2_BYTES / nbytes) + 1)
    reps = []
    for _ in range(n_rep):
        d = {k: v.to(dev).clone() for k, v in x.items()}
        d["q_abs"] = torch.empty(T, H, 576, dtype=torch.bfloat16, device=dev)
        d["o"] = torch.empty(T, H, 128, dtype=torch.bfloat16, device=dev)
        reps.append(d)

    def step(d):
        ops.absorb_query(d["q_nope"], d["q_rope"], d["w_uk"], out=d["q_abs"])
        ops.absorb_output(d["o_latent"], d["w_uv"], out=d["o"])

    for i in range(max(args.warmup, 3)):
        step(reps[i % n_rep])
    torch.cuda.synchronize(dev)
    stream = torch.cuda.Stream(device=dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(args.steps):
            step(reps[i % n_rep])
    graph.replay()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(dev.index)
    load_for(graph, dev, 1.0)  # the sampled clocks describe the load
    group.barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        graph.replay()
        b.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    per_step = group.max(a.elapsed_time(b) * 1e-3 / args.steps)
    graph.reset()
    peaks, peak_kind = load_peaks()
    achieved = nbytes / per_step / 1e9
    res = {
        "config": {"workload": f"absorption products: T={T} tokens, H={H} heads, W^UK and W^UV [H, 128, 512] "
                               f"bf16 ~N(0, 1/fan-in), q_nope [T, H, 128], q_rope [T, H, 64], o_latent [T, H, 512] "
                               f"~N(0,1) bf16, seed {args.seed}"},
        "unit": "GB/s", "value": achieved, "ms_per_step": per_step * 1e3,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"],
                     "traffic": recorded_traffic("absorb", "absorb_gemm_kernel", "absorb_ncu.md"),
                     "peak_source": f"{peak_kind} (hbm_gbs)", "kernel": "absorb_gemm_kernel (both products)",
                     "kernel_ms": per_step * 1e3,
                     "kernel_timing": f"average over a graph of {args.steps} passes (two launches each)",
                     "algorithmic_bytes_per_launch": nbytes, "algorithmic_flops_per_launch": flops,
                     "achieved_tflops": flops / per_step / 1e12},
        "clocks": clocks,
    }
    if cpu_seconds > 0 and not args.no_cpu_baseline:
        import oracle
        t0, runs = time.perf_counter(), 0
        while runs == 0 or time.perf_counter() - t0 < cpu_seconds:
            oracle.absorb_query(x["q_nope"].double().numpy(), x["q_rope"].double().numpy(), x["w_uk"].double().numpy())
            oracle.absorb_output(x["o_latent"].double().numpy(), x["w_uv"].double().numpy())
            runs += 1
        dt = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": runs * nbytes / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
                               "sample": f"the whole pass, {runs} time(s), {dt:.1f} s of fp64 numpy einsum (one thread)"}
    del reps
    torch.cuda.empty_cache()
    return res


MERGE_SHARDS, MERGE_BATCH, MERGE_SQ, MERGE_HQ = 8, 32, 2, 128  # the causal multi-token query shape


def measure_merge(args, dev, group, cpu_seconds):
    """The on-device step of the sequence-sharded decode: the log-sum-exp merge of the
    partials (bf16 out and fp32 lse) that the GPUs of a node exchange, here 8 shards of the
    causal multi-token query shape, their bytes read and the output written against the HBM
    peak.  (The exchange itself, one all-gather, needs several GPUs.)"""
    from paged_mla_decode_11_b200 import ops
    n, b, s_q, h_q = MERGE_SHARDS, MERGE_BATCH, MERGE_SQ, MERGE_HQ
    g = torch.Generator().manual_seed(args.seed)
    o = torch.randn(n, b, s_q, h_q, 512, generator=g).to(torch.bfloat16)
    l = torch.randn(n, b, h_q, s_q, generator=g) * 3
    rows = b * s_q * h_q
    nbytes = n * rows * (512 * 2 + 4) + rows * (512 * 2 + 4)
    n_rep = max(2, math.ceil(1.5 * L2_BYTES / nbytes) + 1)
    reps = [(o.to(dev).clone(), l.to(dev).clone(), torch.empty(b, s_q, h_q, 512, dtype=torch.bfloat16, device=dev),
             torch.empty(b, h_q, s_q, dtype=torch.float32, device=dev)) for _ in range(n_rep)]
    for i in range(max(args.warmup, 3)):
        d = reps[i % n_rep]
        ops.mla_merge_partials(d[0], d[1], out=d[2], lse=d[3])
    torch.cuda.synchronize(dev)
    stream = torch.cuda.Stream(device=dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(args.steps):
            d = reps[i % n_rep]
            ops.mla_merge_partials(d[0], d[1], out=d[2], lse=d[3])
    graph.replay()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(dev.index)
    load_for(graph, dev, 1.0)  # the sampled clocks describe the load
    group.barrier()
    a = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        graph.replay()
        e.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    per_step = group.max(a.elapsed_time(e) * 1e-3 / args.steps)
    graph.reset()
    peaks, peak_kind = load_peaks()
    achieved = nbytes / per_step / 1e9
    res = {
        "config": {"workload": f"shard merge: {n} shards' partials of batch={b}, s_q={s_q}, h_q={h_q} "
                               f"(out bf16 [n, b, s_q, h_q, 512] ~N(0,1), lse fp32 ~N(0,9)), seed {args.seed}"},
        "unit": "GB/s", "value": achieved, "ms_per_step": per_step * 1e3,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": None, "peak_source": f"{peak_kind} (hbm_gbs)",
                     "kernel": "merge_kernel", "kernel_ms": per_step * 1e3,
                     "kernel_timing": f"average over a graph of {args.steps} merge launches",
                     "algorithmic_bytes_per_launch": nbytes},
        "clocks": clocks,
    }
    if cpu_seconds > 0 and not args.no_cpu_baseline:
        import oracle
        on, ln = o.double().numpy(), l.double().numpy().transpose(0, 1, 3, 2)
        t0, runs = time.perf_counter(), 0
        while runs == 0 or time.perf_counter() - t0 < cpu_seconds:
            oracle.combine(ln, on)
            runs += 1
        dt = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": runs * nbytes / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
                               "sample": f"the whole merge, {runs} time(s), {dt:.1f} s of fp64 numpy (one thread)"}
    del reps
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    rank, local_rank, world = dist_env()
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} needs {args.gpus} processes (launch with torchrun)")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    group = RankGroup("nccl", dev)

    if args.only:
        # one supporting product alone (one GPU), e.g. as the command a profiler runs
        if world != 1:
            raise SystemExit("--only runs on one GPU")
        fn = measure_absorb if args.only == "absorb" else measure_merge
        r = fn(args, dev, group, cpu_seconds=0.0 if args.no_cpu_baseline else 2.0)
        group.close()
        print(json.dumps({"only": args.only, **r}), flush=True)
        return
    head = measure(args.workload, args, dev, group, rank, world, with_e2e=True, cpu_seconds=10.0)
    # every workload of the specification on the same line (one GPU only: at N > 1 the
    # per-rank work is the headline workload alone)
    per_workload = None
    if world == 1 and not args.no_per_workload:
        per_workload = {}
        for name in ALL_WORKLOADS:
            r = head if name == args.workload else measure(name, args, dev, group, rank, world,
                                                            with_e2e=False, cpu_seconds=2.0)
            per_workload[name] = {k: r[k] for k in ("config", "unit", "value", "ms_per_step", "roofline",
                                                    "clocks") if k in r}
            per_workload[name]["cpu_baseline"] = r.get("cpu_baseline")
        per_workload["absorb"] = measure_absorb(args, dev, group, cpu_seconds=2.0)
        per_workload["shard_merge"] = measure_merge(args, dev, group, cpu_seconds=2.0)
    group.close()
    if rank != 0:
        return
    cfg = dict(head["config"])
    cfg["l2"] = (f"inputs larger than L2: steps rotate over {head['n_rep']} copies of the inputs "
                 f"({head['per_rep_bytes'] / 1e6:.0f} MB latent pool each); isolated runs flush L2 "
                 f"with a {FLUSH_BYTES >> 20} MB write")
    cfg["parallelism"] = f"dp{world} (independent batches per GPU)"
    cfg["timing"] = (f"{args.steps} steps replayed from one CUDA graph; decode-kernel time from a graph "
                     f"of {args.steps} back-to-back decode launches on the same rotating inputs, and the "
                     f"median of individually timed decode + combine runs after an L2 flush")
    cfg["kernel"] = args.kernel
    line = {
        "metric": METRIC, "value": head["value"], "unit": head["unit"], "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": cfg, "roofline": head["roofline"],
        "cpu_baseline": head.get("cpu_baseline"), "e2e": head["e2e"],
        "gpu_launches": 3 * args.steps, "clocks": head["clocks"],
    }
    if per_workload is not None:
        line["per_workload"] = per_workload
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="memory_bound", choices=sorted(ALL_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="measure only --workload (by default one GPU also measures every workload)")
    ap.add_argument("--only", choices=["absorb", "shard_merge"],
                    help="measure one supporting product alone and print its result (one GPU)")
    ap.add_argument("--kernel", default="auto", choices=["auto", "tcgen05", "warp_mma"],
                    help="decode kernel choice (auto = the library's choice by shape)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
