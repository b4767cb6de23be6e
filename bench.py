"""Benchmark of the CSA2 sparse-attention decode path on one B200 (or N, one
process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]

Workloads (--workload):
  decode    (default) the 1M-token-context 8-layer step: plan [full, reindex,
            reuse, reuse, reindex, reuse, reuse, reuse], pool 16,384, top-512
            + 128-token window, int8 indexer 64x128, FP4 KV d512, 64 query heads.
  tiny      the same path at context 4096 with the small shapes (indexer 4x64,
            pool 1024, top-64, 8 query heads, KV d128), one full layer.
  single    one full layer at context 131,072 with the 1M step's shapes.
  ragged    32 sequences of 32K-262K rows in 64-row pages (shuffled page
            table), one full layer each: queries/s.
  verify    a speculative-verify block of 5 causal queries at the end of the
            1M context, all 8 layers, the index scan shared by the block.
  window    the decode step with a local window cache per layer: every layer
            reads its 128-token window from its own bf16 ring, every reuse
            layer reads the FP4 cache of the layer whose selection it reuses.
  prefill   2048 causal queries at positions 260096-262143 of a 262,144-row
            context: int8 index GEMM, per-query top-512 over the prefix,
            attention.  queries/s and the index stage's int8 TOP/s.
  quantize  the FP4 cache write of 1,048,576 bf16 rows of d512.

A step is one pass of the whole hot path over one batch of synthetic input,
through the library's C ABI (csa2_layer_plan for the decode workloads),
captured once per input replica in a CUDA graph.  Inputs are seeded (synth/),
resident in HBM, and rotate over device replicas whose caches together exceed
the L2, so no step reads another step's data from L2.  The JSON line gives:
  value       units per second (median of 5 repeats of exactly --steps
              timed steps, each repeat bracketed by a barrier and a device
              synchronisation, max over ranks);
  steps100    the same with at least 100 replays per repeat;
  hbm         algorithmic bytes per step, GB/s and fractions of 8 TB/s and of
              the measured copy peak;
  roofline    the dominant kernel alone (the index-score stream), its
              algorithmic bytes per launch over its CUDA-event time;
  e2e         the same metric through the C ABI with host buffers: one pinned
              host-to-device copy of the step's inputs, the plan call, one
              device-to-host copy of its outputs, every step;
  cpu_baseline  the CPU oracle (oracle/) on this host's cores, on a bounded
              sample of the same workload.
With N GPUs every rank runs its own copy of the workload: weak scaling, no
data-path collective.  Rank 0 prints one JSON line.

--impl reference times the CPU oracle on the same workload on this host's
cores; there is no other implementation of this path to compare against.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "decode steps/s and HBM GB/s (% of B200 roofline) at 1M-token context"
WL = synth.C2_1M_PLAN
WL_VERIFY = synth.scaled(synth.C2_1M_PLAN, name="verify_5q_ctx1048576_8layer",
                         prefill=(5, int(synth.C2_1M_PLAN.lengths()[0]) - 5))
WL_WINDOW = synth.scaled(synth.C2_1M_PLAN, name="window_ctx1048576_8layer")
# workloads whose layers read their window from a local bf16 ring and whose
# reuse layers share the global FP4 cache of the layer they reuse
LOCAL_WINDOW_WORKLOADS = ("window",)
# name: (workload, metric, unit, units per step, group the queries of a sequence)
DECODE_WORKLOADS = {
    "decode": (WL, METRIC, "steps/s", 1, False),
    "tiny": (synth.C0_TINY, "decode steps/s and us per step at 4096-token context (small shapes)", "steps/s", 1,
             False),
    "single": (synth.C1_SINGLE, "decode steps/s and HBM GB/s at 131072-token context", "steps/s", 1, False),
    "ragged": (synth.C3_RAGGED, "decode queries/s and HBM GB/s over 32 paged ragged sequences (32K-262K rows)",
               "queries/s", 32, False),
    "verify": (WL_VERIFY, "verify blocks/s (5 queries sharing one index scan) at 1M-token context",
               "blocks/s", 1, True),
    "window": (WL_WINDOW, "decode steps/s at 1M-token context with per-layer local window caches (bf16) and "
                          "reuse layers sharing the global FP4 KV", "steps/s", 1, False),
}
METRIC_PREFILL = "prefill-chunk queries/s and index int8 TOP/s (2048 causal queries, 262144 context)"
WL_PREFILL = synth.C4_PREFILL
METRIC_QUANT = "FP4 cache write rows/s and HBM GB/s (1,048,576 bf16 rows of d512 -> E2M1 + E4M3)"
QUANT_SAMPLE_ROWS = 65536
# DRAM bytes (read + write) of one index-score launch on the 1M decode
# workload, from one ncu capture of this kernel (its summary is kept with the
# profiles); None when that kernel changed after the capture.  The last
# capture (134,281,728 B read + 3,837,440 B written) predates the prologue
# that records which boxes of each group's last tile are visible.
K1_TRAFFIC_BYTES = {"decode": None}
# DRAM bytes (read + write) of one FP4 cache-write launch of 1,048,576 bf16
# rows of d512, from one ncu capture (summary kept with the profiles).
QUANT_TRAFFIC_BYTES = 1_073_840_384 + 268_985_856
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
NOMINAL_HBM_GBS = 8000.0
REPEATS = 5
MAX_REPLICAS = 256


def peaks() -> dict:
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "src": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "src": "fallback"}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def device_facts(dev) -> dict:
    """The device's L2 size, and a read-only HBM stream rate measured here:
    torch.sum over 2 GiB of fp32 (larger than L2), best of 5 after one warm-up,
    CUDA events.  It is a reference beside the copy peak, not the roofline's
    denominator.  Runs after the timed region; anything that fails is None."""
    out = {"l2_bytes": None, "read_only_gbs": None, "read_only_how": "torch.sum of 2 GiB fp32, best of 5"}
    if getattr(dev, "type", None) != "cuda":
        return out
    out["l2_bytes"] = l2_bytes(dev)
    try:
        x = torch.ones(1 << 29, dtype=torch.float32, device=dev)
        best = None
        for i in range(6):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            x.sum()
            b.record()
            b.synchronize()
            if i:
                ms = a.elapsed_time(b)
                best = ms if best is None else min(best, ms)
        del x
        if best:
            out["read_only_gbs"] = (1 << 31) / (best / 1e3) / 1e9
    except Exception:
        pass
    return out


def l2_bytes(dev) -> int:
    try:
        return int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0)) or (126 << 20)
    except Exception:
        return 126 << 20


# ----------------------------------------------------------------- distributed plumbing
def dist_init(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- clocks during the timed region
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu):
        self.gpu = gpu
        self.proc = None
        self.lines: list[str] = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self) -> dict:
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
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_id(dev) -> str:
    """nvidia-smi id of a torch device (its UUID; the index as a fallback)."""
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev.index or 0)


# ----------------------------------------------------------------- timing
def time_replays(graphs, n: int, stream, world: int, dev) -> float:
    """Milliseconds per replay over exactly n replays (rotating over the
    graphs), bracketed by a barrier and a device synchronisation on both
    sides; the max over ranks."""
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for i in range(n):
            graphs[i % len(graphs)].replay()
        b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(a.elapsed_time(b), world, dev) / n


def timed_block(graphs, steps: int, stream, world: int, dev) -> dict:
    """REPEATS repeats of exactly `steps` replays, then REPEATS repeats of at
    least 100 replays: per-step milliseconds of each repeat and the medians."""
    per = [time_replays(graphs, steps, stream, world, dev) for _ in range(REPEATS)]
    n100 = max(100, steps)
    per100 = [time_replays(graphs, n100, stream, world, dev) for _ in range(REPEATS)]
    return {"ms": statistics.median(per), "ms_all": per, "ms100": statistics.median(per100), "ms100_all": per100,
            "replays100": n100}


def load_for(graphs, seconds: float, stream):
    """Untimed replays for about `seconds`, so the clock samples see the GPU
    under this load before the timed repeats."""
    t0 = time.time()
    i = 0
    while time.time() - t0 < seconds:
        with torch.cuda.stream(stream):
            for _ in range(32):
                graphs[i % len(graphs)].replay()
                i += 1
        torch.cuda.synchronize()


def kernels_in(fn, stream) -> int | None:
    """How many of the library's kernels one call of fn launches, counted by
    torch's profiler (CUPTI) outside the timed region; None if unavailable."""
    try:
        from torch.profiler import ProfilerActivity, profile
        torch.cuda.synchronize()
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            with torch.cuda.stream(stream):
                fn()
            torch.cuda.synchronize()
        n = 0
        for ev in prof.events():
            if getattr(ev, "device_type", None) is not None and "csa2" in ev.name and "Memset" not in ev.name:
                if str(ev.device_type).endswith("CUDA"):
                    n += 1
        return n or None
    except Exception:
        return None


# ----------------------------------------------------------------- the CPU oracle
class OracleQuery:
    """One query of a decode workload through the CPU oracle: every layer of
    the plan (full index, pool and selection; reindex; reuse; attention).

    Every step function is the oracle's own (oracle/); this class sequences
    them the way decode_layer_plan does and times them.  The full layer's scan
    of every key row can run on T host threads, each scoring a contiguous
    slice of the rows with the oracle's index_scores; BLAS gets T threads.
    The FP4 rows of each layer's attention set are stored by the oracle's
    quantiser before the timed run (the cache write is not part of a step).
    With ``local``, every layer reads its window from its own ring of bf16
    rows (the oracle's kv_rows_local_window) and every reuse layer reads the
    FP4 rows of the layer whose selection it reuses."""

    def __init__(self, wl, query: int, local: bool = False):
        import oracle as O
        self.O, self.wl = O, wl
        sq, qp = wl.query_positions()
        self.seq, self.pos = int(sq[query]), int(qp[query])
        n = self.pos + 1
        self.rings = None
        if local:   # ring of the query's sequence: position p in row p mod R
            R, a = wl.window, max(0, n - wl.window)
            self.rings = []
            for l in range(len(wl.modes)):
                ring = np.zeros((R, wl.attn_dim), np.float64)
                ring[np.arange(a, n) % R] = synth.local_kv_values(wl, l, self.seq, a, n)
                self.rings.append(ring)
        self.layers = []
        for l, mode in enumerate(wl.modes):
            d = {"q_attn": synth.attn_query(wl, l, query)}
            if mode != synth.REUSE:
                d["keys"] = synth.index_keys(wl, l, self.seq, 0, n)
                d["q"], d["w"] = synth.index_query(wl, l, query)
            self.layers.append(d)
        self.codes = []
        pool = sel = None
        scores0 = O.index_scores(self.layers[0]["q"], self.layers[0]["w"], self.layers[0]["keys"])
        for l, mode in enumerate(wl.modes):                 # FP4 rows the step reads (untimed)
            d = self.layers[l]
            if mode == synth.FULL:
                pool = O.top_k_positions(scores0, np.arange(n), wl.pool)
                sel = O.top_k_positions(scores0[pool], pool, wl.topk)
            elif mode == synth.REINDEX:
                _, sel = O.reindex(d["q"], d["w"], d["keys"], pool, wl.topk)
            if mode != synth.REUSE or not local:
                src = l   # the layer whose FP4 cache this layer reads
            S = O.attention_set(sel, self.pos, wl.window)
            codes = np.zeros((n, wl.attn_dim // 2), np.uint8)
            scales = np.zeros((n, wl.attn_dim // 32), np.uint8)
            x = np.concatenate([synth.kv_values(wl, src, self.seq, int(r), int(r) + 1) for r in S])
            codes[S], scales[S] = O.fp4_quantize(x)
            self.codes.append((codes, scales))

    def _scores(self, d, threads: int, lo: int, hi: int):
        O = self.O
        if threads <= 1:
            return O.index_scores(d["q"], d["w"], d["keys"][lo:hi])
        from concurrent.futures import ThreadPoolExecutor
        cuts = [lo + (hi - lo) * i // threads for i in range(threads + 1)]
        with ThreadPoolExecutor(threads) as ex:
            parts = list(ex.map(lambda i: O.index_scores(d["q"], d["w"], d["keys"][cuts[i]:cuts[i + 1]]),
                                range(threads)))
        return np.concatenate(parts)

    def run(self, threads: int = 1, f: int = 1, slice_i: int = 0) -> float:
        """Seconds of one query.  With f > 1 the full layer's scan is timed
        on slice slice_i of f equal slices of the rows and scaled by f (its
        pool and selection then use the full scores, computed untimed)."""
        from threadpoolctl import threadpool_limits
        O, wl, pos = self.O, self.wl, self.pos
        n = pos + 1
        t_total = 0.0
        with threadpool_limits(threads):
            pool = sel = None
            for l, mode in enumerate(wl.modes):
                d = self.layers[l]
                t0 = time.perf_counter()
                if mode == synth.FULL:
                    if f > 1:
                        lo, hi = n * slice_i // f, n * (slice_i + 1) // f
                        self._scores(d, threads, lo, hi)
                        t_total += (time.perf_counter() - t0) * f
                        s = self._scores(d, threads, 0, n)
                        t0 = time.perf_counter()
                    else:
                        s = self._scores(d, threads, 0, n)
                    pool = O.top_k_positions(s, np.arange(n), wl.pool)
                    sel = O.top_k_positions(s[pool], pool, wl.topk)
                elif mode == synth.REINDEX:
                    _, sel = O.reindex(d["q"], d["w"], d["keys"], pool, wl.topk)
                S = O.attention_set(sel, pos, wl.window)
                codes, scales = self.codes[l]
                if self.rings is None:
                    kv = O.fp4_dequant(codes[S], scales[S], wl.attn_dim)
                else:
                    kv = O.kv_rows_local_window(S, pos, wl.window, codes, scales, wl.attn_dim, self.rings[l])
                O.sparse_attention(d["q_attn"], kv)
                t_total += time.perf_counter() - t0
        return t_total


def oracle_sample(key: str):
    """(OracleQuery, queries of a step it stands for, description) of a
    decode workload's bounded CPU sample."""
    wl, _, _, units, _ = DECODE_WORKLOADS[key]
    sq, qp = wl.query_positions()
    if key == "ragged":
        q = 0
        return OracleQuery(wl, q), 1, f"query 0 of the 32 (sequence 0, {int(qp[q]) + 1} rows), scaled to queries/s"
    if key == "verify":
        q = len(qp) - 1
        return OracleQuery(wl, q), len(qp), "the block's last query (whole 1M prefix) through all 8 layers, x5 per block"
    if key in LOCAL_WINDOW_WORKLOADS:
        return (OracleQuery(wl, 0, local=True), 1,
                f"one whole {len(wl.modes)}-layer decode step of the same workload (window rows from the local rings)")
    return OracleQuery(wl, 0), 1, f"one whole {len(wl.modes)}-layer decode step of the same workload"


def cpu_baseline_decode(key: str, budget_s: float = 60.0) -> dict:
    oq, per_unit, sample = oracle_sample(key)
    cores = host_cores()
    t_all = oq.run(cores)
    out = {"value": 1.0 / (t_all * per_unit), "unit": DECODE_WORKLOADS[key][2], "cores": cores, "kind": "oracle",
           "sample": sample, "cpu_model": cpu_model(),
           "how": "full layer's key scan split over the host threads (oracle index_scores per slice), BLAS on "
                  "the same threads; everything else single-threaded numpy"}
    if key in ("tiny", "single"):
        t1 = oq.run(1)
        out["value_1core"] = 1.0 / (t1 * per_unit)
    return out


# ----------------------------------------------------------------- reference arm (the oracle)
def run_reference(args, rank, world):
    if rank != 0:
        return
    key = args.workload
    if key == "prefill":
        return run_reference_prefill(args)
    if key == "quantize":
        return run_reference_quantize(args)
    wl, metric, unit, units, _ = DECODE_WORKLOADS[key]
    oq, per_unit, sample = oracle_sample(key)
    cores = host_cores()
    t = oq.run(cores)
    budget = 180.0 / (args.steps + args.warmup)   # warm-up + timed steps near 3 minutes
    f = 1
    while t / f > budget and f < 1024 and wl.lengths().max() > 16384:
        f *= 2
    for i in range(args.warmup):
        oq.run(cores, f, i % f)
    ts = [oq.run(cores, f, i % f) * per_unit for i in range(args.steps)]
    sec = statistics.median(ts)
    v = 1.0 / sec
    if f > 1:
        sample += f"; the full layer's scan timed on 1/{f} of the key rows (rotating) and scaled by {f}"
    line = {"impl": "reference", "metric": metric, "value": v, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int64,f64", "data": "synthetic",
            "config": config_dict(key, wl),
            "cpu_baseline": {"value": v, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample,
                             "cpu_model": cpu_model()},
            "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_dict(key: str, wl, n_rep: int | None = None, rep_bytes: int | None = None) -> dict:
    lens = wl.lengths()
    sq, qp = wl.query_positions()
    d = {"workload": wl.name, "ctx": int(lens.max()), "batch": len(lens), "queries": len(qp),
         "layer_plan": ",".join(synth.MODE_NAMES[m] for m in wl.modes), "pool": wl.pool, "topk": wl.topk,
         "window": wl.window, "indexer": f"int8 {wl.idx_heads}x{wl.idx_dim}, w int8",
         "kv": f"FP4 E2M1 d{wl.attn_dim}, E4M3 per 32", "q_heads": wl.attn_heads,
         "parallelism": "one workload per rank"}
    if wl.page_rows:
        d["paged"] = f"{wl.page_rows}-row pages, shuffled page table; lengths {int(lens.min())}..{int(lens.max())}, " \
                     f"sum {int(lens.sum())}"
    if key == "verify":
        d["verify_block"] = f"{len(qp)} causal queries at positions {int(qp[0])}..{int(qp[-1])}, one sequence, " \
                            "index scan shared (group_queries)"
    if key in LOCAL_WINDOW_WORKLOADS:
        d["local_window"] = (f"every layer's last {wl.window} positions from its own bf16 ring of {wl.window} rows; "
                             "reuse layers read the FP4 cache of the layer they reuse")
    if n_rep is not None:
        d["l2"] = (f"inputs rotate over {n_rep} device replicas ({rep_bytes * n_rep / 1e6:.0f} MB of caches, "
                   f"> L2)")
    return d


# ----------------------------------------------------------------- decode workloads
def run_decode(args, rank, world, local):
    from kv_cache_decode_csa2_b200 import csa2 as B
    from kv_cache_decode_csa2_b200 import workloads as W
    key = args.workload
    wl, metric, unit, units, group = DECODE_WORKLOADS[key]
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    t_setup = time.time()
    status = B.new_status(dev)
    base = W.build_decode(wl, dev, status, local_window=key in LOCAL_WINDOW_WORKLOADS)
    rep_bytes = W.state_bytes(base)
    n_rep = args.replicas or max(4, min(MAX_REPLICAS, math.ceil(2 * l2_bytes(dev) / max(rep_bytes, 1))))
    replicas = [base] + [W.clone_decode(base, dev) for _ in range(n_rep - 1)]
    plans = [W.decode_plan(r, group) for r in replicas]
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for p in plans:                       # ordinary calls first (one-time kernel set-up)
            p.run(stream)
    torch.cuda.synchronize()
    B.check_status(status)
    for p in plans:
        B.check_status(p.status)
    alg_bytes, parts = W.algorithmic_bytes(replicas[0])
    n_kernels = kernels_in(lambda: plans[0].run(stream), stream)
    graphs = []
    for p in plans:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            p.run(stream)
        graphs.append(g)
    torch.cuda.synchronize()
    setup_s = time.time() - t_setup

    # ---- timed steps
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            graphs[i % n_rep].replay()
    torch.cuda.synchronize()
    with ClockSampler(gpu_id(dev)) as clk:
        load_for(graphs, 0.4, stream)
        tb = timed_block(graphs, args.steps, stream, world, dev)
    ms_step = tb["ms"]
    value = world * units / (ms_step / 1e3)
    for p in plans:
        B.check_status(p.status)

    # ---- dominant kernel alone: the full layer's index-score stream (scores
    # only), launches rotating over the replicas, captured in a CUDA graph
    f = [r.layers[0] for r in replicas]
    nq = len(base.query_pos)
    ws = [torch.empty(B.lib().csa2_index_full_workspace(nq, base.max_ctx, 0, 0), dtype=torch.uint8, device=dev)
          for _ in f]
    k_per_graph = 4 * n_rep if n_rep <= 16 else n_rep

    def k1_call(i):
        r = i % n_rep
        B.csa2_index_full(f[r].q, f[r].w, f[r].keys, replicas[r].pos_dev, base.max_ctx,
                          seq_of_query=replicas[r].seq_dev, ws=ws[r], status=status, stream=stream)
    with torch.cuda.stream(stream):
        for i in range(n_rep):
            k1_call(i)
    torch.cuda.synchronize()
    kg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(kg, stream=stream):
        for i in range(k_per_graph):
            k1_call(i)
    k_reps = max(3, 200 // k_per_graph)
    with torch.cuda.stream(stream):
        kg.replay()
    k_ms = time_replays([kg], k_reps, stream, world, dev) / k_per_graph
    B.check_status(status)
    del kg
    sq, qp = base.seq_of_query, base.query_pos
    last = {}
    for s_, p_ in zip(sq, qp):
        last[int(s_)] = max(last.get(int(s_), -1), int(p_))
    key_bytes = sum(p + 1 for p in last.values()) * wl.idx_dim + nq * (wl.idx_heads * wl.idx_dim + wl.idx_heads)
    pk = peaks()
    achieved = key_bytes / (k_ms / 1e3) / 1e9

    # ---- end to end through the C ABI with host buffers: one pinned H2D of the
    # step's inputs, the plan call, one D2H of its outputs
    r0, p0 = replicas[0], plans[0]
    in_host = r0.inbuf.cpu().pin_memory()
    out_host = torch.empty(r0.outbuf.shape, dtype=r0.outbuf.dtype, pin_memory=True)

    def e2e_step():
        r0.inbuf.copy_(in_host, non_blocking=True)
        p0.run(stream)
        out_host.copy_(r0.outbuf, non_blocking=True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            e2e_step()
    torch.cuda.synchronize()
    e_steps = max(args.steps, 20)
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(e_steps):
            e2e_step()
        e1.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / e_steps
    B.check_status(p0.status)

    gbs = alg_bytes / (ms_step / 1e3) / 1e9
    line = {"metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": config_dict(key, wl, n_rep, rep_bytes),
            "timing": {"repeats": REPEATS, "steps_per_repeat": args.steps, "ms_per_step_each": tb["ms_all"],
                       "statistic": "median"},
            "steps100": {"replays_per_repeat": tb["replays100"], "repeats": REPEATS, "ms_per_step": tb["ms100"],
                         "ms_per_step_each": tb["ms100_all"], "value": world * units / (tb["ms100"] / 1e3)},
            "hbm": {"algorithmic_bytes_per_step": alg_bytes, "parts": parts, "achieved_gbs": gbs,
                    "frac_of_8tbs": gbs / NOMINAL_HBM_GBS, "frac_of_measured": gbs / pk["hbm_gbs"]},
            "roofline": {"kernel": "index_score_kernel (full-mode index scoring of every key row, scores only)",
                         "bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / pk["hbm_gbs"], "peak_src": pk["src"], "ms_per_launch": k_ms,
                         "bytes_per_launch": key_bytes, "traffic": K1_TRAFFIC_BYTES.get(key)},
            "e2e": {"value": world * units / (e_ms / 1e3), "unit": unit, "h2d_bytes_per_step": in_host.numel(),
                    "d2h_bytes_per_step": out_host.numel(),
                    "path": "one pinned H2D of the packed inputs + csa2_layer_plan + one D2H of the packed outputs, "
                            "no graph"},
            "gpu_launches": (n_kernels or 0) * args.steps, "kernels_per_step": n_kernels,
            "clocks": clk.summary(), "setup_s": round(setup_s, 1)}
    if key == "verify":
        line["verify"] = {"queries_per_block": nq, "us_per_block": ms_step * 1e3,
                          "key_bytes_per_query": key_bytes / nq,
                          "key_passes": "groups of 4 queries share each key tile: 2 passes per 5-query block"}
    line["device"] = device_facts(dev)
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_decode(key)
    del graphs
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- prefill chunk
def peak_int8_tops() -> dict:
    """Dense int8 tensor peak: the measured bf16 GEMM rate times the nominal
    int8/bf16 ratio (4.5 / 2.25 PFLOP/s); the fallback bf16 figure if the
    measured file is absent."""
    try:
        with open(PEAKS_FILE) as f:
            bf16 = float(json.load(f)["bf16_tflops"])
        return {"tops": 2.0 * bf16, "src": "measured bf16 x 2 (nominal int8/bf16 ratio)"}
    except Exception:
        return {"tops": 2.0 * 1590.0, "src": "fallback bf16 x 2 (nominal int8/bf16 ratio)"}


PREFILL_SAMPLE = "the chunk's last query (its whole 262,144-row prefix), through the oracle"


def oracle_prefill_query_seconds(wl, host, qp, threads: int) -> float:
    """Seconds the oracle takes for one query of the chunk (the last, whose
    prefix is the whole context): its scores (split over `threads` host
    threads by row slices), its top-k and its attention.  The FP4 rows of
    its attention set are stored, untimed, in between."""
    import oracle as O
    from concurrent.futures import ThreadPoolExecutor

    from threadpoolctl import threadpool_limits
    keys = synth.index_keys(wl, 0, 0)
    i = len(qp) - 1
    pos = int(qp[i])
    n = pos + 1
    with threadpool_limits(threads):
        t0 = time.perf_counter()
        if threads > 1:
            cuts = [n * j // threads for j in range(threads + 1)]
            with ThreadPoolExecutor(threads) as ex:
                s_ = np.concatenate(list(ex.map(
                    lambda j: O.index_scores(host[1][i], host[2][i], keys[cuts[j]:cuts[j + 1]]), range(threads))))
        else:
            s_ = O.index_scores(host[1][i], host[2][i], keys[:n])
        sel_ = O.top_k_positions(s_, np.arange(n), wl.topk)
        S = O.attention_set(sel_, pos, wl.window)
        t1 = time.perf_counter()
        x = np.concatenate([synth.kv_values(wl, 0, 0, int(r_), int(r_) + 1) for r_ in S])
        c_, sc_ = O.fp4_quantize(x)
        t2 = time.perf_counter()
        O.sparse_attention(host[3][i], O.fp4_dequant(c_, sc_, wl.attn_dim))
        t3 = time.perf_counter()
    return (t1 - t0) + (t3 - t2)


def run_reference_prefill(args):
    from kv_cache_decode_csa2_b200 import workloads as W
    wl = WL_PREFILL
    host = W.prefill_host(wl)
    _, qp = wl.query_positions()
    cores = host_cores()
    ts = [oracle_prefill_query_seconds(wl, host, qp, cores) for _ in range(max(1, min(args.steps, 5)))]
    v = 1.0 / statistics.median(ts)
    line = {"impl": "reference", "metric": METRIC_PREFILL, "value": v, "unit": "queries/s", "n_gpus": args.gpus,
            "steps": len(ts), "warmup": 0, "ms_per_step": 1e3 / v, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int64,f64", "data": "synthetic",
            "config": {"workload": wl.name},
            "cpu_baseline": {"value": v, "unit": "queries/s", "cores": cores, "kind": "oracle",
                             "sample": PREFILL_SAMPLE, "cpu_model": cpu_model()},
            "e2e": {"value": v, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_prefill(args, rank, world, local):
    from kv_cache_decode_csa2_b200 import csa2 as B
    from kv_cache_decode_csa2_b200 import workloads as W
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    wl = WL_PREFILL
    if args.prefill_queries != wl.prefill[0]:   # the last N queries of the chunk (profiling captures)
        n_ctx = int(wl.lengths()[0])
        wl = synth.scaled(wl, prefill=(args.prefill_queries, n_ctx - args.prefill_queries))
    t_setup = time.time()
    sq, qp = wl.query_positions()
    nq = len(qp)
    host = W.prefill_host(wl)
    n = host[0]
    status = B.new_status(dev)
    n_rep = args.replicas or 4
    reps = [W.prefill_replica(wl, host, dev, status) for _ in range(n_rep)]
    pos_dev = torch.from_numpy(qp.astype(np.int32)).to(dev)
    seq_dev = torch.from_numpy(sq.astype(np.int32)).to(dev)
    sel = torch.empty((nq, wl.topk), dtype=torch.int32, device=dev)
    cnt = torch.empty((nq,), dtype=torch.int32, device=dev)
    out = torch.empty((nq, wl.attn_heads, wl.attn_dim), dtype=torch.bfloat16, device=dev)
    L = B.lib()
    ws_i = torch.empty(L.csa2_index_full_workspace(nq, n, 0, wl.topk), dtype=torch.uint8, device=dev)
    ws_a = torch.empty(L.csa2_sparse_attn_workspace(nq, wl.attn_heads, wl.attn_dim, wl.topk, wl.window),
                       dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def index(r):
        B.csa2_index_full(r["q"], r["w"], r["keys"], pos_dev, n, seq_of_query=seq_dev, K=wl.topk, sel_idx=sel,
                          sel_cnt=cnt, status=status, ws=ws_i, stream=stream)

    def attend(r):
        B.csa2_sparse_attn_fp4(r["qa"], r["codes"], r["scales"], pos_dev, sel, out, sel_cnt=cnt,
                               seq_of_query=seq_dev, window=wl.window, status=status, ws=ws_a, stream=stream)

    with torch.cuda.stream(stream):
        for r in reps:                         # ordinary calls first (one-time kernel set-up)
            index(r)
            attend(r)
    torch.cuda.synchronize()
    B.check_status(status)
    n_kernels = kernels_in(lambda: (index(reps[0]), attend(reps[0])), stream)
    graphs, igraphs = [], []
    for r in reps:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            index(r)
            attend(r)
        graphs.append(g)
        gi = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gi, stream=stream):
            index(r)
        igraphs.append(gi)
    torch.cuda.synchronize()
    setup_s = time.time() - t_setup
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            graphs[i % n_rep].replay()
    torch.cuda.synchronize()
    with ClockSampler(gpu_id(dev)) as clk:
        load_for(graphs, 0.4, stream)
        per = [time_replays(graphs, args.steps, stream, world, dev) for _ in range(REPEATS)]
    ms = statistics.median(per)
    ms_index = statistics.median([time_replays(igraphs, max(3, args.steps), stream, world, dev)
                                  for _ in range(REPEATS)])
    B.check_status(status)
    ops = sum((int(p) + 1) * wl.idx_heads * wl.idx_dim * 2 for p in qp)
    tops = ops / (ms_index / 1e3) / 1e12
    pk = peak_int8_tops()

    # end to end: the chunk's queries in from pinned host memory, outputs back
    r0 = reps[0]
    h2d = [r0["q"], r0["w"], r0["qa"]]
    h2d_host = [t.cpu().pin_memory() for t in h2d]
    d2h = [out, sel]
    d2h_host = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in d2h]
    e_steps = max(3, args.steps // 2)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(e_steps):
            for hsrc, ddst in zip(h2d_host, h2d):
                ddst.copy_(hsrc, non_blocking=True)
            index(r0)
            attend(r0)
            for dsrc, hdst in zip(d2h, d2h_host):
                hdst.copy_(dsrc, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / e_steps
    B.check_status(status)

    line = {"metric": METRIC_PREFILL, "value": world * nq / (ms / 1e3), "unit": "queries/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": wl.name, "ctx": n, "queries": nq, "first_pos": int(qp[0]), "topk": wl.topk,
                       "window": wl.window, "indexer": f"int8 {wl.idx_heads}x{wl.idx_dim}, w int8",
                       "kv": f"FP4 E2M1 d{wl.attn_dim}, E4M3 per 32", "q_heads": wl.attn_heads,
                       "l2": f"inputs rotate over {n_rep} device replicas (~180 MB each)",
                       "parallelism": "one chunk per rank"},
            "timing": {"repeats": REPEATS, "steps_per_repeat": args.steps, "ms_per_step_each": per,
                       "statistic": "median"},
            "roofline": {"kernel": "index stage: grouped index_score_kernel + per-query top-512",
                         "bound": "tensor", "achieved": tops, "peak": pk["tops"], "unit": "TOP/s (int8)",
                         "frac": tops / pk["tops"], "peak_src": pk["src"], "ms_per_launch": ms_index,
                         "ops_per_launch": ops, "traffic": None},
            "e2e": {"value": world * nq / (e_ms / 1e3), "unit": "queries/s",
                    "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in h2d_host),
                    "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in d2h_host),
                    "path": "pinned H2D + csa2_index_full + csa2_sparse_attn_fp4 + D2H, no graph"},
            "gpu_launches": (n_kernels or 0) * args.steps, "kernels_per_step": n_kernels,
            "clocks": clk.summary(), "setup_s": round(setup_s, 1)}
    if rank == 0 and not args.no_cpu_baseline:
        cores = host_cores()
        sec = oracle_prefill_query_seconds(wl, host, qp, cores)
        line["cpu_baseline"] = {"value": 1.0 / sec, "unit": "queries/s", "cores": cores, "kind": "oracle",
                                "sample": PREFILL_SAMPLE, "cpu_model": cpu_model()}
    del graphs, igraphs
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- FP4 cache write
def quant_bytes_per_row(D: int) -> int:
    """Algorithmic bytes of storing one bf16 row of D values as FP4: the row
    read (2 D) and the codes (D / 2) and scales (D / 32) written."""
    return 2 * D + D // 2 + D // 32


def oracle_quant_rows_per_s(wl, rows: int, threads: int) -> tuple[float, str]:
    """The oracle's FP4 quantiser on the first ``rows`` rows of layer 0 (bf16
    values), split into `threads` row slices on host threads."""
    import oracle as O
    from concurrent.futures import ThreadPoolExecutor

    from threadpoolctl import threadpool_limits
    x = synth.round_to_bf16(synth.kv_values(wl, 0, 0, 0, rows))
    cuts = [rows * j // threads for j in range(threads + 1)]
    with threadpool_limits(1):
        t0 = time.perf_counter()
        if threads > 1:
            with ThreadPoolExecutor(threads) as ex:
                list(ex.map(lambda j: O.fp4_quantize(x[cuts[j]:cuts[j + 1]]), range(threads)))
        else:
            O.fp4_quantize(x)
        t = time.perf_counter() - t0
    return rows / t, f"{rows} bf16 rows of d{wl.attn_dim} of the same cache, split over {threads} host threads"


def run_reference_quantize(args):
    wl = WL
    cores = host_cores()
    vs = [oracle_quant_rows_per_s(wl, QUANT_SAMPLE_ROWS, cores)[0] for _ in range(max(1, min(args.steps, 5)))]
    v = statistics.median(vs)
    line = {"impl": "reference", "metric": METRIC_QUANT, "value": v, "unit": "rows/s", "n_gpus": args.gpus,
            "steps": len(vs), "warmup": 0, "ms_per_step": 1e3 * (1 << 20) / v, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "fp4_cache_write_1m_rows_d512"},
            "cpu_baseline": {"value": v, "unit": "rows/s", "cores": cores, "kind": "oracle",
                             "sample": f"{QUANT_SAMPLE_ROWS} rows per step", "cpu_model": cpu_model()},
            "e2e": {"value": v, "unit": "rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_quantize(args, rank, world, local):
    """A step stores one layer's latent KV at the 1M context, 1,048,576 bf16
    rows of d512 (1 GiB, far beyond L2), as FP4 codes and E4M3 scales with
    csa2_fp4_quantize (one launch), replayed in a CUDA graph."""
    from kv_cache_decode_csa2_b200 import csa2 as B
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    wl = WL
    t_setup = time.time()
    n, D = int(wl.lengths()[0]), wl.attn_dim
    status = B.new_status(dev)
    x = torch.empty((n, D), dtype=torch.bfloat16, device=dev)
    step_rows = 1 << 17
    for a in range(0, n, step_rows):
        b = min(n, a + step_rows)
        x[a:b] = torch.from_numpy(synth.kv_values(wl, 0, 0, a, b)).to(dev).to(torch.bfloat16)
    codes = torch.empty((n, D // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((n, D // 32), dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        B.csa2_fp4_quantize(x, codes, scales, status=status, stream=stream)
    torch.cuda.synchronize()
    B.check_status(status)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        B.csa2_fp4_quantize(x, codes, scales, status=status, stream=stream)
    torch.cuda.synchronize()
    setup_s = time.time() - t_setup
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g.replay()
    torch.cuda.synchronize()
    with ClockSampler(gpu_id(dev)) as clk:
        load_for([g], 0.4, stream)
        per = [time_replays([g], args.steps, stream, world, dev) for _ in range(REPEATS)]
    ms = statistics.median(per)
    B.check_status(status)
    per_row = quant_bytes_per_row(D)
    achieved = n * per_row / (ms / 1e3) / 1e9
    pk = peaks()

    # end to end: the rows in from pinned host memory, the codes and scales back
    e_steps = 3
    xh = x.cpu().pin_memory()
    ch = torch.empty(codes.shape, dtype=codes.dtype, pin_memory=True)
    sh = torch.empty(scales.shape, dtype=scales.dtype, pin_memory=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(e_steps):
            x.copy_(xh, non_blocking=True)
            B.csa2_fp4_quantize(x, codes, scales, status=status, stream=stream)
            ch.copy_(codes, non_blocking=True)
            sh.copy_(scales, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / e_steps
    B.check_status(status)

    line = {"metric": METRIC_QUANT, "value": world * n / (ms / 1e3), "unit": "rows/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16->fp4", "data": "synthetic",
            "config": {"workload": "fp4_cache_write_1m_rows_d512", "rows": n, "d": D, "input": "bf16",
                       "l2": "1 GiB of input per step, far beyond L2", "parallelism": "one cache per rank"},
            "timing": {"repeats": REPEATS, "steps_per_repeat": args.steps, "ms_per_step_each": per,
                       "statistic": "median"},
            "roofline": {"kernel": "fp4_quantize_kernel<bf16>", "bound": "hbm", "achieved": achieved,
                         "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
                         "peak_src": pk["src"], "ms_per_launch": ms, "bytes_per_launch": n * per_row,
                         "traffic": QUANT_TRAFFIC_BYTES if n == 1 << 20 and D == 512 else None},
            "e2e": {"value": world * n / (e_ms / 1e3), "unit": "rows/s",
                    "h2d_bytes_per_step": xh.numel() * xh.element_size(),
                    "d2h_bytes_per_step": ch.numel() + sh.numel(),
                    "path": "pinned H2D + csa2_fp4_quantize + D2H, no graph"},
            "gpu_launches": args.steps, "kernels_per_step": 1, "clocks": clk.summary(),
            "setup_s": round(setup_s, 1)}
    if rank == 0 and not args.no_cpu_baseline:
        cores = host_cores()
        v, sample = oracle_quant_rows_per_s(wl, QUANT_SAMPLE_ROWS, cores)
        line["cpu_baseline"] = {"value": v, "unit": "rows/s", "cores": cores, "kind": "oracle", "sample": sample,
                                "cpu_model": cpu_model()}
    del g
    if rank == 0:
        print(json.dumps(line), flush=True)


WORKLOAD_NAMES = list(DECODE_WORKLOADS) + ["prefill", "quantize"]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="csa2", choices=["csa2", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default="decode", choices=WORKLOAD_NAMES)
    ap.add_argument("--prefill-queries", type=int, default=WL_PREFILL.prefill[0],
                    help="prefill workload: the last N queries of the chunk (a smaller case for profiling)")
    ap.add_argument("--replicas", type=int, default=0,
                    help="device copies of the state rotated between steps (default: enough to exceed 2x L2)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, local = dist_init(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        elif args.workload == "prefill":
            run_prefill(args, rank, world, local)
        elif args.workload == "quantize":
            run_quantize(args, rank, world, local)
        else:
            run_decode(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
