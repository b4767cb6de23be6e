"""Benchmark of the CSA2 decode step: the 1M-token-context, 8-layer plan
[full, reindex, reuse, reuse, reindex, reuse, reuse, reuse].

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

A step is one pass of the whole hot path over one decode query:
  - full-mode index scoring of all 1,048,576 positions;
  - the 16,384-candidate pool and the layer's top-512;
  - two reindex layers over the pool;
  - FP4 sparse attention (512 selected + 128 window positions) in all 8 layers.
The step runs as one csa2_layer_plan call, captured once into a CUDA graph
per input replica.  Inputs are synthetic (seeded, see synth/), resident in
HBM, and rotate over 4 device replicas of the whole state: about 141 MB read
per step, 564 MB per cycle against a 126 MB L2.  With N GPUs every rank
decodes its own sequence: weak scaling, no data-path collective.  Rank 0
prints one JSON line.

--impl reference times the CPU oracle (oracle/) on the same workload, on this
host's cores; there is no other reference implementation of this path.

    python bench.py --workload prefill [--steps K] [--warmup W]

times the prefill-chunk configuration instead: 2048 causal queries at
positions 260096-262143 of a 262,144-row context, each scoring its whole
prefix with the int8 indexer, keeping its top-512 and attending to them plus
the 128-row window (one csa2_index_full and one csa2_sparse_attn_fp4 call,
captured in a CUDA graph per replica).  It prints queries/s and the int8
TOP/s of the index stage.

    python bench.py --workload quantize [--steps K] [--warmup W]

times the FP4 cache write: 1,048,576 bf16 rows of d512 (one layer's latent KV
at the 1M context) stored as E2M1 codes and E4M3 scales by
csa2_fp4_quantize, in rows/s and HBM GB/s.
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
METRIC_PREFILL = "prefill-chunk queries/s and index int8 TOP/s (2048 causal queries, 262144 context)"
WL_PREFILL = synth.C4_PREFILL
METRIC_QUANT = "FP4 cache write rows/s and HBM GB/s (1,048,576 bf16 rows of d512 -> E2M1 + E4M3)"
QUANT_SAMPLE_ROWS = 16384
# DRAM bytes (read + write) of one index-score launch on the decode workload,
# from one ncu capture of this kernel on it (its summary is kept with the
# profiles); to be reset to None whenever that kernel changes.
K1_TRAFFIC_BYTES = 134_273_792 + 4_593_664
N_REPLICAS = 4
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
NOMINAL_HBM_GBS = 8000.0


def peaks() -> dict:
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "src": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "src": "fallback"}


def device_facts(dev) -> dict:
    """The device's L2 size, and a read-only HBM stream rate measured here:
    torch.sum over 2 GiB of fp32 (larger than L2), best of 5 after one warm-up,
    CUDA events.  It is a reference beside the copy peak, not the roofline's
    denominator.  Runs after the timed region; anything that fails is None."""
    out = {"l2_bytes": None, "read_only_gbs": None, "read_only_how": "torch.sum of 2 GiB fp32, best of 5"}
    if getattr(dev, "type", None) != "cuda":
        return out
    try:
        out["l2_bytes"] = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0)) or None
    except Exception:
        pass
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


# ----------------------------------------------------------------- device state of one replica
def host_inputs(wl):
    """Host arrays of one decode step (everything except the FP4 KV values)."""
    lens = wl.lengths()
    pos = int(lens[0]) - 1
    layers = []
    for l, mode in enumerate(wl.modes):
        d = {"q_attn": synth.attn_query(wl, l, 0)}
        if mode != synth.REUSE:
            d["keys"] = synth.index_keys(wl, l, 0)
            d["q"], d["w"] = synth.index_query(wl, l, 0)
        layers.append(d)
    return pos, layers


def build_device_state(wl, host, dev, status):
    from kv_cache_decode_csa2_b200 import csa2 as B
    pos, hl = host
    n = pos + 1
    layers = []
    for l, mode in enumerate(wl.modes):
        d = hl[l]
        codes = torch.empty((n, wl.attn_dim // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty((n, wl.attn_dim // 32), dtype=torch.uint8, device=dev)
        step = 1 << 17
        for a in range(0, n, step):            # FP4 cache written by the library's quantiser
            b = min(n, a + step)
            x = torch.from_numpy(synth.kv_values(wl, l, 0, a, b)).to(dev, non_blocking=False)
            B.csa2_fp4_quantize(x, codes[a:b], scales[a:b], status=status)
        ly = B.Layer(q_attn=torch.from_numpy(d["q_attn"]).to(dev).to(torch.bfloat16)[None].contiguous(),
                     codes=B.Rows(codes), scales=B.Rows(scales),
                     out=torch.empty((1, wl.attn_heads, wl.attn_dim), dtype=torch.bfloat16, device=dev),
                     lse=None)
        if mode != synth.REUSE:
            ly.keys = B.Rows(torch.from_numpy(d["keys"]).to(dev))
            ly.q = torch.from_numpy(d["q"]).to(dev)[None].contiguous()
            ly.w = torch.from_numpy(d["w"]).to(dev)[None].contiguous()
            ly.sel_idx = torch.empty((1, wl.topk), dtype=torch.int32, device=dev)
            ly.sel_cnt = torch.empty((1,), dtype=torch.int32, device=dev)
        if mode == synth.FULL:
            ly.pool_idx = torch.empty((1, wl.pool), dtype=torch.int32, device=dev)
            ly.pool_cnt = torch.empty((1,), dtype=torch.int32, device=dev)
        layers.append(ly)
    return layers


def clone_layers(layers, dev):
    from kv_cache_decode_csa2_b200 import csa2 as B
    out = []
    for ly in layers:
        c = B.Layer(q_attn=ly.q_attn.clone(), codes=B.Rows(ly.codes.data.clone()),
                    scales=B.Rows(ly.scales.data.clone()), out=torch.empty_like(ly.out))
        if ly.keys is not None:
            c.keys = B.Rows(ly.keys.data.clone())
            c.q, c.w = ly.q.clone(), ly.w.clone()
            c.sel_idx, c.sel_cnt = torch.empty_like(ly.sel_idx), torch.empty_like(ly.sel_cnt)
        if ly.pool_idx is not None:
            c.pool_idx, c.pool_cnt = torch.empty_like(ly.pool_idx), torch.empty_like(ly.pool_cnt)
        out.append(c)
    return out


def algorithmic_bytes(wl, layers, pos) -> tuple[int, dict]:
    """Bytes the method must move per step: the full layer's key rows, the pool
    rows each reindex layer gathers, the FP4 rows of every layer's attention
    set, queries, head weights and outputs.  Scores, histograms and index lists
    are intermediates and are not counted."""
    ctx = pos + 1
    row_idx = wl.idx_dim
    row_fp4 = wl.attn_dim // 2 + wl.attn_dim // 32
    wstart = max(0, pos - wl.window + 1)
    parts = {"full_keys": ctx * row_idx, "reindex_gather": 0, "attn_rows": 0, "q_w_out": 0}
    sel = None
    for l, mode in enumerate(wl.modes):
        ly = layers[l]
        if mode != synth.REUSE:
            sel = ly.sel_idx[0, :int(ly.sel_cnt[0])].cpu().numpy()
            parts["q_w_out"] += wl.idx_heads * wl.idx_dim + wl.idx_heads
        if mode == synth.REINDEX:
            parts["reindex_gather"] += int(layers[0].pool_cnt[0]) * row_idx
        n_s = int((sel < wstart).sum()) + (pos - wstart + 1)
        parts["attn_rows"] += n_s * row_fp4
        parts["q_w_out"] += 2 * wl.attn_heads * wl.attn_dim * 2
    return sum(parts.values()), parts


def kernels_per_step(wl) -> int:
    """Kernels one plan step launches on this workload: one launch that zeroes
    the step's scratch, the index-score stream and the pool select of the full
    layer, one fused scoring + top-k launch for the reindex layers of the pool,
    and one attention launch for all layers (the ncu launch list in profiles/
    shows the same five per step)."""
    n_re = sum(1 for m in wl.modes if m == synth.REINDEX)
    n_full = sum(1 for m in wl.modes if m == synth.FULL)
    return 1 + 2 * n_full + (1 if n_re else 0) + 1


# ----------------------------------------------------------------- the CPU oracle baseline
class OracleStep:
    """One decode step of the CPU oracle on this workload, on one host core.

    Every step function is the oracle's own (oracle/).  This class only
    sequences them the way decode_layer_plan does, so that the context-linear
    part (the full layer's scan of every key row) can be timed on a 1/f slice
    of the positions and scaled by f.  The pool top-k, reindex and attention
    always run in full, over the full layer's real scores (computed once,
    untimed).  With f = 1 a step is exactly one whole oracle decode step."""

    def __init__(self, wl, host):
        import oracle as O
        self.O, self.wl = O, wl
        self.pos, self.hl = host
        n = self.pos + 1
        full = self.hl[0]
        self.scores0 = O.index_scores(full["q"], full["w"], full["keys"][:n])
        self.codes = []
        pool = sel = None
        for l, mode in enumerate(wl.modes):          # FP4 rows the step reads, stored by the oracle
            d = self.hl[l]
            if mode == synth.FULL:
                pool = O.top_k_positions(self.scores0, np.arange(n), wl.pool)
                sel = O.top_k_positions(self.scores0[pool], pool, wl.topk)
            elif mode == synth.REINDEX:
                _, sel = O.reindex(d["q"], d["w"], d["keys"], pool, wl.topk)
            S = O.attention_set(sel, self.pos, wl.window)
            codes = np.zeros((n, wl.attn_dim // 2), np.uint8)
            scales = np.zeros((n, wl.attn_dim // 32), np.uint8)
            x = np.concatenate([synth.kv_values(wl, l, 0, int(r), int(r) + 1) for r in S])
            codes[S], scales[S] = O.fp4_quantize(x)
            self.codes.append((codes, scales))

    def run(self, f: int = 1, slice_i: int = 0) -> tuple[float, float]:
        """Returns (seconds of the step, seconds of the scaled scan part)."""
        from threadpoolctl import threadpool_limits
        O, wl, pos = self.O, self.wl, self.pos
        n = pos + 1
        with threadpool_limits(1):
            full = self.hl[0]
            lo = (n * slice_i) // f
            hi = (n * (slice_i + 1)) // f
            t0 = time.perf_counter()
            O.index_scores(full["q"], full["w"], full["keys"][lo:hi])
            t_scan = (time.perf_counter() - t0) * f
            t1 = time.perf_counter()
            pool = sel = None
            for l, mode in enumerate(wl.modes):
                d = self.hl[l]
                if mode == synth.FULL:
                    pool = O.top_k_positions(self.scores0, np.arange(n), wl.pool)
                    sel = O.top_k_positions(self.scores0[pool], pool, wl.topk)
                elif mode == synth.REINDEX:
                    _, sel = O.reindex(d["q"], d["w"], d["keys"], pool, wl.topk)
                S = O.attention_set(sel, pos, wl.window)
                codes, scales = self.codes[l]
                O.sparse_attention(d["q_attn"], O.fp4_dequant(codes[S], scales[S], wl.attn_dim))
            t_rest = time.perf_counter() - t1
        return t_scan + t_rest, t_scan


def cpu_cores_used() -> int:
    # the timed oracle runs with BLAS limited to one thread; numpy's int64
    # matrix product and its sorts are single-threaded anyway
    return 1


# ----------------------------------------------------------------- arms
def run_reference(args, rank, world):
    if rank != 0:
        return
    wl = WL
    step = OracleStep(wl, host_inputs(wl))
    # size the per-step sample so that warm-up + timed steps stay near 3 minutes
    probe_f = 64
    t_probe, t_scan_probe = step.run(probe_f, 0)
    t_rest = t_probe - t_scan_probe
    budget = 180.0 / (args.steps + args.warmup)
    f = 1
    while t_scan_probe / f + t_rest > budget and f < 1024:
        f *= 2
    for i in range(args.warmup):
        step.run(f, i % f)
    ts = [step.run(f, i % f)[0] for i in range(args.steps)]
    sec = sum(ts) / len(ts)
    v = 1.0 / sec
    sample = ("whole 8-layer decode steps of the 1M-context workload" if f == 1 else
              f"8-layer decode steps of the 1M-context workload; the full layer's scan timed on 1/{f} of "
              f"the key rows (rotating) and scaled by {f}, everything else in full")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "steps/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int64,f64", "data": "synthetic",
            "config": config_dict(wl),
            "cpu_baseline": {"value": v, "unit": "steps/s", "cores": cpu_cores_used(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_dict(wl) -> dict:
    return {"workload": wl.name, "ctx": int(wl.lengths()[0]), "batch": 1,
            "layer_plan": ",".join(synth.MODE_NAMES[m] for m in wl.modes), "pool": wl.pool, "topk": wl.topk,
            "window": wl.window, "indexer": f"int8 {wl.idx_heads}x{wl.idx_dim}, w int8",
            "kv": f"FP4 E2M1 d{wl.attn_dim}, E4M3 per 32", "q_heads": wl.attn_heads,
            "l2": f"inputs rotate over {N_REPLICAS} device replicas (~141 MB read per step, > L2 per cycle)",
            "parallelism": "one sequence per rank"}


def run_gpu(args, rank, world, local):
    from kv_cache_decode_csa2_b200 import csa2 as B
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    wl = WL
    t_setup = time.time()
    host = host_inputs(wl)
    pos = host[0]
    status = B.new_status(dev)
    base = build_device_state(wl, host, dev, status)
    n_rep = max(1, args.replicas)
    replicas = [base] + [clone_layers(base, dev) for _ in range(n_rep - 1)]
    pos_dev = torch.tensor([pos], dtype=torch.int32, device=dev)
    plans = [B.LayerPlan(list(wl.modes), r, query_pos=pos_dev, max_ctx=pos + 1, P=wl.pool, K=wl.topk,
                         window=wl.window) for r in replicas]
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for p in plans:                       # ordinary calls first (one-time kernel set-up)
            p.run()
    torch.cuda.synchronize()
    B.check_status(status)
    for p in plans:
        B.check_status(p.status)
    alg_bytes, parts = algorithmic_bytes(wl, replicas[0], pos)

    graphs = []
    for p in plans:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            p.run()
        graphs.append(g)
    torch.cuda.synchronize()
    setup_s = time.time() - t_setup

    # ---- timed steps (graph replays)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            graphs[i % n_rep].replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id(dev)) as clk:
        time.sleep(0.3)
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for i in range(args.steps):
                graphs[i % n_rep].replay()
            ev1.record(stream)
        torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1)
    barrier(world)
    ms = max_over_ranks(ms, world, dev)
    ms_step = ms / args.steps
    value = world * args.steps / (ms / 1e3)
    for p in plans:
        B.check_status(p.status)

    # ---- dominant kernel alone: the index-score stream over 1M keys.  Its
    # launches (rotating over the replicas) are captured in a CUDA graph, so
    # the CUDA events bracket kernel time, not Python launch overhead.
    f = [r[0] for r in replicas]
    wss = [torch.empty(B.lib().csa2_index_full_workspace(1, pos + 1, 0, 0), dtype=torch.uint8, device=dev)
           for _ in f]
    k_per_graph = 4 * n_rep
    def k1_call(i):
        r = i % n_rep
        B.csa2_index_full(f[r].q, f[r].w, f[r].keys, pos_dev, pos + 1, ws=wss[r], status=status, stream=stream)
    with torch.cuda.stream(stream):
        for i in range(n_rep):
            k1_call(i)
    torch.cuda.synchronize()
    kg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(kg, stream=stream):
        for i in range(k_per_graph):
            k1_call(i)
    k_reps = max(3, args.steps // k_per_graph)
    with torch.cuda.stream(stream):
        kg.replay()
        ka, kb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ka.record(stream)
        for _ in range(k_reps):
            kg.replay()
        kb.record(stream)
    torch.cuda.synchronize()
    k_ms = ka.elapsed_time(kb) / (k_reps * k_per_graph)
    k_ms = max_over_ranks(k_ms, world, dev)
    del kg
    key_bytes = (pos + 1) * wl.idx_dim + wl.idx_heads * wl.idx_dim + wl.idx_heads
    pk = peaks()
    achieved = key_bytes / (k_ms / 1e3) / 1e9

    # ---- end to end through the C ABI with host buffers
    h2d = [l.q_attn for l in replicas[0]] + [t for l in replicas[0] if l.q is not None for t in (l.q, l.w)]
    h2d_host = [t.cpu().pin_memory() for t in h2d]
    d2h = [l.out for l in replicas[0]]
    d2h_host = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in d2h]
    h2d_bytes = sum(t.numel() * t.element_size() for t in h2d_host)
    d2h_bytes = sum(t.numel() * t.element_size() for t in d2h_host)
    e_steps = max(args.steps, 10)
    with torch.cuda.stream(stream):
        for _ in range(2):
            for hsrc, ddst in zip(h2d_host, h2d):
                ddst.copy_(hsrc, non_blocking=True)
            plans[0].run(stream)
            for dsrc, hdst in zip(d2h, d2h_host):
                hdst.copy_(dsrc, non_blocking=True)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(e_steps):
            for hsrc, ddst in zip(h2d_host, h2d):
                ddst.copy_(hsrc, non_blocking=True)
            plans[0].run(stream)
            for dsrc, hdst in zip(d2h, d2h_host):
                hdst.copy_(dsrc, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e = world * e_steps / (e_ms / 1e3)
    B.check_status(plans[0].status)

    gbs = alg_bytes / (ms_step / 1e3) / 1e9
    line = {"metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic", "config": config_dict(wl),
            "hbm": {"algorithmic_bytes_per_step": alg_bytes, "parts": parts, "achieved_gbs": gbs,
                    "frac_of_8tbs": gbs / NOMINAL_HBM_GBS, "frac_of_measured": gbs / pk["hbm_gbs"]},
            "roofline": {"kernel": "index_score_kernel<128,64> (full-mode index scoring of 1M keys)",
                         "bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / pk["hbm_gbs"], "peak_src": pk["src"], "ms_per_launch": k_ms,
                         "bytes_per_launch": key_bytes, "traffic": K1_TRAFFIC_BYTES},
            "e2e": {"value": e2e, "unit": "steps/s", "h2d_bytes_per_step": h2d_bytes,
                    "d2h_bytes_per_step": d2h_bytes, "path": "pinned H2D + csa2_layer_plan + D2H, no graph"},
            "gpu_launches": kernels_per_step(wl) * args.steps,
            "clocks": clk.summary(), "setup_s": round(setup_s, 1)}
    line["device"] = device_facts(dev)
    if rank == 0 and not args.no_cpu_baseline:
        sec, _ = OracleStep(wl, host).run(1, 0)
        line["cpu_baseline"] = {"value": 1.0 / sec, "unit": "steps/s", "cores": cpu_cores_used(), "kind": "oracle",
                                "sample": "one whole 8-layer decode step of the same 1M-context workload"}
    for p in plans:
        B.check_status(p.status)
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


def prefill_replica(wl, host, dev, status):
    """Device state of one prefill chunk: keys, FP4 cache, the queries."""
    from kv_cache_decode_csa2_b200 import csa2 as B
    n, q, w, qa = host
    codes = torch.empty((n, wl.attn_dim // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((n, wl.attn_dim // 32), dtype=torch.uint8, device=dev)
    step = 1 << 17
    for a in range(0, n, step):                # FP4 cache written by the library's quantiser
        b = min(n, a + step)
        x = torch.from_numpy(synth.kv_values(wl, 0, 0, a, b)).to(dev)
        B.csa2_fp4_quantize(x, codes[a:b], scales[a:b], status=status)
    keys = torch.from_numpy(synth.index_keys(wl, 0, 0)).to(dev)
    return {"keys": B.Rows(keys), "codes": B.Rows(codes), "scales": B.Rows(scales),
            "q": torch.from_numpy(q).to(dev), "w": torch.from_numpy(w).to(dev),
            "qa": torch.from_numpy(qa).to(dev).to(torch.bfloat16)}


PREFILL_SAMPLE = "the chunk's last query (its whole 262,144-row prefix), through the oracle one query at a time"


def prefill_host(wl):
    n = int(wl.lengths()[0])
    _, qp = wl.query_positions()
    qs = [synth.index_query(wl, 0, i) for i in range(len(qp))]
    return (n, np.stack([x[0] for x in qs]), np.stack([x[1] for x in qs]),
            np.stack([synth.attn_query(wl, 0, i) for i in range(len(qp))]))


def oracle_prefill_query_seconds(wl, host, qp) -> float:
    """Seconds the oracle takes for one query of the chunk (the last, whose
    prefix is the whole context): its scores, its top-k and its attention.
    The FP4 rows of its attention set are stored, untimed, in between."""
    import oracle as O
    from threadpoolctl import threadpool_limits
    keys = synth.index_keys(wl, 0, 0)
    i = len(qp) - 1
    pos = int(qp[i])
    with threadpool_limits(1):
        t0 = time.perf_counter()
        s_ = O.index_scores(host[1][i], host[2][i], keys[:pos + 1])
        sel_ = O.top_k_positions(s_, np.arange(pos + 1), wl.topk)
        S = O.attention_set(sel_, pos, wl.window)
        t1 = time.perf_counter()
        x = np.concatenate([synth.kv_values(wl, 0, 0, int(r_), int(r_) + 1) for r_ in S])
        c_, sc_ = O.fp4_quantize(x)
        t2 = time.perf_counter()
        O.sparse_attention(host[3][i], O.fp4_dequant(c_, sc_, wl.attn_dim))
        t3 = time.perf_counter()
    return (t1 - t0) + (t3 - t2)


def run_reference_prefill(args, rank, world):
    if rank != 0:
        return
    wl = WL_PREFILL
    host = prefill_host(wl)
    _, qp = wl.query_positions()
    ts = [oracle_prefill_query_seconds(wl, host, qp) for _ in range(max(1, min(args.steps, 3)))]
    v = 1.0 / (sum(ts) / len(ts))
    line = {"impl": "reference", "metric": METRIC_PREFILL, "value": v, "unit": "queries/s", "n_gpus": args.gpus,
            "steps": len(ts), "warmup": 0, "ms_per_step": 1e3 / v, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int64,f64", "data": "synthetic",
            "config": {"workload": wl.name},
            "cpu_baseline": {"value": v, "unit": "queries/s", "cores": cpu_cores_used(), "kind": "oracle",
                             "sample": PREFILL_SAMPLE},
            "e2e": {"value": v, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_prefill(args, rank, world, local):
    from kv_cache_decode_csa2_b200 import csa2 as B
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    wl = WL_PREFILL
    t_setup = time.time()
    sq, qp = wl.query_positions()
    nq = len(qp)
    host = prefill_host(wl)
    n = host[0]
    status = B.new_status(dev)
    n_rep = max(1, args.replicas)
    reps = [prefill_replica(wl, host, dev, status) for _ in range(n_rep)]
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

    def timed(gs, steps):
        with torch.cuda.stream(stream):
            for i in range(args.warmup):
                gs[i % n_rep].replay()
        torch.cuda.synchronize()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            for i in range(steps):
                gs[i % n_rep].replay()
            b.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(a.elapsed_time(b), world, dev) / steps

    with ClockSampler(gpu_id(dev)) as clk:
        time.sleep(0.3)
        ms = timed(graphs, args.steps)
    ms_index = timed(igraphs, max(3, args.steps))
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
            "roofline": {"kernel": "index stage: index_score_kernel<128,64,4> + per-query top-512",
                         "bound": "tensor", "achieved": tops, "peak": pk["tops"], "unit": "TOP/s (int8)",
                         "frac": tops / pk["tops"], "peak_src": pk["src"], "ms_per_launch": ms_index,
                         "ops_per_launch": ops, "traffic": None},
            "e2e": {"value": world * nq / (e_ms / 1e3), "unit": "queries/s",
                    "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in h2d_host),
                    "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in d2h_host),
                    "path": "pinned H2D + csa2_index_full + csa2_sparse_attn_fp4 + D2H, no graph"},
            "gpu_launches": 4 * args.steps,
            "clocks": clk.summary(), "setup_s": round(setup_s, 1)}
    if rank == 0 and not args.no_cpu_baseline:
        sec = oracle_prefill_query_seconds(wl, host, qp)
        line["cpu_baseline"] = {"value": 1.0 / sec, "unit": "queries/s", "cores": cpu_cores_used(), "kind": "oracle",
                                "sample": PREFILL_SAMPLE}
    del graphs, igraphs
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- FP4 cache write
def quant_bytes_per_row(D: int) -> int:
    """Algorithmic bytes of storing one bf16 row of D values as FP4: the row
    read (2 D) and the codes (D / 2) and scales (D / 32) written."""
    return 2 * D + D // 2 + D // 32


def oracle_quant_rows_per_s(wl, rows: int) -> tuple[float, str]:
    """The oracle's FP4 quantiser on the first ``rows`` rows of layer 0 (bf16
    values), timed on one host core."""
    import oracle as O
    from threadpoolctl import threadpool_limits
    x = synth.round_to_bf16(synth.kv_values(wl, 0, 0, 0, rows))
    with threadpool_limits(1):
        t0 = time.perf_counter()
        O.fp4_quantize(x)
        t = time.perf_counter() - t0
    return rows / t, f"{rows} bf16 rows of d{wl.attn_dim} of the same cache, one call"


def run_reference_quantize(args, rank, world):
    if rank != 0:
        return
    wl = WL
    vs = [oracle_quant_rows_per_s(wl, QUANT_SAMPLE_ROWS)[0] for _ in range(max(1, min(args.steps, 3)))]
    v = sum(vs) / len(vs)
    line = {"impl": "reference", "metric": METRIC_QUANT, "value": v, "unit": "rows/s", "n_gpus": args.gpus,
            "steps": len(vs), "warmup": 0, "ms_per_step": 1e3 * (1 << 20) / v, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "fp4_cache_write_1m_rows_d512"},
            "cpu_baseline": {"value": v, "unit": "rows/s", "cores": 1, "kind": "oracle",
                             "sample": f"{QUANT_SAMPLE_ROWS} rows per step"},
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
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id(dev)) as clk:
        time.sleep(0.3)
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for _ in range(args.steps):
                g.replay()
            ev1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev) / args.steps
    barrier(world)
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
            "roofline": {"kernel": "fp4_quantize_kernel<bf16>", "bound": "hbm", "achieved": achieved,
                         "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
                         "peak_src": pk["src"], "ms_per_launch": ms, "bytes_per_launch": n * per_row,
                         "traffic": None},
            "e2e": {"value": world * n / (e_ms / 1e3), "unit": "rows/s",
                    "h2d_bytes_per_step": xh.numel() * xh.element_size(),
                    "d2h_bytes_per_step": ch.numel() + sh.numel(),
                    "path": "pinned H2D + csa2_fp4_quantize + D2H, no graph"},
            "gpu_launches": args.steps, "clocks": clk.summary(), "setup_s": round(setup_s, 1)}
    if rank == 0 and not args.no_cpu_baseline:
        v, sample = oracle_quant_rows_per_s(wl, QUANT_SAMPLE_ROWS)
        line["cpu_baseline"] = {"value": v, "unit": "rows/s", "cores": 1, "kind": "oracle", "sample": sample}
    del g
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="csa2", choices=["csa2", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default="decode", choices=["decode", "prefill", "quantize"],
                    help="decode: the 1M-context 8-layer step (default); prefill: the 2048-query chunk; "
                         "quantize: the FP4 cache write of 1M bf16 rows")
    ap.add_argument("--replicas", type=int, default=N_REPLICAS,
                    help="device copies of the state rotated between steps (4 keep each step's reads out of L2)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, local = dist_init(args.gpus)
    try:
        if args.workload == "quantize":
            (run_reference_quantize if args.impl == "reference" else run_quantize)(args, rank, world, *(
                () if args.impl == "reference" else (local,)))
        elif args.workload == "prefill":
            (run_reference_prefill if args.impl == "reference" else run_prefill)(args, rank, world, *(
                () if args.impl == "reference" else (local,)))
        elif args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_gpu(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
