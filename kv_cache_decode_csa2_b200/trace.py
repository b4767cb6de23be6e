"""Phase tracing of the kernels of one decode step (or one prefill chunk).

    python -m kv_cache_decode_csa2_b200.trace [--workload decode|prefill] [--warmup W] [--save T.npy]

Builds libcsa2_trace.so (the library with its phase markers compiled in, see
csa2_trace_attach in include/csa2.h), sets up the benchmark's workload (workloads.py) through it,
replays the work in a CUDA graph as the benchmark does, and records one replay
after an L2 flush.  It prints, per kernel in launch order, when its CTAs
started and reached each marked point, relative to the start of the first
kernel: the median and the latest CTA.  Times inside a CTA come from its SM
cycle counter (converted at the clock rate the trace itself shows); the
start of each CTA comes from the global timer.

This is a measurement tool: the markers are a few global stores per CTA, so
traced times run slightly above untraced ones, and no bench number comes from
here.
"""
from __future__ import annotations

import argparse
import os
from dataclasses import dataclass

import numpy as np
import torch

KERNELS = 8
CTAS = 1024
POINTS = 16

# Names of the marked points of each kernel (point 0 is kernel entry).
POINT_NAMES = {
    0: ("index_score", ["entry", "prologue done", "first TMA issued", "first stage landed",
                        "first epilogue tile", "last epilogue tile", "histogram flushed", "producer done",
                        "MMA issuer done", "exit", "producer set up"]),
    1: ("select", ["entry", "grid before done", "threshold buckets", "classified", "first grid barrier",
                   "row ties staged", "ties ranked", "second grid barrier", "written"]),
    2: ("reindex_select", ["entry", "own inputs staged", "grid before done", "pool rows gathered", "scored",
                           "published | histogram barrier", "threshold bucket", "tie barrier", "ties ranked",
                           "count barrier", "written"]),
    3: ("sparse_attn", ["entry", "Q staged", "grid before done", "row positions", "rows dequantised", "logits",
                        "softmax", "P V done", "partial written", "group barrier", "merged"]),
    4: ("row_select", ["entry", "threshold buckets", "score bounds", "classified", "ties resolved", "written"]),
    5: ("zero", ["entry", "done"]),
    6: ("reindex_cluster", ["entry", "own inputs staged", "grid before done", "rows gathered", "scored",
                            "histogram barrier", "slice barrier", "threshold", "count barrier", "ties resolved",
                            "written"]),
}


@dataclass
class PointStat:
    name: str
    reached: int          # CTAs that recorded the point
    median_us: float      # median over those CTAs, from the start of the first kernel
    max_us: float         # the latest CTA


@dataclass
class KernelStat:
    kernel: int
    name: str
    ctas: int
    start_us: float       # first CTA entry, from the start of the first kernel
    end_us: float         # latest recorded point of any CTA
    points: list


def clock_ghz(table: np.ndarray, min_span_ns: int = 3000) -> float:
    """SM cycles per ns, the median over CTAs whose recorded span is long
    enough to measure with the global timer; 1.9 if none is."""
    ratios = []
    for k in range(table.shape[0]):
        for c in range(table.shape[1]):
            e = table[k, c]
            if e[0, 0] == 0:
                continue
            hit = np.nonzero(e[:, 0])[0]
            last = hit[-1]
            span = int(e[last, 0]) - int(e[0, 0])
            if last > 0 and span >= min_span_ns and e[last, 1] > 0:
                ratios.append(float(e[last, 1]) / span)
    return float(np.median(ratios)) if ratios else 1.9


def summarize(table: np.ndarray, ghz: float | None = None) -> list[KernelStat]:
    """Per kernel present in `table` (uint64 [KERNELS][CTAS][POINTS][2] =
    {global ns, SM cycles since entry}), the start, end and point times in
    microseconds from the earliest kernel entry, sorted by start."""
    table = np.asarray(table, dtype=np.uint64)
    assert table.shape == (KERNELS, CTAS, POINTS, 2), table.shape
    if ghz is None:
        ghz = clock_ghz(table)
    entries = table[:, :, 0, 0]
    present = entries != 0
    if not present.any():
        return []
    t0 = int(entries[present].min())
    out = []
    for k in range(KERNELS):
        ctas = np.nonzero(present[k])[0]
        if len(ctas) == 0:
            continue
        name, pnames = POINT_NAMES.get(k, (f"kernel{k}", []))
        start = (entries[k, ctas].astype(np.int64) - t0)            # ns per CTA
        pts = []
        end = 0.0
        for p in range(POINTS):
            rec = table[k, ctas, p, 0] != 0
            if not rec.any():
                continue
            t = start[rec] + table[k, ctas[rec], p, 1].astype(np.float64) / ghz
            pts.append(PointStat(pnames[p] if p < len(pnames) else f"point {p}", int(rec.sum()),
                                 float(np.median(t)) / 1e3, float(t.max()) / 1e3))
            end = max(end, float(t.max()) / 1e3)
        out.append(KernelStat(k, name, len(ctas), float(start.min()) / 1e3, end, pts))
    out.sort(key=lambda s: s.start_us)
    return out


def format_report(stats: list[KernelStat], ghz: float) -> str:
    lines = [f"SM clock from the trace: {ghz * 1e3:.0f} MHz; times in us from the first kernel's start"]
    for s in stats:
        lines.append("")
        lines.append(f"{s.name}: {s.ctas} CTAs traced, start {s.start_us:.2f}, end {s.end_us:.2f} "
                     f"({s.end_us - s.start_us:.2f})")
        lines.append(f"  {'point':<24} {'CTAs':>5} {'median':>9} {'latest':>9}")
        for p in s.points:
            lines.append(f"  {p.name:<24} {p.reached:>5} {p.median_us:>9.2f} {p.max_us:>9.2f}")
    return "\n".join(lines)


# ----------------------------------------------------------------- running a workload
def load_traced_library():
    """Builds and loads libcsa2_trace.so in place of libcsa2.so."""
    from . import build as _build
    from . import csa2 as B
    path = _build.build(trace=True)
    B.LIB_PATH = path
    B._lib = None
    return B.lib()


def _decode_work(dev, status):
    import synth

    from . import workloads as W
    st = W.build_decode(synth.C2_1M_PLAN, dev, status)
    plan = W.decode_plan(st)
    return plan.run, [plan.status]


def _prefill_work(dev, status, stream):
    import synth

    from . import csa2 as B
    from . import workloads as W
    wl = synth.C4_PREFILL
    sq, qp = wl.query_positions()
    nq = len(qp)
    host = W.prefill_host(wl)
    n = host[0]
    r = W.prefill_replica(wl, host, dev, status)
    pos_dev = torch.from_numpy(qp.astype(np.int32)).to(dev)
    seq_dev = torch.from_numpy(sq.astype(np.int32)).to(dev)
    sel = torch.empty((nq, wl.topk), dtype=torch.int32, device=dev)
    cnt = torch.empty((nq,), dtype=torch.int32, device=dev)
    out = torch.empty((nq, wl.attn_heads, wl.attn_dim), dtype=torch.bfloat16, device=dev)
    L = B.lib()
    ws_i = torch.empty(L.csa2_index_full_workspace(nq, n, 0, wl.topk), dtype=torch.uint8, device=dev)
    ws_a = torch.empty(L.csa2_sparse_attn_workspace(nq, wl.attn_heads, wl.attn_dim, wl.topk, wl.window),
                       dtype=torch.uint8, device=dev)

    def run():
        B.csa2_index_full(r["q"], r["w"], r["keys"], pos_dev, n, seq_of_query=seq_dev, K=wl.topk, sel_idx=sel,
                          sel_cnt=cnt, status=status, ws=ws_i, stream=stream)
        B.csa2_sparse_attn_fp4(r["qa"], r["codes"], r["scales"], pos_dev, sel, out, sel_cnt=cnt,
                               seq_of_query=seq_dev, window=wl.window, status=status, ws=ws_a, stream=stream)
    return run, []


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", choices=["decode", "prefill"], default="decode")
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--save", default=None, help="also write the raw table (uint64 [8][1024][16][2]) to this .npy")
    args = ap.parse_args(argv)
    L = load_traced_library()
    from . import csa2 as B
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    status = B.new_status(dev)
    stream = torch.cuda.Stream(device=dev)
    table = torch.zeros(L.csa2_trace_table_bytes() // 8, dtype=torch.int64, device=dev)
    B._check(L.csa2_trace_attach(table.data_ptr()), "csa2_trace_attach")
    if args.workload == "decode":
        run, statuses = _decode_work(dev, status)
    else:
        run, statuses = _prefill_work(dev, status, stream)
    with torch.cuda.stream(stream):
        run()                                   # ordinary call first (one-time kernel set-up)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        run()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g.replay()
        flush.zero_()                           # the traced replay starts with a cold L2
        table.zero_()
        g.replay()
    torch.cuda.synchronize()
    for s in [status] + statuses:
        B.check_status(s)
    B._check(L.csa2_trace_attach(None), "csa2_trace_attach")
    t = table.cpu().numpy().view(np.uint64).reshape(KERNELS, CTAS, POINTS, 2)
    if args.save:
        np.save(args.save, t)
    ghz = clock_ghz(t)
    print(f"workload: {args.workload}")
    print(format_report(summarize(t, ghz), ghz))
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
