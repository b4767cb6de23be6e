"""Device state of the benchmark workloads.

The synthetic inputs of ``synth`` placed in HBM the way the library reads
them, for the benchmark (``bench.py``) and the phase-trace tool
(``trace.py``).  Nothing here computes any step of the method: the FP4 cache
is written by the library's own quantiser (csa2_fp4_quantize) and every
other tensor is a copy of the generator's bytes.

A decode state keeps the per-step inputs of every layer (attention queries,
index queries and head weights) as views of ONE device buffer, and every
layer's attention output as a view of ONE more, so an end-to-end step moves
its inputs in with one host-to-device copy and its outputs back with one
device-to-host copy.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

import synth

from . import csa2 as B

_ALIGN = 256


@dataclass
class DecodeState:
    """One replica of a decode workload on the device."""
    wl: synth.Workload
    layers: list                      # B.Layer per layer
    seq_of_query: np.ndarray          # host copies of the query placement
    query_pos: np.ndarray
    pos_dev: torch.Tensor
    seq_dev: torch.Tensor | None      # None for one sequence
    max_ctx: int
    inbuf: torch.Tensor               # uint8: every per-step input, packed
    outbuf: torch.Tensor              # uint8: every layer's output, packed
    extra: dict = field(default_factory=dict)


class _Packer:
    """Carves views of one flat uint8 device buffer, 256-byte aligned."""

    def __init__(self):
        self.parts = []   # (offset, nbytes, shape, dtype)
        self.size = 0

    def add(self, shape, dtype) -> int:
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        off = (self.size + _ALIGN - 1) // _ALIGN * _ALIGN
        self.parts.append((off, n, tuple(shape), dtype))
        self.size = off + n
        return len(self.parts) - 1

    def views(self, buf: torch.Tensor) -> list[torch.Tensor]:
        return [buf[o:o + n].view(dt).view(shape) for o, n, shape, dt in self.parts]


def _fp4_rows(wl, layer, lens, pt, dev, status):
    """The layer's FP4 cache (codes and scales planes), each sequence's values
    stored by csa2_fp4_quantize, 64K rows at a time, at their physical rows."""
    D = wl.attn_dim
    pr = wl.page_rows or 64
    if pt is None:
        seq_rows = int(max(lens))
        n_rows = len(lens) * seq_rows
    else:
        seq_rows = 0
        n_rows = (int(pt.max()) + 1) * pr
    codes = torch.empty((n_rows, D // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((n_rows, D // 32), dtype=torch.uint8, device=dev)
    step = 1 << 17
    for s, n in enumerate(lens):
        for a in range(0, int(n), step):
            b = min(int(n), a + step)
            x = torch.from_numpy(synth.kv_values(wl, layer, s, a, b)).to(dev)
            if pt is None:
                r0 = s * seq_rows + a
                B.csa2_fp4_quantize(x, codes[r0:r0 + (b - a)], scales[r0:r0 + (b - a)], status=status)
            else:
                pos = np.arange(a, b)
                dst = pt[s, pos // pr].astype(np.int64) * pr + pos % pr
                B.csa2_fp4_quantize(x, codes, scales, status=status,
                                    dst_rows=torch.from_numpy(dst.astype(np.int32)).to(dev))
    return codes, scales, seq_rows


def _key_rows(wl, layer, lens, pt, dev):
    """The layer's int8 index-key cache in its physical layout."""
    pr = wl.page_rows or 64
    if pt is None:
        seq_rows = int(max(lens))
        keys = torch.zeros((len(lens) * seq_rows, wl.idx_dim), dtype=torch.int8, device=dev)
        for s, n in enumerate(lens):
            keys[s * seq_rows:s * seq_rows + int(n)] = torch.from_numpy(synth.index_keys(wl, layer, s)).to(dev)
        return keys, seq_rows
    keys = torch.zeros(((int(pt.max()) + 1) * pr, wl.idx_dim), dtype=torch.int8, device=dev)
    for s, n in enumerate(lens):
        n = int(n)
        pos = np.arange(n)
        dst = torch.from_numpy(pt[s, pos // pr].astype(np.int64) * pr + pos % pr).to(dev)
        keys.index_copy_(0, dst, torch.from_numpy(synth.index_keys(wl, layer, s)).to(dev))
    return keys, 0


def local_ring_rows(wl: synth.Workload, layer: int, lens, R: int) -> np.ndarray:
    """float32 [len(lens) * R][attn_dim] local window cache of one layer: a
    ring of R rows per sequence, position p of sequence s in row s R + p mod R,
    holding the last R positions (synth.local_kv_values)."""
    rows = np.zeros((len(lens) * R, wl.attn_dim), np.float32)
    for s, n in enumerate(lens):
        n = int(n)
        a = max(0, n - R)
        rows[s * R + np.arange(a, n) % R] = synth.local_kv_values(wl, layer, s, a, n)
    return rows


def build_decode(wl: synth.Workload, dev, status, local_window: bool = False) -> DecodeState:
    """Builds one replica of a decode workload: one query per sequence at its
    last position, or a block of causal queries of sequence 0 when the
    workload has a query block (a verify block).

    With ``local_window`` every layer reads its window from its own bf16
    ring of ``wl.window`` rows per sequence, and every REUSE layer reads the
    global FP4 cache of the layer whose selection it reuses (the same codes
    and scales views)."""
    lens = wl.lengths()
    sq, qp = wl.query_positions()
    nq = len(qp)
    pt = synth.page_table(wl) if wl.page_rows else None
    pt_dev = torch.from_numpy(pt).to(dev) if pt is not None else None
    pr = wl.page_rows or 64
    D, Hq = wl.attn_dim, wl.attn_heads

    pin, pout = _Packer(), _Packer()
    slots = []
    for mode in wl.modes:
        s = {"qa": pin.add((nq, Hq, D), torch.bfloat16), "out": pout.add((nq, Hq, D), torch.bfloat16)}
        if mode != synth.REUSE:
            s["q"] = pin.add((nq, wl.idx_heads, wl.idx_dim), torch.int8)
            s["w"] = pin.add((nq, wl.idx_heads), torch.int8)
        slots.append(s)
    inbuf = torch.zeros(pin.size, dtype=torch.uint8, device=dev)
    outbuf = torch.zeros(pout.size, dtype=torch.uint8, device=dev)
    vin, vout = pin.views(inbuf), pout.views(outbuf)

    layers = []
    src = 0   # the most recent FULL/REINDEX layer
    for l, mode in enumerate(wl.modes):
        s = slots[l]
        qa = vin[s["qa"]]
        qa.copy_(torch.from_numpy(np.stack([synth.attn_query(wl, l, i) for i in range(nq)])).to(torch.bfloat16))
        if mode != synth.REUSE:
            src = l
        if local_window and mode == synth.REUSE:
            ly = B.Layer(q_attn=qa, codes=layers[src].codes, scales=layers[src].scales, out=vout[s["out"]],
                         lse=None)
        else:
            codes, scales, srows = _fp4_rows(wl, l, lens, pt, dev, status)
            ly = B.Layer(q_attn=qa, codes=B.Rows(codes, pt_dev, pr, srows),
                         scales=B.Rows(scales, pt_dev, pr, srows), out=vout[s["out"]], lse=None)
        if local_window:
            ring = torch.from_numpy(local_ring_rows(wl, l, lens, wl.window)).to(dev).to(torch.bfloat16)
            ly.local_kv = B.Rows(ring, seq_rows=wl.window)
        if mode != synth.REUSE:
            keys, ksr = _key_rows(wl, l, lens, pt, dev)
            ly.keys = B.Rows(keys, pt_dev, pr, ksr)
            qs = [synth.index_query(wl, l, i) for i in range(nq)]
            ly.q = vin[s["q"]]
            ly.q.copy_(torch.from_numpy(np.stack([x[0] for x in qs])))
            ly.w = vin[s["w"]]
            ly.w.copy_(torch.from_numpy(np.stack([x[1] for x in qs])))
            ly.sel_idx = torch.empty((nq, wl.topk), dtype=torch.int32, device=dev)
            ly.sel_cnt = torch.empty((nq,), dtype=torch.int32, device=dev)
        if mode == synth.FULL:
            ly.pool_idx = torch.empty((nq, wl.pool), dtype=torch.int32, device=dev)
            ly.pool_cnt = torch.empty((nq,), dtype=torch.int32, device=dev)
        layers.append(ly)
    multi = len(lens) > 1 or nq > 1
    return DecodeState(wl=wl, layers=layers, seq_of_query=sq, query_pos=qp,
                       pos_dev=torch.from_numpy(qp.astype(np.int32)).to(dev),
                       seq_dev=torch.from_numpy(sq.astype(np.int32)).to(dev) if multi else None,
                       max_ctx=int(lens.max()), inbuf=inbuf, outbuf=outbuf,
                       extra={"pin": pin, "pout": pout, "slots": slots, "page_table": pt_dev})


def clone_decode(st: DecodeState, dev) -> DecodeState:
    """A second replica of the same state: every cache and buffer copied
    (a cache that several layers share stays shared in the copy)."""
    inbuf, outbuf = st.inbuf.clone(), torch.zeros_like(st.outbuf)
    vin, vout = st.extra["pin"].views(inbuf), st.extra["pout"].views(outbuf)
    copies = {}

    def copy(r: "B.Rows") -> "B.Rows":
        if id(r) not in copies:
            copies[id(r)] = B.Rows(r.data.clone(), r.page_table, r.page_rows, r.seq_rows)
        return copies[id(r)]
    layers = []
    for ly, s in zip(st.layers, st.extra["slots"]):
        c = B.Layer(q_attn=vin[s["qa"]], out=vout[s["out"]], lse=None, codes=copy(ly.codes),
                    scales=copy(ly.scales))
        if ly.local_kv is not None:
            c.local_kv = copy(ly.local_kv)
        if ly.keys is not None:
            c.keys = B.Rows(ly.keys.data.clone(), ly.keys.page_table, ly.keys.page_rows, ly.keys.seq_rows)
            c.q, c.w = vin[s["q"]], vin[s["w"]]
            c.sel_idx, c.sel_cnt = torch.empty_like(ly.sel_idx), torch.empty_like(ly.sel_cnt)
        if ly.pool_idx is not None:
            c.pool_idx, c.pool_cnt = torch.empty_like(ly.pool_idx), torch.empty_like(ly.pool_cnt)
        layers.append(c)
    return DecodeState(wl=st.wl, layers=layers, seq_of_query=st.seq_of_query, query_pos=st.query_pos,
                       pos_dev=st.pos_dev.clone(), seq_dev=None if st.seq_dev is None else st.seq_dev.clone(),
                       max_ctx=st.max_ctx, inbuf=inbuf, outbuf=outbuf, extra=st.extra)


def decode_plan(st: DecodeState, group_queries: bool = False) -> "B.LayerPlan":
    wl = st.wl
    return B.LayerPlan(list(wl.modes), st.layers, query_pos=st.pos_dev, seq_of_query=st.seq_dev,
                       max_ctx=st.max_ctx, P=wl.pool, K=wl.topk, window=wl.window, group_queries=group_queries)


def state_bytes(st: DecodeState) -> int:
    """Device bytes of the caches of one replica (a shared cache once)."""
    seen, n = set(), 0
    for ly in st.layers:
        for r in (ly.codes, ly.scales, ly.keys, ly.local_kv):
            if r is not None and id(r.data) not in seen:
                seen.add(id(r.data))
                n += r.data.numel() * r.data.element_size()
    return n


def algorithmic_bytes(st: DecodeState) -> tuple[int, dict]:
    """Bytes the method must move per step, from the selections of a step
    that has run:
      - the key rows of every full-mode layer: per sequence, the rows up to
        the last position any of its queries sees (queries of one sequence
        share one scan);
      - per query and reindex layer, the key rows of the pool it gathers;
      - per query and layer, the FP4 rows of its attention set (selection and
        window, each position once), or with a local window cache the FP4
        rows below the window and the window's bf16 rows;
      - queries, head weights and outputs.
    Scores, histograms and index lists are intermediates and are not counted."""
    wl = st.wl
    row_idx = wl.idx_dim
    row_fp4 = wl.attn_dim // 2 + wl.attn_dim // 32
    sq, qp = st.seq_of_query, st.query_pos
    last = {}
    for s, p in zip(sq, qp):
        last[int(s)] = max(last.get(int(s), -1), int(p))
    n_full = sum(1 for m in wl.modes if m == synth.FULL)
    parts = {"full_keys": n_full * sum(p + 1 for p in last.values()) * row_idx, "reindex_gather": 0,
             "attn_rows": 0, "q_w_out": 0}
    sel_h = {}
    pool_cnt = None
    for l, mode in enumerate(wl.modes):
        ly = st.layers[l]
        if mode == synth.FULL:
            pool_cnt = ly.pool_cnt.cpu().numpy()
        if mode != synth.REUSE:
            cnt = ly.sel_cnt.cpu().numpy()
            idx = ly.sel_idx.cpu().numpy()
            sel_h = {i: idx[i, :int(cnt[i])] for i in range(len(qp))}
            parts["q_w_out"] += len(qp) * (wl.idx_heads * wl.idx_dim + wl.idx_heads)
        if mode == synth.REINDEX:
            parts["reindex_gather"] += int(pool_cnt.sum()) * row_idx
        row_win = 2 * wl.attn_dim if ly.local_kv is not None else row_fp4
        for i, p in enumerate(qp):
            wstart = max(0, int(p) - wl.window + 1)
            parts["attn_rows"] += int((sel_h[i] < wstart).sum()) * row_fp4 + (int(p) - wstart + 1) * row_win
        parts["q_w_out"] += 2 * len(qp) * wl.attn_heads * wl.attn_dim * 2
    return sum(parts.values()), parts


def kernels_per_step(wl: synth.Workload, n_queries: int = 1, grouped: bool = False) -> int:
    """Kernels one plan step launches on a workload whose queries fit one
    co-resident select pass: one launch that zeroes the step's scratch, the
    index-score stream and the pool select of each full layer, one fused
    scoring + top-k launch for the reindex layers of a pool, and one
    attention launch for all layers."""
    n_re = sum(1 for m in wl.modes if m == synth.REINDEX)
    n_full = sum(1 for m in wl.modes if m == synth.FULL)
    return 1 + 2 * n_full + (1 if n_re else 0) + 1


# ----------------------------------------------------------------- prefill chunk
def prefill_host(wl):
    """Host arrays of one prefill chunk: (context rows, q, w, attention q)."""
    n = int(wl.lengths()[0])
    _, qp = wl.query_positions()
    qs = [synth.index_query(wl, 0, i) for i in range(len(qp))]
    return (n, np.stack([x[0] for x in qs]), np.stack([x[1] for x in qs]),
            np.stack([synth.attn_query(wl, 0, i) for i in range(len(qp))]))


def prefill_replica(wl, host, dev, status):
    """Device state of one prefill chunk: keys, FP4 cache, the queries."""
    n, q, w, qa = host
    codes, scales, _ = _fp4_rows(wl, 0, np.array([n]), None, dev, status)
    keys = torch.from_numpy(synth.index_keys(wl, 0, 0)).to(dev)
    return {"keys": B.Rows(keys), "codes": B.Rows(codes), "scales": B.Rows(scales),
            "q": torch.from_numpy(q).to(dev), "w": torch.from_numpy(w).to(dev),
            "qa": torch.from_numpy(qa).to(dev).to(torch.bfloat16)}
