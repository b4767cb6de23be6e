"""Builds one synthetic workload for both sides of a parity test.

Host inputs come from ``synth``.  The oracle gets logical rows per sequence.
The device gets the same bytes, in contiguous or paged physical layout.  The
FP4 cache is stored either by the oracle's quantiser (small cases: the device
then reads exactly the oracle's codes) or by the library's csa2_fp4_quantize
(full-size cases; the test then checks those codes bit-exactly against the
oracle's quantiser on every row the oracle reads).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

import oracle as O
import synth
from kv_cache_decode_csa2_b200 import csa2 as B


@dataclass
class Case:
    wl: synth.Workload
    lens: np.ndarray
    seq_of_query: np.ndarray
    query_pos: np.ndarray
    layers_dev: list = field(default_factory=list)     # B.Layer per layer
    host_keys: dict = field(default_factory=dict)      # (layer, seq) -> int8 rows
    host_q: dict = field(default_factory=dict)         # (layer, query) -> (q, w)
    host_qa: dict = field(default_factory=dict)        # (layer, query) -> float32 [Hq][D]
    fp4_host: dict = field(default_factory=dict)       # (layer, seq) -> (codes, scales) (oracle quantised)
    fp4_on_gpu: bool = False
    status: torch.Tensor | None = None


def _place(rows_by_seq, lens, page_table, page_rows, width, dtype, dev):
    """Physical row array for per-sequence logical rows (contiguous or paged)."""
    if page_table is None:
        seq_rows = int(max(lens))
        out = np.zeros((len(lens) * seq_rows, width), dtype=dtype)
        for s, rows in enumerate(rows_by_seq):
            out[s * seq_rows:s * seq_rows + len(rows)] = rows
        return torch.from_numpy(out).to(dev), seq_rows
    n_pages = int(page_table.max()) + 1
    out = np.zeros((n_pages * page_rows, width), dtype=dtype)
    for s, rows in enumerate(rows_by_seq):
        n = len(rows)
        for pg in range((n + page_rows - 1) // page_rows):
            a = pg * page_rows
            b = min(n, a + page_rows)
            p = int(page_table[s, pg])
            out[p * page_rows:p * page_rows + (b - a)] = rows[a:b]
    return torch.from_numpy(out).to(dev), 0


def build(wl: synth.Workload, *, fp4_on_gpu: bool = False, dev="cuda") -> Case:
    lens = wl.lengths()
    sq, qp = wl.query_positions()
    c = Case(wl, lens, sq, qp, fp4_on_gpu=fp4_on_gpu)
    c.status = B.new_status(dev)
    nq = len(qp)
    pt = synth.page_table(wl) if wl.page_rows else None
    pt_dev = torch.from_numpy(pt).to(dev) if pt is not None else None
    c.seq_dev = torch.from_numpy(sq.astype(np.int32)).to(dev)
    c.pos_dev = torch.from_numpy(qp.astype(np.int32)).to(dev)
    c.max_ctx = int(lens.max())
    for l, mode in enumerate(wl.modes):
        keys_rows = None
        q_dev = w_dev = None
        if mode != synth.REUSE:
            per_seq = [synth.index_keys(wl, l, s) for s in range(len(lens))]
            for s, r in enumerate(per_seq):
                c.host_keys[(l, s)] = r
            kt, srows = _place(per_seq, lens, pt, wl.page_rows or 64, wl.idx_dim, np.int8, dev)
            keys_rows = B.Rows(kt, pt_dev, wl.page_rows or 64, srows)
            qs, ws = [], []
            for i in range(nq):
                q, w = synth.index_query(wl, l, i)
                c.host_q[(l, i)] = (q, w)
                qs.append(q)
                ws.append(w)
            q_dev = torch.from_numpy(np.stack(qs)).to(dev)
            w_dev = torch.from_numpy(np.stack(ws)).to(dev)
        qa = []
        for i in range(nq):
            a = synth.attn_query(wl, l, i)
            c.host_qa[(l, i)] = a
            qa.append(a)
        qa_dev = torch.from_numpy(np.stack(qa)).to(dev).to(torch.bfloat16)
        # FP4 cache of this layer
        D = wl.attn_dim
        if fp4_on_gpu:
            codes_rows, scales_rows = _fp4_gpu(wl, l, lens, pt, dev, c.status)
        else:
            cs, ss = [], []
            for s in range(len(lens)):
                codes, scales = O.fp4_quantize(synth.kv_values(wl, l, s))
                c.fp4_host[(l, s)] = (codes, scales)
                cs.append(codes)
                ss.append(scales)
            ct, srows = _place(cs, lens, pt, wl.page_rows or 64, D // 2, np.uint8, dev)
            st, _ = _place(ss, lens, pt, wl.page_rows or 64, D // 32, np.uint8, dev)
            codes_rows = B.Rows(ct, pt_dev, wl.page_rows or 64, srows)
            scales_rows = B.Rows(st, pt_dev, wl.page_rows or 64, srows)
        out = torch.empty((nq, wl.attn_heads, D), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((nq, wl.attn_heads), dtype=torch.float32, device=dev)
        ly = B.Layer(q_attn=qa_dev, codes=codes_rows, scales=scales_rows, out=out, q=q_dev, w=w_dev,
                     keys=keys_rows, lse=lse)
        if mode == synth.FULL:
            ly.pool_idx = torch.full((nq, wl.pool), -7, dtype=torch.int32, device=dev)
            ly.pool_cnt = torch.full((nq,), -7, dtype=torch.int32, device=dev)
        ly.sel_idx = torch.full((nq, wl.topk), -7, dtype=torch.int32, device=dev)
        ly.sel_cnt = torch.full((nq,), -7, dtype=torch.int32, device=dev)
        c.layers_dev.append(ly)
    return c


def _fp4_gpu(wl, l, lens, pt, dev, status):
    """Stores each sequence's KV values with csa2_fp4_quantize, chunk by chunk."""
    D = wl.attn_dim
    pr = wl.page_rows or 64
    if pt is None:
        seq_rows = int(max(lens))
        n_rows = len(lens) * seq_rows
    else:
        seq_rows = 0
        n_rows = (int(pt.max()) + 1) * pr
    codes = torch.zeros((n_rows, D // 2), dtype=torch.uint8, device=dev)
    scales = torch.zeros((n_rows, D // 32), dtype=torch.uint8, device=dev)
    step = 65536
    for s, n in enumerate(lens):
        for a in range(0, int(n), step):
            b = min(int(n), a + step)
            x = torch.from_numpy(synth.kv_values(wl, l, s, a, b)).to(dev)
            pos = np.arange(a, b)
            if pt is None:
                dst = s * seq_rows + pos
            else:
                dst = pt[s, pos // pr].astype(np.int64) * pr + pos % pr
            B.csa2_fp4_quantize(x, codes, scales, dst_rows=torch.from_numpy(dst.astype(np.int32)).to(dev),
                                status=status)
    return B.Rows(codes, torch.from_numpy(pt).to(dev) if pt is not None else None, pr, seq_rows), \
        B.Rows(scales, torch.from_numpy(pt).to(dev) if pt is not None else None, pr, seq_rows)


def physical_rows(case: Case, seq: int, positions: np.ndarray) -> np.ndarray:
    wl = case.wl
    if wl.page_rows:
        pt = synth.page_table(wl)
        return pt[seq, positions // wl.page_rows].astype(np.int64) * wl.page_rows + positions % wl.page_rows
    return seq * int(max(case.lens)) + positions


def oracle_layers(case: Case, query: int, need_rows=None):
    """Oracle inputs of every layer for one query.  FP4 rows are quantised by
    the oracle from the synth values (all rows for small cases).  If
    ``need_rows[l]`` is given, only those rows are quantised (full-size cases),
    and every other row stays zero."""
    wl = case.wl
    s = int(case.seq_of_query[query])
    n = int(case.lens[s])
    out = []
    for l, mode in enumerate(wl.modes):
        L = {"q_attn": case.host_qa[(l, query)]}
        if mode != synth.REUSE:
            L["q"], L["w"] = case.host_q[(l, query)]
            L["keys"] = case.host_keys[(l, s)]
        if (l, s) in case.fp4_host:
            L["codes"], L["scales"] = case.fp4_host[(l, s)]
        else:
            codes = np.zeros((n, wl.attn_dim // 2), np.uint8)
            scales = np.zeros((n, wl.attn_dim // 32), np.uint8)
            rows = np.unique(np.asarray(need_rows[l], dtype=np.int64))
            x = np.concatenate([synth.kv_values(wl, l, s, int(r), int(r) + 1) for r in rows]) if len(rows) else \
                np.zeros((0, wl.attn_dim), np.float32)
            cq, sq = O.fp4_quantize(x)
            codes[rows], scales[rows] = cq, sq
            L["codes"], L["scales"] = codes, scales
        out.append(L)
    return out


def tol_ok(got: np.ndarray, ref: np.ndarray, atol=2e-3, rtol=1e-2) -> tuple[bool, float]:
    err = np.abs(got.astype(np.float64) - ref)
    return bool(np.all(err <= atol + rtol * np.abs(ref))), float(err.max()) if err.size else 0.0
