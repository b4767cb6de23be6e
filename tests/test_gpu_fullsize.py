"""Parity at the workloads' full sizes, in the launch configuration the bench
times, on outputs the oracle can compute one by one.

- The 1M-context 8-layer decode plan: one csa2_layer_plan call (the zeroing
  launch and programmatic dependent launches of the bench's step).  The pool
  and every layer's selection are compared bit-exactly with the oracle's, and
  every layer's attention output within the attention tolerance; the oracle
  quantises only the FP4 rows of each layer's attention set (its own, not the
  GPU's).
- The 2048-query prefill chunk at the 262,144-row context: the first and the
  last query's top-512 and attention.

Inputs are the seeded synthetic workloads (synth/).
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from kv_cache_decode_csa2_b200 import csa2 as B
from tests import gpu_cases as G

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().cpu().numpy()


def _oracle_attention(wl, layer, seq, q_attn, S):
    """The oracle's attention over rows S of one layer's cache, with the FP4
    rows quantised by the oracle from the synthetic values."""
    x = np.concatenate([synth.kv_values(wl, layer, seq, int(r), int(r) + 1) for r in S])
    codes, scales = O.fp4_quantize(x)
    o, _ = O.sparse_attention(q_attn, O.fp4_dequant(codes, scales, wl.attn_dim))
    return o


def test_full_size_decode_plan_1m_context():
    wl = synth.C2_1M_PLAN
    c = G.build(wl, fp4_on_gpu=True)
    plan = B.csa2_layer_plan(list(wl.modes), c.layers_dev, query_pos=c.pos_dev, max_ctx=c.max_ctx, P=wl.pool,
                             K=wl.topk, window=wl.window)
    B.check_status(plan.status)
    pos = int(c.query_pos[0])
    # the oracle's selections, from the synthetic inputs only
    sels, pool = [], None
    for l, mode in enumerate(wl.modes):
        if mode == synth.FULL:
            q, w = c.host_q[(l, 0)]
            _, pool, sel = O.full_index(q, w, c.host_keys[(l, 0)], pos, wl.pool, wl.topk)
        elif mode == synth.REINDEX:
            q, w = c.host_q[(l, 0)]
            _, sel = O.reindex(q, w, c.host_keys[(l, 0)], pool, wl.topk)
        sels.append(sel)
    full = c.layers_dev[0]
    n = int(_np(full.pool_cnt)[0])
    assert n == len(pool) and np.array_equal(_np(full.pool_idx)[0, :n], pool)
    for l, (ly, sel) in enumerate(zip(c.layers_dev, sels)):
        m = int(_np(ly.sel_cnt)[0])
        assert m == len(sel) and np.array_equal(_np(ly.sel_idx)[0, :m], sel), f"layer {l}"
        S = O.attention_set(sel, pos, wl.window)
        ok, err = G.tol_ok(_np(ly.out[0].float()), _oracle_attention(wl, l, 0, c.host_qa[(l, 0)], S))
        assert ok, f"layer {l}: max abs err {err}"


def test_full_size_prefill_chunk_sampled_queries():
    wl = synth.C4_PREFILL
    c = G.build(wl, fp4_on_gpu=True)
    ly = c.layers_dev[0]
    nq = len(c.query_pos)
    B.check_status(B.csa2_index_full(ly.q, ly.w, ly.keys, c.pos_dev, c.max_ctx, seq_of_query=c.seq_dev,
                                     K=wl.topk, sel_idx=ly.sel_idx, sel_cnt=ly.sel_cnt))
    B.check_status(B.csa2_sparse_attn_fp4(ly.q_attn, ly.codes, ly.scales, c.pos_dev, ly.sel_idx, ly.out,
                                          sel_cnt=ly.sel_cnt, seq_of_query=c.seq_dev, window=wl.window))
    sels, cnts, outs = _np(ly.sel_idx), _np(ly.sel_cnt), _np(ly.out.float())
    keys = c.host_keys[(0, 0)]
    for i in (0, nq - 1):
        q, w = c.host_q[(0, i)]
        pos = int(c.query_pos[i])
        s = O.index_scores(q, w, keys[:pos + 1])
        sel = O.top_k_positions(s, np.arange(pos + 1, dtype=np.int64), wl.topk)
        assert cnts[i] == len(sel) and np.array_equal(sels[i, :cnts[i]], sel), f"query {i}"
        S = O.attention_set(sel, pos, wl.window)
        ok, err = G.tol_ok(outs[i], _oracle_attention(wl, 0, 0, c.host_qa[(0, i)], S))
        assert ok, f"query {i}: max abs err {err}"
