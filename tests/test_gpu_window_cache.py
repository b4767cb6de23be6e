"""GPU parity of attention whose window rows come from the layer's local
window cache (csa2_sparse_attn_fp4_local, and the plan's per-layer local_kv),
and of reuse layers that share the global KV of the layer they reuse.

The local cache is a bf16 ring of R rows per sequence (position p in slot
p mod R) holding the last R positions; its values come from
synth.local_kv_values.  The oracle reads the same bf16 values."""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from kv_cache_decode_csa2_b200 import csa2 as B
from tests import gpu_cases as G

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _np(t):
    return t.detach().cpu().numpy()


def ring_rows(wl, layer, lens, R):
    """(device bf16 [n_seq*R][D] ring, host float64 view of the same values
    per sequence): slot p mod R holds position p for the last R positions."""
    D = wl.attn_dim
    rows = np.zeros((len(lens) * R, D), np.float32)
    for s, n in enumerate(lens):
        a = max(0, int(n) - R)
        x = synth.local_kv_values(wl, layer, s, a, int(n))
        for p in range(a, int(n)):
            rows[s * R + p % R] = x[p - a]
    dev = torch.from_numpy(rows).to(DEV).to(torch.bfloat16)
    host = dev.float().cpu().numpy().astype(np.float64)
    return dev, [host[s * R:(s + 1) * R] for s in range(len(lens))]


@pytest.mark.parametrize("wl,R", [(synth.C0_TINY, 128), (synth.scaled(synth.C1_SINGLE, seq_lens=(3001,)), 128),
                                  (synth.scaled(synth.C1_SINGLE, seq_lens=(3001,)), 160)],
                         ids=["hq8_d128", "hq64_d512", "hq64_d512_ring160"])
def test_local_window_attention_matches_oracle(wl, R):
    c = G.build(wl)
    ly = c.layers_dev[0]
    pos = int(c.query_pos[0])
    q, w = c.host_q[(0, 0)]
    _, _, sel = O.full_index(q, w, c.host_keys[(0, 0)], pos, wl.pool, wl.topk)
    ring_dev, ring_host = ring_rows(wl, 0, c.lens, R)
    codes, scales = c.fp4_host[(0, 0)]
    cases = [sel, np.zeros(0, np.int64), np.arange(pos - 40, pos + 1), np.array([0, 5, pos - 100, pos - 3, pos])]
    for sel_i in cases:
        sel_i = np.asarray(sel_i, dtype=np.int64)
        sel_pad = np.full((1, wl.topk), -1, np.int32)
        sel_pad[0, :len(sel_i)] = sel_i
        B.check_status(B.csa2_sparse_attn_fp4(ly.q_attn, ly.codes, ly.scales, c.pos_dev,
                                              torch.from_numpy(sel_pad).to(DEV), ly.out,
                                              sel_cnt=torch.tensor([len(sel_i)], dtype=torch.int32, device=DEV),
                                              window=wl.window, lse=ly.lse,
                                              local_kv=B.Rows(ring_dev, seq_rows=R)))
        S = O.attention_set(sel_i, pos, wl.window)
        kv = O.kv_rows_local_window(S, pos, wl.window, codes, scales, wl.attn_dim, ring_host[0])
        ref, ref_lse = O.sparse_attention(c.host_qa[(0, 0)], kv)
        ok, err = G.tol_ok(_np(ly.out.float())[0], ref)
        assert ok, f"{len(sel_i)} selected: max abs err {err}"
        assert np.allclose(_np(ly.lse)[0], ref_lse, atol=1e-3, rtol=1e-4)


def test_local_window_batch_of_sequences():
    """Several paged sequences, each with its own ring (contiguous, R rows)."""
    wl = synth.scaled(synth.C3_RAGGED, ragged=(4, 2000, 9000), modes=(synth.FULL,))
    c = G.build(wl)
    ly = c.layers_dev[0]
    R = 128
    ring_dev, ring_host = ring_rows(wl, 0, c.lens, R)
    nq = len(c.query_pos)
    sels = []
    sel_pad = np.full((nq, wl.topk), -1, np.int32)
    cnt = np.zeros(nq, np.int32)
    for i in range(nq):
        s = int(c.seq_of_query[i])
        q, w = c.host_q[(0, i)]
        _, _, sel = O.full_index(q, w, c.host_keys[(0, s)], int(c.query_pos[i]), wl.pool, wl.topk)
        sels.append(sel)
        sel_pad[i, :len(sel)] = sel
        cnt[i] = len(sel)
    B.check_status(B.csa2_sparse_attn_fp4(ly.q_attn, ly.codes, ly.scales, c.pos_dev,
                                          torch.from_numpy(sel_pad).to(DEV), ly.out,
                                          sel_cnt=torch.from_numpy(cnt).to(DEV), seq_of_query=c.seq_dev,
                                          window=wl.window, local_kv=B.Rows(ring_dev, seq_rows=R)))
    out = _np(ly.out.float())
    for i in range(nq):
        s, pos = int(c.seq_of_query[i]), int(c.query_pos[i])
        codes, scales = c.fp4_host[(0, s)]
        S = O.attention_set(sels[i], pos, wl.window)
        kv = O.kv_rows_local_window(S, pos, wl.window, codes, scales, wl.attn_dim, ring_host[s])
        ref, _ = O.sparse_attention(c.host_qa[(0, i)], kv)
        ok, err = G.tol_ok(out[i], ref)
        assert ok, f"query {i}: max abs err {err}"


def test_plan_with_local_rings_and_shared_global_kv():
    """An 8-layer plan in which layers 0, 2 and 5 read their window from a
    local ring, and every REUSE layer reads the global FP4 KV of the layer it
    reuses (the same codes and scales views)."""
    wl = synth.scaled(synth.C2_1M_PLAN, seq_lens=(7001,))
    c = G.build(wl)
    R = 128
    src = 0
    for l, mode in enumerate(wl.modes):
        if mode != synth.REUSE:
            src = l
        else:   # share the global KV of the most recent FULL/REINDEX layer
            c.layers_dev[l].codes = c.layers_dev[src].codes
            c.layers_dev[l].scales = c.layers_dev[src].scales
            c.fp4_host[(l, 0)] = c.fp4_host[(src, 0)]
    rings = {}
    for l in (0, 2, 5):
        ring_dev, ring_host = ring_rows(wl, l, c.lens, R)
        c.layers_dev[l].local_kv = B.Rows(ring_dev, seq_rows=R)
        rings[l] = ring_host[0]
    plan = B.csa2_layer_plan(list(wl.modes), c.layers_dev, query_pos=c.pos_dev, max_ctx=c.max_ctx, P=wl.pool,
                             K=wl.topk, window=wl.window)
    B.check_status(plan.status)
    pos = int(c.query_pos[0])
    layers = G.oracle_layers(c, 0)
    for l, ring in rings.items():
        layers[l]["local_ring"] = ring
    res = O.decode_layer_plan(wl.modes, layers, pos, wl.pool, wl.topk, wl.window)
    for l, (r, ly) in enumerate(zip(res, c.layers_dev)):
        n = int(_np(ly.sel_cnt)[0]) if ly.sel_cnt is not None else len(r.sel_idx)
        assert n == len(r.sel_idx) and np.array_equal(_np(ly.sel_idx)[0, :n], r.sel_idx), f"layer {l}"
        ok, err = G.tol_ok(_np(ly.out[0].float()), r.out)
        assert ok, f"layer {l}: max abs err {err}"
