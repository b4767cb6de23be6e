"""Full-size parity of the single 131,072-context decode step and of the
32-sequence paged ragged batch (sampled sequences), on outputs the oracle
computes one by one."""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from kv_cache_decode_csa2_b200 import csa2 as B
from tests import gpu_cases as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _np(t):
    return t.detach().cpu().numpy()


def _oracle_attention(wl, layer, seq, q_attn, S):
    x = np.concatenate([synth.kv_values(wl, layer, seq, int(r), int(r) + 1) for r in S])
    codes, scales = O.fp4_quantize(x)
    o, _ = O.sparse_attention(q_attn, O.fp4_dequant(codes, scales, wl.attn_dim))
    return o


def test_full_size_single_decode_ctx131072():
    wl = synth.C1_SINGLE
    c = G.build(wl, fp4_on_gpu=True)
    plan = B.csa2_layer_plan(list(wl.modes), c.layers_dev, query_pos=c.pos_dev, max_ctx=c.max_ctx, P=wl.pool,
                             K=wl.topk, window=wl.window)
    B.check_status(plan.status)
    pos = int(c.query_pos[0])
    q, w = c.host_q[(0, 0)]
    _, pool, sel = O.full_index(q, w, c.host_keys[(0, 0)], pos, wl.pool, wl.topk)
    ly = c.layers_dev[0]
    n = int(_np(ly.pool_cnt)[0])
    assert n == len(pool) and np.array_equal(_np(ly.pool_idx)[0, :n], pool)
    m = int(_np(ly.sel_cnt)[0])
    assert m == len(sel) and np.array_equal(_np(ly.sel_idx)[0, :m], sel)
    S = O.attention_set(sel, pos, wl.window)
    ok, err = G.tol_ok(_np(ly.out[0].float()), _oracle_attention(wl, 0, 0, c.host_qa[(0, 0)], S))
    assert ok, f"max abs err {err}"


def test_full_size_ragged_paged_batch_sampled_sequences():
    wl = synth.C3_RAGGED
    c = G.build(wl, fp4_on_gpu=True)
    plan = B.csa2_layer_plan(list(wl.modes), c.layers_dev, query_pos=c.pos_dev, seq_of_query=c.seq_dev,
                             max_ctx=c.max_ctx, P=wl.pool, K=wl.topk, window=wl.window)
    B.check_status(plan.status)
    ly = c.layers_dev[0]
    pools, pcnt, sels, scnt = _np(ly.pool_idx), _np(ly.pool_cnt), _np(ly.sel_idx), _np(ly.sel_cnt)
    outs = _np(ly.out.float())
    lens = c.lens
    for i in sorted({int(np.argmin(lens)), int(np.argmax(lens)), 0}):
        s, pos = int(c.seq_of_query[i]), int(c.query_pos[i])
        q, w = c.host_q[(0, i)]
        _, pool, sel = O.full_index(q, w, c.host_keys[(0, s)], pos, wl.pool, wl.topk)
        assert pcnt[i] == len(pool) and np.array_equal(pools[i, :pcnt[i]], pool), f"query {i}"
        assert scnt[i] == len(sel) and np.array_equal(sels[i, :scnt[i]], sel), f"query {i}"
        S = O.attention_set(sel, pos, wl.window)
        ok, err = G.tol_ok(outs[i], _oracle_attention(wl, 0, s, c.host_qa[(0, i)], S))
        assert ok, f"query {i}: max abs err {err}"
