"""A context-sharded decode step on one GPU: the context split into R slices,
each handled by the library as a GPU that owns that slice would, then merged.

Per slice: the full-mode index scores and the slice's own top-P pool.  The
exchange payload is each slice's pool with its scores and global positions
(what an all-gather would carry); csa2_topk_pool over the concatenation, with
those positions as candidate positions, gives the global pool and the
global top-K exactly (every global member is in its slice's pool).  Attention
runs per slice over the rows of S = selection U window that the slice holds
(window 0, the rows as an explicit list) and csa2_attn_combine merges the R
partial (o, lse).  Everything is compared with the oracle on the whole
context: pools and selections bit-exactly, attention within tolerance."""
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


@pytest.mark.parametrize("ctx,R", [(100000, 4), (70001, 3)])
def test_context_sharded_step_matches_oracle(ctx, R):
    wl = synth.scaled(synth.C1_SINGLE, seq_lens=(ctx,))
    P, K, W = wl.pool, wl.topk, wl.window
    c = G.build(wl, fp4_on_gpu=True)
    ly = c.layers_dev[0]
    pos = int(c.query_pos[0])
    cuts = [ctx * r // R for r in range(R + 1)]
    assert min(b - a for a, b in zip(cuts, cuts[1:])) >= P      # every slice fills its pool
    # ---- per slice: scores and the slice's pool, then the exchange payload
    cand_s, cand_p = [], []
    for lo, hi in zip(cuts, cuts[1:]):
        n = hi - lo
        qpos = torch.tensor([min(pos, hi - 1) - lo], dtype=torch.int32, device=DEV)
        scores = torch.empty((1, n), dtype=torch.int32, device=DEV)
        pool = torch.empty((1, P), dtype=torch.int32, device=DEV)
        cnt = torch.empty((1,), dtype=torch.int32, device=DEV)
        B.check_status(B.csa2_index_full(ly.q, ly.w, B.Rows(ly.keys.data[lo:hi]), qpos, n, scores=scores, P=P,
                                         pool_idx=pool, pool_cnt=cnt))
        assert int(cnt.item()) == P
        cand_s.append(scores[0, pool[0].long()])
        cand_p.append(pool[0] + lo)
    S = torch.cat(cand_s)[None].contiguous()
    Pp = torch.cat(cand_p)[None].contiguous()
    gpool = torch.empty((1, P), dtype=torch.int32, device=DEV)
    gsel = torch.empty((1, K), dtype=torch.int32, device=DEV)
    B.check_status(B.csa2_topk_pool(S, P, gpool, cand_pos=Pp))
    B.check_status(B.csa2_topk_pool(S, K, gsel, cand_pos=Pp))
    q, w = c.host_q[(0, 0)]
    _, ref_pool, ref_sel = O.full_index(q, w, c.host_keys[(0, 0)], pos, P, K)
    assert np.array_equal(_np(gpool)[0], ref_pool)
    assert np.array_equal(_np(gsel)[0], ref_sel)
    # ---- attention per slice over the rows of S it holds, then the combine
    Satt = O.attention_set(ref_sel, pos, W)
    Hq, D = wl.attn_heads, wl.attn_dim
    o_parts = torch.empty((R, 1, Hq, D), dtype=torch.bfloat16, device=DEV)
    lse_parts = torch.empty((R, 1, Hq), dtype=torch.float32, device=DEV)
    for r, (lo, hi) in enumerate(zip(cuts, cuts[1:])):
        rows = Satt[(Satt >= lo) & (Satt < hi)] - lo
        k = max(len(rows), 1)
        sel = torch.full((1, k), -1, dtype=torch.int32, device=DEV)
        sel[0, :len(rows)] = torch.from_numpy(rows.astype(np.int32)).to(DEV)
        scnt = torch.tensor([len(rows)], dtype=torch.int32, device=DEV)
        qpos = torch.tensor([hi - 1 - lo], dtype=torch.int32, device=DEV)
        B.check_status(B.csa2_sparse_attn_fp4(ly.q_attn, B.Rows(ly.codes.data[lo:hi]), B.Rows(ly.scales.data[lo:hi]),
                                              qpos, sel, o_parts[r], sel_cnt=scnt, window=0, lse=lse_parts[r]))
    out = torch.empty((1, Hq, D), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((1, Hq), dtype=torch.float32, device=DEV)
    B.check_status(B.csa2_attn_combine(o_parts, lse_parts, out, lse_out=lse))
    ref = G.oracle_layers(c, 0, need_rows=[Satt])[0]
    ref_o, ref_l = O.sparse_attention(c.host_qa[(0, 0)], O.fp4_dequant(ref["codes"][Satt], ref["scales"][Satt], D))
    ok, err = G.tol_ok(_np(out[0].float()), ref_o)
    assert ok, f"max abs err {err}"
    assert np.allclose(_np(lse[0]), ref_l, rtol=0, atol=1e-3)


def test_combine_of_one_part_is_that_part_and_empty_parts_vanish():
    rng = np.random.default_rng(3)
    Hq, D = 16, 128
    o = torch.from_numpy(rng.standard_normal((1, 2, Hq, D)).astype(np.float32)).to(DEV).to(torch.bfloat16)
    lse = torch.from_numpy(rng.standard_normal((1, 2, Hq)).astype(np.float32)).to(DEV)
    parts = torch.cat([o, torch.zeros_like(o)])                         # part 1 holds no row
    lses = torch.cat([lse, torch.full_like(lse, float("-inf"))])
    out = torch.empty((2, Hq, D), dtype=torch.bfloat16, device=DEV)
    lo = torch.empty((2, Hq), dtype=torch.float32, device=DEV)
    B.check_status(B.csa2_attn_combine(parts, lses, out, lse_out=lo))
    assert torch.equal(out, o[0])
    assert torch.allclose(lo, lse[0], rtol=0, atol=1e-6)
