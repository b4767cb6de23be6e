"""A speculative-verify block through a plan call that groups its queries:
5 queries of one sequence share the key tiles of the index scan (groups of
4 and 1), and every layer's pool, selection and attention match the oracle."""
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


@pytest.mark.parametrize("nq,ctx", [(5, 30000), (2, 20001), (7, 140001)])
def test_plan_verify_block_grouped(nq, ctx):
    wl = synth.scaled(synth.C1_SINGLE, seq_lens=(ctx,), prefill=(nq, ctx - nq),
                      modes=(synth.FULL, synth.REINDEX, synth.REUSE))
    c = G.build(wl)
    assert len(c.query_pos) == nq and (c.seq_of_query == 0).all()
    plan = B.csa2_layer_plan(list(wl.modes), c.layers_dev, query_pos=c.pos_dev, seq_of_query=c.seq_dev,
                             max_ctx=c.max_ctx, P=wl.pool, K=wl.topk, window=wl.window, group_queries=True)
    B.check_status(plan.status)
    for i in range(nq):
        pos = int(c.query_pos[i])
        res = O.decode_layer_plan(wl.modes, G.oracle_layers(c, i), pos, wl.pool, wl.topk, wl.window)
        for l, (r, ly) in enumerate(zip(res, c.layers_dev)):
            if r.pool_idx is not None:
                n = int(_np(ly.pool_cnt)[i])
                assert n == len(r.pool_idx) and np.array_equal(_np(ly.pool_idx)[i, :n], r.pool_idx)
            n = int(_np(ly.sel_cnt)[i])
            assert n == len(r.sel_idx) and np.array_equal(_np(ly.sel_idx)[i, :n], r.sel_idx), f"q{i} layer {l}"
            ok, err = G.tol_ok(_np(ly.out[i].float()), r.out)
            assert ok, f"query {i} layer {l}: max abs err {err}"
