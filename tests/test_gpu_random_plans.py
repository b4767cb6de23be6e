"""Randomised small plans against the oracle: context lengths that are not
multiples of 64 or 128, contexts shorter than the pool, the selection or the
window, K close to P, several sequences (contiguous or paged), random mode
sequences.  Seeded, so a failure names its case."""
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


def _case(seed):
    rng = np.random.default_rng(1000 + seed)
    n_layers = int(rng.integers(1, 6))
    modes = (synth.FULL,) + tuple(int(m) for m in rng.choice([synth.FULL, synth.REINDEX, synth.REUSE],
                                                               size=n_layers - 1, p=[0.2, 0.4, 0.4]))
    H = int(rng.choice([4, 16, 64]))
    D_idx = int(rng.choice([64, 128]))
    Hq = int(rng.choice([8, 16, 32, 64]))
    D = int(rng.choice([128, 512]))
    n_seq = int(rng.integers(1, 4))
    lens = tuple(int(x) for x in rng.integers(1, 5000, size=n_seq))
    P = int(rng.integers(1, 2049))
    K = int(rng.integers(1, min(P, 600) + 1))
    window = int(rng.integers(1, 200))
    paged = bool(rng.integers(0, 2))
    base = synth.C0_TINY if D_idx == 64 else synth.C1_SINGLE
    return synth.scaled(base, name=f"random_plan_{seed}", idx_heads=H, idx_dim=D_idx, attn_heads=Hq, attn_dim=D,
                        pool=P, topk=K, window=window, modes=modes, seq_lens=lens, ragged=None,
                        page_rows=64 if paged else None)


@pytest.mark.parametrize("seed", range(16))
def test_random_plan_matches_oracle(seed):
    wl = _case(seed)
    c = G.build(wl)
    plan = B.csa2_layer_plan(list(wl.modes), c.layers_dev, query_pos=c.pos_dev, seq_of_query=c.seq_dev,
                             max_ctx=c.max_ctx, P=wl.pool, K=wl.topk, window=wl.window)
    B.check_status(plan.status)
    for i in range(len(c.query_pos)):
        pos = int(c.query_pos[i])
        res = O.decode_layer_plan(wl.modes, G.oracle_layers(c, i), pos, wl.pool, wl.topk, wl.window)
        for l, (r, ly) in enumerate(zip(res, c.layers_dev)):
            if r.pool_idx is not None:
                n = int(_np(ly.pool_cnt)[i])
                assert n == len(r.pool_idx) and np.array_equal(_np(ly.pool_idx)[i, :n], r.pool_idx), (wl, i, l)
            n = int(_np(ly.sel_cnt)[i])
            assert n == len(r.sel_idx) and np.array_equal(_np(ly.sel_idx)[i, :n], r.sel_idx), (wl, i, l)
            ok, err = G.tol_ok(_np(ly.out[i].float()), r.out)
            assert ok, f"{wl.name} query {i} layer {l}: max abs err {err}"
