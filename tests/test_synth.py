"""The seeded input generator: deterministic, row-addressable, and drawing the
distributions that the workloads name."""
import numpy as np

import synth


def test_rows_are_addressable_and_deterministic():
    wl = synth.scaled(synth.C1_SINGLE, seq_lens=(5000,))
    full = synth.index_keys(wl, 0, 0)
    assert full.shape == (5000, 128) and full.dtype == np.int8
    assert np.array_equal(synth.index_keys(wl, 0, 0, 1000, 3100), full[1000:3100])
    assert np.array_equal(synth.index_keys(wl, 0, 0), full)
    kv = synth.kv_values(wl, 2, 0)
    assert np.array_equal(synth.kv_values(wl, 2, 0, 4000, 4999), kv[4000:4999])
    assert not np.array_equal(synth.kv_values(wl, 3, 0, 0, 10), kv[:10])   # fresh per layer


def test_distributions():
    wl = synth.scaled(synth.C1_SINGLE, seq_lens=(20000,))
    k = synth.index_keys(wl, 0, 0)
    assert k.min() == -16 and k.max() == 16
    assert abs(k.mean()) < 0.05 and abs(k.astype(np.float64).var() - 90.67) < 1.0
    q, w = synth.index_query(wl, 0, 0)
    assert q.shape == (64, 128) and w.shape == (64,)
    assert w.min() >= 1 and w.max() <= 8
    x = synth.kv_values(wl, 0, 0)
    big = np.abs(x) > 6.5          # beyond what N(0,1) reaches at this size
    assert 0.004 < big.mean() < 0.009
    qa = synth.attn_query(wl, 0, 0)
    assert np.array_equal(qa, synth.round_to_bf16(qa))
    loc = synth.local_kv_values(wl, 0, 0, 19000, 20000)
    assert loc.shape == (1000, 512) and np.array_equal(loc, synth.round_to_bf16(loc))
    assert np.array_equal(synth.local_kv_values(wl, 0, 0, 19500, 19600), loc[500:600])
    assert not np.array_equal(loc, synth.round_to_bf16(x[19000:20000]))   # not the main cache's values
    assert 0.5 < np.abs(loc).mean() < 1.2


def test_ragged_lengths_and_pages():
    wl = synth.C3_RAGGED
    lens = wl.lengths()
    assert len(lens) == 32 and lens.min() >= 32768 and lens.max() <= 262144
    t = synth.page_table(wl)
    used = t[t >= 0]
    assert sorted(used.tolist()) == list(range(int(((lens + 63) // 64).sum())))
    for s, n in enumerate(lens):
        assert (t[s] >= 0).sum() == (n + 63) // 64


def test_workloads_use_the_page_sizes():
    sizes = {}
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "csa2_page_sizes.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, v = line.split()
                sizes[k] = int(v)
    for wl in (synth.C1_SINGLE, synth.C2_1M_PLAN, synth.C3_RAGGED):
        assert (wl.pool, wl.topk, wl.window) == (sizes["pool"], sizes["topk"], sizes["window"])
    assert synth.C4_PREFILL.topk == sizes["topk"] and synth.C4_PREFILL.window == sizes["window"]
    sq, qp = synth.C4_PREFILL.query_positions()
    assert qp[0] == 260096 and qp[-1] == 262143 and (sq == 0).all()
