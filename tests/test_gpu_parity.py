"""GPU parity: libcsa2 (through its C ABI) against the CPU oracle.

Indices, scores and FP4 codes must match bit-exactly.  Attention outputs must
satisfy |gpu - ref| <= 2e-3 + 1e-2 |ref| against the fp64 oracle.  These sizes
finish in seconds on the oracle and still span several tiles and a ragged
tail.  Full-size cases are in test_gpu_fullsize.py.
"""
import math

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


# ------------------------------------------------------------------ K7 quantiser
def test_fp4_quantize_bitexact():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2048, 512)).astype(np.float32)
    x[::7] *= 8
    x[1, :32] = 0                                  # zero block
    x[2, :32] *= 1e-5                              # underflowing scale
    x[3, :32] *= 5000                              # saturating scale
    # exact ties of the E2M1 grid at scale 1: amax 6 pins the scale to 1.0
    x[4, :32] = np.array([6, .25, .75, 1.25, 1.75, 2.5, 3.5, 5, -.25, -.75, -1.25, -1.75, -2.5, -3.5, -5,
                          0, -0.0, 6, -6, 7, 1, 2, 3, 4, .5, 1.5, -1, -2, -3, -4, -.5, -1.5], np.float32)
    # exact E4M3 ties of amax/6: midpoints between adjacent scale values
    v = O.e4m3_decode(np.arange(0x7F))
    mids = (v[:-1] + v[1:]) / 2 * 6
    for i in range(32):
        x[5 + i, :32] = 0
        x[5 + i, 0] = mids[i * 4]
    codes_ref, scales_ref = O.fp4_quantize(x)
    xd = torch.from_numpy(x).to(DEV)
    codes = torch.zeros((2048, 256), dtype=torch.uint8, device=DEV)
    scales = torch.zeros((2048, 16), dtype=torch.uint8, device=DEV)
    st = B.csa2_fp4_quantize(xd, codes, scales)
    B.check_status(st)
    assert np.array_equal(_np(scales), scales_ref)
    assert np.array_equal(_np(codes), codes_ref)


def test_fp4_quantize_one_ulp_from_midpoints():
    """fp32 values one ulp either side of (and exactly on) midpoint x scale,
    for every E2M1 midpoint, both signs and 59 scales: the quotient x/scale
    may round onto the midpoint in fp32, and the code must still be the
    nearest of the exact quotient (ties to even only for exact midpoints)."""
    mids = np.array([.25, .75, 1.25, 1.75, 2.5, 3.5, 5.0])
    scales = O.e4m3_decode(np.arange(8, 126, 2))                   # 59 normal E4M3 scales
    rows = []
    for sv in scales:
        # one block per (scale, sign): element 0 = 6 * scale pins the scale to sv exactly
        for sign in (1.0, -1.0):
            blk = np.zeros(32, np.float64)
            blk[0] = 6 * sv
            k = 1
            for m in mids:
                c = np.float32(m * sv)
                for v in (np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))):
                    blk[k] = sign * float(v)
                    k += 1
            rows.append(blk)
    x = np.stack(rows).astype(np.float32)                          # [120][32]
    assert np.all(np.abs(x[:, 0]) == 6 * np.repeat(scales, 2))
    codes_ref, scales_ref = O.fp4_quantize(x)
    assert np.array_equal(O.e4m3_decode(scales_ref[:, 0]), np.repeat(scales, 2))
    codes = torch.zeros((len(x), 16), dtype=torch.uint8, device=DEV)
    sc = torch.zeros((len(x), 1), dtype=torch.uint8, device=DEV)
    B.check_status(B.csa2_fp4_quantize(torch.from_numpy(x).to(DEV), codes, sc))
    assert np.array_equal(_np(sc), scales_ref)
    assert np.array_equal(_np(codes), codes_ref)


def test_fp4_quantize_scatter_rows():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((100, 128)).astype(np.float32)
    dst = rng.permutation(300)[:100].astype(np.int32)
    codes = torch.zeros((300, 64), dtype=torch.uint8, device=DEV)
    scales = torch.zeros((300, 4), dtype=torch.uint8, device=DEV)
    B.check_status(B.csa2_fp4_quantize(torch.from_numpy(x).to(DEV), codes, scales,
                                       dst_rows=torch.from_numpy(dst).to(DEV)))
    cr, sr = O.fp4_quantize(x)
    assert np.array_equal(_np(codes)[dst], cr) and np.array_equal(_np(scales)[dst], sr)
    untouched = np.setdiff1d(np.arange(300), dst)
    assert not _np(codes)[untouched].any()


# ------------------------------------------------------------------ K1 + K2: full index
def _index_case(wl, nq_check=None):
    c = G.build(wl)
    ly = c.layers_dev[0]
    nq = len(c.query_pos)
    scores = torch.full((nq, c.max_ctx), -123, dtype=torch.int32, device=DEV)
    B.check_status(B.csa2_index_full(ly.q, ly.w, ly.keys, c.pos_dev, c.max_ctx, seq_of_query=c.seq_dev,
                                     scores=scores, P=wl.pool, pool_idx=ly.pool_idx, pool_cnt=ly.pool_cnt,
                                     K=wl.topk, sel_idx=ly.sel_idx, sel_cnt=ly.sel_cnt))
    sc, pool, pcnt, sel, scnt = map(_np, (scores, ly.pool_idx, ly.pool_cnt, ly.sel_idx, ly.sel_cnt))
    for i in range(nq if nq_check is None else nq_check):
        s = int(c.seq_of_query[i])
        pos = int(c.query_pos[i])
        q, w = c.host_q[(0, i)]
        ref_s, ref_pool, ref_sel = O.full_index(q, w, c.host_keys[(0, s)], pos, wl.pool, wl.topk)
        assert np.array_equal(sc[i, :pos + 1], ref_s), f"scores of query {i}"
        assert (sc[i, pos + 1:] == -123).all()
        assert pcnt[i] == len(ref_pool) and np.array_equal(pool[i, :pcnt[i]], ref_pool)
        assert (pool[i, pcnt[i]:] == -1).all()
        assert scnt[i] == len(ref_sel) and np.array_equal(sel[i, :scnt[i]], ref_sel)
        assert (sel[i, scnt[i]:] == -1).all()


def test_index_full_tiny_d64():
    _index_case(synth.C0_TINY)


def test_index_full_ragged_tail_large_path():
    # 20011 positions: many 128-row tiles, a ragged last tile, the multi-CTA top-k
    _index_case(synth.scaled(synth.C1_SINGLE, seq_lens=(20011,)))


@pytest.mark.parametrize("ctx", [1, 2, 100, 129, 1025])
def test_index_full_short_contexts(ctx):
    # context shorter than the pool, the selection and the window
    _index_case(synth.scaled(synth.C0_TINY, seq_lens=(ctx,)))


def test_index_full_paged_ragged_batch():
    wl = synth.scaled(synth.C3_RAGGED, ragged=(5, 3000, 40000))
    _index_case(wl)


def test_index_score_range_error():
    q = torch.full((1, 64, 128), -128, dtype=torch.int8, device=DEV)
    w = torch.full((1, 64), 127, dtype=torch.int8, device=DEV)
    keys = torch.zeros((256, 128), dtype=torch.int8, device=DEV)
    st = B.csa2_index_full(q, w, B.Rows(keys), torch.tensor([255], dtype=torch.int32, device=DEV), 256,
                           scores=torch.zeros((1, 256), dtype=torch.int32, device=DEV))
    assert int(st.item()) == 5       # SCORE_RANGE


def test_index_bad_position_is_reported():
    wl = synth.C0_TINY
    c = G.build(wl)
    ly = c.layers_dev[0]
    bad = torch.tensor([5000], dtype=torch.int32, device=DEV)     # >= max_ctx
    st = B.csa2_index_full(ly.q, ly.w, ly.keys, bad, c.max_ctx, P=16, pool_idx=ly.pool_idx[:, :16].contiguous(),
                           pool_cnt=ly.pool_cnt)
    assert int(st.item()) == 6
    assert int(_np(ly.pool_cnt)[0]) == 0


# ------------------------------------------------------------------ K2: top-k alone
# Sizes cover one select CTA per row (n <= 16384), several co-resident CTAs per
# row (n > 16384), and rows that do not fit on the device at once (3 x 10^6:
# the multi-pass path); spreads 2 and 3 make tie lists too long to rank.
@pytest.mark.parametrize("n,k,spread", [(5000, 700, 3), (16384, 512, 50), (16385, 512, 50),
                                        (70000, 16384, 1000), (70000, 300, 2), (300000, 16384, 10 ** 6),
                                        (1000000, 16384, 25000)])
def test_topk_pool_matches_oracle(n, k, spread):
    rng = np.random.default_rng(n + k)
    nq = 3
    s = rng.integers(-spread, spread + 1, size=(nq, n)).astype(np.int32)
    nv = np.array([n, n // 2 + 1, min(n, k // 2)], dtype=np.int32)
    out = torch.empty((nq, k), dtype=torch.int32, device=DEV)
    cnt = torch.empty((nq,), dtype=torch.int32, device=DEV)
    B.check_status(B.csa2_topk_pool(torch.from_numpy(s).to(DEV), k, out, out_cnt=cnt,
                                    n_valid=torch.from_numpy(nv).to(DEV)))
    o, c = _np(out), _np(cnt)
    for i in range(nq):
        ref = O.top_k_positions(s[i, :nv[i]], np.arange(nv[i]), k)
        assert c[i] == len(ref) and np.array_equal(o[i, :c[i]], ref)
        assert (o[i, c[i]:] == -1).all()


@pytest.mark.parametrize("spread,k", [(10 ** 6, 700), (1000, 512), (2, 600), (0, 512)])
def test_topk_many_long_rows(spread, k):
    """40 rows of up to 50,000 candidates: more rows than fit on the device at
    once, so every row gets one CTA.  Spread 2 and 0 make the tie list too
    long to rank (radix path); ragged valid counts include one below k."""
    rng = np.random.default_rng(spread + k)
    nq, n = 40, 50000
    s = rng.integers(-spread, spread + 1, size=(nq, n)).astype(np.int32)
    nv = rng.integers(n // 2, n + 1, size=nq).astype(np.int32)
    nv[3] = k // 2
    out = torch.empty((nq, k), dtype=torch.int32, device=DEV)
    cnt = torch.empty((nq,), dtype=torch.int32, device=DEV)
    B.check_status(B.csa2_topk_pool(torch.from_numpy(s).to(DEV), k, out, out_cnt=cnt,
                                    n_valid=torch.from_numpy(nv).to(DEV)))
    o, c = _np(out), _np(cnt)
    for i in range(nq):
        ref = O.top_k_positions(s[i, :nv[i]], np.arange(nv[i]), k)
        assert c[i] == len(ref) and np.array_equal(o[i, :c[i]], ref), f"row {i}"
        assert (o[i, c[i]:] == -1).all()


@pytest.mark.parametrize("spread,k,with_pos", [(10 ** 6, 700, False), (1000, 512, True), (2, 600, False),
                                                (0, 512, True)])
def test_topk_one_cta_per_row(spread, k, with_pos):
    """80 rows of up to 50,000 candidates: at least half as many rows as SMs
    and too long for the co-resident select, so each row takes one CTA of the
    row kernel (the 40- and 24-row cases above take the chunked passes).
    Wide spreads keep the few candidates above the sampled cut in shared
    memory; spreads 2 and 0 put too many there (the row is read again) and
    overflow the tie list; ragged valid counts include one below k and one
    inside a single select span."""
    rng = np.random.default_rng(7 * spread + k)
    nq, n = 80, 50000
    s = rng.integers(-spread, spread + 1, size=(nq, n)).astype(np.int32)
    nv = rng.integers(n // 2, n + 1, size=nq).astype(np.int32)
    nv[5], nv[6], nv[7] = k // 2, 9000, n
    pos = None
    if with_pos:
        pos = np.sort(rng.choice(10 ** 7, size=(nq, n), replace=True), axis=1).astype(np.int32)
        pos += np.arange(n, dtype=np.int32)[None]
    out = torch.empty((nq, k), dtype=torch.int32, device=DEV)
    cnt = torch.empty((nq,), dtype=torch.int32, device=DEV)
    B.check_status(B.csa2_topk_pool(torch.from_numpy(s).to(DEV), k, out, out_cnt=cnt,
                                    n_valid=torch.from_numpy(nv).to(DEV),
                                    cand_pos=None if pos is None else torch.from_numpy(pos).to(DEV)))
    o, c = _np(out), _np(cnt)
    for i in range(nq):
        p_i = np.arange(nv[i]) if pos is None else pos[i, :nv[i]]
        ref = O.top_k_positions(s[i, :nv[i]], p_i, k)
        assert c[i] == len(ref) and np.array_equal(o[i, :c[i]], ref), f"row {i}"
        assert (o[i, c[i]:] == -1).all()


@pytest.mark.parametrize("mode,P,K", [("random", 16384, 512), ("half", 16384, 512), ("random", 1024, 256)])
def test_index_full_prefill_pool_and_selection_rows(mode, P, K):
    """80 causal queries at the end of a 50,000-row sequence, each keeping a
    pool and a top-K: the row kernel with both targets in one pass.  A pool
    of 16,384 makes its sampled cut loose (the row is read twice); a pool of
    1,024 keeps the candidates above the cut in shared memory (read once).
    Half-zero keys put thousands of equal zero scores at the pool's
    threshold.  Sampled queries are checked against the oracle one by one."""
    ctx, nq = 50000, 80
    wl = synth.scaled(synth.C1_SINGLE, seq_lens=(ctx,), prefill=(nq, ctx - nq), pool=P, topk=K)
    c = G.build(wl, fp4_on_gpu=True)   # only the index side is checked here
    ly = c.layers_dev[0]
    keys = c.host_keys[(0, 0)].copy()
    if mode == "half":
        keys[::2] = 0
        ly.keys.data[:ctx].copy_(torch.from_numpy(keys))
    pool = torch.full((nq, P), -7, dtype=torch.int32, device=DEV)
    pcnt = torch.full((nq,), -7, dtype=torch.int32, device=DEV)
    sel = torch.full((nq, K), -7, dtype=torch.int32, device=DEV)
    scnt = torch.full((nq,), -7, dtype=torch.int32, device=DEV)
    B.check_status(B.csa2_index_full(ly.q, ly.w, ly.keys, c.pos_dev, c.max_ctx, seq_of_query=c.seq_dev,
                                     P=P, pool_idx=pool, pool_cnt=pcnt, K=K, sel_idx=sel, sel_cnt=scnt))
    po, pc, so, sc = _np(pool), _np(pcnt), _np(sel), _np(scnt)
    for i in (0, 1, 40, 78, 79):
        q, w = c.host_q[(0, i)]
        _, ref_pool, ref_sel = O.full_index(q, w, keys, int(c.query_pos[i]), P, K)
        assert pc[i] == len(ref_pool) and np.array_equal(po[i, :pc[i]], ref_pool), f"query {i} pool"
        assert (po[i, pc[i]:] == -1).all()
        assert sc[i] == len(ref_sel) and np.array_equal(so[i, :sc[i]], ref_sel), f"query {i} selection"
        assert (so[i, sc[i]:] == -1).all()


def test_topk_many_long_rows_with_positions():
    rng = np.random.default_rng(9)
    nq, n = 24, 70000
    s = rng.integers(0, 50, size=(nq, n)).astype(np.int32)
    pos = np.sort(rng.choice(10 ** 7, size=(nq, n), replace=True), axis=1).astype(np.int32)
    pos += np.arange(n, dtype=np.int32)[None]          # strictly ascending per row
    out = torch.empty((nq, 512), dtype=torch.int32, device=DEV)
    B.check_status(B.csa2_topk_pool(torch.from_numpy(s).to(DEV), 512, out,
                                    cand_pos=torch.from_numpy(pos).to(DEV)))
    o = _np(out)
    for i in range(nq):
        assert np.array_equal(o[i], O.top_k_positions(s[i], pos[i], 512)), f"row {i}"


@pytest.mark.parametrize("n", [1000, 16000, 40000])
def test_topk_all_equal_and_two_valued(n):
    for s in (np.zeros((1, n), np.int32), np.where(np.arange(n) % 3 == 0, 7, -7).astype(np.int32)[None]):
        k = 600
        out = torch.empty((1, k), dtype=torch.int32, device=DEV)
        B.check_status(B.csa2_topk_pool(torch.from_numpy(s).to(DEV), k, out))
        assert np.array_equal(_np(out)[0], O.top_k_positions(s[0], np.arange(n), k))


def test_topk_with_candidate_positions():
    rng = np.random.default_rng(5)
    for n in (9000, 30000):
        pos = np.sort(rng.choice(10 ** 6, size=n, replace=False)).astype(np.int32)
        s = rng.integers(0, 40, size=n).astype(np.int32)
        out = torch.empty((1, 512), dtype=torch.int32, device=DEV)
        B.check_status(B.csa2_topk_pool(torch.from_numpy(s[None]).to(DEV), 512, out,
                                        cand_pos=torch.from_numpy(pos[None]).to(DEV)))
        assert np.array_equal(_np(out)[0], O.top_k_positions(s, pos, 512))


def test_topk_rejects_unsorted_candidates():
    s = torch.zeros((1, 100), dtype=torch.int32, device=DEV)
    pos = torch.arange(100, dtype=torch.int32, device=DEV).flip(0)[None].contiguous()
    out = torch.empty((1, 10), dtype=torch.int32, device=DEV)
    st = B.csa2_topk_pool(s, 10, out, cand_pos=pos)
    assert int(st.item()) == 8


# ------------------------------------------------------------------ K3 reindex
@pytest.mark.parametrize("pool", [1024, 16384])
def test_reindex_matches_oracle(pool):
    wl = synth.scaled(synth.C1_SINGLE, seq_lens=(40000,), modes=(synth.FULL, synth.REINDEX), pool=pool)
    c = G.build(wl)
    full, re = c.layers_dev
    B.check_status(B.csa2_index_full(full.q, full.w, full.keys, c.pos_dev, c.max_ctx, P=pool,
                                     pool_idx=full.pool_idx, pool_cnt=full.pool_cnt))
    scores = torch.empty((1, pool), dtype=torch.int32, device=DEV)
    B.check_status(B.csa2_reindex(re.q, re.w, re.keys, full.pool_idx, full.pool_cnt, wl.topk, re.sel_idx,
                                  sel_cnt=re.sel_cnt, scores=scores))
    q0, w0 = c.host_q[(0, 0)]
    _, ref_pool, _ = O.full_index(q0, w0, c.host_keys[(0, 0)], 39999, pool, wl.topk)
    q1, w1 = c.host_q[(1, 0)]
    ref_s, ref_sel = O.reindex(q1, w1, c.host_keys[(1, 0)], ref_pool, wl.topk)
    assert np.array_equal(_np(full.pool_idx)[0], ref_pool)
    assert np.array_equal(_np(scores)[0], ref_s)
    assert np.array_equal(_np(re.sel_idx)[0], ref_sel) and int(_np(re.sel_cnt)[0]) == len(ref_sel)


def test_reindex_flat_scores():
    """All-zero reindex keys: every pool entry scores 0, so the top-K is the K
    lowest pool positions (ties go to the lower position) and the tie list is
    far longer than the ranked one: the radix select decides."""
    wl = synth.scaled(synth.C1_SINGLE, seq_lens=(40000,), modes=(synth.FULL, synth.REINDEX))
    c = G.build(wl)
    full, re = c.layers_dev
    re.keys.data.zero_()
    B.check_status(B.csa2_index_full(full.q, full.w, full.keys, c.pos_dev, c.max_ctx, P=wl.pool,
                                     pool_idx=full.pool_idx, pool_cnt=full.pool_cnt))
    B.check_status(B.csa2_reindex(re.q, re.w, re.keys, full.pool_idx, full.pool_cnt, wl.topk, re.sel_idx,
                                  sel_cnt=re.sel_cnt))
    q1, w1 = c.host_q[(1, 0)]
    pool = _np(full.pool_idx)[0]
    _, ref_sel = O.reindex(q1, w1, np.zeros_like(c.host_keys[(1, 0)]), pool, wl.topk)
    assert np.array_equal(ref_sel, pool[:wl.topk])
    assert np.array_equal(_np(re.sel_idx)[0], ref_sel) and int(_np(re.sel_cnt)[0]) == wl.topk


@pytest.mark.parametrize("flat", [False, True])
def test_reindex_batch_of_many_queries(flat):
    """Eight queries of a 16384-entry pool: more CTAs than fit on the device at
    once, so the last CTA of each pool to finish its scores selects alone.
    flat: all-zero reindex keys, every score ties, and the need-th tie key is
    found by the radix passes over the whole pool."""
    wl = synth.scaled(synth.C3_RAGGED, ragged=(8, 17000, 30000), modes=(synth.FULL, synth.REINDEX), page_rows=0)
    c = G.build(wl)
    full, re = c.layers_dev
    if flat:
        re.keys.data.zero_()
    B.check_status(B.csa2_index_full(full.q, full.w, full.keys, c.pos_dev, c.max_ctx, P=wl.pool,
                                     pool_idx=full.pool_idx, pool_cnt=full.pool_cnt, seq_of_query=c.seq_dev))
    B.check_status(B.csa2_reindex(re.q, re.w, re.keys, full.pool_idx, full.pool_cnt, wl.topk, re.sel_idx,
                                  sel_cnt=re.sel_cnt, seq_of_query=c.seq_dev))
    pools, sels = _np(full.pool_idx), _np(re.sel_idx)
    for i in range(len(c.query_pos)):
        s = int(c.seq_of_query[i])
        q0, w0 = c.host_q[(0, i)]
        _, ref_pool, _ = O.full_index(q0, w0, c.host_keys[(0, s)], int(c.query_pos[i]), wl.pool, wl.topk)
        q1, w1 = c.host_q[(1, i)]
        k1 = np.zeros_like(c.host_keys[(1, s)]) if flat else c.host_keys[(1, s)]
        _, ref_sel = O.reindex(q1, w1, k1, ref_pool, wl.topk)
        if flat:
            assert np.array_equal(ref_sel, ref_pool[:wl.topk])
        assert np.array_equal(pools[i, :len(ref_pool)], ref_pool)
        assert np.array_equal(sels[i, :len(ref_sel)], ref_sel)


def test_index_grouped_queries_of_several_sequences():
    """20 queries over three sequences (runs of 7, 1 and 12 queries): from 16
    queries on, consecutive queries of one sequence share key tiles in groups
    of at most four, so this has partial and single-query groups.  Every
    query's scores and its top-K of the whole prefix must equal the oracle's."""
    wl = synth.scaled(synth.C1_SINGLE, seq_lens=(9000, 5000, 12000), modes=(synth.FULL,))
    lens = wl.lengths()
    seq = np.array([0] * 7 + [1] + [2] * 12, dtype=np.int32)
    pos = np.concatenate([np.arange(8990, 8997), [4999], np.arange(11900, 12000, 9)[:12]]).astype(np.int32)
    keys_host = [synth.index_keys(wl, 0, s_) for s_ in range(len(lens))]
    kt, srows = G._place(keys_host, lens, None, 64, wl.idx_dim, np.int8, DEV)
    keys = B.Rows(kt, None, 64, srows)
    qs = [synth.index_query(wl, 0, i) for i in range(len(pos))]
    q = torch.from_numpy(np.stack([x[0] for x in qs])).to(DEV)
    w = torch.from_numpy(np.stack([x[1] for x in qs])).to(DEV)
    nq, K = len(pos), 300
    max_ctx = int(lens.max())
    scores = torch.full((nq, max_ctx), -7, dtype=torch.int32, device=DEV)
    sel = torch.empty((nq, K), dtype=torch.int32, device=DEV)
    cnt = torch.empty((nq,), dtype=torch.int32, device=DEV)
    B.check_status(B.csa2_index_full(q, w, keys, torch.from_numpy(pos).to(DEV), max_ctx,
                                     seq_of_query=torch.from_numpy(seq).to(DEV), scores=scores, K=K,
                                     sel_idx=sel, sel_cnt=cnt))
    sc, so, co = _np(scores), _np(sel), _np(cnt)
    for i in range(nq):
        ref = O.index_scores(qs[i][0], qs[i][1], keys_host[seq[i]][:pos[i] + 1])
        assert np.array_equal(sc[i, :pos[i] + 1], ref), f"query {i} scores"
        ref_sel = O.top_k_positions(ref, np.arange(pos[i] + 1), K)
        assert co[i] == len(ref_sel) and np.array_equal(so[i, :co[i]], ref_sel), f"query {i} selection"


# ------------------------------------------------------------------ A6 prefill chunk
def test_prefill_chunk_matches_oracle():
    """A causal prefill chunk (the C4 shape, reduced): 96 queries at positions
    8904..8999 of one 9000-row sequence.  Every query scores its own prefix,
    keeps its top-512 of the whole prefix (no pool) and attends to it plus the
    window.  Sampled queries are checked against the oracle one by one."""
    wl = synth.scaled(synth.C4_PREFILL, seq_lens=(9000,), prefill=(96, 8904))
    c = G.build(wl)
    ly = c.layers_dev[0]
    nq = len(c.query_pos)
    B.check_status(B.csa2_index_full(ly.q, ly.w, ly.keys, c.pos_dev, c.max_ctx, seq_of_query=c.seq_dev,
                                     K=wl.topk, sel_idx=ly.sel_idx, sel_cnt=ly.sel_cnt))
    B.check_status(B.csa2_sparse_attn_fp4(ly.q_attn, ly.codes, ly.scales, c.pos_dev, ly.sel_idx, ly.out,
                                          sel_cnt=ly.sel_cnt, seq_of_query=c.seq_dev, window=wl.window,
                                          lse=ly.lse))
    sels, cnts, outs = _np(ly.sel_idx), _np(ly.sel_cnt), _np(ly.out.float())
    keys = c.host_keys[(0, 0)]
    codes, scales = c.fp4_host[(0, 0)]
    for i in (0, 1, 17, 50, 94, 95):
        q, w = c.host_q[(0, i)]
        sel, S, o, _ = O.prefill_query(q, w, keys, c.host_qa[(0, i)], codes, scales, int(c.query_pos[i]),
                                       wl.topk, wl.window)
        assert cnts[i] == len(sel) and np.array_equal(sels[i, :cnts[i]], sel), f"query {i}"
        ok, err = G.tol_ok(outs[i], o)
        assert ok, f"query {i}: max abs err {err}"
    assert nq == 96


# ------------------------------------------------------------------ K4 attention
@pytest.mark.parametrize("wl", [synth.C0_TINY, synth.scaled(synth.C1_SINGLE, seq_lens=(3001,))],
                         ids=["hq8_d128", "hq64_d512"])
def test_sparse_attention_matches_oracle(wl):
    c = G.build(wl)
    ly = c.layers_dev[0]
    pos = int(c.query_pos[0])
    q, w = c.host_q[(0, 0)]
    _, _, sel = O.full_index(q, w, c.host_keys[(0, 0)], pos, wl.pool, wl.topk)
    sel_pad = np.full((1, wl.topk), -1, np.int32)
    sel_pad[0, :len(sel)] = sel
    sel_d = torch.from_numpy(sel_pad).to(DEV)
    cnt_d = torch.tensor([len(sel)], dtype=torch.int32, device=DEV)
    B.check_status(B.csa2_sparse_attn_fp4(ly.q_attn, ly.codes, ly.scales, c.pos_dev, sel_d, ly.out,
                                          sel_cnt=cnt_d, window=wl.window, lse=ly.lse))
    S = O.attention_set(sel, pos, wl.window)
    codes, scales = c.fp4_host[(0, 0)]
    ref, ref_lse = O.sparse_attention(c.host_qa[(0, 0)], O.fp4_dequant(codes[S], scales[S], wl.attn_dim))
    ok, err = G.tol_ok(_np(ly.out.float())[0], ref)
    assert ok, f"max abs err {err}"
    assert np.allclose(_np(ly.lse)[0], ref_lse, atol=1e-3, rtol=1e-4)


def test_sparse_attention_window_only_and_overlap():
    wl = synth.scaled(synth.C0_TINY, seq_lens=(700,))
    c = G.build(wl)
    ly = c.layers_dev[0]
    codes, scales = c.fp4_host[(0, 0)]
    cases = [np.zeros(0, np.int64), np.arange(636, 700), np.array([0, 5, 580, 650, 699])]
    for sel in cases:
        sel_pad = np.full((1, wl.topk), -1, np.int32)
        sel_pad[0, :len(sel)] = sel
        B.check_status(B.csa2_sparse_attn_fp4(ly.q_attn, ly.codes, ly.scales, c.pos_dev,
                                              torch.from_numpy(sel_pad).to(DEV), ly.out,
                                              sel_cnt=torch.tensor([len(sel)], dtype=torch.int32, device=DEV),
                                              window=wl.window))
        S = O.attention_set(sel, 699, wl.window)
        ref, _ = O.sparse_attention(c.host_qa[(0, 0)], O.fp4_dequant(codes[S], scales[S], wl.attn_dim))
        ok, err = G.tol_ok(_np(ly.out.float())[0], ref)
        assert ok, f"max abs err {err}"


# ------------------------------------------------------------------ the whole plan
def _check_plan(c, n_check=None, need_rows_from_oracle=False):
    wl = c.wl
    plan = B.csa2_layer_plan(list(wl.modes), c.layers_dev, query_pos=c.pos_dev, seq_of_query=c.seq_dev,
                             max_ctx=c.max_ctx, P=wl.pool, K=wl.topk, window=wl.window)
    B.check_status(plan.status)
    nq = len(c.query_pos)
    worst = 0.0
    for i in range(nq if n_check is None else n_check):
        pos = int(c.query_pos[i])
        res = O.decode_layer_plan(wl.modes, G.oracle_layers(c, i), pos, wl.pool, wl.topk, wl.window)
        for l, (r, ly) in enumerate(zip(res, c.layers_dev)):
            if r.pool_idx is not None:
                n = int(_np(ly.pool_cnt)[i])
                assert n == len(r.pool_idx) and np.array_equal(_np(ly.pool_idx)[i, :n], r.pool_idx)
            n = int(_np(ly.sel_cnt)[i])
            assert n == len(r.sel_idx) and np.array_equal(_np(ly.sel_idx)[i, :n], r.sel_idx), f"layer {l}"
            ok, err = G.tol_ok(_np(ly.out[i].float()), r.out)
            worst = max(worst, err)
            assert ok, f"query {i} layer {l}: max abs err {err}"
    return worst


def test_plan_8_layers_reduced_context():
    wl = synth.scaled(synth.C2_1M_PLAN, seq_lens=(50003,))
    c = G.build(wl)
    _check_plan(c)


def test_plan_paged_ragged_batch():
    wl = synth.scaled(synth.C3_RAGGED, ragged=(4, 2000, 30000), modes=(synth.FULL, synth.REUSE, synth.REINDEX))
    c = G.build(wl)
    _check_plan(c)


def test_plan_verify_block_of_five_queries():
    """A speculative-verify block: 5 queries of one sequence at consecutive
    positions, each with its own full / reindex / reuse step, through one
    plan call."""
    wl = synth.scaled(synth.C1_SINGLE, seq_lens=(30000,), prefill=(5, 29995),
                      modes=(synth.FULL, synth.REINDEX, synth.REUSE))
    c = G.build(wl)
    assert len(c.query_pos) == 5 and (c.seq_of_query == 0).all()
    _check_plan(c)


@pytest.mark.parametrize("case", ["two_reindex_small_heads", "flat_reindex", "paged_one_sequence"])
def test_plan_one_query_reindex_layers(case):
    """One query with more candidates than one select CTA holds (the
    co-resident select) and one or two reindex layers on its pool (the fused
    reindex launch).  Small heads (4 x d64: 16-column MMA, 64-byte rows) with
    two reindex layers; all-zero reindex keys, where every pool entry ties and
    the radix passes decide; 64-row pages."""
    if case == "two_reindex_small_heads":
        wl = synth.scaled(synth.C0_TINY, seq_lens=(40000,), pool=2000, topk=64,
                          modes=(synth.FULL, synth.REINDEX, synth.REINDEX, synth.REUSE))
    elif case == "flat_reindex":
        wl = synth.scaled(synth.C1_SINGLE, seq_lens=(40000,), modes=(synth.FULL, synth.REINDEX, synth.REUSE))
    else:
        wl = synth.scaled(synth.C3_RAGGED, ragged=(1, 40000, 40000), modes=(synth.FULL, synth.REINDEX))
    c = G.build(wl)
    assert len(c.query_pos) == 1 and c.max_ctx > 16384
    if case == "flat_reindex":
        c.layers_dev[1].keys.data.zero_()
        c.host_keys[(1, 0)][:] = 0
    _check_plan(c)


def test_plan_tiny_config():
    c = G.build(synth.C0_TINY)
    _check_plan(c)


def test_plan_repeat_is_deterministic():
    wl = synth.scaled(synth.C2_1M_PLAN, seq_lens=(30000,), modes=(synth.FULL, synth.REINDEX, synth.REUSE))
    c = G.build(wl)
    plan = B.csa2_layer_plan(list(wl.modes), c.layers_dev, query_pos=c.pos_dev, max_ctx=c.max_ctx,
                             P=wl.pool, K=wl.topk, window=wl.window)
    first = [ly.out.clone() for ly in c.layers_dev]
    for _ in range(3):
        plan.run()
    torch.cuda.synchronize()
    for a, ly in zip(first, c.layers_dev):
        assert torch.equal(a, ly.out)


def test_sparse_attention_long_selection():
    # K = 2000 > the 1024 selection entries a CTA keeps in shared memory,
    # and more than 24 chunks of 64 rows for the combine.
    wl = synth.scaled(synth.C0_TINY, seq_lens=(6000,), topk=2000, pool=3000)
    c = G.build(wl)
    ly = c.layers_dev[0]
    pos = int(c.query_pos[0])
    q, w = c.host_q[(0, 0)]
    _, _, sel = O.full_index(q, w, c.host_keys[(0, 0)], pos, wl.pool, wl.topk)
    sel_d = torch.from_numpy(sel.astype(np.int32)[None]).to(DEV)
    B.check_status(B.csa2_sparse_attn_fp4(ly.q_attn, ly.codes, ly.scales, c.pos_dev, sel_d, ly.out,
                                          sel_cnt=torch.tensor([len(sel)], dtype=torch.int32, device=DEV),
                                          window=wl.window))
    S = O.attention_set(sel, pos, wl.window)
    codes, scales = c.fp4_host[(0, 0)]
    ref, _ = O.sparse_attention(c.host_qa[(0, 0)], O.fp4_dequant(codes[S], scales[S], wl.attn_dim))
    ok, err = G.tol_ok(_np(ly.out.float())[0], ref)
    assert ok, f"max abs err {err}"


# ------------------------------------------------------------------ one query: pool and selection fused
# into the index launch.  Random scores leave a few ties at the threshold
# (gathered and ranked); zero keys make every score 0 (the ties of one CTA
# overflow its slot and the grid's radix select decides); half-zero keys with
# a pool larger than the positive rows split a long tie list of zeros.
@pytest.mark.parametrize("ctx,mode,P,K", [(40000, "random", 16384, 512), (40000, "zero", 16384, 512),
                                          (40000, "half", 30000, 512), (4096, "zero", 1024, 64),
                                          (300000, "random", 16384, 512)])
def test_index_full_one_query_ties(ctx, mode, P, K):
    wl = synth.scaled(synth.C1_SINGLE, seq_lens=(ctx,), pool=P, topk=K)
    c = G.build(wl, fp4_on_gpu=True)   # only the index side is checked here
    ly = c.layers_dev[0]
    keys = c.host_keys[(0, 0)].copy()
    if mode == "zero":
        keys[:] = 0
    elif mode == "half":
        keys[::2] = 0
    ly.keys.data[:ctx].copy_(torch.from_numpy(keys))
    pool = torch.full((1, P), -7, dtype=torch.int32, device=DEV)
    pcnt = torch.full((1,), -7, dtype=torch.int32, device=DEV)
    sel = torch.full((1, K), -7, dtype=torch.int32, device=DEV)
    scnt = torch.full((1,), -7, dtype=torch.int32, device=DEV)
    B.check_status(B.csa2_index_full(ly.q, ly.w, ly.keys, c.pos_dev, c.max_ctx, P=P, pool_idx=pool,
                                     pool_cnt=pcnt, K=K, sel_idx=sel, sel_cnt=scnt))
    q, w = c.host_q[(0, 0)]
    _, ref_pool, ref_sel = O.full_index(q, w, keys, int(c.query_pos[0]), P, K)
    n = int(_np(pcnt)[0])
    assert n == len(ref_pool) and np.array_equal(_np(pool)[0, :n], ref_pool)
    assert (_np(pool)[0, n:] == -1).all()
    m = int(_np(scnt)[0])
    assert m == len(ref_sel) and np.array_equal(_np(sel)[0, :m], ref_sel)
    if mode == "zero":
        assert np.array_equal(ref_pool, np.arange(min(P, ctx)))   # equal scores: the lowest positions
