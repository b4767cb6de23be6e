"""Pins for the CPU oracle: each check compares it with something other
than itself.  The sources are golden tables from public format specifications,
library routines, closed forms, invariants, and a separate brute-force
implementation.  No GPU is needed."""
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from tests import bruteforce as BF

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ------------------------------------------------------------------ index scores
@pytest.mark.parametrize("seed", range(6))
def test_scores_match_bruteforce_loops(seed):
    rng = np.random.default_rng(seed)
    H, D, n = rng.integers(1, 4), rng.integers(1, 9), rng.integers(1, 40)
    q = rng.integers(-128, 128, size=(H, D)).astype(np.int8)
    w = rng.integers(-128, 128, size=H).astype(np.int8)
    keys = rng.integers(-128, 128, size=(n, D)).astype(np.int8)
    got = O.index_scores(q, w, keys)
    want = [BF.score(q.tolist(), w.tolist(), keys[s].tolist()) for s in range(n)]
    assert got.tolist() == want


def test_scores_closed_form_one_hot():
    # q_h = c_h * e_{j_h}: head h sees only column j_h, so
    # score[s] = sum_h w_h * max(0, c_h * keys[s][j_h]).
    D = 8
    c = np.array([3, -2, 5], dtype=np.int64)
    j = np.array([1, 1, 6])
    w = np.array([2, 7, 1], dtype=np.int8)
    q = np.zeros((3, D), dtype=np.int8)
    q[np.arange(3), j] = c
    keys = np.arange(-40, 40, dtype=np.int64).reshape(10, D).astype(np.int8)
    got = O.index_scores(q, w, keys)
    k = keys.astype(np.int64)
    want = 2 * np.maximum(0, 3 * k[:, 1]) + 7 * np.maximum(0, -2 * k[:, 1]) + np.maximum(0, 5 * k[:, 6])
    assert np.array_equal(got, want)


def test_scores_relu_identity():
    # relu(x) - relu(-x) = x, so s(q) - s(-q) = keys . (sum_h w_h q_h).
    rng = np.random.default_rng(11)
    q = rng.integers(-127, 128, size=(16, 32)).astype(np.int8)
    w = rng.integers(-20, 21, size=16).astype(np.int8)
    keys = rng.integers(-128, 128, size=(300, 32)).astype(np.int8)
    lhs = O.index_scores(q, w, keys) - O.index_scores(-q, w, keys)
    comb = (w.astype(np.int64)[:, None] * q.astype(np.int64)).sum(0)
    rhs = np.array([int(sum(int(a) * int(b) for a, b in zip(row, comb))) for row in keys])
    assert np.array_equal(lhs, rhs)


def test_scores_weight_linearity():
    rng = np.random.default_rng(12)
    q = rng.integers(-16, 17, size=(8, 16)).astype(np.int8)
    w1 = rng.integers(-8, 9, size=8).astype(np.int8)
    w2 = rng.integers(-8, 9, size=8).astype(np.int8)
    keys = rng.integers(-16, 17, size=(100, 16)).astype(np.int8)
    s1, s2 = O.index_scores(q, w1, keys), O.index_scores(q, w2, keys)
    assert np.array_equal(O.index_scores(q, (w1 + w2).astype(np.int8), keys), s1 + s2)
    assert np.array_equal(O.index_scores(q, (2 * w1).astype(np.int8), keys), 2 * s1)


def test_score_bound_is_tight():
    H, D = 4, 16
    q = -np.ones((H, D), dtype=np.int8) * 3
    w = np.full(H, 5, dtype=np.int8)
    keys = np.full((1, D), -128, dtype=np.int8)
    assert O.index_scores(q, w, keys)[0] == O.score_bound(q, w) == 128 * 4 * 5 * 3 * 16
    rng = np.random.default_rng(1)
    q = rng.integers(-128, 128, size=(H, D)).astype(np.int8)
    w = rng.integers(-128, 128, size=H).astype(np.int8)
    keys = rng.integers(-128, 128, size=(500, D)).astype(np.int8)
    assert np.abs(O.index_scores(q, w, keys)).max() <= O.score_bound(q, w)


# ------------------------------------------------------------------ exact top-k
@pytest.mark.parametrize("seed", range(8))
def test_topk_matches_repeated_max(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(0, 60))
    positions = np.sort(rng.choice(1000, size=n, replace=False))
    scores = rng.integers(-3, 4, size=n)            # many ties
    for k in (0, 1, 5, n, n + 3):
        got = O.top_k_positions(scores, positions, k)
        want = BF.select(dict(zip(positions.tolist(), scores.tolist())), k)
        assert got.tolist() == want


def test_topk_adversarial():
    pos = np.arange(50)
    assert O.top_k_positions(np.zeros(50), pos, 7).tolist() == list(range(7))
    two = np.where(pos % 2 == 0, 5, 9)
    assert O.top_k_positions(two, pos, 30).tolist() == sorted(list(range(1, 50, 2)) + list(range(0, 10, 2)))
    assert O.top_k_positions(pos, pos, 50).tolist() == list(range(50))
    assert O.top_k_positions(pos, pos, 80).tolist() == list(range(50))
    assert O.top_k_positions(np.zeros(0), np.zeros(0), 4).tolist() == []
    assert O.top_k_positions(-pos, pos, 3).tolist() == [0, 1, 2]


def test_topk_nested():
    rng = np.random.default_rng(3)
    s = rng.integers(0, 40, size=5000)
    pos = np.arange(5000)
    pool = O.top_k_positions(s, pos, 700)
    assert np.array_equal(O.top_k_positions(s[pool], pool, 64), O.top_k_positions(s, pos, 64))


# ------------------------------------------------------------------ FP4 format
def test_e2m1_matches_ocp_table():
    table = _golden("e2m1_ocp_mx.txt")
    codes = np.array([int(c) for c, _ in table])
    want = np.array([float(v) for _, v in table])
    got = O.e2m1_decode(codes)
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.signbit(want))


def test_e2m1_all_codes_match_ml_dtypes():
    """A second, independent decoder of OCP E2M1: ml_dtypes.float4_e2m1fn
    (one code per byte, in the low nibble)."""
    ml = pytest.importorskip("ml_dtypes")
    want = np.arange(16, dtype=np.uint8).view(ml.float4_e2m1fn).astype(np.float64)
    got = O.e2m1_decode(np.arange(16))
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.signbit(want))


def test_e2m1_rounding_matches_ml_dtypes_in_range():
    """Inside the E2M1 range the quantiser's code choice is round to nearest,
    ties to even: on a grid that holds every representable value, every
    midpoint between neighbours and points just beside them, the magnitude
    it stores equals ml_dtypes' float -> float4_e2m1fn conversion (scale 1)."""
    ml = pytest.importorskip("ml_dtypes")
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    mids = (mags[:-1] + mags[1:]) / 2
    pts = np.unique(np.concatenate([mags, mids, mids - 1e-6, mids + 1e-6, np.linspace(0, 6, 241)]))
    x = np.concatenate([pts, -pts])
    # one block per value: the block maximum 6 fixes the scale at exactly 1.0 (E4M3 0x38)
    blocks = np.zeros((len(x), 32))
    blocks[:, 0] = x
    blocks[:, 1] = 6.0
    codes, scales = O.fp4_quantize(blocks)
    assert (scales == 0x38).all()
    got = O.e2m1_decode(codes[:, 0] & 0xF)
    want = x.astype(np.float32).astype(ml.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(np.abs(got), np.abs(want))
    nz = want != 0
    assert np.array_equal(np.sign(got[nz]), np.sign(want[nz]))


def test_e4m3_all_bytes_match_torch():
    b = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    want = b.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_decode(np.arange(256))
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])


def test_e4m3_matches_ofp8_named_values():
    for hexb, val, _ in _golden("e4m3_ofp8.txt"):
        got = O.e4m3_decode(int(hexb, 16))
        if val == "nan":
            assert np.isnan(got)
        else:
            assert got == float(val) and np.signbit(got) == np.signbit(float(val))


def test_e4m3_encode_round_trip_and_ties():
    codes = np.arange(0x7F)
    vals = O.e4m3_decode(codes)
    assert np.array_equal(O.e4m3_encode_rne(vals), codes)
    mids = (vals[:-1] + vals[1:]) / 2                  # exact midpoints
    got = O.e4m3_encode_rne(mids)
    want = np.where(codes[:-1] % 2 == 0, codes[:-1], codes[1:])
    assert np.array_equal(got, want)
    assert O.e4m3_encode_rne(np.array([448.0, 460.0, 1e9]))[0] == 0x7E
    assert np.all(O.e4m3_encode_rne(np.array([460.0, 1e9])) == 0x7E)
    assert O.e4m3_encode_rne(np.array([2.0 ** -10]))[0] == 0      # tie with 0 -> even (0)


def _bf_quant_block(x):
    """Brute force: scale byte minimises |amax/6 - v| over all scale bytes
    (ties to the even byte).  Each code minimises |x/scale - e2m1(code)|
    (ties to the even magnitude index; zero magnitude is +0)."""
    amax = max(abs(v) for v in x)
    target = amax / 6.0
    best = None
    for b in range(0x7F):
        d = abs(target - BF.e4m3(b))
        if best is None or d < best[0] or (d == best[0] and b % 2 == 0):
            best = (d, b)
    sb = best[1] if target < 448 else 0x7E
    s = BF.e4m3(sb)
    codes = []
    for v in x:
        if s == 0:
            codes.append(0)
            continue
        r = abs(v) / s
        bm = None
        for m in range(8):
            d = abs(r - BF.E2M1[m])
            if bm is None or d < bm[0] or (d == bm[0] and m % 2 == 0):
                bm = (d, m)
        m = bm[1] if r < 6 else 7
        codes.append(m | (8 if (v < 0 and m > 0) else 0))
    return sb, codes


@pytest.mark.parametrize("seed", range(4))
def test_fp4_quantize_matches_exhaustive_search(seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((6, 64)).astype(np.float32)
    x[0, :32] *= 8.0
    x[1, :32] = 0.0                     # zero block
    x[2, :32] *= 1e-4                   # scale underflows toward 0
    x[3, :32] *= 3000.0                 # scale saturates
    x[4, 5] = 0.0
    codes, scales = O.fp4_quantize(x)
    for r in range(x.shape[0]):
        for blk in range(2):
            sb, cs = _bf_quant_block(x[r, blk * 32:(blk + 1) * 32].astype(np.float64).tolist())
            assert scales[r, blk] == sb
            for j, c in enumerate(cs):
                e = blk * 32 + j
                nib = (codes[r, e // 2] >> (4 * (e % 2))) & 0xF
                assert nib == c, (r, e)


def test_fp4_round_trip_on_representable_rows():
    rng = np.random.default_rng(5)
    n, D = 40, 128
    sb = rng.integers(0x08, 0x77, size=(n, D // 32)).astype(np.uint8)  # normal scales, 6*s < 448
    codes = rng.integers(0, 256, size=(n, D // 2)).astype(np.uint8)
    codes[:, ::16] = 0x77                # one +6 per block pins amax/6 to the scale
    codes[codes & 0x0F == 0x08] &= 0xF0  # no -0 in the low nibble
    codes[(codes >> 4) == 0x8] &= 0x0F   # no -0 in the high nibble
    x = O.fp4_dequant(codes, sb, D)
    c2, s2 = O.fp4_quantize(x)
    assert np.array_equal(s2, sb) and np.array_equal(c2, codes)


def test_fp4_dequant_nibble_order():
    codes = np.zeros((1, 16), dtype=np.uint8)
    codes[0, 0] = 0x72                   # element 0 -> code 2 (1.0), element 1 -> code 7 (6.0)
    codes[0, 1] = 0x0B                   # element 2 -> code 11 (-1.5), element 3 -> 0
    scales = np.array([[0x40]], dtype=np.uint8)   # 2.0
    v = O.fp4_dequant(codes, scales, 32)[0]
    assert v[:4].tolist() == [2.0, 12.0, -3.0, 0.0]
    assert np.all(v[4:] == 0)


# ------------------------------------------------------------------ attention
@pytest.mark.parametrize("seed", range(3))
def test_attention_matches_torch_sdpa(seed):
    rng = np.random.default_rng(seed)
    Hq, D, m = 8, 64, 37
    q = rng.standard_normal((Hq, D))
    kv = rng.standard_normal((m, D)) * 2
    scale = 1 / math.sqrt(D)
    o, lse = O.sparse_attention(q, kv)
    tq = torch.from_numpy(q)[None, :, None, :]                  # B, H, L=1, D
    tk = torch.from_numpy(kv)[None, None].expand(1, Hq, m, D)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tk, scale=scale)[0, :, 0].numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-12)
    ref_lse = torch.logsumexp(torch.from_numpy(scale * q @ kv.T), dim=1).numpy()
    assert np.allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_attention_closed_forms():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((4, 16))
    row = rng.standard_normal(16)
    o, lse = O.sparse_attention(q, row[None])
    assert np.allclose(o, np.broadcast_to(row, (4, 16)), atol=1e-15)
    assert np.allclose(lse, (q @ row) / 4.0)
    o, _ = O.sparse_attention(q, np.stack([row] * 9))
    assert np.allclose(o, np.broadcast_to(row, (4, 16)), atol=1e-14)
    a, b = rng.standard_normal(16), rng.standard_normal(16)
    o, _ = O.sparse_attention(q, np.stack([a, b]), softmax_scale=0.5)
    pa = 1 / (1 + np.exp(0.5 * (q @ b - q @ a)))
    assert np.allclose(o, pa[:, None] * a + (1 - pa)[:, None] * b, atol=1e-14)


def test_attention_permutation_invariant():
    rng = np.random.default_rng(2)
    q, kv = rng.standard_normal((8, 32)), rng.standard_normal((50, 32))
    perm = rng.permutation(50)
    o1, l1 = O.sparse_attention(q, kv)
    o2, l2 = O.sparse_attention(q, kv[perm])
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(l1, l2, atol=1e-12)


def test_attention_set_window_and_dedup():
    assert O.attention_set(np.array([0, 3]), 5, 128).tolist() == [0, 1, 2, 3, 4, 5]
    assert O.attention_set(np.array([1, 500, 900]), 1000, 4).tolist() == [1, 500, 900, 997, 998, 999, 1000]
    assert O.attention_set(np.array([998]), 1000, 4).tolist() == [997, 998, 999, 1000]
    assert O.attention_set(np.zeros(0, np.int64), 0, 128).tolist() == [0]


# ------------------------------------------------------------------ whole pipeline
def _tiny_layers(rng, n_layers, ctx, H, Di, Hq, D):
    layers = []
    for _ in range(n_layers):
        x = rng.standard_normal((ctx, D)) * np.where(rng.random((ctx, D)) < 0.05, 8, 1)
        codes, scales = O.fp4_quantize(x)
        layers.append(dict(
            q=rng.integers(-8, 9, size=(H, Di)).astype(np.int8),
            w=rng.integers(1, 5, size=H).astype(np.int8),
            keys=rng.integers(-8, 9, size=(ctx, Di)).astype(np.int8),
            q_attn=rng.standard_normal((Hq, D)), codes=codes, scales=scales))
    return layers


@pytest.mark.parametrize("seed", range(4))
def test_plan_matches_bruteforce(seed):
    rng = np.random.default_rng(100 + seed)
    ctx = int(rng.integers(1, 64))
    modes = [0, 1, 2, 1, 2]
    layers = _tiny_layers(rng, len(modes), ctx, H=3, Di=4, Hq=2, D=64)
    pos, pool, topk, window = ctx - 1, 12, 5, 6
    got = O.decode_layer_plan(modes, layers, pos, pool, topk, window)
    bl = [dict(L, codes=L["codes"].tolist(), scales=L["scales"].tolist(),
               q_attn=L["q_attn"].tolist(), keys=L["keys"].tolist()) for L in layers]
    want = BF.decode_step(modes, bl, pos, pool, topk, window)
    for g, (sel, S, out) in zip(got, want):
        assert g.sel_idx.tolist() == sel
        assert g.attn_set.tolist() == S
        assert np.allclose(g.out, np.array(out), rtol=1e-12, atol=1e-12)


def test_reuse_layers_share_selection():
    rng = np.random.default_rng(7)
    modes = [0, 2, 1, 2, 2]
    layers = _tiny_layers(rng, len(modes), 300, H=4, Di=16, Hq=2, D=32)
    r = O.decode_layer_plan(modes, layers, 299, 64, 16, 8)
    assert r[1].sel_idx is r[0].sel_idx
    assert r[3].sel_idx is r[2].sel_idx and r[4].sel_idx is r[2].sel_idx
    assert set(r[2].sel_idx.tolist()) <= set(r[0].pool_idx.tolist())


def test_full_selection_is_global_topk():
    rng = np.random.default_rng(8)
    L = _tiny_layers(rng, 1, 2000, H=4, Di=16, Hq=2, D=32)[0]
    s, pool, sel = O.full_index(L["q"], L["w"], L["keys"], 1999, 256, 32)
    assert np.array_equal(sel, O.top_k_positions(s, np.arange(2000), 32))
    assert len(pool) == 256 and np.all(np.diff(pool) > 0)


def test_prefill_query_equals_single_full_layer_decode():
    rng = np.random.default_rng(9)
    L = _tiny_layers(rng, 1, 500, H=4, Di=16, Hq=2, D=32)[0]
    for pos in (0, 77, 499):
        sel, S, o, lse = O.prefill_query(L["q"], L["w"], L["keys"], L["q_attn"], L["codes"],
                                         L["scales"], pos, 24, 10)
        r = O.decode_layer_plan([0], [L], pos, pos + 1, 24, 10)[0]
        assert np.array_equal(sel, r.sel_idx) and np.array_equal(S, r.attn_set)
        assert np.array_equal(o, r.out)


# ------------------------------------------------------------------ the layer's local window cache
def test_local_window_single_row_is_the_output():
    rng = np.random.default_rng(11)
    D, R = 32, 128
    ring = rng.standard_normal((R, D))
    codes = np.zeros((4, D // 2), np.uint8)
    scales = np.zeros((4, D // 32), np.uint8)
    S = O.attention_set(np.zeros(0, np.int64), 0, 128)          # pos 0: the window is position 0 alone
    rows = O.kv_rows_local_window(S, 0, 128, codes, scales, D, ring)
    assert np.array_equal(rows, ring[:1])
    o, _ = O.sparse_attention(rng.standard_normal((3, D)), rows)
    assert np.allclose(o, np.broadcast_to(ring[0], (3, D)), atol=1e-15)


def test_local_window_uniform_softmax_closed_form():
    # FP4 rows of exactly 1.0 (code 2 = 1.0 in both nibbles, E4M3 0x38 = 1.0);
    # ring slot k holds the constant k + 1; q = 0 makes the softmax uniform,
    # so the output is the plain mean of the rows of S.
    D, R, window, pos = 64, 8, 5, 20
    codes = np.full((pos + 1, D // 2), 0x22, np.uint8)
    scales = np.full((pos + 1, D // 32), 0x38, np.uint8)
    ring = np.repeat(np.arange(1, R + 1, dtype=np.float64)[:, None], D, axis=1)
    sel = np.array([2, 7, 17])                                   # 17 lies in the window 16..20
    S = O.attention_set(sel, pos, window)
    assert S.tolist() == [2, 7, 16, 17, 18, 19, 20]
    rows = O.kv_rows_local_window(S, pos, window, codes, scales, D, ring)
    want = (1.0 + 1.0 + sum((p % R) + 1 for p in range(16, 21))) / 7
    o, _ = O.sparse_attention(np.zeros((2, D)), rows)
    assert np.allclose(o, want, atol=1e-14)
    assert rows[0].tolist() == [1.0] * D and rows[-1].tolist() == [float(20 % R + 1)] * D


def test_local_window_holding_the_fp4_rows_changes_nothing():
    rng = np.random.default_rng(12)
    modes = [0, 1, 2]
    ctx, window, R = 200, 16, 24
    layers = _tiny_layers(rng, len(modes), ctx, H=3, Di=8, Hq=2, D=64)
    pos = ctx - 1
    plain = O.decode_layer_plan(modes, layers, pos, 40, 8, window)
    for L in layers:
        ring = np.zeros((R, 64))
        for p in range(ctx - R, ctx):
            ring[p % R] = O.fp4_dequant(L["codes"][p:p + 1], L["scales"][p:p + 1], 64)[0]
        L["local_ring"] = ring
    local = O.decode_layer_plan(modes, layers, pos, 40, 8, window)
    for a, b in zip(plain, local):
        assert np.array_equal(a.attn_set, b.attn_set)
        assert np.array_equal(a.out, b.out) and np.array_equal(a.lse, b.lse)


@pytest.mark.parametrize("seed", range(3))
def test_plan_with_local_rings_matches_bruteforce(seed):
    rng = np.random.default_rng(200 + seed)
    ctx = int(rng.integers(1, 64))
    modes = [0, 2, 1, 2]
    window, R = 6, 9
    layers = _tiny_layers(rng, len(modes), ctx, H=3, Di=4, Hq=2, D=64)
    for i in (0, 2, 3):                                          # layer 1 keeps reading the FP4 cache
        layers[i]["local_ring"] = rng.standard_normal((R, 64))
    pos, pool, topk = ctx - 1, 12, 5
    got = O.decode_layer_plan(modes, layers, pos, pool, topk, window)
    bl = [dict(L, codes=L["codes"].tolist(), scales=L["scales"].tolist(), q_attn=L["q_attn"].tolist(),
               keys=L["keys"].tolist(),
               local_ring=None if L.get("local_ring") is None else L["local_ring"].tolist()) for L in layers]
    want = BF.decode_step(modes, bl, pos, pool, topk, window)
    for g, (sel, S, out) in zip(got, want):
        assert g.sel_idx.tolist() == sel and g.attn_set.tolist() == S
        assert np.allclose(g.out, np.array(out), rtol=1e-12, atol=1e-12)


def test_local_window_needs_a_ring_as_long_as_the_window():
    with pytest.raises(ValueError):
        O.kv_rows_local_window(np.array([5]), 5, 8, np.zeros((6, 16), np.uint8), np.zeros((6, 1), np.uint8), 32,
                               np.zeros((7, 32)))


def test_plan_rejects_bad_first_mode():
    with pytest.raises(ValueError):
        O.decode_layer_plan([1, 0], [{}, {}], 0, 4, 2, 2)


# ------------------------------------------------------------------ combine of partial attention
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_attention_combine_equals_attention_over_the_union(seed):
    """Softmax attention over a set of rows equals the combine of attention
    over any partition of it (one part left empty): the identity the
    context-sharded decode rests on, checked in fp64."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((8, 64))
    kv = rng.standard_normal((300, 64)) * 2.0
    parts = rng.integers(0, 3, size=300)          # part 3 stays empty
    outs, lses = [], []
    for r in range(4):
        rows = kv[parts == r]
        if len(rows):
            o, l = O.sparse_attention(q, rows)
        else:
            o, l = np.full((8, 64), np.nan), np.full(8, -np.inf)
        outs.append(o)
        lses.append(l)
    got_o, got_l = O.attention_combine(outs, lses)
    want_o, want_l = O.sparse_attention(q, kv)
    assert np.allclose(got_o, want_o, rtol=1e-12, atol=1e-12)
    assert np.allclose(got_l, want_l, rtol=1e-12, atol=1e-12)


def test_attention_combine_single_part_and_all_empty():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((4, 32))
    kv = rng.standard_normal((50, 32))
    o, l = O.sparse_attention(q, kv)
    got_o, got_l = O.attention_combine([o], [l])
    assert np.array_equal(got_o, o) and np.allclose(got_l, l, rtol=0, atol=1e-15)
    e_o, e_l = O.attention_combine([np.ones((4, 32)), np.ones((4, 32))], [np.full(4, -np.inf)] * 2)
    assert (e_o == 0).all() and np.isneginf(e_l).all()
