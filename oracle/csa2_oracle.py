"""CSA2 hierarchical sparse-attention decode: the CPU oracle.

TEST INFRASTRUCTURE.  This is the plain, slow, obviously correct statement
of what the CUDA library computes.  Only the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it.  The product path never
does, and it shares no code, table or constant with the CUDA sources.

Integer steps (index scores, selections) are computed in int64 and are exact.
Attention is computed in float64.  Library primitives (a matrix product, a
stable sort) serve as single steps.  Nothing is blocked, fused or reordered
beyond the definitions below.

Sources (web pages on DeepSeek V4.1-Flash; cited by title and section):
  [AD] "DeepSeek V4.1-Flash: 552B runs like 16B" (the-agent-daily.org deep
       dive), sections "Act 2: CSA2 & Hierarchical Sparse Indexing" and
       "Act 3: FP4 KV & SWA Bounded Replay".
  [AS] "DeepSeek V4.1 Flash: the most insane optimization so far"
       (artofsm.art digest), third paragraph (full / reindex / reuse modes).
  [YS] "How DeepSeek V4.1 Flash Actually Works: A Deep Dive"
       (youtubesummary.com), section "The three KV-cache optimizations",
       item 2 "Compress Sparse Attention / CA2" and item 3 (deployment-time
       cache management: the per-layer local cache of the latest tokens).
  [DA] "DeepSeek Has Done It Again..." (youtubesummary.com), section
       "Architecture and inference efficiency", bullet "Sparse attention for
       long context".
  [ST] "Deepseek just did the impossible" (summarytube.com), section "Memory
       and Compute Optimization".

The pages give no formulas, number formats beyond "FP4", or head sizes.  The
library fixes: an int8 indexer whose integer head weights make scores exact
integers; FP4 E2M1 values in 32-element blocks with one FP8 E4M3 scale each
(both as the OCP MX / OFP8 specifications define them); bf16 queries and
outputs.  Each reading of the pages is marked READING below.

Pin status (what checks each function against something other than itself;
see tests/test_oracle_pins.py):
  index_scores        pinned: brute-force loops, closed forms, the identity
                      s(q) - s(-q) = keys . (sum_h w_h q_h).  The formula
                      itself is READING 1 (parity unpinned by the pages).
  top_k_positions     pinned: repeated-maximum extraction, adversarial ties.
  e2m1_decode         pinned: OCP MX E2M1 table (tests/golden) and
                      ml_dtypes' float4_e2m1fn decoder on all 16 codes.
  e4m3_decode         pinned: torch.float8_e4m3fn on all 256 bytes, OFP8 table.
  fp4_quantize        pinned: exhaustive nearest-code search, round trips,
                      ml_dtypes' float -> float4_e2m1fn rounding inside the range.
  sparse_attention    pinned: torch scaled_dot_product_attention (fp64) when
                      the set is the whole context; closed forms.
  full_index, reindex, attention_set
                      compositions of the pinned functions above (scores, then
                      the top-k of all positions or of the pool; the set
                      selection U window); pinned with the plan's brute force.
  decode_layer_plan   pinned: separate pure-Python brute force on tiny inputs.
                      Which keys a reindex layer reads and what the full layer
                      attends to are READINGS 3 and 4 (parity unpinned by the
                      pages).
  prefill_query       pinned: equals decode at the same position (property).
  attention_combine   pinned: equals sparse_attention over the union on random
                      partitions (one set empty), and the single-set identity.
  kv_rows_local_window  pinned: closed forms (one window row, uniform
                      softmax over ring slots and FP4 rows), the separate
                      brute force of the plan with local rings, and equality
                      with the FP4-only rows when the ring holds them.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

FULL, REINDEX, REUSE = 0, 1, 2


# =============================================================== step 1: index score
def index_scores(q: np.ndarray, w: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """Indexer score of every key row for one query.

    score[s] = sum_h w[h] * max(0, sum_d q[h][d] * keys[s][d])

    q int8 [H][D], w int8 [H], keys int8 [n][D] -> int64 [n].

    [AD] Act 2: the first full-mode indexing layer searches the whole context;
    [YS] item 2: "an indexing layer scans full context once".
    READING 1: the pages give no formula.  This is an integer multi-head
    indexer: one shared key row per position, ReLU per head, integer head
    weights.  Without the ReLU, the heads would collapse into one dot product.
    READING 2: one key row per position, shared by all indexer heads.
    """
    k = np.asarray(keys, dtype=np.int64)
    qq = np.asarray(q, dtype=np.int64)
    ww = np.asarray(w, dtype=np.int64)
    dots = k @ qq.T                       # [n][H]
    return np.maximum(dots, 0) @ ww       # [n]


def score_bound(q: np.ndarray, w: np.ndarray) -> int:
    """Upper bound on |score| for any int8 keys: 128 * sum_h |w_h| * sum_d |q_hd|.
    The library reports an error when this bound reaches 2**31, because then an
    int32 score could overflow."""
    qq = np.abs(np.asarray(q, dtype=np.int64))
    ww = np.abs(np.asarray(w, dtype=np.int64))
    return int(128 * np.sum(ww * qq.sum(axis=1)))


# =============================================================== step 2: exact top-k
def top_k_positions(scores: np.ndarray, positions: np.ndarray, k: int) -> np.ndarray:
    """The k highest-scoring positions, with ties going to the lower position.
    The result is returned in ascending position order.

    If k exceeds the number of candidates, every candidate is returned.  The
    order is: score descending, then position ascending.  The first k
    entries are taken and then sorted by position.
    READING 5: ties go to the lower index, and selections are reported in
    ascending position order.
    """
    scores = np.asarray(scores, dtype=np.int64)
    positions = np.asarray(positions, dtype=np.int64)
    assert scores.shape == positions.shape
    if k <= 0 or scores.size == 0:
        return np.zeros(0, dtype=np.int64)
    order = np.lexsort((positions, -scores))      # last key is primary
    return np.sort(positions[order[:k]])


# =============================================================== steps 1-4: the index pipeline
def full_index(q, w, keys, pos: int, pool: int, topk: int):
    """A full-mode layer for a query at position ``pos``.

    Scores every visible position 0..pos.  Keeps the candidate pool (the
    ``pool`` best positions) and the layer's own selection (the ``topk`` best
    positions in the pool, under the same scores).
    Returns (scores int64 [pos+1], pool_idx ascending, sel_idx ascending).

    [AD] Act 2: "searches the large context and builds a candidate pool".
    [YS] item 2: the pool holds up to 16,384 positions.
    READING 4: the full layer attends to the top-k of its own pool.  That is
    the same set as the top-k of all positions.
    """
    s = index_scores(q, w, keys[:pos + 1])
    positions = np.arange(pos + 1, dtype=np.int64)
    pool_idx = top_k_positions(s, positions, pool)
    sel_idx = top_k_positions(s[pool_idx], pool_idx, topk)
    return s, pool_idx, sel_idx


def reindex(q, w, keys, pool_idx: np.ndarray, topk: int):
    """A reindex layer: score only the pool positions (with this layer's q, w
    and index keys) and keep the ``topk`` best.
    Returns (pool scores int64 [len(pool)], sel_idx ascending).

    [AD] Act 2: "later layers search only that much smaller pool instead of
    rescanning everything"; [YS] item 2: "later layers search within that
    shortlist".
    READING 3: a reindex layer reads its own index-key cache, at pool rows only.
    """
    pool_idx = np.asarray(pool_idx, dtype=np.int64)
    s = index_scores(q, w, keys[pool_idx]) if pool_idx.size else np.zeros(0, np.int64)
    return s, top_k_positions(s, pool_idx, topk)


def attention_set(sel_idx: np.ndarray, pos: int, window: int) -> np.ndarray:
    """The selected global positions plus the sliding window
    [max(0, pos-window+1), pos], each counted once, in ascending order.

    [YS] item 2: "512 most relevant KV entries, plus a local 128-token window";
    [DA]: "up to 512 global positions, alongside a local window of the most
    recent 128 tokens".
    READING 6: a position that is both selected and in the window is used once.
    """
    win = np.arange(max(0, pos - window + 1), pos + 1, dtype=np.int64)
    return np.union1d(np.asarray(sel_idx, dtype=np.int64), win)


# =============================================================== FP4 storage format
# E2M1 (OCP MX): 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit.
def e2m1_decode(code) -> np.ndarray:
    """Value of 4-bit E2M1 codes (array of ints 0..15), from the bit fields:
    exponent 0 gives a subnormal m * 0.5; otherwise 2**(e-1) * (1 + m/2)."""
    code = np.asarray(code, dtype=np.int64)
    sign = np.where(code & 0x8, -1.0, 1.0)
    e = (code >> 1) & 0x3
    m = code & 0x1
    mag = np.where(e == 0, m * 0.5, np.ldexp(1.0 + m / 2.0, (e - 1).astype(np.int64)))
    return sign * mag


# E4M3 "fn" (OCP OFP8): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits,
# no infinities, S.1111.111 is NaN, largest finite 448.
def e4m3_decode(byte) -> np.ndarray:
    """Value of E4M3 bytes (array of ints 0..255), from the bit fields."""
    b = np.asarray(byte, dtype=np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 0x7
    normal = np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = np.ldexp(m / 8.0, -6)
    val = sign * np.where(e == 0, sub, normal)
    return np.where((e == 15) & (m == 7), np.nan, val)


FP4_BLOCK = 32


def fp4_dequant(codes: np.ndarray, scales: np.ndarray, dim: int) -> np.ndarray:
    """Dequantise FP4 rows to float64.

    codes  uint8 [n][dim/2]: element 2i sits in the low nibble of byte i and
           element 2i+1 in the high nibble.
    scales uint8 [n][dim/32]: one E4M3 scale per block of 32 elements.
    value[j] = e2m1(code j) * e4m3(scale of block j // 32).

    [AD] Act 3: "FP4 main KV caching"; [YS] item 2: "KV values are compressed
    from FP8 (8 bits) to FP4 (4 bits)".  READING 9: the nibble order and the
    two-plane row layout.
    """
    codes = np.asarray(codes, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.uint8)
    n = codes.shape[0]
    nib = np.empty((n, dim), dtype=np.int64)
    nib[:, 0::2] = codes[:, :dim // 2] & 0xF
    nib[:, 1::2] = codes[:, :dim // 2] >> 4
    scale = np.repeat(e4m3_decode(scales[:, :dim // FP4_BLOCK]), FP4_BLOCK, axis=1)
    return e2m1_decode(nib) * scale


_E2M1_MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])    # codes 0..7
_E4M3_POS = e4m3_decode(np.arange(0x7F))                           # codes 0..126, ascending


def _nearest_even(values: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the grid value nearest to each (non-negative) value.
    A tie goes to the even index, which is the even mantissa; values above
    the grid saturate to the last index."""
    hi = np.clip(np.searchsorted(grid, values, side="left"), 1, len(grid) - 1)
    lo = hi - 1
    d_lo = values - grid[lo]
    d_hi = grid[hi] - values
    pick = np.where(d_lo < d_hi, lo, np.where(d_hi < d_lo, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(values >= grid[-1], len(grid) - 1, pick)
    return np.where(values <= grid[0], 0, pick)


def e4m3_encode_rne(a: np.ndarray) -> np.ndarray:
    """Non-negative float64 values -> nearest E4M3 byte (ties to even),
    saturating at 448 (0x7E)."""
    return _nearest_even(np.asarray(a, dtype=np.float64), _E4M3_POS).astype(np.uint8)


def fp4_quantize(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Store float rows [n][dim] as FP4: returns (codes [n][dim/2], scales [n][dim/32]).

    Each block of 32 values is encoded as follows:
      amax  = max |x|
      scale = E4M3 nearest to amax/6 (ties to even, saturating at 448)
      code  = E2M1 nearest to x/scale (ties to even, saturating at +-6)
    If the scale decodes to 0, every code in the block is 0.  A value that
    rounds to magnitude 0 is stored as +0 (code 0).
    READING 10: the scale is rounded to nearest, so the block maximum can be
    clipped to 6*scale.  This is the cache-write side of the FP4 main KV cache
    ([AD] Act 3).
    """
    x = np.asarray(x, dtype=np.float64)
    n, dim = x.shape
    blocks = x.reshape(n, dim // FP4_BLOCK, FP4_BLOCK)
    amax = np.abs(blocks).max(axis=2)
    scale_b = e4m3_encode_rne(amax / 6.0)
    scale = e4m3_decode(scale_b)[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(scale > 0, np.abs(blocks) / np.where(scale > 0, scale, 1.0), 0.0)
    mag = _nearest_even(v, _E2M1_MAGS).astype(np.int64)
    sign = np.where((blocks < 0) & (mag > 0), 8, 0)
    nib = (mag | sign).reshape(n, dim)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return codes, scale_b.astype(np.uint8)


# =============================================================== step 5: sparse attention
def sparse_attention(q: np.ndarray, kv_rows: np.ndarray, softmax_scale: float | None = None):
    """Softmax attention of every query head over the given latent rows.

    q float [Hq][D], kv_rows float64 [m][D].  The rows are the dequantised
    cache rows of the attention set, and each row is both key and value.
      logit[h][s] = softmax_scale * (q[h] . kv[s])
      o[h]        = sum_s softmax_s(logit[h]) * kv[s]
    Returns (o float64 [Hq][D], lse float64 [Hq]).  The lse is the natural log
    of sum_s exp(logit).

    [YS] item 2 / [DA]: attention reads the selected global positions plus the
    local window.  READING 8: the default scale is 1/sqrt(D).  There is no
    positional rotation, sink or bias.
    """
    q = np.asarray(q, dtype=np.float64)
    kv = np.asarray(kv_rows, dtype=np.float64)
    if softmax_scale is None or softmax_scale <= 0:
        softmax_scale = 1.0 / math.sqrt(q.shape[1])
    logits = softmax_scale * (q @ kv.T)                 # [Hq][m]
    mx = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - mx)
    l = p.sum(axis=1, keepdims=True)
    o = (p @ kv) / l
    return o, (mx + np.log(l))[:, 0]


def attention_combine(outs, lses):
    """Attention over the union of disjoint row sets, from the result of each
    set.

    outs float [R][Hq][D] and lses float [R][Hq] are sparse_attention's
    (o, lse) over R disjoint sets of rows; an empty set has lse = -inf (its o
    is ignored).  Softmax over the union is each set's softmax scaled by that
    set's share of the total mass:
      LSE = log sum_r exp(lse_r),   o = sum_r exp(lse_r - LSE) o_r.
    Returns (o float64 [Hq][D], LSE float64 [Hq]).  A head whose sets are all
    empty gets o = 0 and LSE = -inf.
    READING 16: a context split over several GPUs attends slice by slice and
    combines the slices' results.  The pages scale context by selection
    ([AD] Act 2) and do not say how a sharded context is attended.
    """
    outs = np.asarray(outs, dtype=np.float64)
    lses = np.asarray(lses, dtype=np.float64)
    M = lses.max(axis=0)                                            # [Hq]
    some = np.isfinite(M)
    w = np.where(np.isfinite(lses), np.exp(lses - np.where(some, M, 0.0)), 0.0)   # [R][Hq]
    L = w.sum(axis=0)
    safe = np.where(L > 0, L, 1.0)
    outs = np.where(np.isfinite(lses)[:, :, None], outs, 0.0)      # an empty set's o is not used
    o = np.einsum("rh,rhd->hd", w, outs) / safe[:, None]
    return np.where(some[:, None], o, 0.0), np.where(some, M + np.log(safe), -np.inf)


# =============================================================== the layer's local window cache
def kv_rows_local_window(S, pos: int, window: int, codes, scales, D: int, local_ring) -> np.ndarray:
    """Key/value rows of the attention set S (ascending positions, as
    attention_set gives it) for a layer that keeps its own cache of the most
    recent tokens beside the FP4 main cache.

    The positions of the window [max(0, pos-window+1), pos] are read from
    ``local_ring``, float [R][D] with R >= window: position p sits in slot
    p mod R.  Every other position of S is read from the FP4 main cache
    (codes, scales) and dequantised.  Returns float64 [len(S)][D].

    [YS] "The three KV-cache optimizations", item 3: besides the global KV,
    V4 kept a separate per-layer local KV for the latest 128 tokens, and
    V4.1 keeps that local cache while a session is active.
    READING 15: the pages give the local cache no number format and state FP4
    for the global KV only, so the local cache holds the rows as they are
    (bf16 values in the library), in a ring of R rows per sequence.
    """
    S = np.asarray(S, dtype=np.int64)
    ring = np.asarray(local_ring, dtype=np.float64)
    R = ring.shape[0]
    if R < window:
        raise ValueError(f"local ring of {R} rows cannot hold a window of {window}")
    wstart = max(0, pos - window + 1)
    rows = np.empty((len(S), D), dtype=np.float64)
    local = S >= wstart
    far = S[~local]
    if far.size:
        rows[~local] = fp4_dequant(np.asarray(codes)[far], np.asarray(scales)[far], D)
    rows[local] = ring[S[local] % R]
    return rows


# =============================================================== the layer plan
@dataclass
class LayerResult:
    mode: int
    pool_idx: np.ndarray | None     # FULL layers only
    sel_idx: np.ndarray             # positions this layer attends to globally
    attn_set: np.ndarray            # sel_idx together with the window
    out: np.ndarray                 # float64 [Hq][D]
    lse: np.ndarray                 # float64 [Hq]
    scores: np.ndarray | None = None


def decode_layer_plan(modes, layers, pos: int, pool: int, topk: int, window: int,
                      softmax_scale: float | None = None) -> list[LayerResult]:
    """One decode step through a sequence of CSA2 layers.

    ``layers[i]`` holds the inputs of layer i:
      'q', 'w', 'keys'    int8 indexer query, head weights and key rows
                          (needed by FULL and REINDEX layers),
      'q_attn'            float [Hq][D] query (bf16 values),
      'codes', 'scales'   the FP4 cache planes of that layer,
      'local_ring'        optional float [R][D]: the layer's local cache of
                          the most recent tokens; the window reads it (see
                          kv_rows_local_window).
    Modes: FULL scores every position and builds the pool.  REINDEX re-scores
    the most recent FULL layer's pool.  REUSE takes the selection of the most
    recent FULL or REINDEX layer unchanged.

    [AD] Act 2, [AS] and [ST]: layers are full, reindex or reuse.  Reuse
    layers share indices with the layer they reuse ([YS] item 2: "selection
    reuse").  READING 3/4: see full_index and reindex.
    """
    modes = list(modes)
    if not modes or modes[0] != FULL:
        raise ValueError("the first layer must be a full-mode layer")
    results: list[LayerResult] = []
    pool_idx = sel = None
    for mode, L in zip(modes, layers):
        scores = None
        layer_pool = None
        if mode == FULL:
            scores, pool_idx, sel = full_index(L["q"], L["w"], L["keys"], pos, pool, topk)
            layer_pool = pool_idx
        elif mode == REINDEX:
            scores, sel = reindex(L["q"], L["w"], L["keys"], pool_idx, topk)
        elif mode != REUSE:
            raise ValueError(f"unknown mode {mode}")
        S = attention_set(sel, pos, window)
        D = np.asarray(L["q_attn"]).shape[1]
        if L.get("local_ring") is not None:
            kv = kv_rows_local_window(S, pos, window, L["codes"], L["scales"], D, L["local_ring"])
        else:
            kv = fp4_dequant(L["codes"][S], L["scales"][S], D)
        o, lse = sparse_attention(L["q_attn"], kv, softmax_scale)
        results.append(LayerResult(mode, layer_pool, sel, S, o, lse, scores))
    return results


def prefill_query(q, w, keys, q_attn, codes, scales, pos: int, topk: int, window: int,
                  softmax_scale: float | None = None):
    """One query of a causal prefill chunk at position ``pos``.  Its top-k is
    taken over its whole causal prefix 0..pos (there is no pool), and it then
    attends to that top-k together with the window.
    Returns (sel_idx, attn_set, o, lse).

    READING 14: every query of the chunk sees rows 0..pos only, for the index,
    the window and the attention, and keeps its top-k of the whole prefix.
    READING 7 (as for decode): the cache already holds the token at pos."""
    s = index_scores(q, w, keys[:pos + 1])
    sel = top_k_positions(s, np.arange(pos + 1, dtype=np.int64), topk)
    S = attention_set(sel, pos, window)
    kv = fp4_dequant(codes[S], scales[S], np.asarray(q_attn).shape[1])
    o, lse = sparse_attention(q_attn, kv, softmax_scale)
    return sel, S, o, lse
