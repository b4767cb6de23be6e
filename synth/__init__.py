"""Seeded synthetic inputs for the CSA2 sparse-attention decode path.

This module holds the workload recipes (shapes, sizes, value distributions,
ragged lengths, page placement) and the seeded random draws that realise them.
It holds none of the method's arithmetic: no index scoring, no selection, no
FP4 encoding or decoding and no attention.  The oracle-side tests and the
benchmark both draw their inputs here, so both sides of every parity check
consume the same bytes.

Every tensor is split into chunks of ``CHUNK_ROWS`` rows.  Each chunk comes
from its own Philox stream keyed by (base seed, workload, layer, tensor name,
sequence, chunk), so any row range can be regenerated alone and chunks can be
drawn in parallel threads without changing a single value.
"""
from __future__ import annotations

import hashlib
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from typing import Sequence

import numpy as np

CHUNK_ROWS = 1024

FULL, REINDEX, REUSE = 0, 1, 2
MODE_NAMES = {FULL: "full", REINDEX: "reindex", REUSE: "reuse"}


@dataclass(frozen=True)
class Workload:
    """One synthetic decode (or prefill) workload.

    idx_*   : the int8 indexer (heads x head dim, value range of q and keys,
              range of the integer head weights).
    pool/topk/window : candidate-pool size, selected global positions and the
              sliding-window length.
    attn_*  : bf16 query heads sharing one latent K=V row of ``attn_dim``
              values, stored as FP4 with one scale per 32 values.
    outlier_p / outlier_mul : probability that one cache value is multiplied
              by ``outlier_mul`` before it is stored.
    modes   : per-layer CSA2 mode (FULL / REINDEX / REUSE).
    seq_lens: fixed lengths, or None with ``ragged`` = (n_seq, lo, hi).
    page_rows: rows per KV page (None = one contiguous block per sequence).
    prefill : (n_queries, first_pos) for a causal prefill chunk, else None.
    """

    name: str
    idx_heads: int
    idx_dim: int
    idx_range: tuple[int, int]
    w_range: tuple[int, int]
    pool: int
    topk: int
    window: int
    attn_heads: int
    attn_dim: int
    outlier_p: float = 0.0
    outlier_mul: float = 8.0
    modes: tuple[int, ...] = (FULL,)
    seq_lens: tuple[int, ...] | None = None
    ragged: tuple[int, int, int] | None = None
    page_rows: int | None = None
    prefill: tuple[int, int] | None = None
    seed: int = 0

    @property
    def n_layers(self) -> int:
        return len(self.modes)

    def lengths(self) -> np.ndarray:
        """Context length of each sequence (int64)."""
        if self.seq_lens is not None:
            return np.asarray(self.seq_lens, dtype=np.int64)
        n_seq, lo, hi = self.ragged
        g = _gen(self, "seq_lens", 0, 0, 0)
        return g.integers(lo, hi, size=n_seq, endpoint=True, dtype=np.int64)

    def query_positions(self) -> tuple[np.ndarray, np.ndarray]:
        """(seq_of_query, query_pos) for every query of one step.

        Decode: one query per sequence at its last cached position (the cache
        already holds the current token).  Prefill: ``n_queries`` consecutive
        positions of sequence 0 starting at ``first_pos``.
        """
        lens = self.lengths()
        if self.prefill is not None:
            nq, first = self.prefill
            return (np.zeros(nq, dtype=np.int64),
                    np.arange(first, first + nq, dtype=np.int64))
        return np.arange(len(lens), dtype=np.int64), lens - 1


def _key(wl: Workload, tensor: str, layer: int, seq: int, chunk: int) -> list[int]:
    text = f"csa2|{wl.seed}|{wl.name}|{tensor}|{layer}|{seq}|{chunk}".encode()
    digest = hashlib.blake2b(text, digest_size=16).digest()
    return [int.from_bytes(digest[:8], "little"), int.from_bytes(digest[8:], "little")]


def _gen(wl: Workload, tensor: str, layer: int, seq: int, chunk: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=_key(wl, tensor, layer, seq, chunk)))


def _threads() -> int:
    try:
        return max(1, min(32, len(os.sched_getaffinity(0))))
    except AttributeError:  # pragma: no cover
        return max(1, min(32, os.cpu_count() or 1))


def _chunked(fill, n_rows: int, row0: int, row1: int, width: int, dtype) -> np.ndarray:
    """Rows [row0, row1) of a chunked tensor whose chunk c is ``fill(c)``."""
    assert 0 <= row0 <= row1 <= n_rows
    out = np.empty((row1 - row0, width), dtype=dtype)
    if row1 == row0:
        return out
    c0, c1 = row0 // CHUNK_ROWS, (row1 - 1) // CHUNK_ROWS

    def one(c: int) -> None:
        lo = c * CHUNK_ROWS
        rows = fill(c, min(CHUNK_ROWS, n_rows - lo))
        a, b = max(row0, lo), min(row1, lo + CHUNK_ROWS)
        out[a - row0:b - row0] = rows[a - lo:b - lo]

    if c1 - c0 < 4:
        for c in range(c0, c1 + 1):
            one(c)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(one, range(c0, c1 + 1)))
    return out


# ---------------------------------------------------------------- index side
def index_keys(wl: Workload, layer: int, seq: int, row0: int = 0, row1: int | None = None) -> np.ndarray:
    """int8 [row1-row0][idx_dim] index-key rows of one sequence, uniform on
    the inclusive range ``idx_range``."""
    n = int(wl.lengths()[seq])
    row1 = n if row1 is None else row1
    lo, hi = wl.idx_range

    def fill(c: int, rows: int) -> np.ndarray:
        g = _gen(wl, "idx_keys", layer, seq, c)
        return g.integers(lo, hi, size=(rows, wl.idx_dim), endpoint=True, dtype=np.int8)

    return _chunked(fill, n, row0, row1, wl.idx_dim, np.int8)


def index_query(wl: Workload, layer: int, query: int) -> tuple[np.ndarray, np.ndarray]:
    """(q int8 [idx_heads][idx_dim], w int8 [idx_heads]) of one query."""
    g = _gen(wl, "idx_query", layer, query, 0)
    lo, hi = wl.idx_range
    q = g.integers(lo, hi, size=(wl.idx_heads, wl.idx_dim), endpoint=True, dtype=np.int8)
    wlo, whi = wl.w_range
    w = g.integers(wlo, whi, size=wl.idx_heads, endpoint=True, dtype=np.int8)
    return q, w


# ---------------------------------------------------------------- attention side
def kv_values(wl: Workload, layer: int, seq: int, row0: int = 0, row1: int | None = None) -> np.ndarray:
    """float32 [row1-row0][attn_dim] latent KV values before FP4 storage:
    N(0,1), each value independently multiplied by ``outlier_mul`` with
    probability ``outlier_p`` (drawn as one of 1/outlier_p equally likely
    integers being zero)."""
    n = int(wl.lengths()[seq])
    row1 = n if row1 is None else row1
    period = int(round(1.0 / wl.outlier_p)) if wl.outlier_p > 0 else 0

    def fill(c: int, rows: int) -> np.ndarray:
        g = _gen(wl, "kv", layer, seq, c)
        x = g.standard_normal((rows, wl.attn_dim), dtype=np.float32)
        if period:
            hit = g.integers(0, period, size=(rows, wl.attn_dim), dtype=np.uint16) == 0
            x[hit] *= np.float32(wl.outlier_mul)
        return x

    return _chunked(fill, n, row0, row1, wl.attn_dim, np.float32)


def local_kv_values(wl: Workload, layer: int, seq: int, row0: int, row1: int) -> np.ndarray:
    """float32 [row1-row0][attn_dim] rows of a layer's local window cache for
    positions row0..row1-1 of one sequence: the same distribution as
    kv_values (its own stream: the local rows are not the main cache's
    values), rounded to the nearest bf16 value, the format the local cache
    stores."""
    n = int(wl.lengths()[seq])
    period = int(round(1.0 / wl.outlier_p)) if wl.outlier_p > 0 else 0

    def fill(c: int, rows: int) -> np.ndarray:
        g = _gen(wl, "local_kv", layer, seq, c)
        x = g.standard_normal((rows, wl.attn_dim), dtype=np.float32)
        if period:
            hit = g.integers(0, period, size=(rows, wl.attn_dim), dtype=np.uint16) == 0
            x[hit] *= np.float32(wl.outlier_mul)
        return x

    return round_to_bf16(_chunked(fill, n, row0, row1, wl.attn_dim, np.float32))


def attn_query(wl: Workload, layer: int, query: int) -> np.ndarray:
    """float32 [attn_heads][attn_dim] N(0,1) query, already rounded to the
    nearest bf16 value (ties to even), so it is exactly a bf16 tensor."""
    g = _gen(wl, "attn_query", layer, query, 0)
    x = g.standard_normal((wl.attn_heads, wl.attn_dim), dtype=np.float32)
    return round_to_bf16(x)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest bf16 value (ties to even), returned as float32.
    Input preparation only (the queries are bf16 by definition)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


# ---------------------------------------------------------------- paged placement
def page_table(wl: Workload) -> np.ndarray:
    """int32 [n_seq][max_pages]: physical page of each logical page.

    Physical pages are one seeded random permutation of
    [0, sum_i ceil(len_i / page_rows)), handed out in sequence order; unused
    slots hold -1."""
    lens = wl.lengths()
    pr = wl.page_rows
    pages = (lens + pr - 1) // pr
    total = int(pages.sum())
    perm = _gen(wl, "page_perm", 0, 0, 0).permutation(total).astype(np.int32)
    table = np.full((len(lens), int(pages.max())), -1, dtype=np.int32)
    at = 0
    for s, n in enumerate(pages):
        table[s, :n] = perm[at:at + n]
        at += int(n)
    return table


# ---------------------------------------------------------------- the workloads
C0_TINY = Workload(
    name="tiny_decode_ctx4096", idx_heads=4, idx_dim=64, idx_range=(-8, 8), w_range=(1, 4),
    pool=1024, topk=64, window=128, attn_heads=8, attn_dim=128, seq_lens=(4096,))

C1_SINGLE = Workload(
    name="decode_ctx131072", idx_heads=64, idx_dim=128, idx_range=(-16, 16), w_range=(1, 8),
    pool=16384, topk=512, window=128, attn_heads=64, attn_dim=512, outlier_p=0.01,
    seq_lens=(131072,))

C2_1M_PLAN = Workload(
    name="decode_ctx1048576_8layer", idx_heads=64, idx_dim=128, idx_range=(-16, 16), w_range=(1, 8),
    pool=16384, topk=512, window=128, attn_heads=64, attn_dim=512, outlier_p=0.01,
    modes=(FULL, REINDEX, REUSE, REUSE, REINDEX, REUSE, REUSE, REUSE), seq_lens=(1048576,))

C3_RAGGED = Workload(
    name="ragged_decode_32seq_paged", idx_heads=64, idx_dim=128, idx_range=(-16, 16), w_range=(1, 8),
    pool=16384, topk=512, window=128, attn_heads=64, attn_dim=512, outlier_p=0.01,
    ragged=(32, 32768, 262144), page_rows=64)

C4_PREFILL = Workload(
    name="prefill_2048q_ctx262144", idx_heads=64, idx_dim=128, idx_range=(-16, 16), w_range=(1, 8),
    pool=0, topk=512, window=128, attn_heads=64, attn_dim=512, outlier_p=0.01,
    seq_lens=(262144,), prefill=(2048, 260096))

WORKLOADS = {wl.name: wl for wl in (C0_TINY, C1_SINGLE, C2_1M_PLAN, C3_RAGGED, C4_PREFILL)}


def scaled(wl: Workload, **changes) -> Workload:
    """A copy of ``wl`` with some fields replaced (for reduced-size tests)."""
    from dataclasses import replace
    return replace(wl, **changes)
