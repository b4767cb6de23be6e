"""The benchmark's byte accounting for the decode workloads, on the CPU.

The roofline fraction the benchmark reports divides these algorithmic bytes
by the measured step time, so they are pinned here to their closed form: the
full layer's key rows (once per sequence, however many of its queries share
the scan), one pool gather per query and reindex layer, the FP4 rows of every
layer's attention set (selected rows below the window plus the window, 272
bytes each at d=512) and the queries, weights and outputs.
"""
import importlib.util
import os

import numpy as np
import torch

import synth
from kv_cache_decode_csa2_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_accounting", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


class _Layer:
    local_kv = None

    def __init__(self, sels, pool_cnt=None):
        K = max(len(s) for s in sels)
        self.sel_idx = torch.tensor([list(s) + [-1] * (K - len(s)) for s in sels], dtype=torch.int32)
        self.sel_cnt = torch.tensor([len(s) for s in sels], dtype=torch.int32)
        self.pool_cnt = None if pool_cnt is None else torch.tensor(pool_cnt, dtype=torch.int32)


def _state(wl, sels):
    sq, qp = wl.query_positions()
    nq = len(qp)
    layers = [_Layer(sels, pool_cnt=[wl.pool] * nq if m == synth.FULL else None) for m in wl.modes]
    return W.DecodeState(wl=wl, layers=layers, seq_of_query=sq, query_pos=qp, pos_dev=None, seq_dev=None,
                         max_ctx=int(wl.lengths().max()), inbuf=None, outbuf=None)


def test_algorithmic_bytes_of_the_1m_step():
    wl = synth.C2_1M_PLAN
    pos = int(wl.lengths()[0]) - 1
    sel = list(range(0, 512 * 1000, 1000))            # 512 selected rows, all below the window
    total, parts = W.algorithmic_bytes(_state(wl, [sel]))
    row_fp4 = wl.attn_dim // 2 + wl.attn_dim // 32    # 256 code bytes + 16 scale bytes
    assert parts["full_keys"] == (pos + 1) * wl.idx_dim == 134_217_728
    assert parts["reindex_gather"] == 2 * wl.pool * wl.idx_dim == 4_194_304
    assert parts["attn_rows"] == 8 * (512 + wl.window) * row_fp4 == 1_392_640
    n_index_layers = sum(1 for m in wl.modes if m != synth.REUSE)
    assert parts["q_w_out"] == (n_index_layers * (wl.idx_heads * wl.idx_dim + wl.idx_heads)
                                + 8 * 2 * wl.attn_heads * wl.attn_dim * 2) == 1_073_344
    assert total == 140_878_016


def test_window_overlap_is_counted_once():
    wl = synth.C2_1M_PLAN
    pos = int(wl.lengths()[0]) - 1
    sel = list(range(pos - 511, pos + 1))              # every selected row inside the window
    _, parts = W.algorithmic_bytes(_state(wl, [sel]))
    row_fp4 = wl.attn_dim // 2 + wl.attn_dim // 32
    below = 512 - wl.window                            # selected rows before the window start
    assert parts["attn_rows"] == 8 * (below + wl.window) * row_fp4


def test_local_window_rows_are_counted_as_bf16():
    """With a local window cache the window's rows are bf16 (2 bytes per
    value) and only the selected rows below the window are FP4."""
    bench = _bench()
    wl = bench.WL_WINDOW
    pos = int(wl.lengths()[0]) - 1
    sel = list(range(0, 384 * 1000, 1000)) + list(range(pos - 127, pos + 1))   # 384 below, 128 in the window
    st = _state(wl, [sel])
    for ly in st.layers:
        ly.local_kv = object()
    _, parts = W.algorithmic_bytes(st)
    row_fp4 = wl.attn_dim // 2 + wl.attn_dim // 32
    assert parts["attn_rows"] == 8 * (384 * row_fp4 + wl.window * 2 * wl.attn_dim)
    assert "window" in bench.LOCAL_WINDOW_WORKLOADS and bench.DECODE_WORKLOADS["window"][0] is wl


def test_local_ring_places_the_last_positions():
    """Ring row s R + p mod R holds position p of sequence s for the last R
    positions (the other rows stay zero)."""
    wl = synth.scaled(synth.C0_TINY, seq_lens=(300, 90))
    R = 128
    rows = W.local_ring_rows(wl, 0, wl.lengths(), R)
    assert rows.shape == (2 * R, wl.attn_dim)
    for s, n in enumerate(wl.lengths()):
        a = max(0, int(n) - R)
        x = synth.local_kv_values(wl, 0, s, a, int(n))
        for p in range(a, int(n)):
            assert np.array_equal(rows[s * R + p % R], x[p - a])
    assert not rows[R + 90:2 * R].any()


def test_verify_block_reads_the_keys_once_per_sequence():
    bench = _bench()
    wl = bench.WL_VERIFY
    sq, qp = wl.query_positions()
    assert len(qp) == 5 and (sq == 0).all() and int(qp[-1]) == int(wl.lengths()[0]) - 1
    sels = [list(range(0, 512 * 1000, 1000))] * 5
    _, parts = W.algorithmic_bytes(_state(wl, sels))
    assert parts["full_keys"] == int(wl.lengths()[0]) * wl.idx_dim        # one shared scan, not five
    assert parts["reindex_gather"] == 5 * 2 * wl.pool * wl.idx_dim


def test_ragged_batch_counts_every_sequence():
    wl = synth.C3_RAGGED
    lens = wl.lengths()
    sq, qp = wl.query_positions()
    sels = [list(range(0, 512 * 32, 32))] * len(qp)
    _, parts = W.algorithmic_bytes(_state(wl, sels))
    assert parts["full_keys"] == int(lens.sum()) * wl.idx_dim
    assert parts["reindex_gather"] == 0
    row_fp4 = wl.attn_dim // 2 + wl.attn_dim // 32
    assert parts["attn_rows"] == len(qp) * (512 + wl.window) * row_fp4


def test_decode_workloads_name_their_configs():
    bench = _bench()
    assert bench.DECODE_WORKLOADS["decode"][0] is synth.C2_1M_PLAN
    assert bench.DECODE_WORKLOADS["tiny"][0] is synth.C0_TINY
    assert bench.DECODE_WORKLOADS["single"][0] is synth.C1_SINGLE
    assert bench.DECODE_WORKLOADS["ragged"][0] is synth.C3_RAGGED
    assert bench.DECODE_WORKLOADS["ragged"][3] == len(synth.C3_RAGGED.lengths())
    assert bench.METRIC == "decode steps/s and HBM GB/s (% of B200 roofline) at 1M-token context"


def test_device_facts_without_a_gpu_are_none():
    bench = _bench()
    f = bench.device_facts(torch.device("cpu"))
    assert f["l2_bytes"] is None and f["read_only_gbs"] is None and "2 GiB" in f["read_only_how"]


def test_fp4_cache_write_bytes_per_row():
    bench = _bench()
    assert bench.quant_bytes_per_row(512) == 1024 + 256 + 16     # bf16 row in, codes and scales out
    assert bench.quant_bytes_per_row(128) == 256 + 64 + 4


def test_packer_aligns_views_of_one_buffer():
    p = W._Packer()
    a = p.add((3, 5), torch.bfloat16)
    b = p.add((7,), torch.int8)
    c = p.add((2, 4), torch.bfloat16)
    buf = torch.zeros(p.size, dtype=torch.uint8)
    v = p.views(buf)
    assert [tuple(x.shape) for x in v] == [(3, 5), (7,), (2, 4)]
    offs = [x.data_ptr() - buf.data_ptr() for x in v]
    assert offs == [0, 256, 512] and all(o % 256 == 0 for o in offs)
    v[b].fill_(3)
    assert int(buf[256:263].sum()) == 21 and int(buf[:30].sum()) == 0
    assert a == 0 and c == 2
