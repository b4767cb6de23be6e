"""The bench's byte and launch accounting for the 1M-context 8-layer step,
on the CPU.

The roofline fraction the bench reports divides these algorithmic bytes by
the measured step time, so they are pinned here to their closed form: the
full layer's key rows, one pool gather per reindex layer, the FP4 rows of
every layer's attention set (512 selected rows below the window plus the
128-row window, 272 bytes each at d=512) and the queries, weights and
outputs.
"""
import importlib.util
import os

import torch

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_accounting", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


class _Layer:
    def __init__(self, sel, pool_cnt=None):
        self.sel_idx = torch.tensor([sel], dtype=torch.int32)
        self.sel_cnt = torch.tensor([len(sel)], dtype=torch.int32)
        self.pool_cnt = None if pool_cnt is None else torch.tensor([pool_cnt], dtype=torch.int32)


def test_algorithmic_bytes_of_the_1m_step():
    bench = _bench()
    wl = synth.C2_1M_PLAN
    pos = int(wl.lengths()[0]) - 1
    sel = list(range(0, 512 * 1000, 1000))            # 512 selected rows, all below the window
    layers = [_Layer(sel, pool_cnt=wl.pool if m == synth.FULL else None) for m in wl.modes]
    total, parts = bench.algorithmic_bytes(wl, layers, pos)
    row_fp4 = wl.attn_dim // 2 + wl.attn_dim // 32    # 256 code bytes + 16 scale bytes
    assert parts["full_keys"] == (pos + 1) * wl.idx_dim == 134_217_728
    assert parts["reindex_gather"] == 2 * wl.pool * wl.idx_dim == 4_194_304
    assert parts["attn_rows"] == 8 * (512 + wl.window) * row_fp4 == 1_392_640
    n_index_layers = sum(1 for m in wl.modes if m != synth.REUSE)
    assert parts["q_w_out"] == (n_index_layers * (wl.idx_heads * wl.idx_dim + wl.idx_heads)
                                + 8 * 2 * wl.attn_heads * wl.attn_dim * 2) == 1_073_344
    assert total == 140_878_016


def test_window_overlap_is_counted_once():
    bench = _bench()
    wl = synth.C2_1M_PLAN
    pos = int(wl.lengths()[0]) - 1
    sel = list(range(pos - 511, pos + 1))              # every selected row inside the window
    layers = [_Layer(sel, pool_cnt=wl.pool if m == synth.FULL else None) for m in wl.modes]
    _, parts = bench.algorithmic_bytes(wl, layers, pos)
    row_fp4 = wl.attn_dim // 2 + wl.attn_dim // 32
    below = 512 - wl.window                            # selected rows before the window start
    assert parts["attn_rows"] == 8 * (below + wl.window) * row_fp4


def test_five_launches_per_decode_step():
    assert _bench().kernels_per_step(synth.C2_1M_PLAN) == 5


def test_device_facts_without_a_gpu_are_none():
    import torch
    bench = _bench()
    f = bench.device_facts(torch.device("cpu"))
    assert f["l2_bytes"] is None and f["read_only_gbs"] is None and "2 GiB" in f["read_only_how"]


def test_fp4_cache_write_bytes_per_row():
    bench = _bench()
    assert bench.quant_bytes_per_row(512) == 1024 + 256 + 16     # bf16 row in, codes and scales out
    assert bench.quant_bytes_per_row(128) == 256 + 64 + 4
