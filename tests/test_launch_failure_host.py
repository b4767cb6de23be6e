"""Launch failures surface as CSA2_ERR_CUDA, on a machine without a GPU.

Every call below passes the argument checks: aligned pointers, supported
shapes, enough workspace.  With no CUDA device, the library's first CUDA
call fails, and the entry point must return CSA2_ERR_CUDA (4) without
touching the fake pointers or crashing.  Where a GPU is present these
pointers would reach real kernels, so the test runs only without one."""
import ctypes

import pytest
import torch

import kv_cache_decode_csa2_b200 as K
from kv_cache_decode_csa2_b200 import csa2 as B

pytestmark = pytest.mark.skipif(torch.cuda.is_available(), reason="fake device pointers: only without a GPU")

A = 1 << 20          # a 16-byte (and 256-byte) aligned fake device address
BIG = 1 << 40        # a workspace size every call accepts


def _rows(row_bytes, n_rows=4096, seq_rows=4096):
    r = B.csa2_rows()
    r.base, r.row_bytes, r.n_rows = A, row_bytes, n_rows
    r.page_table, r.page_rows, r.max_pages, r.seq_rows = None, 0, 0, seq_rows
    return r


def test_index_full_reports_the_failed_launch():
    L = K.lib()
    keys = _rows(128)
    assert L.csa2_index_full(A, A, ctypes.byref(keys), None, A, 1, 64, 128, 4096, None, 0, 1024, A, A, 64, A, A,
                             A, BIG, A, None) == 4


def test_topk_and_reindex_report_the_failed_launch():
    L = K.lib()
    assert L.csa2_topk_pool(A, 4096, None, None, 1, 4096, 64, A, A, A, BIG, A, None) == 4      # one-CTA path
    assert L.csa2_topk_pool(A, 1 << 20, None, None, 1, 1 << 20, 512, A, A, A, BIG, A, None) == 4
    keys = _rows(128)
    assert L.csa2_reindex(A, A, ctypes.byref(keys), None, A, A, 1, 64, 128, 16384, 512, A, A, None, A, BIG, A,
                          None) == 4


def test_attention_and_quantiser_report_the_failed_launch():
    L = K.lib()
    codes, scales, ring = _rows(256), _rows(16), _rows(1024, n_rows=128, seq_rows=128)
    assert L.csa2_sparse_attn_fp4(A, ctypes.byref(codes), ctypes.byref(scales), None, A, A, A, 1, 64, 512, 512,
                                  128, 0.0, A, None, A, BIG, A, None) == 4
    assert L.csa2_sparse_attn_fp4_local(A, ctypes.byref(codes), ctypes.byref(scales), ctypes.byref(ring), None, A,
                                        A, A, 1, 64, 512, 512, 128, 0.0, A, None, A, BIG, A, None) == 4
    assert L.csa2_fp4_quantize(A, 16, 512, 512, None, A, 256, A, 16, 16, A, None) == 4
    assert L.csa2_fp4_quantize_bf16(A, 16, 512, 512, None, A, 256, A, 16, 16, A, None) == 4


def test_wait_selftest_reports_the_failed_launch():
    L = K.lib()
    assert L.csa2_selftest_wait(0, 1000, A, A, None) == 4
    assert L.csa2_selftest_wait(1, 1000, None, A, None) == 4


def test_plan_reports_the_failed_launch():
    L = K.lib()
    modes = (ctypes.c_int32 * 3)(0, 1, 2)
    layers = (B.csa2_layer * 3)()
    for i, ly in enumerate(layers):
        ly.q, ly.w, ly.q_attn, ly.out = A, A, A, A
        ly.keys, ly.codes, ly.scales = _rows(128), _rows(256), _rows(16)
    s = B.csa2_plan_shape(nq=1, H=64, D_idx=128, Hq=64, D=512, P=1024, K=64, window=128, max_ctx=4096,
                          softmax_scale=0.0, seq_of_query=None, query_pos=A)
    assert L.csa2_layer_plan(modes, 3, layers, ctypes.byref(s), A, BIG, A, None) == 4
