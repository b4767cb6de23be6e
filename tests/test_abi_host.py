"""Host-only checks of the C ABI: the library loads, exports every function
include/csa2.h declares, sizes workspaces, and rejects bad arguments with the
documented codes before it touches a GPU.  No kernel is launched here."""
import ctypes
import os
import re

import pytest

import kv_cache_decode_csa2_b200 as K
from kv_cache_decode_csa2_b200 import csa2 as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "csa2.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(csa2_\w+)\s*\(", text, re.M)))


def test_library_exports_every_declared_function():
    L = K.lib()
    names = _declared()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(B.EXPORTS)


def test_version_and_status_strings():
    L = K.lib()
    assert L.csa2_version() == 200
    for code in range(9):
        assert L.csa2_status_string(code)
    assert L.csa2_status_string(6) == b"position, page or row out of range"
    assert L.csa2_status_string(99) == b"unknown status"


def test_workspace_sizes():
    L = K.lib()
    small = L.csa2_index_full_workspace(1, 4096, 1024, 64)
    big = L.csa2_index_full_workspace(1, 1 << 20, 16384, 512)
    assert 4096 * 4 < small < big
    assert big >= (1 << 20) * 4                       # the score row
    assert L.csa2_index_full_workspace(0, 10, 1, 1) == 0
    assert L.csa2_topk_pool_workspace(1, 16384, 512) == 256     # one-CTA path, no scratch
    assert L.csa2_topk_pool_workspace(1, 16385, 512) > 256
    assert L.csa2_reindex_workspace(1, 16384, 512) >= 16384 * 4
    a = L.csa2_sparse_attn_workspace(1, 64, 512, 512, 128)
    assert a >= 8 * 64 * 512 * 4                      # fp32 partial O of 8 row slices per head
    modes = (ctypes.c_int32 * 8)(0, 1, 2, 2, 1, 2, 2, 2)
    s = B.csa2_plan_shape(nq=1, H=64, D_idx=128, Hq=64, D=512, P=16384, K=512, window=128,
                          max_ctx=1 << 20, softmax_scale=0.0, seq_of_query=None, query_pos=None)
    assert L.csa2_layer_plan_workspace(modes, 8, ctypes.byref(s)) > big + 8 * a
    bad = (ctypes.c_int32 * 2)(1, 0)                  # a plan must start with a full layer
    assert L.csa2_layer_plan_workspace(bad, 2, ctypes.byref(s)) == 0


def _rows(base=16, row_bytes=128, n_rows=10):
    r = B.csa2_rows()
    r.base, r.row_bytes, r.n_rows = base, row_bytes, n_rows
    r.page_table, r.page_rows, r.max_pages, r.seq_rows = None, 0, 0, 0
    return r


def test_rejects_bad_arguments_before_any_launch():
    L = K.lib()
    keys = _rows()
    # NULL q
    assert L.csa2_index_full(None, 16, ctypes.byref(keys), None, 16, 1, 64, 128, 10, None, 0, 0, None, None,
                             0, None, None, 256, 1 << 20, 16, None) == 1
    # unsupported indexer head dim
    assert L.csa2_index_full(16, 16, ctypes.byref(keys), None, 16, 1, 64, 96, 10, None, 0, 0, None, None,
                             0, None, None, 256, 1 << 20, 16, None) == 2
    # misaligned key rows
    bad = _rows(row_bytes=136)
    assert L.csa2_index_full(16, 16, ctypes.byref(bad), None, 16, 1, 64, 128, 10, None, 0, 0, None, None,
                             0, None, None, 256, 1 << 20, 16, None) == 1
    # workspace too small
    assert L.csa2_index_full(16, 16, ctypes.byref(keys), None, 16, 1, 64, 128, 10, None, 0, 0, None, None,
                             0, None, None, 256, 8, 16, None) == 3
    # more queries than one launch's work list holds
    assert L.csa2_index_full(16, 16, ctypes.byref(keys), None, 16, 4097, 64, 128, 10, None, 0, 0, None, None,
                             0, None, None, 256, 1 << 20, 16, None) == 2
    # top-k: k out of range; more queries than a grid dimension holds
    assert L.csa2_topk_pool(16, 10, None, None, 1, 10, 0, 16, None, None, 0, 16, None) == 1
    assert L.csa2_topk_pool(16, 10, None, None, 65536, 10, 4, 16, None, None, 0, 16, None) == 2
    assert L.csa2_topk_pool_noalloc(16, 10, None, None, 65536, 10, 4, 16, None, 16, None) == 2
    # reindex: K > P
    assert L.csa2_reindex(16, 16, ctypes.byref(keys), None, 16, 16, 1, 64, 128, 8, 9, 16, None, None, 256,
                          1 << 20, 16, None) == 1
    # attention: unsupported D and head count
    codes, scales = _rows(row_bytes=256), _rows(row_bytes=16)
    assert L.csa2_sparse_attn_fp4(16, ctypes.byref(codes), ctypes.byref(scales), None, 16, 16, None, 1, 64,
                                  256, 8, 128, 0.0, 16, None, 256, 1 << 20, 16, None) == 2
    assert L.csa2_sparse_attn_fp4(16, ctypes.byref(codes), ctypes.byref(scales), None, 16, 16, None, 1, 12,
                                  512, 8, 128, 0.0, 16, None, 256, 1 << 20, 16, None) == 2
    # quantiser: D not a multiple of 32
    assert L.csa2_fp4_quantize(16, 4, 48, 48, None, 16, 32, 16, 2, 4, 16, None) == 2
    # bf16 rows must start on 16 bytes: ld_x a multiple of 8 values (fp32: of 4)
    assert L.csa2_fp4_quantize_bf16(16, 4, 64, 68, None, 16, 32, 16, 2, 4, 16, None) == 1


def test_local_window_cache_is_checked():
    L = K.lib()
    codes, scales = _rows(row_bytes=256), _rows(row_bytes=16)
    args = (None, 16, 16, None, 1, 64, 512, 8, 128, 0.0, 16, None, 256, 1 << 20, 16, None)

    def call(local):
        return L.csa2_sparse_attn_fp4_local(16, ctypes.byref(codes), ctypes.byref(scales),
                                            ctypes.byref(local) if local is not None else None, *args)

    ring = _rows(row_bytes=1024, n_rows=256)
    ring.seq_rows = 128
    assert call(ring) == 3                       # a good ring: only the (too small) workspace is left
    assert call(None) == 1                       # the local entry point needs the cache
    ring.seq_rows = 127                          # a ring shorter than the 128-row window
    assert call(ring) == 1
    ring.seq_rows, ring.row_bytes = 128, 512     # rows shorter than D bf16 values
    assert call(ring) == 1
    ring.row_bytes = 1024
    ring.page_table, ring.page_rows, ring.max_pages = 16, 64, 4   # a ring is not paged
    assert call(ring) == 1
    # the same call through the plain entry point with a bad head count still says so first
    assert L.csa2_sparse_attn_fp4(16, ctypes.byref(codes), ctypes.byref(scales), None, 16, 16, None, 1, 12,
                                  512, 8, 128, 0.0, 16, None, 256, 1 << 20, 16, None) == 2


def test_wait_selftest_checks_its_arguments():
    L = K.lib()
    assert L.csa2_selftest_wait(2, 1000, 16, 16, None) == 1                    # no such kind
    assert L.csa2_selftest_wait(0, 1000, None, 16, None) == 1                  # the barrier needs a counter
    assert L.csa2_selftest_wait(1, 1000, None, None, None) == 1                # and every kind a status word
    assert L.csa2_selftest_wait(1, 10 ** 10 + 1, None, 16, None) == 1          # limits above 10 s are refused


def test_plan_rejects_too_many_queries_times_layers():
    L = K.lib()
    n = 16
    modes = (ctypes.c_int32 * n)(*([0] + [2] * (n - 1)))
    layers = (B.csa2_layer * n)()
    s = B.csa2_plan_shape(nq=4096, H=64, D_idx=128, Hq=64, D=512, P=16384, K=512, window=128, max_ctx=1 << 20,
                          softmax_scale=0.0, seq_of_query=None, query_pos=16)
    assert L.csa2_layer_plan(modes, n, layers, ctypes.byref(s), 256, 1 << 20, 16, None) == 2


def test_plan_rejects_reindex_first():
    L = K.lib()
    modes = (ctypes.c_int32 * 2)(1, 2)
    layers = (B.csa2_layer * 2)()
    s = B.csa2_plan_shape(nq=1, H=4, D_idx=64, Hq=8, D=128, P=16, K=4, window=8, max_ctx=32)
    assert L.csa2_layer_plan(modes, 2, layers, ctypes.byref(s), 256, 1 << 20, 16, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(B, "_lib", None)
    monkeypatch.setattr(B, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        B.lib()


def test_noalloc_capacity_matches_its_documented_bounds():
    """The fixed array of csa2_topk_pool_noalloc holds the scratch of 8 queries
    of up to 10^6 candidates or 7 of up to 2^24, and not one query more."""
    L = B.lib()
    cap = 4 << 20
    for nq, n in [(8, 10 ** 6), (7, 2 ** 24), (2, 4194304)]:
        assert L.csa2_topk_pool_workspace(nq, n, 16384) <= cap, (nq, n)
    for nq, n in [(9, 10 ** 6), (8, 2 ** 24)]:
        assert L.csa2_topk_pool_workspace(nq, n, 16384) > cap, (nq, n)
