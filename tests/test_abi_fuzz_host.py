"""Seeded random arguments through the C ABI's argument checks, on a machine
without a GPU: every call that has work to do must come back with a
documented error code (an argument, shape or workspace error, or
CSA2_ERR_CUDA once the checks pass and the first CUDA call fails), and none
may crash the process.  Pointers are NULL or
fake aligned or misaligned addresses, so the test runs only without a GPU,
where none of them can reach a kernel."""
import ctypes
import random

import pytest
import torch

import kv_cache_decode_csa2_b200 as K
from kv_cache_decode_csa2_b200 import csa2 as B

pytestmark = pytest.mark.skipif(torch.cuda.is_available(), reason="fake device pointers: only without a GPU")

CODES = {1, 2, 3, 4}


def _ptr(r):
    return r.choice([None, 1 << 20, (1 << 20) + 4, (1 << 20) + 8])


def _int(r, hi=1 << 20):
    return r.choice([-1, 0, 1, 2, 7, 16, 63, 64, 65, 127, 128, 512, 4096, 4097, 16384, 65536, 65537, hi])


def _rows(r):
    v = B.csa2_rows()
    v.base = _ptr(r)
    v.row_bytes = r.choice([0, 8, 16, 32, 64, 68, 128, 256, 1024])
    v.n_rows = r.choice([0, 1, 100, 1 << 20, 1 << 31])
    if r.random() < 0.3:
        v.page_table, v.page_rows, v.max_pages = _ptr(r), r.choice([0, 32, 64, 128]), r.choice([0, 1, 8])
    v.seq_rows = r.choice([-1, 0, 64, 4096])
    return v


def test_random_arguments_return_documented_codes():
    L = K.lib()
    rng = random.Random(7)
    for _ in range(400):
        keys, codes, scales, local = _rows(rng), _rows(rng), _rows(rng), _rows(rng)
        calls = [
            lambda: L.csa2_index_full(_ptr(rng), _ptr(rng), ctypes.byref(keys), _ptr(rng), _ptr(rng), _int(rng),
                                      _int(rng), rng.choice([32, 64, 128]), _int(rng), _ptr(rng), _int(rng),
                                      _int(rng), _ptr(rng), _ptr(rng), _int(rng), _ptr(rng), _ptr(rng), _ptr(rng),
                                      _int(rng, 1 << 40), _ptr(rng), None),
            lambda: L.csa2_topk_pool(_ptr(rng), _int(rng), _ptr(rng), _ptr(rng), _int(rng), _int(rng), _int(rng),
                                     _ptr(rng), _ptr(rng), _ptr(rng), _int(rng, 1 << 40), _ptr(rng), None),
            lambda: L.csa2_reindex(_ptr(rng), _ptr(rng), ctypes.byref(keys), _ptr(rng), _ptr(rng), _ptr(rng),
                                   _int(rng), _int(rng), rng.choice([64, 128]), _int(rng), _int(rng), _ptr(rng),
                                   _ptr(rng), _ptr(rng), _ptr(rng), _int(rng, 1 << 40), _ptr(rng), None),
            lambda: L.csa2_sparse_attn_fp4(_ptr(rng), ctypes.byref(codes), ctypes.byref(scales), _ptr(rng),
                                           _ptr(rng), _ptr(rng), _ptr(rng), _int(rng), rng.choice([8, 12, 64]),
                                           rng.choice([128, 256, 512]), _int(rng), _int(rng), 0.0, _ptr(rng),
                                           _ptr(rng), _ptr(rng), _int(rng, 1 << 40), _ptr(rng), None),
            lambda: L.csa2_sparse_attn_fp4_local(_ptr(rng), ctypes.byref(codes), ctypes.byref(scales),
                                                 ctypes.byref(local), _ptr(rng), _ptr(rng), _ptr(rng), _ptr(rng),
                                                 _int(rng), 64, 512, _int(rng), _int(rng), 0.0, _ptr(rng), None,
                                                 _ptr(rng), _int(rng, 1 << 40), _ptr(rng), None),
            lambda: L.csa2_fp4_quantize(_ptr(rng), _int(rng) or 1, rng.choice([16, 32, 512]), _int(rng),
                                        _ptr(rng), _ptr(rng), _int(rng), _ptr(rng), _int(rng), _int(rng), _ptr(rng),
                                        None),
            lambda: L.csa2_fp4_quantize_bf16(_ptr(rng), _int(rng) or 1, rng.choice([16, 32, 512]), _int(rng),
                                             _ptr(rng), _ptr(rng), _int(rng), _ptr(rng), _int(rng), _int(rng),
                                             _ptr(rng), None),
            lambda: L.csa2_selftest_wait(rng.choice([-1, 0, 1, 2]), rng.choice([0, 1000, 10 ** 11]), _ptr(rng),
                                         _ptr(rng), None),
        ]
        for call in calls:
            assert call() in CODES
    # zero rows is the one call here with nothing to launch: it succeeds without a device
    assert L.csa2_fp4_quantize(1 << 20, 0, 512, 512, None, 1 << 20, 256, 1 << 20, 16, 16, 1 << 20, None) == 0


def test_random_plans_return_documented_codes():
    L = K.lib()
    rng = random.Random(11)
    for _ in range(300):
        n = rng.choice([0, 1, 2, 3, 8, 16, 17])
        size = max(n, 1)
        modes = (ctypes.c_int32 * size)(*[rng.choice([-1, 0, 0, 1, 2, 3]) for _ in range(size)])
        layers = (B.csa2_layer * size)()
        for ly in layers:
            ly.q, ly.w, ly.q_attn, ly.out = _ptr(rng), _ptr(rng), _ptr(rng), _ptr(rng)
            ly.keys, ly.codes, ly.scales = _rows(rng), _rows(rng), _rows(rng)
            if rng.random() < 0.3:
                ly.local_kv = _rows(rng)
        s = B.csa2_plan_shape(nq=_int(rng), H=_int(rng), D_idx=rng.choice([64, 128, 96]), Hq=rng.choice([8, 64, 12]),
                              D=rng.choice([128, 512, 256]), P=_int(rng), K=_int(rng), window=_int(rng),
                              max_ctx=_int(rng), softmax_scale=0.0, seq_of_query=_ptr(rng), query_pos=_ptr(rng),
                              group_queries=rng.choice([0, 1]))
        args = (modes if rng.random() < 0.95 else None, n, layers if rng.random() < 0.95 else None,
                ctypes.byref(s) if rng.random() < 0.95 else None)
        assert L.csa2_layer_plan(*args, _ptr(rng), _int(rng, 1 << 40), _ptr(rng), None) in CODES
        assert L.csa2_layer_plan_workspace(args[0], n, args[3]) >= 0
