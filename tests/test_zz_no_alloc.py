"""csa2_topk_pool_noalloc against csa2_topk_pool, through the C ABI.

The no-allocation entry point is for callers that cannot allocate device
memory.  Examples are code running inside a host framework that only passes
it input and output buffers, and serving loops that reserved all device memory
at start-up.  Its scratch is one fixed array inside the library.  This test
checks that two calls in a row give exactly the same pool as the workspace
entry point (indices are integers, so the match must be exact), and that
the second call is not disturbed by what the first left in the shared
array.  It runs last so that a failure here never hides the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from kv_cache_decode_csa2_b200 import csa2 as B

pytestmark = pytest.mark.gpu


def _call_noalloc(L, scores, n_valid, k, out, cnt, status):
    nq, ld = scores.shape
    return L.csa2_topk_pool_noalloc(scores.data_ptr(), ld, n_valid.data_ptr(), None, nq, ld, k, out.data_ptr(),
                                    cnt.data_ptr(), status.data_ptr(), torch.cuda.current_stream().cuda_stream)


def _call_ws(L, scores, n_valid, k, out, cnt, status):
    nq, ld = scores.shape
    need = L.csa2_topk_pool_workspace(nq, ld, k)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
    return L.csa2_topk_pool(scores.data_ptr(), ld, n_valid.data_ptr(), None, nq, ld, k, out.data_ptr(),
                            cnt.data_ptr(), ws.data_ptr(), ws.numel(), status.data_ptr(),
                            torch.cuda.current_stream().cuda_stream)


# Sizes: co-resident select CTAs (300,000 candidates), the one-CTA path
# (16,384), and rows too long for the co-resident select (4,194,304: the
# multi-pass path, whose chunk counts and candidate lists take most of the
# fixed array).
@pytest.mark.parametrize("nq,n,k,spread", [(3, 300000, 16384, 25000), (3, 16384, 512, 40),
                                           (2, 4194304, 16384, 10 ** 6)])
def test_noalloc_matches_workspace_entry_point_twice(nq, n, k, spread):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    L = B.lib()
    rng = np.random.default_rng(n)
    for call in range(2):          # two calls in a row, different data each time
        s = rng.integers(-spread, spread + 1, size=(nq, n)).astype(np.int32) + 10 ** 5 * call
        nv = np.array([n, n // 3, n - 7][:nq], dtype=np.int32)
        scores = torch.from_numpy(s).cuda()
        n_valid = torch.from_numpy(nv).cuda()
        outs = []
        for fn in (_call_noalloc, _call_ws):
            out = torch.full((nq, k), -5, dtype=torch.int32, device="cuda")
            cnt = torch.full((nq,), -5, dtype=torch.int32, device="cuda")
            status = torch.zeros(1, dtype=torch.int32, device="cuda")
            assert fn(L, scores, n_valid, k, out, cnt, status) == 0
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            outs.append((out.cpu().numpy(), cnt.cpu().numpy()))
        assert np.array_equal(outs[0][1], outs[1][1])
        assert np.array_equal(outs[0][0], outs[1][0])


def test_noalloc_rejects_sizes_beyond_its_array():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    L = B.lib()
    n, nq, k = 10 ** 6, 20, 512
    assert L.csa2_topk_pool_workspace(nq, n, k) > (4 << 20)
    scores = torch.zeros((nq, 16), dtype=torch.int32, device="cuda")   # never read: rejected first
    out = torch.empty((nq, k), dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = L.csa2_topk_pool_noalloc(scores.data_ptr(), n, None, None, nq, n, k, out.data_ptr(), None,
                                  status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 3          # CSA2_ERR_WORKSPACE, nothing launched
