"""The give-up path of the bounded waits, on the GPU: a wait that nothing
satisfies records CSA2_ERR_TIMEOUT after its limit and its kernel returns;
the device stays usable for the next call."""
import time

import numpy as np
import pytest
import torch

from kv_cache_decode_csa2_b200 import csa2 as B

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("kind", [0, 1], ids=["grid_barrier", "mbarrier"])
def test_wait_gives_up_and_the_device_stays_usable(kind):
    status = B.new_status(DEV)
    counter = torch.zeros(1, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    t0 = time.time()
    B.csa2_selftest_wait(kind, 5_000_000, counter=counter, status=status)   # 5 ms
    torch.cuda.synchronize()
    took = time.time() - t0
    assert int(status.item()) == 7                    # CSA2_ERR_TIMEOUT
    assert took < 2.0
    if kind == 0:
        assert int(counter.item()) == 1               # the one CTA arrived, nobody else
    # the next call works: an exact top-k of 5000 candidates
    rng = np.random.default_rng(0)
    s = torch.from_numpy(rng.integers(-1000, 1000, size=(1, 5000)).astype(np.int32)).to(DEV)
    out = torch.empty((1, 64), dtype=torch.int32, device=DEV)
    cnt = torch.empty((1,), dtype=torch.int32, device=DEV)
    st2 = B.csa2_topk_pool(s, 64, out, out_cnt=cnt)
    B.check_status(st2)
    keys = [(-int(v), j) for j, v in enumerate(s[0].cpu().numpy())]
    want = sorted(j for _, j in sorted(keys)[:64])
    assert int(cnt.item()) == 64 and out[0].cpu().numpy().tolist() == want
