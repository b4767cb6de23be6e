"""The FP4 cache write from bf16 rows (csa2_fp4_quantize_bf16) against the
oracle's quantiser on the same values: bit-exact codes and scales."""
import numpy as np
import pytest
import torch

import oracle as O
from kv_cache_decode_csa2_b200 import csa2 as B

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def test_fp4_quantize_from_bf16_bitexact():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1024, 512)).astype(np.float32)
    x[::7] *= 8
    x[1, :32] = 0
    x[2, :32] *= 1e-5
    x[3, :32] *= 5000
    x[4, :32] = np.array([6, .25, .75, 1.25, 1.75, 2.5, 3.5, 5, -.25, -.75, -1.25, -1.75, -2.5, -3.5, -5,
                          0, -0.0, 6, -6, 7, 1, 2, 3, 4, .5, 1.5, -1, -2, -3, -4, -.5, -1.5], np.float32)
    xb = torch.from_numpy(x).to(DEV).to(torch.bfloat16)
    vals = xb.float().cpu().numpy()                  # the exact bf16 values the kernel reads
    codes_ref, scales_ref = O.fp4_quantize(vals)
    codes = torch.zeros((1024, 256), dtype=torch.uint8, device=DEV)
    scales = torch.zeros((1024, 16), dtype=torch.uint8, device=DEV)
    B.check_status(B.csa2_fp4_quantize(xb, codes, scales))
    assert np.array_equal(scales.cpu().numpy(), scales_ref)
    assert np.array_equal(codes.cpu().numpy(), codes_ref)
    # the same values as fp32 give the same bytes
    c2 = torch.zeros_like(codes)
    s2 = torch.zeros_like(scales)
    B.check_status(B.csa2_fp4_quantize(torch.from_numpy(vals).to(DEV), c2, s2))
    assert torch.equal(c2, codes) and torch.equal(s2, scales)
