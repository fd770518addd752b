"""w3a16_gemm_noalloc (fixed library scratch, no allocation) against w3a16_gemm.

Kept in its own file, named to run after the other GPU tests.  Two calls in a
row on one stream must each give exactly the bits of the allocating entry point,
including shapes whose tiles are shared between CTAs (partial sums in scratch).
"""
import numpy as np
import pytest
import torch

from gpu_helpers import device_problem, from_dev_bf16
from w3a16_gemv_b200 import build, w3_check_device_error, w3_pack, w3a16_gemm, w3a16_gemm_noalloc
from w3a16_gemv_b200.inputs import make_problem

pytestmark = pytest.mark.gpu

CASES = [
    (8, 28672, 8192),   # gate_proj shape, tiles split over 148 CTAs
    (16, 1024, 8192),   # k/v_proj shape: every tile shared by several CTAs
    (5, 300, 1152),     # ragged N, K of 9 groups
    (1, 4096, 4096),    # a shape that needs no scratch (falls through to the decode kernels)
    (32, 28672, 8192),  # the 32-wide decode: twice the partial-sum scratch per CTA
    (20, 1024, 8192),
]


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("case", CASES, ids=[f"M{m}_N{n}_K{k}" for m, n, k in CASES])
def test_noalloc_matches_allocating_entry_twice(case):
    M, N, K = case
    p = make_problem(M, N, K, "uniform8", "lognormal", "normal", seed=21)
    x, codes, scales = device_problem(p)
    packed = w3_pack(codes)
    ref = from_dev_bf16(w3a16_gemm(x, packed, scales))
    y1 = from_dev_bf16(w3a16_gemm_noalloc(x, packed, scales))
    y2 = from_dev_bf16(w3a16_gemm_noalloc(x, packed, scales))
    w3_check_device_error()
    assert np.array_equal(y1, ref)
    assert np.array_equal(y2, ref)
