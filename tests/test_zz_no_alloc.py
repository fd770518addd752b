"""w3a16_gemm_noalloc (fixed library scratch, no allocation) against w3a16_gemm.

Kept in its own file, named to run after the other GPU tests.  Two calls in a
row on one stream must each give exactly the bits of the allocating entry point,
including shapes whose tiles are shared between CTAs (partial sums in scratch)
and a batch above 32 rows with K < 256, which runs as 16-row tensor-core passes
on the same fixed scratch.  One case is also checked against the CPU oracle.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_within_bound, bound, device_problem, from_dev_bf16
from w3a16_gemv_b200 import build, w3_check_device_error, w3_pack, w3a16_gemm, w3a16_gemm_noalloc, w3a16_gemm_route
from w3a16_gemv_b200.inputs import make_problem

pytestmark = pytest.mark.gpu

CASES = [
    (8, 28672, 8192),   # gate_proj shape, tiles split over 148 CTAs
    (16, 1024, 8192),   # k/v_proj shape: every tile shared by several CTAs
    (5, 300, 1152),     # ragged N, K of 9 groups
    (1, 4096, 4096),    # a shape that needs no scratch (falls through to the decode kernels)
    (32, 28672, 8192),  # the 32-wide decode: twice the partial-sum scratch per CTA
    (20, 1024, 8192),
    (40, 28672, 128),   # M > 32 with K < 256: 16-row passes of the tensor-core decode on the fixed scratch
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


def test_noalloc_within_the_oracle_bound(orc):
    M, N, K = 24, 1024, 8192  # every row tile shared between CTAs: the partial sums live in the scratch
    assert w3a16_gemm_route(M, N, K) == "decode_tc32"
    p = make_problem(M, N, K, "gsq_5level", "absnormal", "normal_outliers", seed=22)
    x, codes, scales = device_problem(p)
    packed = w3_pack(codes)
    y = from_dev_bf16(w3a16_gemm_noalloc(x, packed, scales))
    w3_check_device_error()
    ref_packed = orc.pack(p.codes)
    ref = orc.gemm_f64(p.x_bf16, ref_packed, p.scales_bf16, threads=0)
    assert_within_bound(y, ref, bound(p.x_bf16, orc.weight_row_norms(ref_packed, p.scales_bf16, K), K), "noalloc")
