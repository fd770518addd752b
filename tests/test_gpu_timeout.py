"""Failure detection: a bounded device-side wait that runs out is reported, not hung.

Every wait in the library's kernels (on an mbarrier: a TMA copy, a tensor-core
commit, a neighbour warp) gives up after a fixed number of SM cycles, records a
timeout bit in a per-device flag and lets the kernel return; the host reads it
with w3_check_device_error.  Here a test variant of the library (built with a
test-only kernel and a wait limit of about a millisecond) waits on an mbarrier
phase that nothing ever completes.  Nothing faults and nothing hangs: the wait
runs out, the flag is reported once and cleared, and the context stays usable.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

from gpu_helpers import assert_within_bound, bound, device_problem, from_dev_bf16
from w3a16_gemv_b200 import build, w3_pack
from w3a16_gemv_b200.inputs import make_problem

pytestmark = pytest.mark.gpu

W3_OK, W3_ERR_TIMEOUT = 0, 6
VARIANT = os.path.join(os.path.dirname(build.LIB), "libw3a16_testhooks.so")


@pytest.fixture(scope="module")
def hooks():
    path = build.build(out=VARIANT, defines=["W3_TEST_HOOKS=1", "W3_WAIT_LIMIT_CYCLES=2000000ll"])
    lib = ctypes.CDLL(path)
    lib.w3_test_wait_timeout.argtypes = [ctypes.c_void_p]
    lib.w3_test_wait_timeout.restype = ctypes.c_int
    lib.w3_check_device_error.argtypes = [ctypes.c_void_p]
    lib.w3_check_device_error.restype = ctypes.c_int
    lib.w3a16_gemm.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64] * 3 + [ctypes.c_void_p]
    lib.w3a16_gemm.restype = ctypes.c_int
    return lib


def test_wait_that_runs_out_is_reported_once(hooks):
    stream = torch.cuda.current_stream().cuda_stream
    assert hooks.w3_check_device_error(stream) == W3_OK  # nothing pending
    assert hooks.w3_test_wait_timeout(stream) == W3_OK  # the launch itself succeeds
    assert hooks.w3_check_device_error(stream) == W3_ERR_TIMEOUT
    assert hooks.w3_check_device_error(stream) == W3_OK  # reported once, then cleared


def test_context_usable_after_a_timeout(hooks, orc):
    stream = torch.cuda.current_stream().cuda_stream
    assert hooks.w3_test_wait_timeout(stream) == W3_OK
    assert hooks.w3_check_device_error(stream) == W3_ERR_TIMEOUT
    M, N, K = 4, 300, 1024
    p = make_problem(M, N, K, seed=31)
    x, codes, scales = device_problem(p)
    packed = w3_pack(codes)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert hooks.w3a16_gemm(x.data_ptr(), packed.data_ptr(), scales.data_ptr(), y.data_ptr(), M, N, K, stream) == W3_OK
    assert hooks.w3_check_device_error(stream) == W3_OK
    ref_packed = orc.pack(p.codes)
    ref = orc.gemm_f64(p.x_bf16, ref_packed, p.scales_bf16)
    assert_within_bound(from_dev_bf16(y), ref, bound(p.x_bf16, orc.weight_row_norms(ref_packed, p.scales_bf16, K), K),
                        "after a timeout")
