"""GPU parity of w3_repack_ct4 (4-bit container -> exact-width uint3) against the CPU oracle.

The container layout is the reading written in include/w3a16.h and the oracle
(eight LSB-first 4-bit fields per int32, level + 8); the checks are bit-exact:
the re-packed words, the clamp of levels outside -4..3 and its count, and the
product of a re-packed weight.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import device_problem, from_dev_bf16
from w3a16_gemv_b200 import build, w3_check_device_error, w3_pack, w3_repack_ct4, w3a16_gemm
from w3a16_gemv_b200.inputs import make_problem

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available()


def _dev_u32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).cuda()


SHAPES = [(1, 128), (3, 384), (17, 1152), (1000, 4096), (4096, 8192)]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"N{n}_K{k}" for n, k in SHAPES])
def test_repack_in_range_matches_oracle(orc, shape):
    N, K = shape
    rng = np.random.Generator(np.random.PCG64(31 + N))
    codes = rng.integers(0, 8, size=(N, K), dtype=np.uint8)
    ct4 = orc.pack_ct4(codes)
    packed, count = w3_repack_ct4(_dev_u32(ct4), K, count_out_of_range=True)
    w3_check_device_error()
    assert int(count.item()) == 0
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), orc.pack(codes))


def test_repack_clamps_and_counts_like_the_oracle(orc):
    N, K = 77, 1280
    rng = np.random.Generator(np.random.PCG64(32))
    ct4 = rng.integers(0, 2**32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)  # every field 0..15
    want, want_count = orc.repack_ct4(ct4, K)
    assert want_count > 0
    packed, count = w3_repack_ct4(_dev_u32(ct4), K, count_out_of_range=True)
    w3_check_device_error()
    assert int(count.item()) == want_count
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), want)
    # without a counter the words are the same
    again = w3_repack_ct4(_dev_u32(ct4), K)
    assert np.array_equal(again.cpu().numpy().view(np.uint32), want)


def test_repacked_weight_gives_the_same_product(orc):
    p = make_problem(4, 512, 2048, "gsq_5level", "absnormal", "normal", seed=33)
    x, codes, scales = device_problem(p)
    direct = w3_pack(codes)
    repacked = w3_repack_ct4(_dev_u32(orc.pack_ct4(p.codes)), 2048)
    assert torch.equal(direct, repacked)
    assert np.array_equal(from_dev_bf16(w3a16_gemm(x, repacked, scales)), from_dev_bf16(w3a16_gemm(x, direct, scales)))
