"""The kernel-native block order on the GPU, against the CPU oracle.

* w3_pack_native, w3_native_from_packed and w3_packed_from_native are bit-exact
  with the oracle's permutation (padded rows zero).
* w3a16_gemm_native is within the product bound of the fp64 oracle, on ragged
  shapes that reach both of its kernels (the stream-K decode for M <= 4 on many
  rows, the split decode otherwise), on x = e_k position probes, and on the
  full-size gate_proj decode step (every output).
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_within_bound, bound, device_problem, from_dev_bf16
from w3a16_gemv_b200 import (W3Error, build, w3_check_device_error, w3_native_from_packed, w3_pack, w3_pack_native,
                             w3_packed_from_native, w3a16_gemm, w3a16_gemm_native, w3a16_gemm_route)
from w3a16_gemv_b200.inputs import make_problem, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("N,K", [(32, 128), (40, 256), (300, 1152), (4800, 384), (28672, 8192)])
def test_native_order_bit_exact(orc, N, K):
    p = make_problem(1, N, K, seed=31)
    codes = torch.from_numpy(p.codes).cuda()
    ref = orc.native_from_packed(orc.pack(p.codes), K)
    nat = w3_pack_native(codes)
    assert np.array_equal(nat.cpu().numpy().view(np.uint32), ref)
    packed = w3_pack(codes)
    nat2 = w3_native_from_packed(packed, K)
    assert np.array_equal(nat2.cpu().numpy().view(np.uint32), ref)
    back = w3_packed_from_native(nat2, N, K)
    assert np.array_equal(back.cpu().numpy(), packed.cpu().numpy())


# (M, N, K): the stream-K decode (M <= 4, one 32-row block per SM or more) and the split decode
NATIVE_SHAPES = [
    (1, 4800, 384), (3, 5000, 1152), (4, 6000, 640), (1, 300, 1024), (2, 64, 128), (5, 300, 384),
    (8, 1000, 2048), (12, 77, 768), (16, 512, 1152), (16, 4800, 256), (1, 40, 28672),
]


@pytest.mark.parametrize("case", NATIVE_SHAPES, ids=[f"M{m}_N{n}_K{k}" for m, n, k in NATIVE_SHAPES])
def test_native_product_parity(orc, case):
    M, N, K = case
    p = make_problem(M, N, K, "uniform8", "lognormal", "normal_outliers", seed=32)
    x, codes, scales = device_problem(p)
    nat = w3_pack_native(codes)
    y = from_dev_bf16(w3a16_gemm_native(x, nat, scales, N))
    w3_check_device_error()
    ref_packed = orc.pack(p.codes)
    ref = orc.gemm_f64(p.x_bf16, ref_packed, p.scales_bf16, threads=0)
    assert_within_bound(y, ref, bound(p.x_bf16, orc.weight_row_norms(ref_packed, p.scales_bf16, K), K), str(case))
    # where the row-major call runs the same kernel (with the same plan), the results are bit-identical
    if w3a16_gemm_route(M, N, K) in ("decode_sk", "decode_split"):
        y_rm = from_dev_bf16(w3a16_gemm(x, w3_pack(codes), scales))
        assert np.array_equal(y, y_rm), "native and row-major decode differ"


@pytest.mark.parametrize("M,N,K", [(1, 4800, 256), (4, 4800, 256), (16, 300, 384)])
def test_native_position_probe(orc, M, N, K):
    p = make_problem(M, N, K, seed=33)
    _, codes, scales = device_problem(p)
    nat = w3_pack_native(codes)
    w = orc.dequant_f32(orc.pack(p.codes), p.scales_bf16, K)
    for k0 in range(0, K, M):
        rows = min(M, K - k0)
        eye = np.zeros((M, K), dtype=np.float32)
        eye[np.arange(rows), k0 + np.arange(rows)] = 1.0
        x = torch.from_numpy(eye).to(torch.bfloat16).cuda()
        y = oracle.bf16_to_f64(from_dev_bf16(w3a16_gemm_native(x, nat, scales, N)))
        want = w[:, k0:k0 + rows].T.astype(np.float64)
        assert np.all(np.abs(y[:rows] - want) <= 2.0 ** -8 * np.abs(want) + 1e-30), k0
    w3_check_device_error()


@pytest.mark.parametrize("name", ["gate_28672x8192_m1", "gate_28672x8192_m4", "gate_28672x8192_m16"])
def test_native_full_size_full_parity(orc, name):
    wl = workloads()[name]
    p = wl.problem()
    x, codes, scales = device_problem(p)
    y = from_dev_bf16(w3a16_gemm_native(x, w3_pack_native(codes), scales, wl.N))
    w3_check_device_error()
    ref_packed = orc.pack(p.codes)
    ref = orc.gemm_f64(p.x_bf16, ref_packed, p.scales_bf16, threads=0)
    worst = assert_within_bound(y, ref, bound(p.x_bf16, orc.weight_row_norms(ref_packed, p.scales_bf16, wl.K), wl.K),
                                name)
    print(f"{name} native: worst |err|/bound = {worst:.3g}")


def test_native_rejects_unsupported_shapes():
    p = make_problem(17, 64, 128, seed=34)
    x, codes, scales = device_problem(p)
    nat = w3_pack_native(codes)
    with pytest.raises(W3Error, match="UNSUPPORTED"):
        w3a16_gemm_native(x, nat, scales, 64)  # M = 17: prefill batches use the row-major words
