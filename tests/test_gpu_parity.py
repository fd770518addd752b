"""GPU parity: the CUDA library, called through its C ABI, against the CPU oracle.

* pack / unpack / fp32 dequant: bit-exact.
* y = x W^T: every checked element within |y - y_ref| <= 1e-2*||x_m||*||w_n||/sqrt(K) + 1e-3
  of the fp64 oracle.
Small shapes are checked in full (several tiles, ragged edges, every decode
batch size).  The full-size decode workloads (every M <= 16 configuration the
benchmark times, and the mid-batch ones) are checked in full against the oracle;
the M = 2048, 1024 and 512 prefill workloads on 64 whole rows of y plus 4096
sampled entries.
Position probes (x = e_k) go through every kernel route, each asserted with
w3a16_gemm_route, so that a bit-order or placement mistake in any one kernel
shows up as a wrong weight in a known place.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_within_bound, bound, device_problem, from_dev_bf16
from w3a16_gemv_b200 import (build, w3_check_device_error, w3_dequant_f32, w3_pack, w3_unpack, w3a16_gemm,
                             w3a16_gemm_route)
from w3a16_gemv_b200.inputs import make_problem, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available()


# (M, N, K, codes, scales, x): odd and ragged sizes, one group, odd group counts,
# every M the decode path handles, and batches above 16.
SMALL = [
    (1, 1, 128, "uniform8", "lognormal", "normal"),
    (1, 17, 128, "uniform8", "lognormal", "normal"),
    (2, 64, 384, "gsq_uniform", "absnormal", "normal"),
    (3, 100, 1152, "uniform8", "lognormal", "normal_outliers"),
    (4, 250, 640, "gsq_5level", "absnormal", "normal"),
    (5, 64, 4096, "uniform8", "lognormal", "normal"),
    (7, 129, 256, "uniform8", "lognormal", "normal"),
    (8, 333, 2048, "uniform8", "absnormal", "normal_outliers"),
    (9, 77, 768, "gsq_uniform", "lognormal", "normal"),
    (12, 300, 1024, "uniform8", "lognormal", "normal"),
    (16, 129, 256, "uniform8", "lognormal", "normal"),
    (16, 1000, 8192, "uniform8", "lognormal", "normal"),
    (6, 200, 1152, "gsq_uniform", "lognormal", "normal"),         # K split 5 + 4 groups
    (10, 256, 4224, "uniform8", "absnormal", "normal_outliers"),  # K split 8 ways, last rank idle
    (13, 28672, 256, "uniform8", "lognormal", "normal"),          # many row tiles, two groups
    (1, 2000, 128, "uniform8", "lognormal", "normal"),
    (1, 64, 28672, "gsq_5level", "absnormal", "normal_outliers"),
    # many 32-row blocks: ragged last block, odd group counts, blocks split between warps and
    # K split over thread-block clusters
    (1, 4800, 384, "uniform8", "lognormal", "normal"),
    (3, 5000, 1152, "gsq_5level", "absnormal", "normal_outliers"),
    (4, 6000, 640, "uniform8", "lognormal", "normal"),
    (2, 4736, 3968, "gsq_uniform", "lognormal", "normal"),
    # a single group (K = 128) on every path: the split decode, the 32-wide tcgen05 decode, 16-row
    # passes above 32
    (8, 512, 128, "uniform8", "lognormal", "normal"),
    (24, 512, 128, "uniform8", "lognormal", "normal"),
    (40, 300, 128, "gsq_5level", "absnormal", "normal"),
    (17, 50, 512, "uniform8", "lognormal", "normal"),
    (40, 96, 1280, "uniform8", "lognormal", "normal"),
    (256, 256, 256, "uniform8", "lognormal", "normal"),
    (300, 1000, 1024, "gsq_5level", "absnormal", "normal_outliers"),
    (513, 200, 384, "uniform8", "lognormal", "normal"),
    (32, 28672, 1024, "uniform8", "lognormal", "normal"),   # 128 tiles at once: packed-word buffer reuse
    (32, 448, 8192, "gsq_5level", "absnormal", "normal"),   # 32 packed-word copies per tile
    # the 32-wide tensor-core decode (17 <= M <= 32, N >= 256)
    (17, 256, 1152, "uniform8", "lognormal", "normal"),           # one row tile, K split over CTAs
    (20, 1000, 4224, "gsq_5level", "absnormal", "normal_outliers"),
    (24, 28672, 256, "uniform8", "lognormal", "normal"),          # many row tiles, two groups
    (31, 300, 8192, "uniform8", "lognormal", "normal"),
    (200, 1000, 1024, "gsq_5level", "absnormal", "normal_outliers"),
    (129, 600, 512, "uniform8", "lognormal", "normal"),
]

# (route, M, N, K, codes, scales, x): shapes the dispatch sends to a given kernel (asserted with
# w3a16_gemm_route), checked in full.
ROUTED = [
    # 2..4 batch rows over a K too tall for the stream-K decode's prepared x: the split decode
    ("decode_split", 4, 4800, 12416, "uniform8", "lognormal", "normal"),
    ("decode_split", 2, 4800, 24704, "gsq_5level", "absnormal", "normal_outliers"),
    # the shared-memory prefill: one 128-row MMA tile of x; a ragged second one; a ragged third
    # 256-row batch tile; four batch tiles; ragged last W tiles (N = 20001)
    ("prefill", 33, 20001, 256, "uniform8", "lognormal", "normal"),
    ("prefill", 200, 20001, 256, "gsq_5level", "absnormal", "normal_outliers"),
    ("prefill", 129, 20001, 512, "uniform8", "lognormal", "normal"),
    ("prefill", 600, 20480, 256, "uniform8", "absnormal", "normal"),
    ("prefill", 1024, 8192, 256, "gsq_uniform", "lognormal", "normal"),
    # the tensor-memory prefill below 256 rows of x (UMMA N = M rounded up to 16) and above
    ("prefill_ab", 33, 1000, 1024, "uniform8", "lognormal", "normal"),
    ("prefill_ab", 64, 8192, 512, "gsq_5level", "absnormal", "normal_outliers"),
    ("prefill_ab", 128, 4096, 1024, "uniform8", "lognormal", "normal"),
    ("prefill_ab", 255, 600, 512, "uniform8", "lognormal", "normal_outliers"),
    ("prefill_ab", 200, 1000, 1024, "gsq_uniform", "absnormal", "normal"),
    ("prefill_ab", 300, 1000, 1024, "uniform8", "lognormal", "normal"),
    ("prefill_ab", 1100, 8192, 256, "uniform8", "lognormal", "normal"),
]


def _id(c):
    return f"M{c[0]}_N{c[1]}_K{c[2]}_{c[3]}"


@pytest.mark.parametrize("case", SMALL, ids=[_id(c) for c in SMALL])
def test_small_shapes_full_parity(orc, case):
    _full_parity(orc, case)


@pytest.mark.parametrize("case", ROUTED, ids=[f"{c[0]}_{_id(c[1:])}" for c in ROUTED])
def test_routed_shapes_full_parity(orc, case):
    assert w3a16_gemm_route(*case[1:4]) == case[0]
    _full_parity(orc, case[1:])


def _full_parity(orc, case):
    M, N, K, cd, sd, xd = case
    p = make_problem(M, N, K, cd, sd, xd, seed=11)
    x, codes, scales = device_problem(p)
    packed = w3_pack(codes)
    ref_packed = orc.pack(p.codes)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), ref_packed)
    assert np.array_equal(w3_unpack(packed, K).cpu().numpy(), p.codes)
    w = w3_dequant_f32(packed, scales, K).cpu().numpy()
    assert np.array_equal(w.view(np.uint32), orc.dequant_f32(ref_packed, p.scales_bf16, K).view(np.uint32))
    y = w3a16_gemm(x, packed, scales)
    w3_check_device_error()
    ref = orc.gemm_f64(p.x_bf16, ref_packed, p.scales_bf16, threads=0)
    tol = bound(p.x_bf16, orc.weight_row_norms(ref_packed, p.scales_bf16, K), K)
    assert_within_bound(from_dev_bf16(y), ref, tol, _id(case))


def test_all_levels_exact_dequant_and_gsq_levels(orc):
    # every code value at every block position, and the GSQ levels -2..2 for codes 2..6
    N, K = 8, 256
    codes = (np.arange(N * K).reshape(N, K) % 8).astype(np.uint8)
    codes[1] = np.arange(K) // 32 % 8
    p = make_problem(1, N, K, "uniform8", "lognormal", "normal", seed=12)
    _, _, scales = device_problem(p)
    packed = w3_pack(torch.from_numpy(codes).cuda())
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), orc.pack(codes))
    w = w3_dequant_f32(packed, scales, K).cpu().numpy()
    s = oracle.bf16_to_f64(p.scales_bf16)
    want = (codes.astype(np.float64) - 4.0) * np.repeat(s, 128, axis=1)
    assert np.array_equal(w.astype(np.float64), want)


def test_deterministic_repeated_calls():
    p = make_problem(4, 3000, 4096, seed=13)
    x, codes, scales = device_problem(p)
    packed = w3_pack(codes)
    ys = [from_dev_bf16(w3a16_gemm(x, packed, scales)) for _ in range(3)]
    assert all(np.array_equal(ys[0], y) for y in ys[1:])


def test_batch_rows_match_single_row_calls(orc):
    """Row m of an M=16 call against the M=1 call on that row: both within the bound;
    bit-identity is reported (not required: the split of K may differ with M)."""
    p = make_problem(16, 512, 2048, seed=14)
    x, codes, scales = device_problem(p)
    packed = w3_pack(codes)
    yb = from_dev_bf16(w3a16_gemm(x, packed, scales))
    ref = orc.gemm_f64(p.x_bf16, orc.pack(p.codes), p.scales_bf16)
    tol = bound(p.x_bf16, orc.weight_row_norms(orc.pack(p.codes), p.scales_bf16, 2048), 2048)
    same = 0
    for m in range(16):
        y1 = from_dev_bf16(w3a16_gemm(x[m:m + 1].contiguous(), packed, scales))
        assert_within_bound(y1, ref[m:m + 1], tol[m:m + 1], f"row {m}")
        same += int(np.array_equal(y1[0], yb[m]))
    print(f"batch-invariance: {same}/16 rows bit-identical between M=1 and M=16")


def _probe(orc, M, N, K, seed):
    """x = e_k in every batch row (row i picks column k0 + i): y[i, n] must be the dequantized
    weight W[n, k0 + i] rounded once to bf16, for every n and every k."""
    p = make_problem(M, N, K, seed=seed)
    _, codes, scales = device_problem(p)
    packed = w3_pack(codes)
    w = orc.dequant_f32(orc.pack(p.codes), p.scales_bf16, K)
    for k0 in range(0, K, M):
        rows = min(M, K - k0)
        eye = np.zeros((M, K), dtype=np.float32)
        eye[np.arange(rows), k0 + np.arange(rows)] = 1.0
        x = torch.from_numpy(eye).to(torch.bfloat16).cuda()
        y = oracle.bf16_to_f64(from_dev_bf16(w3a16_gemm(x, packed, scales)))
        want = w[:, k0:k0 + rows].T.astype(np.float64)
        got = y[:rows]
        assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 1e-30), (M, N, K, k0)
        assert np.all(y[rows:] == 0.0), (M, N, K, k0)  # rows of x that are zero give zero
    w3_check_device_error()


# (route, M, N, K): one probe shape per kernel route; the route is asserted first
PROBES = [
    ("decode_sk", 1, 4800, 256),
    ("decode_sk", 4, 4800, 384),
    ("decode_sk", 1, 4768, 1152),   # 149 blocks over 28 CTAs (5 or 6 each), split between warps
    ("decode", 1, 20, 512),
    ("decode_split", 1, 300, 256),
    ("decode_split", 4, 1024, 1152),
    ("decode", 16, 20, 256),
    ("decode_split", 5, 300, 384),
    ("decode_split", 8, 1000, 256),
    ("decode_split", 12, 64, 1152),
    ("decode_split", 16, 512, 384),
    ("decode_split", 16, 40, 128),
    ("decode_tc32", 32, 300, 512),
    ("prefill", 64, 20001, 256),
    ("prefill", 300, 20480, 256),
    ("prefill_ab", 33, 1000, 256),
    ("prefill_ab", 256, 1024, 1024),
    ("passes", 40, 300, 128),
]


@pytest.mark.parametrize("route,M,N,K", PROBES, ids=[f"{r}_M{m}_N{n}_K{k}" for r, m, n, k in PROBES])
def test_position_probe(orc, route, M, N, K):
    assert w3a16_gemm_route(M, N, K) == route
    _probe(orc, M, N, K, seed=15)


def test_row_concatenated_weights_are_one_weight(orc):
    """q, k, v weights concatenated along N run as one call: each part of the result is within
    the bound of the oracle of its own weight (the format's rows are independent)."""
    K = 2048
    parts = [make_problem(1, n, K, "uniform8", "lognormal", "normal", seed=40 + i) for i, n in enumerate((768, 256, 256))]
    x, _, _ = device_problem(parts[0])
    packs, scs = [], []
    for p in parts:
        _, codes, scales = device_problem(p)
        packs.append(w3_pack(codes))
        scs.append(scales)
    y = from_dev_bf16(w3a16_gemm(x, torch.cat(packs), torch.cat(scs)))
    w3_check_device_error()
    n0 = 0
    for p in parts:
        ref_packed = orc.pack(p.codes)
        ref = orc.gemm_f64(parts[0].x_bf16, ref_packed, p.scales_bf16)
        tol = bound(parts[0].x_bf16, orc.weight_row_norms(ref_packed, p.scales_bf16, K), K)
        assert_within_bound(y[:, n0:n0 + p.N], ref, tol, f"part N={p.N}")
        n0 += p.N


def _device_run(orc, wl):
    p = wl.problem()
    x, codes, scales = device_problem(p)
    packed = w3_pack(codes)
    ref_packed = orc.pack(p.codes)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), ref_packed), "pack differs from the oracle"
    del codes
    y = from_dev_bf16(w3a16_gemm(x, packed, scales))
    w3_check_device_error()
    return p, ref_packed, y


FULL = [n for n in workloads() if not n.startswith("prefill")]


@pytest.mark.parametrize("name", FULL)
def test_full_size_full_parity(orc, name):
    """Every output of the full-size decode workload against the fp64 oracle (all cores)."""
    wl = workloads()[name]
    p, ref_packed, y = _device_run(orc, wl)
    ref = orc.gemm_f64(p.x_bf16, ref_packed, p.scales_bf16, threads=0)
    tol = bound(p.x_bf16, orc.weight_row_norms(ref_packed, p.scales_bf16, wl.K), wl.K)
    worst = assert_within_bound(y, ref, tol, name)
    print(f"{name} ({w3a16_gemm_route(wl.M, wl.N, wl.K)}): worst |err|/bound = {worst:.3g} over {y.size} outputs")


def _rows_and_entries_check(orc, name, n_rows=64, n_samples=4096, seed=0):
    """64 random whole rows of y (every n) plus 4096 random (m, n) entries against the oracle."""
    wl = workloads()[name]
    p, ref_packed, y = _device_run(orc, wl)
    rng = np.random.Generator(np.random.PCG64(seed))
    rows = np.sort(rng.choice(wl.M, size=n_rows, replace=False))
    rows[-1] = wl.M - 1  # always the last row
    norms = orc.weight_row_norms(ref_packed, p.scales_bf16, wl.K)
    ref_rows = orc.gemm_f64(p.x_bf16[rows], ref_packed, p.scales_bf16, threads=0)
    worst = assert_within_bound(y[rows], ref_rows, bound(p.x_bf16[rows], norms, wl.K), f"{name} rows")
    ms = np.concatenate([rng.integers(0, wl.M, n_samples), [0, wl.M - 1, 0, wl.M - 1]])
    ns = np.concatenate([rng.integers(0, wl.N, n_samples), [0, 0, wl.N - 1, wl.N - 1]])
    ref = orc.gemm_f64_entries(p.x_bf16, ref_packed, p.scales_bf16, ms, ns)
    xf = oracle.bf16_to_f64(p.x_bf16[ms])
    tol = 1e-2 * np.sqrt(np.sum(xf * xf, axis=1)) * norms[ns] / np.sqrt(wl.K) + 1e-3
    worst = max(worst, assert_within_bound(y[ms, ns][None, :], ref[None, :], tol[None, :], name))
    print(f"{name} ({w3a16_gemm_route(wl.M, wl.N, wl.K)}): worst |err|/bound = {worst:.3g} over {n_rows} rows "
          f"and {ms.size} entries")


def test_prefill_full_size_rows_and_entries(orc):
    _rows_and_entries_check(orc, "prefill_2048x28672x8192")


def test_prefill_tensor_memory_kernel_full_size_rows_and_entries(orc):
    # M = 1024 on gate_proj: the weights-in-tensor-memory prefill kernel is the one launched
    assert w3a16_gemm_route(1024, 28672, 8192) == "prefill_ab"
    _rows_and_entries_check(orc, "prefill_1024x28672x8192")


def test_prefill_shared_memory_kernel_full_size_rows_and_entries(orc):
    # M = 512 on gate_proj: the shared-memory prefill kernel is the one launched
    assert w3a16_gemm_route(512, 28672, 8192) == "prefill"
    _rows_and_entries_check(orc, "prefill_512x28672x8192")
