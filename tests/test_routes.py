"""Kernel selection of w3a16_gemm, asked through the C ABI without a GPU.

w3a16_gemm_route depends only on the shape and the SM count, so the dispatch
rules can be checked on the host: which kernel serves each batch size of the
benchmarked shapes, the batch-size boundaries between routes, how many kernels
a call launches, and that invalid shapes have no route.
"""
import pytest

from w3a16_gemv_b200 import _binding, build, w3a16_gemm_launches, w3a16_gemm_route

SMS = 148  # B200

ROUTES = {"decode_split", "decode_sk", "decode", "decode_tc32", "prefill", "prefill_ab", "passes"}


@pytest.fixture(scope="module", autouse=True)
def lib():
    build.build()
    return _binding.lib()


def test_invalid_shapes_have_no_route(lib):
    f = lib.w3a16_gemm_route
    assert f(0, 16, 128, SMS) is None
    assert f(1, 0, 128, SMS) is None
    assert f(1, 16, 192, SMS) is None
    assert f(1, 16, 0, SMS) is None
    assert f(1, 16, 128, 0) is None


@pytest.mark.parametrize("M", list(range(1, 70)) + [128, 255, 256, 257, 1024, 2048, 4096])
@pytest.mark.parametrize("N,K", [(28672, 8192), (8192, 28672), (8192, 8192), (1024, 8192), (4096, 4096),
                                 (300, 1152), (40, 256), (28672, 128)])
def test_every_shape_has_a_known_route(M, N, K):
    r = w3a16_gemm_route(M, N, K, num_sms=SMS)
    assert r in ROUTES
    if 5 <= M <= 16:
        # the split decode wherever its shared memory holds a K slice of x, a ring and the
        # cluster's partial sums; the older cluster decode otherwise
        assert r in (("decode_split", "decode") if N >= 32 else ("decode",))
    if M <= 4:
        assert r in ("decode_sk", "decode_split", "decode")
    if r == "decode":  # fewer than 32 rows, or a split plan that does not fit (K above 8192 here)
        assert N < 32 or K > 8192
    if r == "decode_sk":
        assert M <= 4 and N >= 32 * SMS
    if r == "decode_tc32":
        assert N >= 256
    if r == "decode_tc32":
        assert 17 <= M <= 32
    if r in ("prefill", "prefill_ab"):
        assert M > 16 and K >= 256
    if r == "passes":
        assert M > 16 and K < 256


def test_benchmarked_shapes():
    # the gate_proj decode step M = 1, 4, 16 and the M = 2048 prefill
    assert w3a16_gemm_route(1, 28672, 8192, SMS) == "decode_sk"
    assert w3a16_gemm_route(4, 28672, 8192, SMS) == "decode_sk"
    assert w3a16_gemm_route(16, 28672, 8192, SMS) == "decode_split"
    assert w3a16_gemm_route(24, 28672, 8192, SMS) == "decode_tc32"
    assert w3a16_gemm_route(2048, 28672, 8192, SMS) in ("prefill", "prefill_ab")
    # fewer 32-row blocks than SMs at M <= 4: the split decode; fewer than 32 rows: the older decode
    assert w3a16_gemm_route(1, 1024, 8192, SMS) == "decode_split"
    assert w3a16_gemm_route(1, 4096, 4096, SMS) == "decode_split"
    assert w3a16_gemm_route(8, 20, 8192, SMS) == "decode"


def test_split_decode_where_its_plan_fits():
    for M in (5, 8, 12, 16):
        for N, K in ((28672, 8192), (8192, 8192), (1024, 8192), (4096, 4096), (300, 1152)):
            assert w3a16_gemm_route(M, N, K, SMS) == "decode_split", (M, N, K)
    assert w3a16_gemm_route(8, 8192, 28672, SMS) == "decode_split"
    # 16 batch rows over K = 28672: x of an eighth of K, the ring and the partial sums do not fit
    assert w3a16_gemm_route(16, 8192, 28672, SMS) == "decode"
    # one SM: no cluster split, and x of the whole K range does not fit
    assert w3a16_gemm_route(16, 4096, 8192, 1) == "decode"
    assert w3a16_gemm_route(16, 4096, 1024, 1) == "decode_split"


# (M, N, K) -> the faster prefill kernel on B200 (each timed alone, device time per call)
MEASURED_PREFILL = {
    (64, 8192, 8192): "prefill_ab",      # 42.4 us against 66.5
    (256, 8192, 28672): "prefill_ab",    # 139.6 against 254.5
    (256, 4096, 4096): "prefill_ab",     # 27.9 against 42.1
    (256, 1024, 8192): "prefill_ab",     # 46.1 against 77.2
    (64, 28672, 8192): "prefill",        # 81.0 against 84.8
    (128, 28672, 8192): "prefill",       # 82.0 against 90.6
    (160, 28672, 8192): "prefill_ab",    # 91.7 against 101.9
    (512, 28672, 8192): "prefill",       # 197.5 against 228.7
    (1024, 28672, 8192): "prefill_ab",   # 421.7 against 479.8
    (3072, 28672, 8192): "prefill_ab",   # 1214.3 against 1393.8
    (1024, 8192, 28672): "prefill",      # 353.5 against 421.9
    (1024, 8192, 8192): "prefill",       # 109.3 against 118.5
    (256, 57344, 8192): "prefill",       # 196.7 against 215.9
}


@pytest.mark.parametrize("shape", sorted(MEASURED_PREFILL))
def test_prefill_dispatch_picks_the_measured_faster_kernel(shape):
    assert w3a16_gemm_route(*shape, SMS) == MEASURED_PREFILL[shape]


@pytest.mark.parametrize("M", [33, 64, 100, 128, 160, 200, 255, 256, 300, 512, 768, 1024, 2048, 4096])
@pytest.mark.parametrize("N", [300, 1024, 4096, 8192, 14336, 28672, 57344])
def test_prefill_dispatch_does_not_depend_on_k(M, N):
    routes = {w3a16_gemm_route(M, N, K, SMS) for K in (256, 1024, 4096, 8192, 28672, 65536)}
    assert len(routes) == 1 and routes <= {"prefill", "prefill_ab"}, routes


def test_tall_k_small_batches_take_the_split_decode():
    # down_proj at 2..4 batch rows: the stream-K decode's prepared x of all of K does not fit
    assert w3a16_gemm_route(1, 8192, 28672, SMS) == "decode_sk"
    for M in (2, 3, 4):
        assert w3a16_gemm_route(M, 8192, 28672, SMS) == "decode_split"
    assert w3a16_gemm_route(4, 28672, 8192, SMS) == "decode_sk"
    assert w3a16_gemm_route(4, 1024, 28672, SMS) == "decode_split"


def test_route_depends_on_the_sm_count():
    # the stream-K decode needs one 32-row block per SM
    assert w3a16_gemm_route(1, 4800, 1024, 148) == "decode_sk"
    assert w3a16_gemm_route(1, 4800, 1024, 160) == "decode_split"


def test_kernels_per_call():
    """One kernel per call, plus the fix-up kernel where the tensor-core decode splits row tiles
    between CTAs, and one per 16-row pass."""
    f = w3a16_gemm_launches
    assert f(1, 28672, 8192, SMS) == 1 and f(4, 28672, 8192, SMS) == 1  # stream-K decode
    assert f(16, 28672, 8192, SMS) == 1  # split decode
    assert f(24, 28672, 8192, SMS) == 2  # tensor-core decode and its fix-up
    assert f(64, 28672, 8192, SMS) == 1 and f(2048, 28672, 8192, SMS) == 1  # prefill kernels
    # passes: M = 36 with K = 128 is two 16-row passes and one 4-row pass
    assert w3a16_gemm_route(36, 28672, 128, num_sms=SMS) == "passes"
    assert f(36, 28672, 128, SMS) == 3
    for args in ((0, 16, 128, SMS), (1, 0, 128, SMS), (1, 16, 192, SMS), (1, 16, 128, 0)):
        assert _binding.lib().w3a16_gemm_launches(*args) == -1
