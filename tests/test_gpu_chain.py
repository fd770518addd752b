"""Back-to-back calls that feed each other, with no synchronisation between them.

Every decode kernel starts its set-up while the previous kernel in the stream is
still running (programmatic dependent launch) and waits for it only before it
reads x or writes y.  Here each call's x is the previous call's y, so a kernel
that read x too early, or wrote y while the next kernel was already reading it,
would produce a product of the wrong input.  After the whole chain the inputs
each call actually saw are read back, and each output is checked against the
fp64 oracle of its own input.  The chains cover every kernel route (the route of
each call is asserted), and mixed chains alternate routes as a model's layers do.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_within_bound, bound, from_dev_bf16, to_dev_bf16
from w3a16_gemv_b200 import build, w3_check_device_error, w3_pack, w3a16_gemm, w3a16_gemm_route
from w3a16_gemv_b200.inputs import make_problem

pytestmark = pytest.mark.gpu

S = 4864  # square weights (N = K) so that y of one call is x of the next; 152 blocks of 32 rows


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available()


def _weights(n, seed):
    """n square weights [S, S]: packed on the GPU, and their codes and scales for the oracle."""
    out = []
    for i in range(n):
        p = make_problem(1, S, S, "gsq_5level", "absnormal", "normal", seed=seed + i)
        out.append((w3_pack(torch.from_numpy(p.codes).cuda()), to_dev_bf16(p.scales_bf16), p))
    return out


def _check_chain(orc, batches, weights):
    """Run the chain (call j on the output of call j-1, batch rows batches[j] taken from the
    front of the previous output) without synchronising, then check every call."""
    M0 = batches[0]
    x0 = make_problem(M0, 8, S, seed=99).x_bf16  # only x is used
    xs = [to_dev_bf16(x0)]
    ys = []
    for j, (M, (packed, scales, _)) in enumerate(zip(batches, weights)):
        assert xs[-1].shape[0] >= M
        x = xs[-1][:M]  # the leading rows: a contiguous view, no copy between the calls
        xs[-1] = x
        y = w3a16_gemm(x, packed, scales)
        ys.append(y)
        xs.append(y)
    torch.cuda.synchronize()
    w3_check_device_error()
    for j, (M, (_, _, p)) in enumerate(zip(batches, weights)):
        x_bits = from_dev_bf16(xs[j])
        ref_packed = orc.pack(p.codes)
        ref = orc.gemm_f64(x_bits, ref_packed, p.scales_bf16, threads=0)
        tol = bound(x_bits, orc.weight_row_norms(ref_packed, p.scales_bf16, S), S)
        assert_within_bound(from_dev_bf16(ys[j]), ref, tol, f"call {j} (M={M}, {w3a16_gemm_route(M, S, S)})")


CHAINS = {
    "decode_sk": [1, 1, 1, 1],
    "decode_sk_m4": [4, 4, 4],
    "decode_split": [16, 16, 16],
    "decode_tc32": [24, 24, 24],
    "prefill": [64, 64, 64],
    # each call takes the first rows of the previous output: tensor-memory prefill, 32-wide
    # tcgen05 decode, split decode, stream-K decode
    "mixed": [64, 24, 16, 4, 1],
}


@pytest.mark.parametrize("name", sorted(CHAINS))
def test_chained_calls_read_the_finished_input(orc, name):
    batches = CHAINS[name]
    routes = {w3a16_gemm_route(M, S, S) for M in batches}
    if name != "mixed":
        assert len(routes) == 1
        if name.startswith("decode_sk"):
            assert routes == {"decode_sk"}
        elif name == "prefill":
            assert routes <= {"prefill", "prefill_ab"}
        else:
            assert routes == {name}
    else:
        assert {"decode_sk", "decode_split", "decode_tc32"} <= routes
    _check_chain(orc, batches, _weights(len(batches), seed=200))
