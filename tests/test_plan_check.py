"""The kernels' launch plans and work splits, checked on the host (no GPU needed).

tests/plan_check.cu includes the kernel headers, calls only their __host__
functions and compares each rule with ground truth computed from the unit
intervals: the 32-wide tensor-core decode's stream-K ranges and the fix-up
rule that finishes every shared 256-row tile exactly once from the right
partial-sum slots; the split decode's cluster, K-slice and warp ranges, its
shared-memory budget, and that whether a plan exists does not depend on the
device's occupancy answer; the stream-K decode's plan; and that both prefill
grids cover every output once.
"""
import os
import subprocess

import pytest

from w3a16_gemv_b200 import build

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "plan_check.cu")


@pytest.fixture(scope="module")
def plan_check_binary(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("plan_check") / "plan_check")
    # host code only is run: a PTX-only device target keeps the build short
    subprocess.check_call([build.nvcc(), "-std=c++17", "-O1", "--expt-relaxed-constexpr",
                           "-gencode", "arch=compute_100a,code=compute_100a", "-o", out, SRC])
    return out


def test_launch_plans_and_work_splits(plan_check_binary):
    r = subprocess.run([plan_check_binary], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert "0 failures" in r.stdout
