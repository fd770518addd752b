"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module draws raw material only -- unpacked 3-bit codes, bf16 scales and
bf16 activations -- and holds none of the format's arithmetic (no packing, no
dequantization, no product).  The CUDA path packs the codes with ``w3_pack``;
the oracle packs them with its own bit-level packer; the tests compare the two.

Recipe (one ``numpy.random.Generator(PCG64(seed))`` per workload, seed 0 unless
stated, draws in the fixed order x -> codes -> scales -> outlier mask; fp32
draws are rounded to bf16 with round-to-nearest-even):

* x: standard normal, [M, K]; for ``x="normal_outliers"`` a Bernoulli(0.01)
  mask multiplies the chosen entries by 20 in fp32 before rounding.
* codes, [N, K] uint8:
  - ``"gsq_uniform"``: uniform over {2..6} (the GSQ levels -2..+2 under q = c-4);
  - ``"uniform8"``: uniform over the full uint3 range 0..7;
  - ``"gsq_5level"``: {2,3,4,5,6} with probabilities 0.1/0.2/0.4/0.2/0.1.
* scales, [N, K/128] bf16:
  - ``"absnormal"``: |N(0, 0.02)| + 1e-4;
  - ``"lognormal"``: lognormal(mu=-4, sigma=0.5).

The shapes are the Llama-3.1-70B projection shapes of the GSQ model card
("Storage layout", the gate_proj example [28672, 8192]) and the other linear
layers of that architecture.  No checkpoint or dataset is used.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

GROUP = 128


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round finite float32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = ((u >> 16) & 1) + 0x7FFF
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(b).view(np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class Problem:
    """One seeded problem: activations, raw codes and scales (bit patterns)."""

    x_bf16: np.ndarray  # uint16 [M, K]
    codes: np.ndarray  # uint8 [N, K], values 0..7
    scales_bf16: np.ndarray  # uint16 [N, K/128]

    @property
    def M(self) -> int:
        return self.x_bf16.shape[0]

    @property
    def N(self) -> int:
        return self.codes.shape[0]

    @property
    def K(self) -> int:
        return self.codes.shape[1]


def draw_codes(rng: np.random.Generator, N: int, K: int, dist: str) -> np.ndarray:
    if dist == "gsq_uniform":
        return rng.integers(2, 7, size=(N, K), dtype=np.uint8)
    if dist == "uniform8":
        return rng.integers(0, 8, size=(N, K), dtype=np.uint8)
    if dist == "gsq_5level":
        u = rng.random(size=(N, K), dtype=np.float32)
        c = np.full((N, K), 2, dtype=np.uint8)
        for edge in (0.1, 0.3, 0.7, 0.9):  # cumulative 0.1/0.2/0.4/0.2/0.1
            c += (u >= np.float32(edge)).astype(np.uint8)
        return c
    raise ValueError(f"unknown code distribution {dist!r}")


def draw_scales(rng: np.random.Generator, N: int, G: int, dist: str) -> np.ndarray:
    if dist == "absnormal":
        s = np.abs(rng.normal(0.0, 0.02, size=(N, G))) + 1e-4
    elif dist == "lognormal":
        s = rng.lognormal(mean=-4.0, sigma=0.5, size=(N, G))
    else:
        raise ValueError(f"unknown scale distribution {dist!r}")
    return f32_to_bf16_bits(s.astype(np.float32))


def make_problem(M: int, N: int, K: int, codes: str = "uniform8", scales: str = "lognormal",
                 x: str = "normal", seed: int = 0) -> Problem:
    """Draw one problem with the recipe in the module docstring."""
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    rng = np.random.Generator(np.random.PCG64(seed))
    xf = rng.standard_normal(size=(M, K), dtype=np.float32)
    c = draw_codes(rng, N, K, codes)
    s = draw_scales(rng, N, K // GROUP, scales)
    if x == "normal_outliers":
        mask = rng.random(size=(M, K)) < 0.01
        xf = np.where(mask, xf * np.float32(20.0), xf).astype(np.float32)
    elif x != "normal":
        raise ValueError(f"unknown activation distribution {x!r}")
    return Problem(f32_to_bf16_bits(xf), c, s)


@dataclass(frozen=True)
class Workload:
    """A named shape + value recipe."""

    name: str
    M: int
    N: int
    K: int
    codes: str
    scales: str
    x: str = "normal"

    def problem(self, seed: int = 0) -> Problem:
        return make_problem(self.M, self.N, self.K, self.codes, self.scales, self.x, seed)


# Llama-3.1-70B projection shapes (out_features N, in_features K).
LLAMA70B_LAYER = (
    ("q_proj", 8192, 8192),
    ("k_proj", 1024, 8192),
    ("v_proj", 1024, 8192),
    ("o_proj", 8192, 8192),
    ("gate_proj", 28672, 8192),
    ("up_proj", 28672, 8192),
    ("down_proj", 8192, 28672),
)


def workloads() -> dict[str, Workload]:
    """Every measured and parity-tested workload, by name."""
    w = {}
    w["gemv_4096_m1"] = Workload("gemv_4096_m1", 1, 4096, 4096, "gsq_uniform", "absnormal")
    for m in (1, 4, 16):
        w[f"gate_28672x8192_m{m}"] = Workload(f"gate_28672x8192_m{m}", m, 28672, 8192, "uniform8", "lognormal")
    for m in (1, 8):
        w[f"down_8192x28672_m{m}"] = Workload(f"down_8192x28672_m{m}", m, 8192, 28672, "gsq_5level",
                                              "absnormal", "normal_outliers")
    for name, n, k in LLAMA70B_LAYER:
        w[f"layer_{name}_m1"] = Workload(f"layer_{name}_m1", 1, n, k, "uniform8", "lognormal")
    # mid-size batches on gate_proj and q_proj: the 32-wide tensor-core decode (M = 24) and
    # both prefill kernels (the dispatch picks per shape)
    for m in (24, 33, 64, 128, 160, 255):
        w[f"mid_gate_28672x8192_m{m}"] = Workload(f"mid_gate_28672x8192_m{m}", m, 28672, 8192, "uniform8",
                                                  "lognormal")
    w["mid_q_8192x8192_m64"] = Workload("mid_q_8192x8192_m64", 64, 8192, 8192, "gsq_5level", "absnormal",
                                        "normal_outliers")
    w["prefill_2048x28672x8192"] = Workload("prefill_2048x28672x8192", 2048, 28672, 8192, "uniform8", "lognormal")
    # batches at which each prefill kernel is the one launched
    w["prefill_1024x28672x8192"] = Workload("prefill_1024x28672x8192", 1024, 28672, 8192, "uniform8", "lognormal")
    w["prefill_512x28672x8192"] = Workload("prefill_512x28672x8192", 512, 28672, 8192, "uniform8", "lognormal")
    return w
