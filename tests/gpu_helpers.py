"""Helpers for the GPU parity tests: device copies of seeded problems and the output bound."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from w3a16_gemv_b200.inputs import Problem


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def from_dev_bf16(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def device_problem(p: Problem):
    """x bf16 [M,K], codes uint8 [N,K], scales bf16 [N,K/128] on the GPU."""
    return to_dev_bf16(p.x_bf16), torch.from_numpy(p.codes).cuda(), to_dev_bf16(p.scales_bf16)


def bound(x_bf16: np.ndarray, w_row_norms: np.ndarray, K: int) -> np.ndarray:
    """The accumulation bound 1e-2 * ||x_m||_2 * ||w_n||_2 / sqrt(K) + 1e-3 (per element, [M,N])."""
    xf = oracle.bf16_to_f64(x_bf16)
    xn = np.sqrt(np.sum(xf * xf, axis=1))
    return 1e-2 * np.outer(xn, w_row_norms) / np.sqrt(K) + 1e-3


def half_ulp_bf16(v: np.ndarray) -> np.ndarray:
    """Half the bf16 spacing at |v|: the error of rounding v to the bf16 output type."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.ldexp(1.0, (e - 8).astype(np.int64))  # spacing 2^(e-7), half of it


def assert_within_bound(y_bits: np.ndarray, y_ref: np.ndarray, tol: np.ndarray, what: str) -> float:
    """Every element within its bound; returns the worst |err|/bound ratio.

    The bound is the accumulation bound plus the unavoidable rounding of the
    result to bf16 (half a bf16 ulp of the larger of |y|, |y_ref|): a correctly
    rounded bf16 output can exceed the accumulation bound alone wherever |y| is
    more than about 3 x ||x_m|| ||w_n|| / sqrt(K)."""
    y = oracle.bf16_to_f64(y_bits)
    err = np.abs(y - y_ref)
    tol = tol + half_ulp_bf16(np.maximum(np.abs(y), np.abs(y_ref)))
    ratio = err / tol
    worst = float(np.max(ratio)) if ratio.size else 0.0
    if not np.all(np.isfinite(y)) or worst > 1.0:
        idx = np.unravel_index(int(np.nanargmax(np.where(np.isfinite(ratio), ratio, np.inf))), ratio.shape)
        raise AssertionError(f"{what}: worst element {idx}: y={y[idx]!r} ref={y_ref[idx]!r} "
                             f"bound={tol[idx]!r} ratio={worst:.3g}")
    return worst
