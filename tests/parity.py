"""Shared helpers of the parity tests: moving seeded problems to the GPU in the
library's argument layout, and the tolerance check.

Tolerance (stated for this GEMM): per output tensor
    calc_diff = 1 - 2*sum(x*y) / sum(x^2 + y^2) <= 1e-3
and per element, after bf16 rounding of both sides,
    |gpu - oracle| <= 1e-2 * (|oracle| + 1e-2).
Placement and masking are bit-exact: rows the method must not write keep a
sentinel pattern.
"""
from __future__ import annotations

import numpy as np
import torch

import dg_inputs as gi

SENTINEL = 0x7FC1          # a bf16 NaN pattern no computation produces
CALC_DIFF_MAX = 1e-3
REL_TOL = 1e-2
ABS_FLOOR = 1e-2


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double().numpy()


def calc_diff(x: np.ndarray, y: np.ndarray) -> float:
    x = x.astype(np.float64).ravel()
    y = y.astype(np.float64).ravel()
    denom = float((x * x + y * y).sum())
    if denom == 0.0:
        return 0.0
    return 1.0 - 2.0 * float((x * y).sum()) / denom


def assert_close(got_bits: np.ndarray, ref_bits: np.ndarray, what: str = ""):
    got = bf16_bits_to_f64(got_bits)
    ref = bf16_bits_to_f64(ref_bits)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bound = REL_TOL * (np.abs(ref) + ABS_FLOOR)
    bad = err > bound
    if bad.any():
        i = np.argmax(err / bound)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements beyond tolerance; worst at flat "
            f"{int(i)}: got {got.ravel()[i]!r} oracle {ref.ravel()[i]!r}")
    cd = calc_diff(got, ref)
    assert cd <= CALC_DIFF_MAX, f"{what}: calc_diff {cd:.3e} > {CALC_DIFF_MAX}"
    return cd


def assert_close_f32(got: np.ndarray, ref: np.ndarray, what: str = ""):
    """The same tolerance for fp32 outputs (the accumulate form)."""
    got = got.astype(np.float64)
    ref = ref.astype(np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bound = REL_TOL * (np.abs(ref) + ABS_FLOOR)
    bad = err > bound
    if bad.any():
        i = np.argmax(err / bound)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements beyond tolerance; worst at flat "
            f"{int(i)}: got {got.ravel()[i]!r} oracle {ref.ravel()[i]!r}")
    cd = calc_diff(got, ref)
    assert cd <= CALC_DIFF_MAX, f"{what}: calc_diff {cd:.3e} > {CALC_DIFF_MAX}"
    return cd


def dev_dense(p):
    """Dense problem -> device tensors in the library layout (+ D prefilled)."""
    dev = torch.device("cuda")
    A = torch.from_numpy(p["A"]).to(dev)
    B = torch.from_numpy(p["B"]).to(dev)
    sA = torch.from_numpy(gi.sa_to_kernel_layout(p["sA"])).to(dev)
    sB = torch.from_numpy(p["sB"]).to(dev)
    D = torch.full((p["M"], p["N"]), SENTINEL, dtype=torch.int16, device=dev).view(torch.bfloat16)
    return A, sA, B, sB, D


def dev_contiguous(p):
    dev = torch.device("cuda")
    A = torch.from_numpy(p["A"]).to(dev)
    B = torch.from_numpy(p["B"]).to(dev)
    sA = torch.from_numpy(gi.sa_to_kernel_layout(p["sA"])).to(dev)
    sB = torch.from_numpy(p["sB"]).to(dev)
    mi = torch.from_numpy(p["m_indices"]).to(dev)
    D = torch.full((p["M"], p["N"]), SENTINEL, dtype=torch.int16, device=dev).view(torch.bfloat16)
    return A, sA, B, sB, D, mi


def dev_masked(p):
    dev = torch.device("cuda")
    A = torch.from_numpy(p["A"]).to(dev)
    B = torch.from_numpy(p["B"]).to(dev)
    sA = torch.from_numpy(gi.sa_to_kernel_layout(p["sA"])).to(dev)
    sB = torch.from_numpy(p["sB"]).to(dev)
    mm = torch.from_numpy(p["masked_m"]).to(dev)
    D = torch.full((p["G"], p["max_m"], p["N"]), SENTINEL, dtype=torch.int16,
                   device=dev).view(torch.bfloat16)
    return A, sA, B, sB, D, mm


def bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)
