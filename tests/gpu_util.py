"""Shared helpers of the GPU parity tests: upload seeded inputs, read results
back as the same uint16/uint8 views the oracle uses, and the GEMM tolerance.

GEMM tolerance: outputs are compared with the fp64 oracle rounded to the
output dtype.  Required: relative Frobenius error <= 1e-3, and relative error
<= 1e-2 on every element whose rounded reference exceeds 1e-3 in magnitude
(one bf16 ulp is 2^-7 ~ 7.8e-3 relative, so a last-bit rounding difference of
the fp32 accumulator passes; a wrong term or index does not)."""
import numpy as np
import torch

import oracle
import synthetic_inputs as si

FRO_TOL = 1e-3
ELEM_TOL = 1e-2
ELEM_FLOOR = 1e-3


def bits_of(t: torch.Tensor) -> np.ndarray:
    return si.bits16(t.detach().cpu())


def f64_of(t: torch.Tensor, dtype: str) -> np.ndarray:
    return oracle.to_f64(bits_of(t), dtype)


def gemm_errors(got: np.ndarray, ref_q: np.ndarray):
    fro = np.linalg.norm(got - ref_q) / max(np.linalg.norm(ref_q), 1e-300)
    big = np.abs(ref_q) > ELEM_FLOOR
    elem = float(np.max(np.abs(got[big] - ref_q[big]) / np.abs(ref_q[big]))) if big.any() else 0.0
    return float(fro), elem


def assert_gemm_close(got: np.ndarray, ref_f64: np.ndarray, dtype: str, what: str = ""):
    ref_q = oracle.round_to(ref_f64, dtype)
    fro, elem = gemm_errors(got, ref_q)
    assert fro <= FRO_TOL, f"{what}: relative Frobenius error {fro:.3e} > {FRO_TOL}"
    assert elem <= ELEM_TOL, f"{what}: max element relative error {elem:.3e} > {ELEM_TOL}"
    return fro, elem


def assert_gemm_within_accumulation_bound(got: np.ndarray, ref_f64: np.ndarray, abs_prod: np.ndarray, n: int,
                                          dtype: str, what: str = ""):
    """Long contractions over whole matrices: the relative Frobenius bound above, and on every
    element |got - ref| <= n 2^-24 sum_k |a_k b_k| + 2 ulp(ref) of the output dtype (the
    textbook bound of an fp32 sum of n products, plus the output rounding).  abs_prod is
    |A| |B|, the sum of the products' magnitudes.  Near-cancelling elements, whose relative
    error the fixed floor above would judge, get their absolute error budget instead; a wrong
    or missing term in every element still moves the Frobenius error far past 1e-3."""
    ref_q = oracle.round_to(ref_f64, dtype)
    fro, _ = gemm_errors(got, ref_q)
    assert fro <= FRO_TOL, f"{what}: relative Frobenius error {fro:.3e} > {FRO_TOL}"
    ulp = 2.0 ** (-10 if dtype == "f16" else -7)
    bound = n * 2.0 ** -24 * abs_prod + 2 * ulp * np.abs(ref_q) + 2.0 ** -24
    worst = float(np.max(np.abs(got - ref_q) / bound))
    assert worst <= 1.0, f"{what}: an element exceeds the accumulation bound ({worst:.3f} of it)"
