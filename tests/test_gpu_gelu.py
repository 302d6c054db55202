"""GPU check of the GEMM epilogues' GELU and GELU' against the exact erf form.

The epilogues evaluate the Gaussian tail as exp(-z^2) R(z) with a fitted
polynomial for R (relative error ~1e-5).  With one-hot activations each output is a single weight
(forward) or a single mask bit (input gradient), so the epilogue's value can
be compared element by element with the oracle's fp64 GELU rounded to the
output dtype: at most one unit in the last place apart wherever the rounded
reference exceeds 1e-3 in magnitude, and within 1e-6 absolute below that
(where fp32 arithmetic, not the output dtype, sets the accuracy).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
import structured_sparse_transformer_b200 as sp

pytestmark = pytest.mark.gpu


def _check(got_bits, ref_bits, dtype):
    got = oracle.to_f64(got_bits, dtype)
    ref = oracle.to_f64(ref_bits, dtype)
    big = np.abs(ref) > 1e-3
    d = _ulp_distance(got_bits, ref_bits)
    assert d[big].max() <= 1, f"max ulp distance {d[big].max()} where |ref| > 1e-3"
    assert np.abs(got - ref)[~big].max(initial=0.0) <= 1e-6


def _ulp_distance(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    def key(u):
        u = u.astype(np.int32)
        return np.where(u & 0x8000, -(u & 0x7FFF), u & 0x7FFF)
    return np.abs(key(a_bits) - key(b_bits))


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_gelu_epilogue_matches_exact_erf(dtype):
    n = 256
    tdt = si.DTYPES[dtype]
    vals = torch.linspace(-8.0, 8.0, n * n, dtype=torch.float32)
    perm = torch.randperm(n * n, generator=torch.Generator().manual_seed(0))
    w = vals[perm].reshape(n, n).to(tdt)
    wd = w.cuda()
    idx = torch.empty(n // 4, n // 4, dtype=torch.uint8, device="cuda")
    c = sp.alloc_compressed(n, n, tdt)
    sp.sp24_mask_step(wd, idx, None, None, *c)
    x = torch.eye(n, dtype=tdt).cuda()
    h = torch.empty(n, n, dtype=tdt, device="cuda")
    pre = torch.empty(n, n, dtype=tdt, device="cuda")
    sp.sp24_gemm_fwd(x, c[0], c[1], n, h, "gelu", pre)
    torch.cuda.synchronize()
    keep = oracle.dense_mask(idx.cpu().numpy())
    pre_ref = np.where(keep, oracle.to_f64(si.bits16(w), dtype), 0.0).T
    assert np.array_equal(oracle.to_f64(si.bits16(pre.cpu()), dtype), pre_ref)   # single exact products
    ref_bits = si.bits16(torch.from_numpy(oracle.gelu(pre_ref)).to(tdt))
    _check(si.bits16(h.cpu()), ref_bits, dtype)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_dgelu_epilogue_matches_exact_erf(dtype):
    n = 256
    tdt = si.DTYPES[dtype]
    w = torch.ones(n, n, dtype=tdt)
    idx = torch.empty(n // 4, n // 4, dtype=torch.uint8, device="cuda")
    c = sp.alloc_compressed(n, n, tdt)
    sp.sp24_mask_step(w.cuda(), idx, None, None, *c)
    aux_vals = torch.linspace(-8.0, 8.0, n * n, dtype=torch.float32).reshape(n, n).to(tdt)
    dy = torch.eye(n, dtype=tdt).cuda()
    dx = torch.empty(n, n, dtype=tdt, device="cuda")
    sp.sp24_gemm_dgrad(dy, c[2], c[3], n, dx, "dgelu", aux_vals.cuda())
    torch.cuda.synchronize()
    keep = oracle.dense_mask(idx.cpu().numpy())
    ref = np.where(keep, oracle.gelu_grad(oracle.to_f64(si.bits16(aux_vals), dtype)), 0.0)
    ref_bits = si.bits16(torch.from_numpy(ref).to(tdt))
    _check(si.bits16(dx.cpu()), ref_bits, dtype)


@pytest.mark.parametrize("dense", [False, True])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_derivative_saving_pair_matches_exact_erf(dtype, dense):
    """SP24_EPI_GELU_DERIV stores gelu(acc) as out and gelu'(acc) as aux; SP24_EPI_MUL_AUX
    multiplies by aux.  One-hot activations make every accumulator a single weight, so both
    outputs of the forward are checked element by element against the fp64 GELU and GELU'
    rounded to the dtype, and the input gradient (dY one-hot) against the stored derivative
    rounded once more (the product acc * aux with acc exactly one value)."""
    n = 256
    tdt = si.DTYPES[dtype]
    vals = torch.linspace(-8.0, 8.0, n * n, dtype=torch.float32)
    perm = torch.randperm(n * n, generator=torch.Generator().manual_seed(1))
    w = vals[perm].reshape(n, n).to(tdt)
    wd = w.cuda()
    idx = torch.empty(n // 4, n // 4, dtype=torch.uint8, device="cuda")
    c = sp.alloc_compressed(n, n, tdt)
    sp.sp24_mask_step(wd, idx, None, None, *c)
    keep = oracle.dense_mask(idx.cpu().numpy())
    x = torch.eye(n, dtype=tdt).cuda()
    h = torch.empty(n, n, dtype=tdt, device="cuda")
    deriv = torch.empty(n, n, dtype=tdt, device="cuda")
    if dense:   # the dense path sees the masked weight as a plain matrix
        wm = torch.from_numpy(np.where(keep, oracle.to_f64(si.bits16(w), dtype), 0.0)).to(tdt).cuda()
        sp.sp24_gemm_dense(x, wm, h, "gelu_deriv", deriv)
    else:
        sp.sp24_gemm_fwd(x, c[0], c[1], n, h, "gelu_deriv", deriv)
    torch.cuda.synchronize()
    pre_ref = np.where(keep, oracle.to_f64(si.bits16(w), dtype), 0.0).T
    _check(si.bits16(h.cpu()), si.bits16(torch.from_numpy(oracle.gelu(pre_ref)).to(tdt)), dtype)
    _check(si.bits16(deriv.cpu()), si.bits16(torch.from_numpy(oracle.gelu_grad(pre_ref)).to(tdt)), dtype)
    # input gradient: dY one-hot, all-ones weight, so acc is the mask bit; out = bit * aux
    ones = torch.ones(n, n, dtype=tdt)
    c1 = sp.alloc_compressed(n, n, tdt)
    idx1 = torch.empty_like(idx)
    sp.sp24_mask_step(ones.cuda(), idx1, None, None, *c1)
    dy = torch.eye(n, dtype=tdt).cuda()
    dx = torch.empty(n, n, dtype=tdt, device="cuda")
    if dense:
        k1 = oracle.dense_mask(idx1.cpu().numpy())
        wt = torch.from_numpy(np.where(k1, 1.0, 0.0).T.copy()).to(tdt).cuda()
        sp.sp24_gemm_dense(dy, wt, dx, "mul_aux", deriv)
    else:
        sp.sp24_gemm_dgrad(dy, c1[2], c1[3], n, dx, "mul_aux", deriv)
    torch.cuda.synchronize()
    k1 = oracle.dense_mask(idx1.cpu().numpy())
    ref = np.where(k1, 1.0, 0.0) * oracle.to_f64(si.bits16(deriv.cpu()), dtype)   # IEEE: 0 * negative = -0
    assert np.array_equal(si.bits16(dx.cpu()), si.bits16(torch.from_numpy(ref).to(tdt)))
