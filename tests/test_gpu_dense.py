"""GPU parity of the dense fine-tuning GEMM and the transpose against the oracle.

"Accelerating Transformer Pre-training with 2:4 Sparsity", abstract (a dense
fine-tuning procedure near the end of pre-training) and Experiment Setup row
(dense fine-tuning takes the last 1/6 of the total steps): the FFN products
run dense, on the same tcgen05 pipeline as the 2:4 GEMMs.  The input gradient
reads W as stored (sp24_gemm_dgrad_dense, W loaded MN-major) or takes W^T from
the transpose kernel (sp24_gemm_dense).  Tolerances as in gpu_util.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
import structured_sparse_transformer_b200 as sp
from gpu_util import assert_gemm_close, assert_gemm_within_accumulation_bound, f64_of

pytestmark = pytest.mark.gpu


def _dt(t):
    return "bf16" if t.dtype == torch.bfloat16 else "f16"


def _transpose(w):
    out = torch.empty(w.shape[1], w.shape[0], dtype=w.dtype, device="cuda")
    sp.sp24_transpose(w, out)
    return out


@pytest.mark.parametrize("R,C,dtype", [(4096, 1024, "f16"), (37, 100, "bf16"), (1, 7, "f16"), (300, 33, "f16")])
def test_transpose_bit_exact(R, C, dtype):
    w = si.normal((R, C), 1.0, R + C, dtype)
    wt = _transpose(w.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(si.bits16(wt.cpu()), np.ascontiguousarray(si.bits16(w).T))


@pytest.mark.parametrize("T,N,K,dtype", [(128, 128, 128, "f16"), (200, 256, 384, "f16"), (77, 144, 400, "bf16"),
                                         (1, 16, 16, "f16"), (300, 1600, 208, "f16"), (513, 208, 1600, "bf16")])
def test_dense_fwd_and_dgrad_small(T, N, K, dtype):
    w = si.normal((N, K), 0.02, N + K, dtype)
    x = si.normal((T, K), 1.0, T, dtype)
    dy = si.normal((T, N), 1.0, T + 1, dtype)
    wd = w.cuda()
    y = torch.empty(T, N, dtype=w.dtype, device="cuda")
    dx = torch.empty(T, K, dtype=w.dtype, device="cuda")
    sp.sp24_gemm_dense(x.cuda(), wd, y)
    sp.sp24_gemm_dense(dy.cuda(), _transpose(wd), dx)
    torch.cuda.synchronize()
    wf = oracle.to_f64(si.bits16(w), dtype)
    assert_gemm_close(f64_of(y, dtype), oracle.dense_fwd(oracle.to_f64(si.bits16(x), dtype), wf), dtype, "fwd")
    assert_gemm_close(f64_of(dx, dtype), oracle.dense_dgrad(oracle.to_f64(si.bits16(dy), dtype), wf), dtype, "dgrad")


@pytest.mark.parametrize("wl", [si.GPT2_355M, si.GPT2_774M], ids=lambda w: w.name)
def test_dense_ffn_chain_with_gelu_sampled_rows(wl):
    """fwd1 (+GELU, aux = pre-activation) -> fwd2; dY -> dgrad2 (+dGELU) -> dgrad1, all dense."""
    dt = wl.dtype
    W1, W2 = wl.weights()
    X, dY = wl.activations()
    T, d, ff = wl.tokens, wl.d, wl.ff
    W1d, W2d = W1.cuda(), W2.cuda()
    tdt = W1.dtype
    H = torch.empty(T, ff, dtype=tdt, device="cuda")
    Hpre = torch.empty(T, ff, dtype=tdt, device="cuda")
    Y = torch.empty(T, d, dtype=tdt, device="cuda")
    dH = torch.empty(T, ff, dtype=tdt, device="cuda")
    dX = torch.empty(T, d, dtype=tdt, device="cuda")
    sp.sp24_gemm_dense(X.cuda(), W1d, H, "gelu", Hpre)
    sp.sp24_gemm_dense(H, W2d, Y)
    sp.sp24_gemm_dgrad_dense(dY.cuda(), W2d, dH, "dgelu", Hpre)
    sp.sp24_gemm_dgrad_dense(dH, W1d, dX)
    torch.cuda.synchronize()
    rows = np.arange(3, T, 32)
    w1f, w2f = oracle.to_f64(si.bits16(W1), dt), oracle.to_f64(si.bits16(W2), dt)
    pre = oracle.dense_fwd(oracle.to_f64(si.bits16(X)[rows], dt), w1f)
    assert_gemm_close(f64_of(Hpre, dt)[rows], pre, dt, "fwd1 pre-activation")
    assert_gemm_close(f64_of(H, dt)[rows], oracle.gelu(pre), dt, "fwd1 gelu")
    assert_gemm_close(f64_of(Y, dt)[rows], oracle.dense_fwd(f64_of(H, dt)[rows], w2f), dt, "fwd2")
    dh_ref = oracle.dense_dgrad(oracle.to_f64(si.bits16(dY)[rows], dt), w2f) * oracle.gelu_grad(f64_of(Hpre, dt)[rows])
    assert_gemm_close(f64_of(dH, dt)[rows], dh_ref, dt, "dgrad2 dgelu")
    assert_gemm_close(f64_of(dX, dt)[rows], oracle.dense_dgrad(f64_of(dH, dt)[rows], w1f), dt, "dgrad1")


@pytest.mark.parametrize("T,N,K,dtype", [(128, 128, 128, "f16"), (200, 256, 384, "f16"), (77, 144, 400, "bf16"),
                                         (1, 16, 16, "f16"), (300, 1600, 208, "f16"), (513, 208, 1600, "bf16"),
                                         (1000, 6400, 1600, "f16"), (640, 1600, 6400, "f16")])
def test_dense_dgrad_reads_w_as_stored(T, N, K, dtype):
    """dX = dY W with W [N x K] loaded MN-major (ragged T, K tiles of 64-column atoms, K steps
    past N): every element against the fp64 product within the fp32 accumulation bound, and
    the same bits as the product with W^T from the transpose (the same MMAs in the same K
    order; only the shared-memory layout of A differs)."""
    w = si.normal((N, K), 0.02, N + K + 1, dtype)
    dy = si.normal((T, N), 1.0, T + 2, dtype)
    wd, dyd = w.cuda(), dy.cuda()
    dx = torch.full((T, K), float("nan"), dtype=w.dtype, device="cuda")
    sp.sp24_gemm_dgrad_dense(dyd, wd, dx)
    dx_t = torch.empty_like(dx)
    sp.sp24_gemm_dense(dyd, _transpose(wd), dx_t)
    torch.cuda.synchronize()
    assert sp.sp24_device_status() == 0
    assert torch.equal(dx.view(torch.int16), dx_t.view(torch.int16))
    dyf, wf = oracle.to_f64(si.bits16(dy), dtype), oracle.to_f64(si.bits16(w), dtype)
    ref = oracle.dense_dgrad(dyf, wf)
    assert_gemm_within_accumulation_bound(f64_of(dx, dtype), ref, np.abs(dyf) @ np.abs(wf), N, dtype,
                                          f"dgrad, W as stored {T}x{N}x{K}")


@pytest.mark.parametrize("epi", ["dgelu", "mul_aux"])
def test_dense_dgrad_epilogues_read_w_as_stored(epi):
    """The input-gradient epilogues on the MN-major weight: dGELU of a stored pre-activation,
    and the product with a stored derivative."""
    T, N, K, dtype = 456, 512, 1040, "f16"
    w = si.normal((N, K), 0.02, 9, dtype)
    dy = si.normal((T, N), 1.0, 10, dtype)
    aux = si.normal((T, K), 1.0, 11, dtype)
    dx = torch.empty(T, K, dtype=w.dtype, device="cuda")
    sp.sp24_gemm_dgrad_dense(dy.cuda(), w.cuda(), dx, epi, aux.cuda())
    torch.cuda.synchronize()
    assert sp.sp24_device_status() == 0
    acc = oracle.dense_dgrad(oracle.to_f64(si.bits16(dy), dtype), oracle.to_f64(si.bits16(w), dtype))
    a = oracle.to_f64(si.bits16(aux), dtype)
    ref = acc * (oracle.gelu_grad(a) if epi == "dgelu" else a)
    assert_gemm_close(f64_of(dx, dtype), ref, dtype, f"dgrad {epi}, W as stored")


def test_dense_zero_tokens_is_a_no_op():
    w = si.normal((128, 128), 0.02, 3).cuda()
    x = torch.empty(0, 128, dtype=torch.float16, device="cuda")
    y = torch.empty(0, 128, dtype=torch.float16, device="cuda")
    sp.sp24_gemm_dense(x, w, y)
    sp.sp24_gemm_dgrad_dense(x, w, y)
    sp.sp24_gemm_dgrad_dense(x, w, y, "mul_aux", y)
    torch.cuda.synchronize()
    assert sp.sp24_device_status() == 0


def _check_wgrad(dw, ref, what=""):
    """fp32 weight gradient against the fp64 product: relative Frobenius <= 1e-4 and the
    largest entry error <= 1e-3 of max |dW| (only the fp32 accumulation rounds)."""
    got = dw.double().cpu().numpy()
    fro = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    mx = np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-300)
    assert fro <= 1e-4, f"{what}: relative Frobenius error {fro:.3e}"
    assert mx <= 1e-3, f"{what}: largest entry error {mx:.3e}"


@pytest.mark.parametrize("T,N,K,dtype", [(128, 256, 256, "f16"), (256, 272, 200, "f16"), (144, 160, 520, "bf16"),
                                         (16, 16, 8, "f16"), (2048, 512, 1024, "f16")])
def test_dense_weight_grad(T, N, K, dtype):
    """dW = dY^T X with both operands read as stored (ragged M, N and K tiles)."""
    dy = si.normal((T, N), 1.0, T + 5, dtype)
    x = si.normal((T, K), 1.0, T + 6, dtype)
    dw = torch.empty(N, K, dtype=torch.float32, device="cuda")
    sp.sp24_gemm_wgrad_dense(x.cuda(), dy.cuda(), dw)
    torch.cuda.synchronize()
    assert sp.sp24_device_status() == 0
    ref = oracle.dense_weight_grad(oracle.to_f64(si.bits16(dy), dtype), oracle.to_f64(si.bits16(x), dtype))
    _check_wgrad(dw, ref, f"dense wgrad {T}x{N}x{K}")


@pytest.mark.parametrize("wl", [si.GPT2_355M, si.GPT2_774M], ids=lambda w: w.name)
def test_dense_weight_grads_full_size_sampled_rows(wl):
    X, dY = wl.activations()
    H, dH = wl.hidden()
    rng = np.random.default_rng(2)
    for g, b in ((dY, H), (dH, X)):
        N, K = g.shape[1], b.shape[1]
        dw = torch.empty(N, K, dtype=torch.float32, device="cuda")
        sp.sp24_gemm_wgrad_dense(b.cuda(), g.cuda(), dw)
        torch.cuda.synchronize()
        assert sp.sp24_device_status() == 0
        rows = np.sort(rng.choice(N, 64, replace=False))
        gf = oracle.to_f64(si.bits16(g), wl.dtype)[:, rows]
        ref = oracle.dense_weight_grad(gf, oracle.to_f64(si.bits16(b), wl.dtype))
        _check_wgrad(dw[torch.from_numpy(rows).cuda()], ref, f"dense dW [{N}x{K}] sampled rows")
