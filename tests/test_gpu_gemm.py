"""GPU parity of the 2:4 sparse FFN GEMMs (tcgen05) against the fp64 oracle.

"Accelerating Transformer Pre-training with 2:4 Sparsity": Software
Dependencies row (2:4 sparse matrix multiplications) and abstract
(transposable masks: the input-gradient product is 2:4 too).  Each GEMM is
checked on the GPU's own inputs (a chain's later GEMM consumes the GPU's
earlier output), with the tolerance in gpu_util.  Small shapes cover several
tiles with ragged M, N and K edges; the GPT-2 FFN shapes are checked on
sampled token rows.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
import structured_sparse_transformer_b200 as sp
from gpu_util import assert_gemm_close, f64_of

pytestmark = pytest.mark.gpu


def _prep(w_cpu):
    """Mask (oracle-independent GPU search) and both compressed orientations of W on the device."""
    R, C = w_cpu.shape
    wd = w_cpu.cuda()
    idx = torch.empty(R // 4, C // 4, dtype=torch.uint8, device="cuda")
    bufs = sp.alloc_compressed(R, C, w_cpu.dtype)
    sp.sp24_mask_step(wd, idx, None, None, *bufs)
    torch.cuda.synchronize()
    return idx, bufs


def _dt(t):
    return "bf16" if t.dtype == torch.bfloat16 else "f16"


def _keep(idx):
    return oracle.dense_mask(idx.cpu().numpy())


@pytest.mark.parametrize("T,N,K,dtype", [(128, 128, 128, "f16"), (200, 256, 384, "f16"), (77, 144, 400, "bf16"),
                                         (1, 16, 16, "f16"), (300, 1600, 208, "f16"), (1024, 3072, 768, "f16"),
                                         (513, 208, 1600, "bf16")])
def test_fwd_and_dgrad_small(T, N, K, dtype):
    w = si.normal((N, K), 0.02, N + K, dtype)
    x = si.normal((T, K), 1.0, T, dtype)
    dy = si.normal((T, N), 1.0, T + 1, dtype)
    idx, (vr, mr, vc, mc) = _prep(w)
    keep = _keep(idx)
    wf = oracle.to_f64(si.bits16(w), dtype)
    y = torch.empty(T, N, dtype=w.dtype, device="cuda")
    dx = torch.empty(T, K, dtype=w.dtype, device="cuda")
    sp.sp24_gemm_fwd(x.cuda(), vr, mr, N, y)
    sp.sp24_gemm_dgrad(dy.cuda(), vc, mc, K, dx)
    torch.cuda.synchronize()
    xf = oracle.to_f64(si.bits16(x), dtype)
    dyf = oracle.to_f64(si.bits16(dy), dtype)
    assert_gemm_close(f64_of(y, dtype), oracle.sparse_fwd(xf, wf, keep), dtype, "fwd")
    assert_gemm_close(f64_of(dx, dtype), oracle.sparse_dgrad(dyf, wf, keep), dtype, "dgrad")


def test_one_hot_tokens_return_pruned_weight_rows():
    N, K = 256, 256
    w = si.normal((N, K), 0.02, 42)
    idx, (vr, mr, vc, mc) = _prep(w)
    eye = torch.eye(K, dtype=torch.float16).cuda()
    y = torch.empty(K, N, dtype=torch.float16, device="cuda")
    sp.sp24_gemm_fwd(eye, vr, mr, N, y)
    torch.cuda.synchronize()
    pruned = oracle.prune(si.bits16(w), idx.cpu().numpy())
    assert np.array_equal(si.bits16(y.cpu()), np.ascontiguousarray(pruned.T))


@pytest.mark.parametrize("wl", [si.GPT2_355M, si.GPT2_774M], ids=lambda w: w.name)
def test_ffn_chain_with_gelu_sampled_rows(wl):
    """fwd1 (+GELU, aux = pre-activation) -> fwd2; dY -> dgrad2 (+dGELU with aux) -> dgrad1."""
    dt = wl.dtype
    W1, W2 = wl.weights()
    X, dY = wl.activations()
    T, d, ff = wl.tokens, wl.d, wl.ff
    i1, (vr1, mr1, vc1, mc1) = _prep(W1)
    i2, (vr2, mr2, vc2, mc2) = _prep(W2)
    tdt = W1.dtype
    H = torch.empty(T, ff, dtype=tdt, device="cuda")
    Hpre = torch.empty(T, ff, dtype=tdt, device="cuda")
    Y = torch.empty(T, d, dtype=tdt, device="cuda")
    dH = torch.empty(T, ff, dtype=tdt, device="cuda")
    dX = torch.empty(T, d, dtype=tdt, device="cuda")
    Xd, dYd = X.cuda(), dY.cuda()
    sp.sp24_gemm_fwd(Xd, vr1, mr1, ff, H, "gelu", Hpre)
    sp.sp24_gemm_fwd(H, vr2, mr2, d, Y)
    sp.sp24_gemm_dgrad(dYd, vc2, mc2, ff, dH, "dgelu", Hpre)
    sp.sp24_gemm_dgrad(dH, vc1, mc1, d, dX)
    torch.cuda.synchronize()
    rows = np.arange(0, T, 16)
    k1, k2 = _keep(i1), _keep(i2)
    w1f, w2f = oracle.to_f64(si.bits16(W1), dt), oracle.to_f64(si.bits16(W2), dt)
    xs = oracle.to_f64(si.bits16(X)[rows], dt)
    pre = oracle.sparse_fwd(xs, w1f, k1)
    assert_gemm_close(f64_of(Hpre, dt)[rows], pre, dt, "fwd1 pre-activation")
    hpre_gpu = f64_of(Hpre, dt)[rows]
    assert_gemm_close(f64_of(H, dt)[rows], oracle.gelu(pre), dt, "fwd1 gelu")
    h_gpu = f64_of(H, dt)[rows]
    assert_gemm_close(f64_of(Y, dt)[rows], oracle.sparse_fwd(h_gpu, w2f, k2), dt, "fwd2")
    dys = oracle.to_f64(si.bits16(dY)[rows], dt)
    dh_ref = oracle.sparse_dgrad(dys, w2f, k2) * oracle.gelu_grad(hpre_gpu)
    assert_gemm_close(f64_of(dH, dt)[rows], dh_ref, dt, "dgrad2 dgelu")
    dh_gpu = f64_of(dH, dt)[rows]
    assert_gemm_close(f64_of(dX, dt)[rows], oracle.sparse_dgrad(dh_gpu, w1f, k1), dt, "dgrad1")


def test_gemm_1p5b_shapes_sampled_rows():
    wl = si.GPT2_1P5B
    W1, W2 = wl.weights()
    X, dY = wl.activations()
    T, d, ff = wl.tokens, wl.d, wl.ff
    i1, (vr1, mr1, vc1, mc1) = _prep(W1)
    i2, (vr2, mr2, vc2, mc2) = _prep(W2)
    H = torch.empty(T, ff, dtype=W1.dtype, device="cuda")
    dX = torch.empty(T, d, dtype=W1.dtype, device="cuda")
    Xd = X.cuda()
    sp.sp24_gemm_fwd(Xd, vr1, mr1, ff, H)
    sp.sp24_gemm_dgrad(H, vc1, mc1, d, dX)
    torch.cuda.synchronize()
    rows = np.arange(7, T, 64)
    w1f = oracle.to_f64(si.bits16(W1), "f16")
    k1 = _keep(i1)
    assert_gemm_close(f64_of(H, "f16")[rows], oracle.sparse_fwd(oracle.to_f64(si.bits16(X)[rows], "f16"), w1f, k1),
                      "f16", "fwd 1.5B")
    assert_gemm_close(f64_of(dX, "f16")[rows], oracle.sparse_dgrad(f64_of(H, "f16")[rows], w1f, k1), "f16",
                      "dgrad 1.5B")


def test_wait_timeout_reports_status_and_context_survives():
    N, K, T = 256, 512, 256
    w = si.normal((N, K), 0.02, 1)
    x = si.normal((T, K), 1.0, 2).cuda()
    idx, (vr, mr, vc, mc) = _prep(w)
    y = torch.zeros(T, N, dtype=torch.float16, device="cuda")
    assert sp.sp24_device_status() == 0
    sp.sp24_set_wait_budget(0)
    try:
        sp.sp24_gemm_fwd(x, vr, mr, N, y)
        assert sp.sp24_device_status() == 6          # SP24_ERR_TIMEOUT
    finally:
        sp.sp24_set_wait_budget(1 << 32)
    sp.sp24_gemm_fwd(x, vr, mr, N, y)
    assert sp.sp24_device_status() == 0
    ref = oracle.sparse_fwd(oracle.to_f64(si.bits16(x.cpu()), "f16"), oracle.to_f64(si.bits16(w), "f16"), _keep(idx))
    assert_gemm_close(f64_of(y, "f16"), ref, "f16", "after timeout")


def test_zero_tokens_is_a_no_op():
    w = si.normal((128, 128), 0.02, 3)
    _, (vr, mr, vc, mc) = _prep(w)
    x = torch.empty(0, 128, dtype=torch.float16, device="cuda")
    y = torch.empty(0, 128, dtype=torch.float16, device="cuda")
    sp.sp24_gemm_fwd(x, vr, mr, 128, y)
    assert sp.sp24_device_status() == 0


def test_metadata_layout_probe():
    """The tensor cores read the metadata exactly where the host layout map says.

    All-ones kept values and code 0x4 (keep offsets 0, 1) everywhere give
    out[t][m] = 1 for t % 4 in {0, 1}.  Setting one nibble of the device buffer
    to 0xE (keep 2, 3) must move exactly that row's group to offsets 2, 3, at the
    (row, group) that sp24_meta_to_canonical assigns to that nibble."""
    M = Kd = 128
    vals = torch.ones(M, Kd // 2, dtype=torch.float16, device="cuda")
    x = torch.eye(Kd, dtype=torch.float16, device="cuda")
    base = np.full(2048, 0x44, dtype=np.uint8)
    probes = [(L, 0, 0) for L in range(0, 128, 3)] + [(0, kk, e) for kk in range(4) for e in range(8)] + \
             [(L, kk, e) for L in (5, 13, 21, 77, 126) for kk in (1, 3) for e in (3, 4, 7)]
    for (L, kk, e) in probes:
        meta = base.copy()
        pos = L * 16 + kk * 4 + e // 2
        meta[pos] = (meta[pos] & 0xF0) | 0x0E if e % 2 == 0 else (meta[pos] & 0x0F) | 0xE0
        y = torch.empty(Kd, M, dtype=torch.float16, device="cuda")
        sp.sp24_gemm_fwd(x, vals, torch.from_numpy(meta).cuda(), M, y)
        torch.cuda.synchronize()
        canon = sp.sp24_meta_to_canonical(meta.tobytes(), M, Kd)
        rows, words = np.nonzero(canon != 0x4444)
        assert len(rows) == 1
        r, w = int(rows[0]), int(words[0])
        nib = [k for k in range(4) if (canon[r, w] >> (4 * k)) & 0xF == 0xE]
        assert len(nib) == 1
        g = 4 * w + nib[0]
        expect = np.zeros((Kd, M), np.float32)
        expect[np.arange(Kd) % 4 < 2, :] = 1.0
        expect[4 * g:4 * g + 2, r] = 0.0
        expect[4 * g + 2:4 * g + 4, r] = 1.0
        assert np.array_equal(y.float().cpu().numpy(), expect), (L, kk, e, r, g)
