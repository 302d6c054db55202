"""Pins of the oracle's canonical compression and fp64 FFN GEMMs.

Compression: the pages only name the semi-structured conversion routines
("Accelerating Transformer Pre-training with 2:4 Sparsity", abstract page, code
samples), so the canonical layout is pinned by hand-built examples and by the
round trip ``decompress(compress(W, m)) == W * m``.  GEMMs: software
dependencies row (2:4 sparse matrix multiplications) and the abstract
(transposable masks keep the backward product 2:4); pinned by one-hot inputs,
exact integer arithmetic and a contraction identity.
"""
import math

import numpy as np
import torch

import oracle
import synthetic_inputs as si


def _bits(x, dtype="f16"):
    return si.bits16(torch.tensor(np.asarray(x, np.float32)).to(si.DTYPES[dtype]))


def test_compress_hand_example():
    # Row: groups [a 0 b 0], [0 c d 0], [0 0 e f], [g 0 0 h] with masks
    # (0,2), (1,2), (2,3), (0,3) -> nibbles 0x8, 0x9, 0xE, 0xC.
    row = np.array([[1, 0, 2, 0, 0, 3, 4, 0, 0, 0, 5, 6, 7, 0, 0, 8]], np.float32)
    keep = row != 0
    vals, meta = oracle.compress_rows(_bits(row), keep)
    assert np.array_equal(oracle.to_f64(vals, "f16"), [[1, 2, 3, 4, 5, 6, 7, 8]])
    assert meta.tolist() == [[0x8 | 0x9 << 4 | 0xE << 8 | 0xC << 12]]


def test_kept_zero_keeps_its_slot():
    row = np.array([[0, 0, 2, 0]], np.float32)
    keep = np.array([[True, False, True, False]])
    vals, meta = oracle.compress_rows(_bits(row), keep)
    assert meta[0, 0] & 0xF == 0x8
    assert oracle.to_f64(vals, "f16").tolist() == [[0.0, 2.0]]


def test_compress_roundtrip_and_codes_both_orientations():
    w = si.normal((96, 160), 0.02, seed=5, dtype="bf16")
    bits = si.bits16(w)
    idx = oracle.mask_search(bits, "bf16")
    (vr, mr), (vc, mc) = oracle.compress_both(bits, idx)
    pruned = oracle.prune(bits, idx)
    assert np.array_equal(oracle.decompress_rows(vr, mr, 160), pruned)
    assert np.array_equal(oracle.decompress_rows(vc, mc, 96), np.ascontiguousarray(pruned.T))
    for meta in (mr, mc):
        nibbles = np.stack([(meta >> (4 * k)) & 0xF for k in range(4)]).reshape(-1)
        assert set(np.unique(nibbles).tolist()) <= set(oracle.NIBBLE_CODES)
    assert vr.shape == (96, 80) and vc.shape == (160, 48)


def test_fwd_with_identity_returns_pruned_weight():
    w = si.normal((32, 48), 0.02, seed=2, dtype="f16")
    bits = si.bits16(w)
    idx = oracle.mask_search(bits, "f16")
    keep = oracle.dense_mask(idx)
    wf = oracle.to_f64(bits, "f16")
    y = oracle.sparse_fwd(np.eye(48), wf, keep)            # [48 tokens, 32 out]
    assert np.array_equal(y, oracle.to_f64(oracle.prune(bits, idx), "f16").T)
    dx = oracle.sparse_dgrad(np.eye(32), wf, keep)         # [32 tokens, 48 in]
    assert np.array_equal(dx, oracle.to_f64(oracle.prune(bits, idx), "f16"))


def test_gemm_exact_on_small_integers():
    rng = np.random.default_rng(0)
    T, N, K = 5, 8, 12
    x = rng.integers(-9, 10, (T, K)).astype(np.float64)
    dy = rng.integers(-9, 10, (T, N)).astype(np.float64)
    w = rng.integers(-9, 10, (N, K)).astype(np.float64)
    keep = oracle.dense_mask(rng.integers(0, 90, (N // 4, K // 4)).astype(np.uint8))
    y = oracle.sparse_fwd(x, w, keep)
    dx = oracle.sparse_dgrad(dy, w, keep)
    for t in range(T):
        for n in range(N):
            assert y[t, n] == sum(int(x[t, k]) * int(w[n, k]) for k in range(K) if keep[n, k])
        for k in range(K):
            assert dx[t, k] == sum(int(dy[t, n]) * int(w[n, k]) for n in range(N) if keep[n, k])


def test_fwd_dgrad_adjoint_identity():
    # <dY, X (W*m)^T> == <dY (W*m), X>: the two products use the same pruned matrix.
    rng = np.random.default_rng(1)
    x, dy = rng.normal(size=(7, 64)), rng.normal(size=(7, 32))
    w = rng.normal(size=(32, 64))
    keep = oracle.dense_mask(rng.integers(0, 90, (8, 16)).astype(np.uint8))
    lhs = np.sum(dy * oracle.sparse_fwd(x, w, keep))
    rhs = np.sum(oracle.sparse_dgrad(dy, w, keep) * x)
    assert abs(lhs - rhs) < 1e-10 * max(1.0, abs(lhs))


def test_gelu_closed_forms():
    phi1 = 0.5 * (1 + math.erf(1 / math.sqrt(2)))
    assert abs(phi1 - 0.8413447460685429) < 1e-15            # standard normal CDF at 1
    g = oracle.gelu(np.array([0.0, 1.0, -1.0, 30.0, -30.0]))
    assert g[0] == 0.0
    assert abs(g[1] - 0.8413447460685429) < 1e-15
    assert abs(g[2] + 0.15865525393145707) < 1e-15
    assert g[3] == 30.0 and abs(g[4]) < 1e-150
    x = np.linspace(-6, 6, 101)
    assert np.allclose(oracle.gelu(x) - oracle.gelu(-x), x, atol=1e-14)
    h = 1e-5
    fd = (oracle.gelu(x + h) - oracle.gelu(x - h)) / (2 * h)
    assert np.allclose(oracle.gelu_grad(x), fd, atol=1e-9)
    assert abs(oracle.gelu_grad(np.array([0.0]))[0] - 0.5) < 1e-15


def test_dense_gemms_exact_on_small_integers_and_adjoint():
    """Dense fine-tuning products: exact integer sums by explicit loops, the
    adjoint identity, and the one-hot case returning W (and W^T) itself."""
    rng = np.random.default_rng(3)
    T, N, K = 4, 8, 12
    x = rng.integers(-9, 10, (T, K)).astype(np.float64)
    dy = rng.integers(-9, 10, (T, N)).astype(np.float64)
    w = rng.integers(-9, 10, (N, K)).astype(np.float64)
    y, dx = oracle.dense_fwd(x, w), oracle.dense_dgrad(dy, w)
    for t in range(T):
        for n in range(N):
            assert y[t, n] == sum(int(x[t, k]) * int(w[n, k]) for k in range(K))
        for k in range(K):
            assert dx[t, k] == sum(int(dy[t, n]) * int(w[n, k]) for n in range(N))
    xr, dyr, wr = rng.normal(size=(5, 24)), rng.normal(size=(5, 16)), rng.normal(size=(16, 24))
    lhs = np.sum(dyr * oracle.dense_fwd(xr, wr))
    rhs = np.sum(oracle.dense_dgrad(dyr, wr) * xr)
    assert abs(lhs - rhs) < 1e-10 * max(1.0, abs(lhs))
    assert np.array_equal(oracle.dense_fwd(np.eye(K), w), w.T)
    assert np.array_equal(oracle.dense_dgrad(np.eye(N), w), w)


def test_dense_weight_grad_is_the_adjoint_of_the_forward_product():
    """<dW, W> = <dY, X W^T> for any W: the weight gradient of the dense phase is the
    gradient of <dY, Y> with respect to W.  Exact on small integers; explicit loops too."""
    rng = np.random.default_rng(7)
    T, N, K = 6, 5, 7
    x = rng.integers(-9, 10, (T, K)).astype(np.float64)
    dy = rng.integers(-9, 10, (T, N)).astype(np.float64)
    dw = oracle.dense_weight_grad(dy, x)
    assert dw.shape == (N, K)
    for n in range(N):
        for k in range(K):
            assert dw[n, k] == sum(int(dy[t, n]) * int(x[t, k]) for t in range(T))
    for _ in range(3):
        w = rng.integers(-9, 10, (N, K)).astype(np.float64)
        assert np.sum(dw * w) == np.sum(dy * oracle.dense_fwd(x, w))


def test_gate_up_interleave_and_split_are_inverse():
    rng = np.random.default_rng(5)
    wg, wu = rng.normal(size=(48, 8)), rng.normal(size=(48, 8))
    w = oracle.interleave_gate_up(wg, wu)
    assert np.array_equal(w[0:16], wg[0:16]) and np.array_equal(w[16:32], wu[0:16])
    assert np.array_equal(w[32:48], wg[16:32]) and np.array_equal(w[80:96], wu[32:48])
    # the columns of X W^T split back into X W_gate^T and X W_up^T
    x = rng.normal(size=(5, 8))
    g, u = oracle.split_gate_up(x @ w.T)
    assert np.allclose(g, x @ wg.T, rtol=0, atol=1e-12) and np.allclose(u, x @ wu.T, rtol=0, atol=1e-12)


def test_geglu_closed_forms_and_finite_differences():
    assert oracle.geglu(np.array([0.0]), np.array([3.0]))[0] == 0.0
    assert oracle.geglu(np.array([2.0]), np.array([0.0]))[0] == 0.0
    dg, du = oracle.geglu_grad(np.array([1.0]), np.array([0.0]), np.array([3.0]))
    assert dg[0] == 1.5 and du[0] == 0.0                  # gelu'(0) = 1/2, gelu(0) = 0
    rng = np.random.default_rng(6)
    g, u, dh = rng.normal(size=64) * 2, rng.normal(size=64), rng.normal(size=64)
    eps = 1e-6
    fd_g = (oracle.geglu(g + eps, u) - oracle.geglu(g - eps, u)) / (2 * eps)
    fd_u = (oracle.geglu(g, u + eps) - oracle.geglu(g, u - eps)) / (2 * eps)
    dg, du = oracle.geglu_grad(dh, g, u)
    assert np.allclose(dg, dh * fd_g, rtol=1e-6, atol=1e-8)
    assert np.allclose(du, dh * fd_u, rtol=1e-6, atol=1e-8)
