"""GPU parity of the MVUE sparsification of dY^T and of the weight-gradient GEMM.

"Accelerating Transformer Pre-training with 2:4 Sparsity", reproducibility
table, Software Dependencies row (the MVUE kernel, the 2:4 sparse matrix
multiplications).  The sparsified operand is integer-decided work (which two
of four tokens, in fp64 on both sides, from the same Philox draws), so its
values and metadata must equal the oracle's bit for bit.  The weight gradient
dW = Yhat X is fp32 out of fp32 tensor-core accumulation over T tokens; it is
compared with the fp64 product of the GPU's own Yhat with a relative Frobenius
error <= 1e-4 and a largest entry error <= 1e-3 of the largest |dW| (fp16/bf16
products are exact in fp32, so only the accumulation rounds: about
sqrt(T) * 2^-24 relative, 5e-6 at T = 8192).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
import structured_sparse_transformer_b200 as sp

pytestmark = pytest.mark.gpu

FRO_TOL = 1e-4
MAX_TOL = 1e-3


def _alloc(N, T, dtype):
    vb, mb = sp.sp24_compressed_size(N, T)
    return (torch.empty(N, T // 2, dtype=si.DTYPES[dtype], device="cuda"),
            torch.empty(mb, dtype=torch.uint8, device="cuda"))


def _yhat_of(vals, meta, N, T, dtype):
    """Dense bits [N, T] of the GPU's compressed operand (host index maps only)."""
    canon = sp.sp24_meta_to_canonical(meta.cpu().numpy().tobytes(), N, T)
    return oracle.decompress_rows(si.bits16(vals.cpu()), canon, T), canon


def _mixed_dy(T, N, dtype, seed):
    """N(0, 1) with planted special groups: all zero, one, two or three nonzeros,
    one dominant entry (the capped case) and equal magnitudes (ties)."""
    x = si.normal((T, N), 1.0, seed, dtype).float()
    g = torch.Generator().manual_seed(seed + 1)
    kind = torch.randint(0, 7, (T // 4, N), generator=g)
    grp = x.reshape(T // 4, 4, N).permute(0, 2, 1)          # [group, column, 4], a view of x
    grp[kind == 1] = 0.0
    grp[..., 1:][kind == 2] = 0.0
    grp[..., 2:][kind == 3] = 0.0
    grp[..., 0][kind == 4] *= 50.0
    grp[kind == 5] = 0.5 * torch.sign(grp[kind == 5])
    grp[..., 3][kind == 6] = 0.0
    return x.to(si.DTYPES[dtype]).contiguous()


@pytest.mark.parametrize("T,N,dtype", [(128, 64, "f16"), (256, 128, "f16"), (144, 200, "bf16"), (16, 8, "f16"),
                                       (1040, 776, "f16"), (512, 256, "bf16")])
def test_mvue_bit_exact(T, N, dtype):
    dy = _mixed_dy(T, N, dtype, T + N)
    vals, meta = _alloc(N, T, dtype)
    sp.sp24_mvue_sparsify(dy.cuda(), 17, 5, vals, meta)
    torch.cuda.synchronize()
    assert sp.sp24_device_status() == 0
    bits, keep, _ = oracle.mvue_sparsify_t(si.bits16(dy), dtype, 17, 5)
    ovals, ometa = oracle.compress_rows(bits, keep)
    assert np.array_equal(si.bits16(vals.cpu()), ovals)
    got, canon = _yhat_of(vals, meta, N, T, dtype)
    assert np.array_equal(canon, ometa)
    assert np.array_equal(got, bits)


def test_mvue_leading_dimension_and_wide_bf16_groups():
    T, N, ld = 64, 16, 40
    base = torch.zeros(T, ld)
    base[:, :N] = torch.randn(T, N, generator=torch.Generator().manual_seed(3))
    base[0::4, :N] *= 1e30        # groups spanning ~100 binades
    base[1::4, :N] *= 1e-30
    dy = base.to(torch.bfloat16)
    vals, meta = _alloc(N, T, "bf16")
    sp.sp24_mvue_sparsify(dy.cuda()[:, :N], 1, 2, vals, meta)
    torch.cuda.synchronize()
    bits, keep, _ = oracle.mvue_sparsify_t(si.bits16(dy[:, :N].contiguous()), "bf16", 1, 2)
    got, _ = _yhat_of(vals, meta, N, T, "bf16")
    assert np.array_equal(got, bits)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_mvue_raw_bit_groups_over_wide_exponent_spans(dtype):
    """Groups of raw bits whose nonzero exponent fields span 0 to 24 binades, with
    subnormals, zeros, the largest finite values (whose estimates S/2 overflow to
    infinity on both sides) and random signs."""
    T, N = 512, 192
    mant, emax_field = (10, 30) if dtype == "f16" else (7, 254)
    rng = np.random.default_rng(23 if dtype == "f16" else 24)
    G = T // 4 * N
    span = rng.integers(0, 25, G)
    top = rng.integers(np.minimum(span, emax_field - 1), emax_field + 1)   # largest exponent field
    e = top[:, None] - rng.integers(0, span[:, None] + 1, (G, 4))
    e[:, 0] = np.where(rng.random(G) < 0.5, top, e[:, 0])
    e = np.clip(e, 0, emax_field)
    m = rng.integers(0, 1 << mant, (G, 4))
    m[rng.random((G, 4)) < 0.05] = (1 << mant) - 1                        # with e = top: the largest finite
    bits = (e << mant) | m
    bits[rng.random((G, 4)) < 0.1] = 0
    bits |= rng.integers(0, 2, (G, 4)) << 15
    bits = bits.astype(np.uint16).reshape(T // 4, N, 4).transpose(0, 2, 1).reshape(T, N)
    dy = torch.from_numpy(bits.view(np.int16)).view(si.DTYPES[dtype])
    vals, meta = _alloc(N, T, dtype)
    sp.sp24_mvue_sparsify(dy.cuda(), 5, 9, vals, meta)
    torch.cuda.synchronize()
    assert sp.sp24_device_status() == 0
    obits, keep, _ = oracle.mvue_sparsify_t(np.ascontiguousarray(bits), dtype, 5, 9)
    ovals, ometa = oracle.compress_rows(obits, keep)
    assert np.array_equal(si.bits16(vals.cpu()), ovals)
    got, canon = _yhat_of(vals, meta, N, T, dtype)
    assert np.array_equal(canon, ometa)


def test_mvue_draws_depend_on_seed_and_offset_only():
    T, N = 256, 64
    dy = si.normal((T, N), 1.0, 9, "f16").cuda()
    outs = []
    for seed, off in ((1, 1), (1, 1), (1, 2), (2, 1)):
        vals, meta = _alloc(N, T, "f16")
        sp.sp24_mvue_sparsify(dy, seed, off, vals, meta)
        torch.cuda.synchronize()
        outs.append(meta.cpu().numpy())
    assert np.array_equal(outs[0], outs[1])
    assert not np.array_equal(outs[0], outs[2]) and not np.array_equal(outs[0], outs[3])


def _check_wgrad(dw, ref, what=""):
    got = dw.double().cpu().numpy()
    fro = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    mx = np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-300)
    assert fro <= FRO_TOL, f"{what}: relative Frobenius error {fro:.3e}"
    assert mx <= MAX_TOL, f"{what}: largest entry error {mx:.3e} of max |dW|"


@pytest.mark.parametrize("T,N,K,dtype", [(128, 256, 256, "f16"), (256, 272, 200, "f16"), (144, 160, 520, "bf16"),
                                         (16, 16, 8, "f16"), (2048, 512, 1024, "f16"), (400, 1040, 264, "bf16")])
def test_wgrad_small(T, N, K, dtype):
    dy = si.normal((T, N), 1.0, T + 3, dtype)
    x = si.normal((T, K), 1.0, T + 4, dtype)
    vals, meta = _alloc(N, T, dtype)
    dw = torch.empty(N, K, dtype=torch.float32, device="cuda")
    sp.sp24_mvue_sparsify(dy.cuda(), 11, 0, vals, meta)
    sp.sp24_gemm_wgrad(x.cuda(), vals, meta, N, dw)
    torch.cuda.synchronize()
    assert sp.sp24_device_status() == 0
    yhat, _ = _yhat_of(vals, meta, N, T, dtype)
    ref = oracle.weight_grad(oracle.to_f64(yhat, dtype), oracle.to_f64(si.bits16(x), dtype))
    _check_wgrad(dw, ref, f"wgrad {T}x{N}x{K}")


@pytest.mark.parametrize("T,N,K,dtype", [(1024, 2560, 2048, "f16"), (896, 2608, 1800, "bf16")])
def test_wgrad_stream_k_full_matrix(T, N, K, dtype):
    """dW with more tiles than CTA pairs and not a multiple of them (80 and 88 tiles of
    256 x 256 on 74 pairs): the stream-K schedule, where two pairs share a tile's K
    steps and one adds the other's partial.  Every entry against the fp64 product
    of the GPU's own Yhat, and the same bits from a second call."""
    dy = si.normal((T, N), 1.0, T + 5, dtype)
    x = si.normal((T, K), 1.0, T + 6, dtype)
    vals, meta = _alloc(N, T, dtype)
    sp.sp24_mvue_sparsify(dy.cuda(), 13, 2, vals, meta)
    xd = x.cuda()
    dw = torch.empty(N, K, dtype=torch.float32, device="cuda")
    again = torch.full((N, K), float("nan"), dtype=torch.float32, device="cuda")
    sp.sp24_gemm_wgrad(xd, vals, meta, N, dw)
    sp.sp24_gemm_wgrad(xd, vals, meta, N, again)
    torch.cuda.synchronize()
    assert sp.sp24_device_status() == 0
    assert torch.equal(dw.view(torch.int32), again.view(torch.int32))
    yhat, _ = _yhat_of(vals, meta, N, T, dtype)
    ref = oracle.weight_grad(oracle.to_f64(yhat, dtype), oracle.to_f64(si.bits16(x), dtype))
    _check_wgrad(dw, ref, f"wgrad {T}x{N}x{K}")


def test_wgrad_stream_k_timeout_reports_status_and_next_call_is_exact():
    """A zero wait budget makes the stream-K launch give up (no bounded wait can
    succeed late); the status reports it and clears any ready counter left raised,
    so the next launch with the normal budget gives the same bits as before."""
    T, N, K, dtype = 1024, 2560, 2048, "f16"
    dy = si.normal((T, N), 1.0, 41, dtype)
    x = si.normal((T, K), 1.0, 42, dtype).cuda()
    vals, meta = _alloc(N, T, dtype)
    sp.sp24_mvue_sparsify(dy.cuda(), 3, 4, vals, meta)
    good = torch.empty(N, K, dtype=torch.float32, device="cuda")
    sp.sp24_gemm_wgrad(x, vals, meta, N, good)
    assert sp.sp24_device_status() == 0
    dw = torch.zeros(N, K, dtype=torch.float32, device="cuda")
    sp.sp24_set_wait_budget(0)
    try:
        sp.sp24_gemm_wgrad(x, vals, meta, N, dw)
        assert sp.sp24_device_status() == 6          # SP24_ERR_TIMEOUT
    finally:
        sp.sp24_set_wait_budget(1 << 32)
    sp.sp24_gemm_wgrad(x, vals, meta, N, dw)
    assert sp.sp24_device_status() == 0
    assert torch.equal(dw.view(torch.int32), good.view(torch.int32))


def test_wgrad_zero_tokens_gives_zeros():
    N, K = 32, 16
    dw = torch.full((N, K), 7.0, device="cuda")
    x = torch.empty(0, K, dtype=torch.float16, device="cuda")
    vals, meta = _alloc(N, 16, "f16")
    sp.sp24_gemm_wgrad(x, vals, meta, N, dw)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dw).item() == 0


@pytest.mark.parametrize("wl", [si.GPT2_355M], ids=lambda w: w.name)
def test_ffn_weight_grads_full_size_sampled(wl):
    """Both weight gradients of the FFN at full size: dW2 = MVUE(dY^T) H and
    dW1 = MVUE(dH^T) X.  The sparsified operands are compared in full; dW on
    96 sampled rows (all columns) against the fp64 oracle."""
    dt = wl.dtype
    X, dY = wl.activations()
    H, dH = wl.hidden()
    T = wl.tokens
    rng = np.random.default_rng(0)
    for (g, b, N, K, off) in ((dY, H, wl.d, wl.ff, 1), (dH, X, wl.ff, wl.d, 2)):
        vals, meta = _alloc(N, T, dt)
        dw = torch.empty(N, K, dtype=torch.float32, device="cuda")
        sp.sp24_mvue_sparsify(g.cuda(), wl.seeds["mvue"], off, vals, meta)
        sp.sp24_gemm_wgrad(b.cuda(), vals, meta, N, dw)
        torch.cuda.synchronize()
        assert sp.sp24_device_status() == 0
        bits, keep, _ = oracle.mvue_sparsify_t(si.bits16(g), dt, wl.seeds["mvue"], off)
        ovals, _ = oracle.compress_rows(bits, keep)
        assert np.array_equal(si.bits16(vals.cpu()), ovals)
        rows = np.sort(rng.choice(N, 96, replace=False))
        ref = oracle.weight_grad(oracle.to_f64(bits[rows], dt), oracle.to_f64(si.bits16(b), dt))
        _check_wgrad(dw[torch.from_numpy(rows).cuda()], ref, f"dW [{N}x{K}] sampled rows")


@pytest.mark.parametrize("wl", [si.GPT2_774M], ids=lambda w: w.name)
def test_ffn_weight_grads_full_size_column_sample(wl):
    """Both weight gradients of the 774M FFN (bf16, 16384 tokens) at full size; the
    sparsified operands are compared on 160 sampled columns of dY / dH (the oracle draws
    from the columns' indices in the full matrices), dW on the same 160 rows."""
    dt = wl.dtype
    X, dY = wl.activations()
    H, dH = wl.hidden()
    T = wl.tokens
    rng = np.random.default_rng(1)
    for (g, b, N, K, off) in ((dY, H, wl.d, wl.ff, 3), (dH, X, wl.ff, wl.d, 4)):
        vals, meta = _alloc(N, T, dt)
        dw = torch.empty(N, K, dtype=torch.float32, device="cuda")
        sp.sp24_mvue_sparsify(g.cuda(), wl.seeds["mvue"], off, vals, meta)
        sp.sp24_gemm_wgrad(b.cuda(), vals, meta, N, dw)
        torch.cuda.synchronize()
        assert sp.sp24_device_status() == 0
        start = int(rng.integers(0, N // 32)) * 32
        rows = np.arange(start, start + 160) % N
        gb = si.bits16(g)
        bf = oracle.to_f64(si.bits16(b), dt)
        got_vals = si.bits16(vals.cpu())
        for r0 in range(0, 160, 32):
            cols = rows[r0:r0 + 32]
            if cols[-1] < cols[0]:
                continue
            bits, keep, _ = oracle.mvue_sparsify_t(np.ascontiguousarray(gb[:, cols[0]:cols[-1] + 1]), dt,
                                                   wl.seeds["mvue"], off, col0=int(cols[0]))
            ovals, _ = oracle.compress_rows(bits, keep)
            assert np.array_equal(got_vals[cols[0]:cols[-1] + 1], ovals)
            ref = oracle.weight_grad(oracle.to_f64(bits, dt), bf)
            _check_wgrad(dw[int(cols[0]):int(cols[-1]) + 1], ref, f"dW [{N}x{K}] rows {cols[0]}..")


def test_ffn_weight_grads_1p5b_sampled_rows_and_columns():
    """Both weight gradients of the 1.5B FFN (fp16, 32768 tokens) at full size: dW1 [6400 x 1600]
    has a ragged last column tile (1600 = 6 x 256 + 64).  The sparsified operand is compared on
    64 columns of dY / dH, dW on those 64 rows x 96 columns (the last 32 in the ragged tile)."""
    wl = si.GPT2_1P5B
    dt = wl.dtype
    X, dY = wl.activations()
    H, dH = wl.hidden()
    T = wl.tokens
    rng = np.random.default_rng(5)
    for (g, b, N, K, off) in ((dY, H, wl.d, wl.ff, 5), (dH, X, wl.ff, wl.d, 6)):
        vals, meta = _alloc(N, T, dt)
        dw = torch.empty(N, K, dtype=torch.float32, device="cuda")
        sp.sp24_mvue_sparsify(g.cuda(), wl.seeds["mvue"], off, vals, meta)
        sp.sp24_gemm_wgrad(b.cuda(), vals, meta, N, dw)
        torch.cuda.synchronize()
        assert sp.sp24_device_status() == 0
        r0 = int(rng.integers(0, (N - 64) // 32)) * 32
        cols = np.concatenate([np.sort(rng.choice(K - 32, 64, replace=False)), np.arange(K - 32, K)])
        bits, keep, _ = oracle.mvue_sparsify_t(np.ascontiguousarray(si.bits16(g)[:, r0:r0 + 64]), dt,
                                               wl.seeds["mvue"], off, col0=r0)
        ovals, _ = oracle.compress_rows(bits, keep)
        assert np.array_equal(si.bits16(vals[r0:r0 + 64].cpu()), ovals)
        bf = oracle.to_f64(np.ascontiguousarray(si.bits16(b)[:, cols]), dt)
        ref = oracle.weight_grad(oracle.to_f64(bits, dt), bf)
        got = dw[r0:r0 + 64][:, torch.from_numpy(cols).cuda()]
        _check_wgrad(got, ref, f"dW [{N}x{K}] rows {r0}.. sampled columns")


@pytest.mark.parametrize("T,N,K,dtype", [(256, 128, 136, "f16"), (512, 272, 520, "bf16"), (1024, 4096, 1024, "f16"),
                                         (2048, 1600, 6400, "f16"), (0, 64, 64, "f16")])
def test_wgrad_decay_fused_equals_separate_passes(T, N, K, dtype):
    """sp24_gemm_wgrad_decay = sp24_gemm_wgrad then sp24_masked_decay, bit for bit, and that
    equals the oracle's masked decay (an fp32 fused multiply-add per pruned entry) of the
    GPU's own undecayed gradient.  Ragged dW tiles (N, K not multiples of 256) included."""
    tdt = si.DTYPES[dtype]
    w = si.normal((N, K), 0.02, N + K, dtype)
    x = si.normal((max(T, 16), K), 1.0, T + 3, dtype)[:T].contiguous()
    dy = si.normal((max(T, 16), N), 1.0, T + 4, dtype)[:T].contiguous()
    wd, xd = w.cuda(), x.cuda()
    idx = torch.empty(N // 4, K // 4, dtype=torch.uint8, device="cuda")
    sp.sp24_mask_search(wd, idx)
    vals, meta = _alloc(N, max(T, 16), dtype)
    if T:
        sp.sp24_mvue_sparsify(dy.cuda(), 31, 7, vals, meta)
    lam = 6e-5
    plain = torch.empty(N, K, dtype=torch.float32, device="cuda")
    fused = torch.full((N, K), float("nan"), dtype=torch.float32, device="cuda")
    if T:
        sp.sp24_gemm_wgrad(xd, vals, meta, N, plain)
        sp.sp24_gemm_wgrad_decay(xd, vals, meta, N, wd, idx, lam, fused)
    else:
        # an empty token range: the decay of a zero gradient
        lib = sp.lib()
        import ctypes
        z = ctypes.c_void_p(0)
        plain.zero_()
        st = lib.sp24_gemm_wgrad_decay(z, 0, K, z, z, N, 0, ctypes.c_void_p(wd.data_ptr()),
                                       ctypes.c_void_p(idx.data_ptr()), ctypes.c_float(lam),
                                       ctypes.c_void_p(fused.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0
    undecayed = plain.cpu().numpy().copy()
    sp.sp24_masked_decay(plain, wd, idx, lam)
    torch.cuda.synchronize()
    assert sp.sp24_device_status() == 0
    got = fused.cpu().numpy()
    assert np.array_equal(got.view(np.uint32), plain.cpu().numpy().view(np.uint32))
    ref = oracle.masked_decay(undecayed, si.bits16(w), dtype, idx.cpu().numpy(), lam)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    assert np.array_equal(idx.cpu().numpy(), oracle.mask_search(si.bits16(w), dtype))
