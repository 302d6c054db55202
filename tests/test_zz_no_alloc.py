"""GPU checks of sp24_gemm_wgrad_noalloc: the weight gradient through the library's
fixed static scratch instead of its per-stream workspace.

The entry point runs the same kernel with the same split of the last wave's tiles
as sp24_gemm_wgrad, so its results must be the same bits, call after call.  Its
scratch holds the partial sums of 128 CTAs: a split tail of r tiles in s parts
uses 2 r s of them, and a call that would need more is rejected before anything
is launched.  The file sorts last so that it also runs after every other test.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
import structured_sparse_transformer_b200 as sp

pytestmark = pytest.mark.gpu

SCRATCH_CTAS = 128


def _pairs():
    # CTA pairs of one wave: one pair per two SMs (one CTA per SM at this kernel's shared memory).
    return torch.cuda.get_device_properties(0).multi_processor_count // 2


def _split_ctas(T, N, K):
    """CTAs whose partial slots a call uses (0 without a split tail), by the split rule of
    sp24_gemm_wgrad: r = tiles mod P tail tiles in s = min(P // r, 8, ceil(T / 128)) parts."""
    P = _pairs()
    tiles = -(-N // 256) * -(-K // 256)
    r = tiles % P
    if r == 0:
        return 0
    s = min(P // r, 8, -(-T // 128))
    return 2 * r * s if s > 1 else 0


def _operands(T, N, K, dtype, seed):
    dy = si.normal((T, N), 1.0, seed, dtype)
    x = si.normal((T, K), 1.0, seed + 1, dtype)
    vb, mb = sp.sp24_compressed_size(N, T)
    vals = torch.empty(N, T // 2, dtype=si.DTYPES[dtype], device="cuda")
    meta = torch.empty(mb, dtype=torch.uint8, device="cuda")
    sp.sp24_mvue_sparsify(dy.cuda(), 21, 3, vals, meta)
    return x, x.cuda(), vals, meta


@pytest.mark.parametrize("T,N,K,dtype", [(2048, 6400, 1600, "f16"),   # 175 tiles: a split tail
                                         (1024, 1024, 4096, "bf16"),  # 64 tiles: one partial wave, no split
                                         (2048, 512, 1024, "f16")])   # 8 tiles split 8 ways
def test_noalloc_equals_wgrad_on_two_calls(T, N, K, dtype):
    need = _split_ctas(T, N, K)
    if need > SCRATCH_CTAS:
        pytest.skip(f"this device's split tail uses {need} CTAs, more than the scratch holds")
    x, xd, vals, meta = _operands(T, N, K, dtype, T + N + K)
    ref = torch.empty(N, K, dtype=torch.float32, device="cuda")
    sp.sp24_gemm_wgrad(xd, vals, meta, N, ref)
    outs = []
    for _ in range(2):
        dw = torch.full((N, K), float("nan"), dtype=torch.float32, device="cuda")
        sp.sp24_gemm_wgrad_noalloc(xd, vals, meta, N, dw)
        outs.append(dw)
    torch.cuda.synchronize()
    assert sp.sp24_device_status() == 0
    for dw in outs:
        assert torch.equal(dw.view(torch.int32), ref.view(torch.int32))
    # and against the fp64 product of the GPU's own sparsified operand on sampled rows
    canon = sp.sp24_meta_to_canonical(meta.cpu().numpy().tobytes(), N, T)
    yhat = oracle.decompress_rows(si.bits16(vals.cpu()), canon, T)
    rows = np.sort(np.random.default_rng(0).choice(N, 32, replace=False))
    want = oracle.weight_grad(oracle.to_f64(yhat[rows], dtype), oracle.to_f64(si.bits16(x), dtype))
    got = outs[1][torch.from_numpy(rows).cuda()].double().cpu().numpy()
    assert np.linalg.norm(got - want) <= 1e-4 * np.linalg.norm(want)


def test_noalloc_rejects_a_split_tail_larger_than_its_scratch():
    P = _pairs()
    T = 256
    # the smallest tail r whose split needs more than the scratch: tiles = P + r, one column tile
    r = next((r for r in range(1, P) if 2 * r * min(P // r, 8, T // 128) > SCRATCH_CTAS
              and min(P // r, 8, T // 128) > 1), None)
    if r is None:
        pytest.skip("no split tail on this device exceeds the scratch")
    N, K = 256 * (P + r), 256
    assert _split_ctas(T, N, K) > SCRATCH_CTAS
    _, xd, vals, meta = _operands(T, N, K, "f16", 7)
    dw = torch.full((N, K), float("nan"), dtype=torch.float32, device="cuda")
    with pytest.raises(sp.Sp24Error, match="SP24_ERR_SCRATCH_TOO_SMALL"):
        sp.sp24_gemm_wgrad_noalloc(xd, vals, meta, N, dw)
    torch.cuda.synchronize()
    assert torch.isnan(dw).all()          # nothing was launched
    assert sp.sp24_device_status() == 0


def test_noalloc_takes_no_device_memory_on_a_new_stream():
    """On a stream the library has not seen, sp24_gemm_wgrad would allocate its workspace
    (the device's free memory drops); sp24_gemm_wgrad_noalloc leaves it unchanged."""
    T, N, K = 2048, 6400, 1600
    if not 0 < _split_ctas(T, N, K) <= SCRATCH_CTAS:
        pytest.skip("no split tail that fits the scratch at this shape on this device")
    _, xd, vals, meta = _operands(T, N, K, "f16", 11)
    dw = torch.empty(N, K, dtype=torch.float32, device="cuda")
    sp.sp24_gemm_wgrad_noalloc(xd, vals, meta, N, dw)     # first use: kernels and scratch loaded
    torch.cuda.synchronize()
    fresh = torch.cuda.Stream()
    free0, _ = torch.cuda.mem_get_info()
    with torch.cuda.stream(fresh):
        sp.sp24_gemm_wgrad_noalloc(xd, vals, meta, N, dw, stream=fresh)
        sp.sp24_gemm_wgrad_noalloc(xd, vals, meta, N, dw, stream=fresh)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    other = torch.cuda.Stream()
    with torch.cuda.stream(other):
        sp.sp24_gemm_wgrad(xd, vals, meta, N, dw, stream=other)
    torch.cuda.synchronize()
    free2, _ = torch.cuda.mem_get_info()
    assert free0 - free2 >= 16 << 20       # the workspace of the new stream
    assert sp.sp24_device_status() == 0
