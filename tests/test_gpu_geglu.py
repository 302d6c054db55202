"""GPU parity of the gated FFN (GEGLU) on the 2:4 GEMMs.

"Accelerating Transformer Pre-training with 2:4 Sparsity", abstract
(accelerating gated activation functions by reducing GPU L2 cache misses) and
the Software Dependencies row (GEGLU kernel).  The gate and up projections are
one stacked 2:4 weight whose rows alternate in groups of 16; the forward GEMM's
epilogue forms gelu(gate) * up where both accumulators are produced, and the
input-gradient GEMM of the down projection forms the two pre-activation
gradients in its epilogue, so no gate, up or dH tensor makes a round trip
through memory between the GEMMs.  Tolerances as in gpu_util.
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
    R, C = w_cpu.shape
    idx = torch.empty(R // 4, C // 4, dtype=torch.uint8, device="cuda")
    bufs = sp.alloc_compressed(R, C, w_cpu.dtype)
    sp.sp24_mask_step(w_cpu.cuda(), idx, None, None, *bufs)
    torch.cuda.synchronize()
    return oracle.dense_mask(idx.cpu().numpy()), bufs


def _stack(wg, wu):
    return torch.from_numpy(oracle.interleave_gate_up(si.bits16(wg), si.bits16(wu)).view(np.int16)).view(wg.dtype)


@pytest.mark.parametrize("T,d,ff,dtype,rows", [(77, 144, 208, "bf16", None), (300, 256, 512, "f16", None),
                                               (8192, 1024, 4096, "f16", 24)])
def test_geglu_ffn_chain(T, d, ff, dtype, rows):
    """H = gelu(X Wg^T) * (X Wu^T), Y = H Wd^T; dGU = gated gradients of dY Wd; dX = dGU Wgu."""
    wg = si.normal((ff, d), 0.02, 11, dtype)
    wu = si.normal((ff, d), 0.02, 12, dtype)
    wd = si.normal((d, ff), 0.02, 13, dtype)
    x = si.normal((T, d), 1.0, 14, dtype)
    dy = si.normal((T, d), 1.0, 15, dtype)
    wgu = _stack(wg, wu)
    k_gu, (vr_gu, mr_gu, vc_gu, mc_gu) = _prep(wgu)
    k_d, (vr_d, mr_d, vc_d, mc_d) = _prep(wd)
    tdt = wg.dtype
    H = torch.empty(T, ff, dtype=tdt, device="cuda")
    GU = torch.empty(T, 2 * ff, dtype=tdt, device="cuda")
    Y = torch.empty(T, d, dtype=tdt, device="cuda")
    dGU = torch.empty(T, 2 * ff, dtype=tdt, device="cuda")
    dX = torch.empty(T, d, dtype=tdt, device="cuda")
    sp.sp24_gemm_fwd(x.cuda(), vr_gu, mr_gu, 2 * ff, H, "geglu", GU)
    sp.sp24_gemm_fwd(H, vr_d, mr_d, d, Y)
    sp.sp24_gemm_dgrad(dy.cuda(), vc_d, mc_d, ff, dGU, "dgeglu", GU)
    sp.sp24_gemm_dgrad(dGU, vc_gu, mc_gu, d, dX)
    torch.cuda.synchronize()
    sel = np.arange(T) if rows is None else np.arange(5, T, rows)
    dt = dtype
    wgu_f, wd_f = oracle.to_f64(si.bits16(wgu), dt), oracle.to_f64(si.bits16(wd), dt)
    pre = oracle.sparse_fwd(oracle.to_f64(si.bits16(x)[sel], dt), wgu_f, k_gu)
    gu_gpu = f64_of(GU, dt)[sel]
    assert_gemm_close(gu_gpu, pre, dt, "gate/up pre-activations")
    # The epilogue gates the fp32 accumulators, so the reference gates the exact
    # pre-activations; the gradient epilogue reads the stored (rounded) ones.
    assert_gemm_close(f64_of(H, dt)[sel], oracle.geglu(*oracle.split_gate_up(pre)), dt, "geglu")
    gate, up = oracle.split_gate_up(gu_gpu)
    assert_gemm_close(f64_of(Y, dt)[sel], oracle.sparse_fwd(f64_of(H, dt)[sel], wd_f, k_d), dt, "down")
    dh = oracle.sparse_dgrad(oracle.to_f64(si.bits16(dy)[sel], dt), wd_f, k_d)
    dg, du = oracle.geglu_grad(dh, gate, up)
    dgu_ref = oracle.interleave_gate_up(dg.T, du.T).T
    assert_gemm_close(f64_of(dGU, dt)[sel], dgu_ref, dt, "gated gradients")
    assert_gemm_close(f64_of(dX, dt)[sel], oracle.sparse_dgrad(f64_of(dGU, dt)[sel], wgu_f, k_gu), dt, "dX")
