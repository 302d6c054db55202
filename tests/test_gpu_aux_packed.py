"""GPU checks of the derivative-saving GELU pair with the derivative in the packed
chunk layout (SP24_EPI_GELU_DERIV_PACKED / SP24_EPI_MUL_AUX_PACKED).

Both kernels compute exactly what the row-major pair computes (the same fp32
arithmetic and roundings); only where the derivative is kept differs.  So the
forward's output must equal the row-major forward's bit for bit, the packed
derivative must unpack to the row-major derivative bit for bit, and the input
gradient that multiplies by the packed derivative must equal the one that
multiplies by the row-major derivative.  The row-major pair itself is checked
against the oracle in test_gpu_gelu and test_gpu_gemm.  Shapes include token
counts and widths that are not multiples of the 16 x 32 blocks.
"""
import numpy as np
import pytest
import torch

import synthetic_inputs as si
import structured_sparse_transformer_b200 as sp

pytestmark = pytest.mark.gpu


def _bits(t):
    return si.bits16(t.cpu())


@pytest.mark.parametrize("dense", [False, True])
@pytest.mark.parametrize("T,d,ff,dtype", [(1000, 1600, 6400, "f16"), (300, 400, 208, "bf16"), (77, 64, 48, "f16"),
                                          (4096, 1024, 4096, "bf16"), (1, 32, 16, "f16")])
def test_packed_pair_equals_the_row_major_pair(T, d, ff, dtype, dense):
    tdt = si.DTYPES[dtype]
    W1 = si.normal((ff, d), 0.02, T + ff, dtype).cuda()     # layer 1: X [T, d] -> H [T, ff]
    W2 = si.normal((d, ff), 0.02, T + d, dtype).cuda()      # layer 2's input gradient: dY [T, d] -> dH [T, ff]
    X = si.normal((T, d), 1.0, T + 1, dtype).cuda()
    dY = si.normal((T, d), 1.0, T + 2, dtype).cuda()
    H1, H2 = (torch.empty(T, ff, dtype=tdt, device="cuda") for _ in range(2))
    D1 = torch.empty(T, ff, dtype=tdt, device="cuda")
    P = torch.full((sp.sp24_aux_packed_size(T, ff) // 2,), float("nan"), dtype=tdt, device="cuda")
    dH1, dH2 = (torch.full((T, ff), float("nan"), dtype=tdt, device="cuda") for _ in range(2))
    if dense:
        sp.sp24_gemm_dense(X, W1, H1, "gelu_deriv", D1)
        sp.sp24_gemm_dense(X, W1, H2, "gelu_deriv_packed", P)
        sp.sp24_gemm_dgrad_dense(dY, W2, dH1, "mul_aux", D1)
        sp.sp24_gemm_dgrad_dense(dY, W2, dH2, "mul_aux_packed", P)
    else:
        idx = [torch.empty(r // 4, c // 4, dtype=torch.uint8, device="cuda") for r, c in ((ff, d), (d, ff))]
        c1, c2 = sp.alloc_compressed(ff, d, tdt), sp.alloc_compressed(d, ff, tdt)
        sp.sp24_mask_step(W1, idx[0], None, None, *c1)
        sp.sp24_mask_step(W2, idx[1], None, None, *c2)
        sp.sp24_gemm_fwd(X, c1[0], c1[1], ff, H1, "gelu_deriv", D1)
        sp.sp24_gemm_fwd(X, c1[0], c1[1], ff, H2, "gelu_deriv_packed", P)
        sp.sp24_gemm_dgrad(dY, c2[2], c2[3], ff, dH1, "mul_aux", D1)
        sp.sp24_gemm_dgrad(dY, c2[2], c2[3], ff, dH2, "mul_aux_packed", P)
    torch.cuda.synchronize()
    assert sp.sp24_device_status() == 0
    assert np.array_equal(_bits(H2), _bits(H1))
    assert np.array_equal(sp.sp24_aux_unpack(_bits(P), T, ff), _bits(D1))
    assert np.array_equal(_bits(dH2), _bits(dH1))


def test_packed_input_gradient_reads_a_host_packed_derivative():
    """A derivative packed on the host (sp24_aux_pack) gives the same input gradient as
    the same values row-major, so the host map and the kernel's reads agree."""
    T, d, ff, dtype = 200, 256, 272, "f16"
    tdt = si.DTYPES[dtype]
    W2 = si.normal((d, ff), 0.02, 5, dtype).cuda()
    dY = si.normal((T, d), 1.0, 6, dtype).cuda()
    aux = si.normal((T, ff), 1.0, 7, dtype)
    packed = torch.from_numpy(sp.sp24_aux_pack(si.bits16(aux), T, ff).view(np.int16)).view(tdt).cuda()
    idx = torch.empty(d // 4, ff // 4, dtype=torch.uint8, device="cuda")
    c2 = sp.alloc_compressed(d, ff, tdt)
    sp.sp24_mask_step(W2, idx, None, None, *c2)
    dH1, dH2 = (torch.empty(T, ff, dtype=tdt, device="cuda") for _ in range(2))
    sp.sp24_gemm_dgrad(dY, c2[2], c2[3], ff, dH1, "mul_aux", aux.cuda())
    sp.sp24_gemm_dgrad(dY, c2[2], c2[3], ff, dH2, "mul_aux_packed", packed)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(dH2), _bits(dH1))
