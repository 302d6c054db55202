"""The C ABI on a machine without a GPU: the library loads, exports every entry
point that include/sp24.h declares, rejects bad arguments on the host before any
CUDA call, and its host-side metadata maps agree with the oracle's canonical
layout.  No kernel is launched here."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import synthetic_inputs as si
import structured_sparse_transformer_b200 as sp

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "sp24.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SP24_API[^;(]*?\b(sp24_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 14
    lib = sp.lib()
    for n in names:
        assert hasattr(lib, n), n
    expected = {"sp24_mask_search", "sp24_prune_compress", "sp24_gemm_fwd", "sp24_gemm_dgrad",
                "sp24_masked_decay", "sp24_flip_rate"}
    assert expected <= set(names)


def test_status_strings():
    for code, name in sp.STATUS.items():
        assert sp.sp24_status_string(code) == name
    assert sp.sp24_status_string(99) == "SP24_UNKNOWN_STATUS"


def test_pattern_table_matches_oracle():
    assert sp.sp24_pattern_table() == [int(b) for b in oracle.pattern_bits()]


def test_compressed_size():
    assert sp.sp24_compressed_size(6400, 1600) == (6400 * 800 * 2, 50 * 13 * 2048)
    assert sp.sp24_compressed_size(1600, 6400) == (1600 * 3200 * 2, 13 * 50 * 2048)
    assert sp.sp24_compressed_size(0, 0) == (0, 0)
    with pytest.raises(sp.Sp24Error):
        sp.sp24_compressed_size(6, 8)


def _raw(name, *args):
    return getattr(sp.lib(), name)(*args)


def test_host_validation_rejects_bad_arguments_without_a_device():
    fake = ctypes.c_void_p(0x10000)          # aligned, never dereferenced: checks run first
    odd = ctypes.c_void_p(0x10008)
    E = {v: k for k, v in sp.STATUS.items()}
    # mask search: shapes, dtype, alignment, null pointers
    assert _raw("sp24_mask_search", fake, 0, 6, 8, 8, fake, None) == E["SP24_ERR_UNSUPPORTED_SHAPE"]
    assert _raw("sp24_mask_search", fake, 7, 8, 8, 8, fake, None) == E["SP24_ERR_UNSUPPORTED_DTYPE"]
    assert _raw("sp24_mask_search", odd, 0, 8, 8, 8, fake, None) == E["SP24_ERR_MISALIGNED"]
    assert _raw("sp24_mask_search", fake, 0, 8, 8, 10, fake, None) == E["SP24_ERR_MISALIGNED"]
    assert _raw("sp24_mask_search", fake, 0, 8, 8, 4, fake, None) == E["SP24_ERR_INVALID_ARG"]
    assert _raw("sp24_mask_search", None, 0, 8, 8, 8, fake, None) == E["SP24_ERR_INVALID_ARG"]
    # compression needs multiples of 16
    assert _raw("sp24_prune_compress", fake, 0, 8, 16, 16, fake, fake, fake, fake, fake, None) == \
        E["SP24_ERR_UNSUPPORTED_SHAPE"]
    assert _raw("sp24_mask_step", fake, 0, 16, 16, 16, fake, fake, None, None, None, None, None, None) == \
        E["SP24_ERR_INVALID_ARG"]
    # GEMMs
    assert _raw("sp24_gemm_fwd", fake, 8, 24, fake, fake, 16, 0, fake, 0, None, None) == \
        E["SP24_ERR_UNSUPPORTED_SHAPE"]
    assert _raw("sp24_gemm_fwd", fake, 8, 32, fake, fake, 16, 0, fake, 1, None, None) == \
        E["SP24_ERR_INVALID_ARG"]                       # GELU without aux
    assert _raw("sp24_gemm_fwd", fake, 8, 32, fake, fake, 16, 0, fake, 2, fake, None) == \
        E["SP24_ERR_INVALID_ARG"]                       # DGELU is not a forward epilogue
    assert _raw("sp24_gemm_dgrad", fake, 8, 32, fake, fake, 16, 0, fake, 1, fake, None) == \
        E["SP24_ERR_INVALID_ARG"]                       # GELU is not an input-gradient epilogue
    assert _raw("sp24_gemm_dgrad", fake, 8, 32, fake, fake, 16, 0, fake, 8, fake, None) == \
        E["SP24_ERR_INVALID_ARG"]                       # the packed GELU' writer is a forward epilogue
    assert _raw("sp24_gemm_fwd", fake, 8, 32, fake, fake, 16, 0, fake, 9, fake, None) == \
        E["SP24_ERR_INVALID_ARG"]                       # the packed multiply is an input-gradient epilogue
    assert _raw("sp24_gemm_fwd", fake, 8, 32, fake, fake, 16, 0, fake, 8, None, None) == \
        E["SP24_ERR_INVALID_ARG"]                       # packed GELU' without aux
    assert _raw("sp24_gemm_fwd", fake, 8, 32, fake, fake, 48, 0, fake, 3, fake, None) == \
        E["SP24_ERR_UNSUPPORTED_SHAPE"]                # GEGLU needs whole gate/up row groups
    assert _raw("sp24_gemm_fwd", fake, 8, 32, fake, fake, 64, 0, fake, 4, fake, None) == \
        E["SP24_ERR_INVALID_ARG"]                       # DGEGLU is not a forward epilogue
    assert _raw("sp24_gemm_dgrad", fake, 8, 32, fake, fake, 64, 0, fake, 3, fake, None) == \
        E["SP24_ERR_INVALID_ARG"]                       # GEGLU is not an input-gradient epilogue
    assert _raw("sp24_gemm_dense", fake, 8, 32, fake, 64, 0, fake, 3, fake, None) == \
        E["SP24_ERR_INVALID_ARG"]                       # gated epilogues serve the 2:4 GEMMs
    assert _raw("sp24_gemm_fwd", odd, 8, 32, fake, fake, 16, 0, fake, 0, None, None) == \
        E["SP24_ERR_MISALIGNED"]
    assert _raw("sp24_gemm_fwd", fake, -1, 32, fake, fake, 16, 0, fake, 0, None, None) == \
        E["SP24_ERR_INVALID_ARG"]
    # dense fine-tuning GEMM and transpose
    assert _raw("sp24_gemm_dense", fake, 8, 24, fake, 16, 0, fake, 0, None, None) == \
        E["SP24_ERR_UNSUPPORTED_SHAPE"]
    assert _raw("sp24_gemm_dense", fake, 8, 32, fake, 16, 0, fake, 2, None, None) == \
        E["SP24_ERR_INVALID_ARG"]                       # DGELU without aux
    assert _raw("sp24_gemm_dense", fake, 8, 32, fake, 16, 0, fake, 3, fake, None) == \
        E["SP24_ERR_INVALID_ARG"]                       # no such epilogue
    assert _raw("sp24_gemm_dense", fake, 8, 32, odd, 16, 0, fake, 0, None, None) == \
        E["SP24_ERR_MISALIGNED"]
    assert _raw("sp24_gemm_dgrad_dense", fake, 8, 24, fake, 16, 0, fake, 0, None, None) == \
        E["SP24_ERR_UNSUPPORTED_SHAPE"]                # N (the contraction) % 16
    assert _raw("sp24_gemm_dgrad_dense", fake, 8, 32, fake, 24, 0, fake, 0, None, None) == \
        E["SP24_ERR_UNSUPPORTED_SHAPE"]                # K (the output width) % 16
    assert _raw("sp24_gemm_dgrad_dense", fake, 8, 32, fake, 16, 0, fake, 1, fake, None) == \
        E["SP24_ERR_INVALID_ARG"]                       # GELU is not an input-gradient epilogue
    assert _raw("sp24_gemm_dgrad_dense", fake, 8, 32, fake, 16, 0, fake, 7, None, None) == \
        E["SP24_ERR_INVALID_ARG"]                       # MUL_AUX without aux
    assert _raw("sp24_gemm_dgrad_dense", fake, 8, 32, odd, 16, 0, fake, 0, None, None) == \
        E["SP24_ERR_MISALIGNED"]
    assert _raw("sp24_transpose", fake, 8, 8, 5, fake, None) == E["SP24_ERR_UNSUPPORTED_DTYPE"]
    assert _raw("sp24_transpose", None, 8, 8, 0, fake, None) == E["SP24_ERR_INVALID_ARG"]
    assert _raw("sp24_transpose", fake, -2, 8, 0, fake, None) == E["SP24_ERR_INVALID_ARG"]
    assert _raw("sp24_transpose", odd, 8, 8, 0, fake, None) == E["SP24_ERR_MISALIGNED"]
    # MVUE sparsification and the weight-gradient GEMM
    assert _raw("sp24_mvue_sparsify", fake, 24, 64, 64, 0, 1, 2, fake, fake, None) == \
        E["SP24_ERR_UNSUPPORTED_SHAPE"]                # tokens must be a multiple of 16
    assert _raw("sp24_mvue_sparsify", fake, 32, 12, 16, 0, 1, 2, fake, fake, None) == \
        E["SP24_ERR_UNSUPPORTED_SHAPE"]                # columns must be a multiple of 8
    assert _raw("sp24_mvue_sparsify", fake, 32, 64, 32, 0, 1, 2, fake, fake, None) == \
        E["SP24_ERR_INVALID_ARG"]                       # ldy < N
    assert _raw("sp24_mvue_sparsify", fake, 32, 64, 68, 0, 1, 2, fake, fake, None) == \
        E["SP24_ERR_MISALIGNED"]                        # ldy not a multiple of 8
    assert _raw("sp24_mvue_sparsify", fake, 32, 64, 64, 9, 1, 2, fake, fake, None) == \
        E["SP24_ERR_UNSUPPORTED_DTYPE"]
    assert _raw("sp24_mvue_sparsify", fake, 32, 64, 64, 0, 1, 2, None, fake, None) == \
        E["SP24_ERR_INVALID_ARG"]
    assert _raw("sp24_gemm_wgrad", fake, 24, 64, fake, fake, 64, 0, fake, None) == \
        E["SP24_ERR_UNSUPPORTED_SHAPE"]                # tokens (the contraction) % 16
    assert _raw("sp24_gemm_wgrad", fake, 32, 60, fake, fake, 64, 0, fake, None) == \
        E["SP24_ERR_UNSUPPORTED_SHAPE"]                # dW columns % 8
    assert _raw("sp24_gemm_wgrad", fake, 32, 64, fake, fake, 40, 0, fake, None) == \
        E["SP24_ERR_UNSUPPORTED_SHAPE"]                # dW rows % 16
    assert _raw("sp24_gemm_wgrad", fake, 32, 64, fake, fake, 64, 0, None, None) == \
        E["SP24_ERR_INVALID_ARG"]
    assert _raw("sp24_gemm_wgrad", fake, 32, 64, odd, fake, 64, 0, fake, None) == \
        E["SP24_ERR_MISALIGNED"]
    assert _raw("sp24_gemm_wgrad_decay", fake, 32, 64, fake, fake, 64, 0, None, fake, ctypes.c_float(1e-4),
                fake, None) == E["SP24_ERR_INVALID_ARG"]          # no weight
    assert _raw("sp24_gemm_wgrad_decay", fake, 32, 64, fake, fake, 64, 0, fake, None, ctypes.c_float(1e-4),
                fake, None) == E["SP24_ERR_INVALID_ARG"]          # no mask
    assert _raw("sp24_gemm_wgrad_decay", fake, 32, 64, fake, fake, 64, 0, odd, fake, ctypes.c_float(1e-4),
                fake, None) == E["SP24_ERR_MISALIGNED"]
    assert _raw("sp24_gemm_wgrad_decay", fake, 24, 64, fake, fake, 64, 0, fake, fake, ctypes.c_float(1e-4),
                fake, None) == E["SP24_ERR_UNSUPPORTED_SHAPE"]
    assert _raw("sp24_gemm_wgrad_dense", fake, 24, 64, fake, 64, 0, fake, None) == \
        E["SP24_ERR_UNSUPPORTED_SHAPE"]
    assert _raw("sp24_gemm_wgrad_dense", fake, 32, 64, None, 64, 0, fake, None) == E["SP24_ERR_INVALID_ARG"]
    assert _raw("sp24_gemm_wgrad_dense", fake, 32, 64, fake, 64, 0, odd, None) == E["SP24_ERR_MISALIGNED"]
    # decay and flip
    assert _raw("sp24_masked_decay", fake, fake, 0, 6, 8, fake, ctypes.c_float(1.0), None) == \
        E["SP24_ERR_UNSUPPORTED_SHAPE"]
    assert _raw("sp24_flip_rate", fake, fake, -1, fake, None) == E["SP24_ERR_INVALID_ARG"]
    assert _raw("sp24_flip_rate", fake, fake, 4, None, None) == E["SP24_ERR_INVALID_ARG"]


def test_binding_rejects_views_that_are_not_row_major():
    """Layout is checked before anything else (here on CPU tensors, so no device is needed)."""
    import torch
    w = torch.zeros(64, 64, dtype=torch.float16)
    idx = torch.zeros(16, 16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="row-major"):
        sp.sp24_mask_search(w.t(), idx)                     # column-major view of W
    with pytest.raises(ValueError, match="contiguous"):
        sp.sp24_gemm_fwd(w[:, ::2], w, idx, 64, w)          # strided activations
    with pytest.raises(ValueError, match="contiguous"):
        sp.sp24_masked_decay(torch.zeros(64, 64).t(), w, idx, 1e-4)
    with pytest.raises(ValueError, match="row-major"):
        sp.sp24_mvue_sparsify(w[:, ::2], 0, 0, w, idx)
    # a row-pitched W passes the layout check and stops at the device check
    with pytest.raises(ValueError, match="CUDA"):
        sp.sp24_mask_search(torch.zeros(64, 96, dtype=torch.float16)[:, :64], idx)


def test_binding_rejects_wrong_dtype_and_short_buffers():
    """Every buffer's dtype and size is checked against what the C call will touch, before the
    call (CPU tensors: the checks run before the device check)."""
    import torch
    f16, u8, f32, i64 = torch.float16, torch.uint8, torch.float32, torch.int64
    R, C, T = 64, 128, 32
    w = torch.zeros(R, C, dtype=f16)
    idx = torch.zeros(R // 4, C // 4, dtype=u8)
    vr, mr = sp.sp24_compressed_size(R, C)
    vc, mc = sp.sp24_compressed_size(C, R)
    comp = [torch.zeros(R, C // 2, dtype=f16), torch.zeros(mr, dtype=u8),
            torch.zeros(C, R // 2, dtype=f16), torch.zeros(mc, dtype=u8)]
    cnt = torch.zeros(1, dtype=i64)

    def bad(fn, *a, match):
        with pytest.raises(ValueError, match=match):
            fn(*a)

    def ok_until_device(fn, *a):
        with pytest.raises(ValueError, match="CUDA"):
            fn(*a)

    ok_until_device(sp.sp24_mask_step, w, idx, idx, cnt, *comp)
    bad(sp.sp24_mask_search, w, idx[:8], match="idx")
    bad(sp.sp24_mask_search, w, idx.to(torch.int8), match="idx")
    bad(sp.sp24_mask_step, w, idx, idx[:4], cnt, *comp, match="idx_prev")
    bad(sp.sp24_mask_step, w, idx, idx, cnt.to(torch.int32), *comp, match="flip_count")
    bad(sp.sp24_mask_step, w, idx, idx, cnt, comp[0][:10], *comp[1:], match="row-compressed values")
    bad(sp.sp24_mask_step, w, idx, idx, cnt, comp[0], comp[1][:100], *comp[2:], match="row-compressed metadata")
    bad(sp.sp24_prune_compress, w, idx, comp[0], comp[1], comp[2].to(torch.bfloat16), comp[3],
        match="column-compressed values")
    x = torch.zeros(T, C, dtype=f16)
    y = torch.zeros(T, R, dtype=f16)
    ok_until_device(sp.sp24_gemm_fwd, x, comp[0], comp[1], R, y, "gelu", y.clone())
    bad(sp.sp24_gemm_fwd, x, comp[0], comp[1], R, y[:-1], match="Y")
    bad(sp.sp24_gemm_fwd, x, comp[0], comp[1], R, y, "gelu", y[:, :R // 2].contiguous(), match="aux")
    bad(sp.sp24_gemm_fwd, x, comp[0], comp[1], R, y.float(), match="Y")
    ok_until_device(sp.sp24_gemm_fwd, x, comp[0], comp[1], R, torch.zeros(T, R // 2, dtype=f16), "geglu", y)
    ok_until_device(sp.sp24_gemm_dgrad, y, comp[2], comp[3], C, x, "dgelu", x.clone())
    pk = torch.zeros(sp.sp24_aux_packed_size(T, C) // 2, dtype=f16)
    ok_until_device(sp.sp24_gemm_dgrad, y, comp[2], comp[3], C, x, "mul_aux_packed", pk)
    bad(sp.sp24_gemm_dgrad, y, comp[2], comp[3], C, x, "mul_aux_packed", pk[:-8].clone(), match="aux")
    bad(sp.sp24_gemm_dgrad, y, comp[2], comp[3], C, x[:1], match="dX")
    bad(sp.sp24_gemm_dgrad, y, comp[2], comp[3], C, x, "dgeglu", x.clone(), match="dX")
    bad(sp.sp24_gemm_dgrad, y, comp[2][:10], comp[3], C, x, match="W\\^T values")
    ok_until_device(sp.sp24_gemm_dense, x, w, y)
    bad(sp.sp24_gemm_dense, x, w[:, :64].contiguous(), y, match="A:")
    bad(sp.sp24_transpose, w, torch.zeros(C, R - 4, dtype=f16), match="out")
    ok_until_device(sp.sp24_gemm_dgrad_dense, y, w, x, "mul_aux", x.clone())
    bad(sp.sp24_gemm_dgrad_dense, y, w[:32].contiguous(), x, match="W has 32 rows")
    bad(sp.sp24_gemm_dgrad_dense, y, w, x[:, :64].contiguous(), match="dX")
    bad(sp.sp24_gemm_dgrad_dense, y, w, x, "mul_aux", x[:1].clone(), match="aux")
    # weight gradient: MVUE(dY^T) [R x T] compressed along T, dW fp32 [R x C]
    dy = torch.zeros(T, R, dtype=f16)
    yv = torch.zeros(R, T // 2, dtype=f16)
    ym = torch.zeros(sp.sp24_compressed_size(R, T)[1], dtype=u8)
    dw = torch.zeros(R, C, dtype=f32)
    ok_until_device(sp.sp24_mvue_sparsify, dy, 0, 0, yv, ym)
    bad(sp.sp24_mvue_sparsify, dy, 0, 0, yv[:4], ym, match="values")
    ok_until_device(sp.sp24_gemm_wgrad, x, yv, ym, R, dw)
    bad(sp.sp24_gemm_wgrad, x, yv, ym, R, dw[:10], match="dW")
    bad(sp.sp24_gemm_wgrad, x, yv, ym, R, dw.half(), match="dW")
    bad(sp.sp24_gemm_wgrad_dense, x, torch.zeros(T, R, dtype=f16), dw.double(), match="dW")
    bad(sp.sp24_gemm_wgrad_dense, x, torch.zeros(R, T, dtype=f16), dw, match="rows")
    wt = torch.zeros(R, C, dtype=f16)
    ok_until_device(sp.sp24_gemm_wgrad_decay, x, yv, ym, R, wt, idx.reshape(-1)[:(R // 4) * (C // 4)].clone(), 1e-4, dw)
    bad(sp.sp24_gemm_wgrad_decay, x, yv, ym, R, wt[:, :64].contiguous(), idx, 1e-4, dw, match="W:")
    bad(sp.sp24_gemm_wgrad_decay, x, yv, ym, R, wt, idx[:1], 1e-4, dw, match="idx")
    g = torch.zeros(R, C, dtype=f32)
    ok_until_device(sp.sp24_masked_decay, g, w, idx, 1e-4)
    bad(sp.sp24_masked_decay, g.half(), w, idx, 1e-4, match="grad")
    bad(sp.sp24_masked_decay, g[:8], w, idx, 1e-4, match="grad")
    bad(sp.sp24_masked_decay, g, w, idx[:2], 1e-4, match="idx")
    ok_until_device(sp.sp24_flip_rate, idx, idx, cnt)
    bad(sp.sp24_flip_rate, idx[:3], idx, cnt, match="idx_prev")
    bad(sp.sp24_flip_rate, idx, idx, torch.zeros(0, dtype=i64), match="count")


def test_valid_call_without_a_device_reports_no_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    fake = ctypes.c_void_p(0x10000)
    assert _raw("sp24_mask_search", fake, 0, 8, 8, 8, fake, None) == 7


@pytest.mark.parametrize("rows,cols", [(16, 16), (48, 80), (128, 256), (144, 400)])
def test_meta_layout_roundtrip_and_padding(rows, cols):
    w = si.normal((rows, cols), 0.02, seed=rows + cols, dtype="f16")
    bits = si.bits16(w)
    idx = oracle.mask_search(bits, "f16")
    (_, canon_row), (_, canon_col) = oracle.compress_both(bits, idx)
    for canon, r, c in ((canon_row, rows, cols), (canon_col, cols, rows)):
        dev = sp.sp24_meta_from_canonical(canon, r, c)
        assert dev.size == sp.sp24_compressed_size(r, c)[1]
        back = sp.sp24_meta_to_canonical(dev.tobytes(), r, c)
        assert np.array_equal(back, canon)
        nibbles = np.stack([(dev >> 4) & 0xF, dev & 0xF]).reshape(-1)
        assert set(np.unique(nibbles).tolist()) <= set(oracle.NIBBLE_CODES)
        # every byte that no (row, group) maps to keeps the padding code 0x44
        assert (dev == 0x44).sum() >= dev.size - r * (c // 4) // 2


def test_meta_layout_is_a_permutation():
    # Distinct canonical inputs map to distinct device bytes: the map is injective.
    rows, cols = 128, 128
    rng = np.random.default_rng(0)
    codes = np.array(oracle.NIBBLE_CODES, dtype=np.uint16)
    canon = np.zeros((rows, cols // 16), np.uint16)
    for k in range(4):
        canon |= codes[rng.integers(0, 6, canon.shape)] << (4 * k)
    dev = sp.sp24_meta_from_canonical(canon, rows, cols)
    assert dev.size == 2048
    flipped = canon.copy()
    flipped[37, 3] ^= 0x0040            # 0x4 <-> 0x0 in one nibble changes exactly one device nibble
    dev2 = sp.sp24_meta_from_canonical(flipped, rows, cols)
    assert np.count_nonzero(dev != dev2) == 1
