"""Python binding of libsp24.so -- argument marshalling only.

Each ``sp24_*`` function here has the name of the C entry point it calls
(``include/sp24.h``), takes torch CUDA tensors (or raw pointers for the host
helpers), passes their data pointers, sizes and the current CUDA stream, and
raises ``Sp24Error`` on a non-OK status.  Every step of the computation runs in
the library's kernels; there is no fallback of any kind.  Importing the package
raises if ``libsp24.so`` is missing: build it with
``python structured_sparse_transformer_b200/build.py``.

Operations from "Accelerating Transformer Pre-training with 2:4 Sparsity":
transposable 2:4 mask search (reproducibility table, Pseudocode row,
Algorithm 1), pruning/compression and the 2:4 sparse FFN GEMMs (Software
Dependencies row), masked decay and flip rate (abstract), and the dense GEMM
of the dense fine-tuning phase (abstract; Experiment Setup row).
"""
from __future__ import annotations

import ctypes
import os

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libsp24.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing; build it with `python structured_sparse_transformer_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

P, I64, I32, U64, F32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint64, ctypes.c_float
_SIGNATURES = {
    "sp24_pattern_table": [P],
    "sp24_mask_search": [P, I32, I64, I64, I64, P, P],
    "sp24_compressed_size": [I64, I64, I32, P, P],
    "sp24_prune_compress": [P, I32, I64, I64, I64, P, P, P, P, P, P],
    "sp24_mask_step": [P, I32, I64, I64, I64, P, P, P, P, P, P, P, P],
    "sp24_gemm_fwd": [P, I64, I64, P, P, I64, I32, P, I32, P, P],
    "sp24_gemm_dgrad": [P, I64, I64, P, P, I64, I32, P, I32, P, P],
    "sp24_gemm_dense": [P, I64, I64, P, I64, I32, P, I32, P, P],
    "sp24_gemm_dgrad_dense": [P, I64, I64, P, I64, I32, P, I32, P, P],
    "sp24_transpose": [P, I64, I64, I32, P, P],
    "sp24_mvue_sparsify": [P, I64, I64, I64, I32, U64, U64, P, P, P],
    "sp24_gemm_wgrad": [P, I64, I64, P, P, I64, I32, P, P],
    "sp24_gemm_wgrad_noalloc": [P, I64, I64, P, P, I64, I32, P, P],
    "sp24_gemm_wgrad_decay": [P, I64, I64, P, P, I64, I32, P, P, F32, P, P],
    "sp24_gemm_wgrad_dense": [P, I64, I64, P, I64, I32, P, P],
    "sp24_masked_decay": [P, P, I32, I64, I64, P, F32, P],
    "sp24_flip_rate": [P, P, I64, P, P],
    "sp24_meta_to_canonical": [P, I64, I64, P],
    "sp24_aux_packed_size": [I64, I64, P],
    "sp24_aux_pack": [P, I64, I64, P],
    "sp24_aux_unpack": [P, I64, I64, P],
    "sp24_meta_from_canonical": [P, I64, I64, P],
    "sp24_device_status": [P],
    "sp24_set_wait_budget": [U64],
}
for _name, _args in _SIGNATURES.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = I32
_lib.sp24_status_string.argtypes = [I32]
_lib.sp24_status_string.restype = ctypes.c_char_p

STATUS = {0: "SP24_OK", 1: "SP24_ERR_INVALID_ARG", 2: "SP24_ERR_UNSUPPORTED_SHAPE",
          3: "SP24_ERR_UNSUPPORTED_DTYPE", 4: "SP24_ERR_MISALIGNED", 5: "SP24_ERR_CUDA",
          6: "SP24_ERR_TIMEOUT", 7: "SP24_ERR_NO_DEVICE", 8: "SP24_ERR_SCRATCH_TOO_SMALL"}
SP24_F16, SP24_BF16 = 0, 1
SP24_EPI_NONE, SP24_EPI_GELU, SP24_EPI_DGELU = 0, 1, 2
EPILOGUES = {None: 0, "none": 0, "gelu": 1, "dgelu": 2, "geglu": 3, "dgeglu": 4, "gelu_deriv": 6, "mul_aux": 7,
             "gelu_deriv_packed": 8, "mul_aux_packed": 9}
PACKED_EPILOGUES = ("gelu_deriv_packed", "mul_aux_packed")


class Sp24Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {sp24_status_string(status)}")


def lib() -> ctypes.CDLL:
    """The loaded ctypes library, for callers that marshal raw pointers themselves."""
    return _lib


def sp24_status_string(status: int) -> str:
    return _lib.sp24_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != 0:
        raise Sp24Error(fn, status)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float16:
        return SP24_F16
    if t.dtype == torch.bfloat16:
        return SP24_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need_rowmajor(*ts, pitched=()):
    """The library reads every buffer as row-major: contiguous tensors, except those in
    `pitched` (2-D, unit stride along rows, the row pitch passed as a leading dimension)."""
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("sp24 takes contiguous (row-major) tensors")
    for t in pitched:
        if t is not None and (t.dim() != 2 or t.stride(1) != 1):
            raise ValueError("sp24 takes 2-D row-major tensors with unit stride along rows")


def _need_device(*ts):
    """Every tensor passed to a kernel lives on a CUDA device (checked after layout, dtype and
    size, so those checks also run on CPU tensors)."""
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("sp24 kernels take CUDA tensors only")


def _expect(t, name: str, dtype, numel: int):
    """Raises ValueError unless tensor `t` has `dtype` and holds at least `numel` elements:
    the kernels read and write exactly the sizes passed to the C call, so a short or
    mistyped buffer would be accessed out of bounds (a longer one is left alone past them)."""
    if t is None:
        return
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected dtype {dtype}, got {t.dtype}")
    n = t.numel()
    if n < numel:
        raise ValueError(f"{name}: expected at least {numel} elements, got {n}")


def _expect_compressed(vals, meta, rows: int, cols: int, dtype, what: str):
    """vals [rows x cols/2] of `dtype` and the metadata bytes of an [rows x cols] operand."""
    import torch
    _expect(vals, f"{what} values", dtype, rows * (cols // 2))
    _expect(meta, f"{what} metadata", torch.uint8, sp24_compressed_size(rows, cols)[1])


def _shape2(t, name: str):
    if t.dim() != 2:
        raise ValueError(f"{name}: expected a 2-D tensor, got {t.dim()}-D")
    return t.shape


# ------------------------------------------------------------ host helpers

def sp24_pattern_table():
    """The 90 candidate patterns as a list of uint16 bit sets (bit 4*i+j = row i, column j)."""
    out = (ctypes.c_uint16 * 90)()
    _check("sp24_pattern_table", _lib.sp24_pattern_table(out))
    return list(out)


def sp24_compressed_size(rows: int, cols: int, dtype: int = SP24_F16):
    """(vals_bytes, meta_bytes) of one orientation of an [rows x cols] matrix compressed along rows."""
    v, m = ctypes.c_size_t(), ctypes.c_size_t()
    _check("sp24_compressed_size", _lib.sp24_compressed_size(rows, cols, dtype, ctypes.byref(v), ctypes.byref(m)))
    return v.value, m.value


def sp24_aux_packed_size(T: int, M: int) -> int:
    """Bytes of a 16-bit [T, M] matrix in the packed chunk layout (the _packed epilogues' aux)."""
    out = ctypes.c_size_t(0)
    _check("sp24_aux_packed_size", _lib.sp24_aux_packed_size(T, M, ctypes.byref(out)))
    return out.value


def aux_elements(T: int, M: int, epi) -> int:
    """16-bit elements of the aux buffer of a [T, M] product with epilogue epi."""
    return sp24_aux_packed_size(T, M) // 2 if epi in PACKED_EPILOGUES else T * M


def sp24_aux_pack(rowmajor, T: int, M: int):
    """Row-major uint16 [T, M] (numpy, host) -> the packed chunk layout (numpy uint16, padding 0)."""
    import numpy as np
    src = np.ascontiguousarray(rowmajor, dtype=np.uint16).reshape(T, M)
    out = np.zeros(sp24_aux_packed_size(T, M) // 2, dtype=np.uint16)
    _check("sp24_aux_pack", _lib.sp24_aux_pack(src.ctypes.data, T, M, out.ctypes.data))
    return out


def sp24_aux_unpack(packed, T: int, M: int):
    """The packed chunk layout (numpy uint16, host) -> row-major uint16 [T, M] (numpy)."""
    import numpy as np
    src = np.ascontiguousarray(packed, dtype=np.uint16).reshape(-1)
    if src.size * 2 < sp24_aux_packed_size(T, M):
        raise ValueError(f"packed aux has {src.size} elements, needs {sp24_aux_packed_size(T, M) // 2}")
    out = np.zeros((T, M), dtype=np.uint16)
    _check("sp24_aux_unpack", _lib.sp24_aux_unpack(src.ctypes.data, T, M, out.ctypes.data))
    return out


def sp24_meta_to_canonical(meta_bytes: bytes, rows: int, cols: int):
    """Device-layout metadata (host bytes) -> canonical uint16 words [rows][cols/16] (numpy)."""
    import numpy as np
    src = np.frombuffer(bytes(meta_bytes), dtype=np.uint8).copy()
    out = np.zeros((rows, cols // 16), dtype=np.uint16)
    _check("sp24_meta_to_canonical", _lib.sp24_meta_to_canonical(src.ctypes.data, rows, cols, out.ctypes.data))
    return out


def sp24_meta_from_canonical(canon, rows: int, cols: int):
    """Canonical uint16 words (numpy [rows][cols/16]) -> device-layout metadata bytes (numpy uint8)."""
    import numpy as np
    canon = np.ascontiguousarray(canon, dtype=np.uint16)
    out = np.zeros(sp24_compressed_size(rows, cols)[1], dtype=np.uint8)
    _check("sp24_meta_from_canonical",
           _lib.sp24_meta_from_canonical(canon.ctypes.data, rows, cols, out.ctypes.data))
    return out


# ------------------------------------------------------------ device calls

def sp24_mask_search(W, idx, stream=None):
    """idx[R/4, C/4] (uint8, CUDA) <- Algorithm 1 on W [R, C] (fp16/bf16, CUDA, row-major)."""
    import torch
    _need_rowmajor(idx, pitched=(W,))
    R, C = _shape2(W, "W")
    _dtype_code(W)
    _expect(idx, "idx", torch.uint8, (R // 4) * (C // 4))
    _need_device(idx, W)
    _check("sp24_mask_search", _lib.sp24_mask_search(_ptr(W), _dtype_code(W), R, C, W.stride(0), _ptr(idx),
                                                     _stream(stream)))


def sp24_prune_compress(W, idx, vals_row, meta_row, vals_col, meta_col, stream=None):
    import torch
    _need_rowmajor(idx, vals_row, meta_row, vals_col, meta_col, pitched=(W,))
    R, C = _shape2(W, "W")
    _dtype_code(W)
    _expect(idx, "idx", torch.uint8, (R // 4) * (C // 4))
    _expect_compressed(vals_row, meta_row, R, C, W.dtype, "row-compressed")
    _expect_compressed(vals_col, meta_col, C, R, W.dtype, "column-compressed")
    _need_device(idx, vals_row, meta_row, vals_col, meta_col, W)
    _check("sp24_prune_compress",
           _lib.sp24_prune_compress(_ptr(W), _dtype_code(W), R, C, W.stride(0), _ptr(idx), _ptr(vals_row),
                                    _ptr(meta_row), _ptr(vals_col), _ptr(meta_col), _stream(stream)))


def sp24_mask_step(W, idx, idx_prev=None, flip_count=None, vals_row=None, meta_row=None, vals_col=None,
                   meta_col=None, stream=None):
    import torch
    _need_rowmajor(idx, idx_prev, flip_count, vals_row, meta_row, vals_col, meta_col, pitched=(W,))
    R, C = _shape2(W, "W")
    _dtype_code(W)
    _expect(idx, "idx", torch.uint8, (R // 4) * (C // 4))
    _expect(idx_prev, "idx_prev", torch.uint8, (R // 4) * (C // 4))
    _expect(flip_count, "flip_count", torch.int64, 1)
    _expect_compressed(vals_row, meta_row, R, C, W.dtype, "row-compressed")
    _expect_compressed(vals_col, meta_col, C, R, W.dtype, "column-compressed")
    _need_device(idx, idx_prev, flip_count, vals_row, meta_row, vals_col, meta_col, W)
    _check("sp24_mask_step",
           _lib.sp24_mask_step(_ptr(W), _dtype_code(W), R, C, W.stride(0), _ptr(idx), _ptr(idx_prev),
                               _ptr(flip_count), _ptr(vals_row), _ptr(meta_row), _ptr(vals_col),
                               _ptr(meta_col), _stream(stream)))


def sp24_gemm_fwd(X, vals_row, meta_row, N: int, Y, epi=None, aux=None, stream=None):
    """Y[T, N] <- X[T, K] (W*m)^T, W given compressed along K; epi None, 'gelu' (aux <- pre-activation),
    'gelu_deriv' (aux <- gelu' of the pre-activation) or 'geglu' (W the stacked gate/up weight:
    Y[T, N/2] <- gelu(gate) * up, aux[T, N] <- pre-activations)."""
    _need_rowmajor(X, vals_row, meta_row, Y, aux)
    T, K = _shape2(X, "X")
    _dtype_code(X)
    _expect_compressed(vals_row, meta_row, N, K, X.dtype, "W")
    _expect(Y, "Y", X.dtype, T * (N // 2 if epi == "geglu" else N))
    _expect(aux, "aux", X.dtype, aux_elements(T, N, epi))
    _need_device(X, vals_row, meta_row, Y, aux)
    _check("sp24_gemm_fwd",
           _lib.sp24_gemm_fwd(_ptr(X), T, K, _ptr(vals_row), _ptr(meta_row), N, _dtype_code(X), _ptr(Y),
                              EPILOGUES[epi], _ptr(aux), _stream(stream)))


def sp24_gemm_dgrad(dY, vals_col, meta_col, K: int, dX, epi=None, aux=None, stream=None):
    """dX[T, K] <- dY[T, N] (W*m), W^T given compressed along N; epi None, 'dgelu' (multiplies by gelu' of
    the pre-activation in aux [T, K]), 'mul_aux' (multiplies by aux [T, K], the derivative 'gelu_deriv'
    stored) or 'dgeglu' (dX[T, 2K] <- gradients of the gated pre-activations in aux [T, 2K])."""
    _need_rowmajor(dY, vals_col, meta_col, dX, aux)
    T, N = _shape2(dY, "dY")
    _dtype_code(dY)
    _expect_compressed(vals_col, meta_col, K, N, dY.dtype, "W^T")
    width = 2 * K if epi == "dgeglu" else K
    _expect(dX, "dX", dY.dtype, T * width)
    _expect(aux, "aux", dY.dtype, aux_elements(T, width, epi))
    _need_device(dY, vals_col, meta_col, dX, aux)
    _check("sp24_gemm_dgrad",
           _lib.sp24_gemm_dgrad(_ptr(dY), T, N, _ptr(vals_col), _ptr(meta_col), K, _dtype_code(dY), _ptr(dX),
                                EPILOGUES[epi], _ptr(aux), _stream(stream)))


def sp24_gemm_dense(B, A, out, epi=None, aux=None, stream=None):
    """out[T, M] <- B[T, Kd] A[M, Kd]^T on the dense tensor-core path; epi None, 'gelu', 'dgelu',
    'gelu_deriv' or 'mul_aux'."""
    _need_rowmajor(B, A, out, aux)
    T, Kd = _shape2(B, "B")
    M = _shape2(A, "A")[0]
    _dtype_code(B)
    _expect(A, "A", B.dtype, M * Kd)
    _expect(out, "out", B.dtype, T * M)
    _expect(aux, "aux", B.dtype, aux_elements(T, M, epi))
    _need_device(B, A, out, aux)
    _check("sp24_gemm_dense",
           _lib.sp24_gemm_dense(_ptr(B), T, Kd, _ptr(A), M, _dtype_code(B), _ptr(out), EPILOGUES[epi], _ptr(aux),
                                _stream(stream)))


def sp24_gemm_dgrad_dense(dY, W, dX, epi=None, aux=None, stream=None):
    """dX[T, K] <- dY[T, N] W[N, K] on the dense tensor-core path with W read as stored;
    epi None, 'dgelu' or 'mul_aux'."""
    _need_rowmajor(dY, W, dX, aux)
    T, N = _shape2(dY, "dY")
    N2, K = _shape2(W, "W")
    if N2 != N:
        raise ValueError(f"W has {N2} rows, dY has {N} columns")
    _dtype_code(dY)
    _expect(W, "W", dY.dtype, N * K)
    _expect(dX, "dX", dY.dtype, T * K)
    _expect(aux, "aux", dY.dtype, aux_elements(T, K, epi))
    _need_device(dY, W, dX, aux)
    _check("sp24_gemm_dgrad_dense",
           _lib.sp24_gemm_dgrad_dense(_ptr(dY), T, N, _ptr(W), K, _dtype_code(dY), _ptr(dX), EPILOGUES[epi],
                                      _ptr(aux), _stream(stream)))


def sp24_transpose(x, out, stream=None):
    """out[C, R] <- x[R, C]^T (16-bit elements, bit copy)."""
    _need_rowmajor(x, out)
    R, C = _shape2(x, "x")
    _dtype_code(x)
    _expect(out, "out", x.dtype, R * C)
    _need_device(x, out)
    _check("sp24_transpose", _lib.sp24_transpose(_ptr(x), R, C, _dtype_code(x), _ptr(out), _stream(stream)))


def sp24_mvue_sparsify(dY, seed: int, offset: int, vals, meta, stream=None):
    """vals/meta <- dY[T, N]^T compressed 2:4 along T with the MVUE draws of (seed, offset)."""
    _need_rowmajor(vals, meta, pitched=(dY,))
    T, N = _shape2(dY, "dY")
    _dtype_code(dY)
    _expect_compressed(vals, meta, N, T, dY.dtype, "MVUE(dY^T)")
    _need_device(vals, meta, dY)
    _check("sp24_mvue_sparsify",
           _lib.sp24_mvue_sparsify(_ptr(dY), T, N, dY.stride(0), _dtype_code(dY), int(seed) & (2**64 - 1),
                                   int(offset) & (2**64 - 1), _ptr(vals), _ptr(meta), _stream(stream)))


def sp24_gemm_wgrad(X, vals, meta, N: int, dW, stream=None):
    """dW[N, K] (fp32) <- Yhat[N, T] X[T, K] with Yhat from sp24_mvue_sparsify."""
    import torch
    _need_rowmajor(X, vals, meta, dW)
    T, K = _shape2(X, "X")
    _dtype_code(X)
    _expect_compressed(vals, meta, N, T, X.dtype, "MVUE(dY^T)")
    _expect(dW, "dW", torch.float32, N * K)
    _need_device(X, vals, meta, dW)
    _check("sp24_gemm_wgrad",
           _lib.sp24_gemm_wgrad(_ptr(X), T, K, _ptr(vals), _ptr(meta), N, _dtype_code(X), _ptr(dW),
                                _stream(stream)))


def sp24_gemm_wgrad_noalloc(X, vals, meta, N: int, dW, stream=None):
    """sp24_gemm_wgrad through the library's fixed static scratch: no device allocation in the
    call; calls overlapping in time race on the scratch; SP24_ERR_SCRATCH_TOO_SMALL when the
    split tail would need more than it holds."""
    import torch
    _need_rowmajor(X, vals, meta, dW)
    T, K = _shape2(X, "X")
    _dtype_code(X)
    _expect_compressed(vals, meta, N, T, X.dtype, "MVUE(dY^T)")
    _expect(dW, "dW", torch.float32, N * K)
    _need_device(X, vals, meta, dW)
    _check("sp24_gemm_wgrad_noalloc",
           _lib.sp24_gemm_wgrad_noalloc(_ptr(X), T, K, _ptr(vals), _ptr(meta), N, _dtype_code(X), _ptr(dW),
                                        _stream(stream)))


def sp24_gemm_wgrad_decay(X, vals, meta, N: int, W, idx, lam: float, dW, stream=None):
    """dW[N, K] (fp32) <- Yhat[N, T] X[T, K], then dW + lam * W on the entries W's mask prunes."""
    import torch
    _need_rowmajor(X, vals, meta, W, idx, dW)
    T, K = _shape2(X, "X")
    _dtype_code(X)
    _expect_compressed(vals, meta, N, T, X.dtype, "MVUE(dY^T)")
    _expect(W, "W", X.dtype, N * K)
    _expect(idx, "idx", torch.uint8, (N // 4) * (K // 4))
    _expect(dW, "dW", torch.float32, N * K)
    _need_device(X, vals, meta, W, idx, dW)
    _check("sp24_gemm_wgrad_decay",
           _lib.sp24_gemm_wgrad_decay(_ptr(X), T, K, _ptr(vals), _ptr(meta), N, _dtype_code(X), _ptr(W), _ptr(idx),
                                      float(lam), _ptr(dW), _stream(stream)))


def sp24_gemm_wgrad_dense(X, dY, dW, stream=None):
    """dW[N, K] (fp32) <- dY[T, N]^T X[T, K] on the dense tensor-core path (dY as stored)."""
    import torch
    _need_rowmajor(X, dY, dW)
    T, K = _shape2(X, "X")
    T2, N = _shape2(dY, "dY")
    if T2 != T:
        raise ValueError(f"dY has {T2} rows, X has {T}")
    _dtype_code(X)
    _expect(dY, "dY", X.dtype, N * T)
    _expect(dW, "dW", torch.float32, N * K)
    _need_device(X, dY, dW)
    _check("sp24_gemm_wgrad_dense",
           _lib.sp24_gemm_wgrad_dense(_ptr(X), T, K, _ptr(dY), N, _dtype_code(X), _ptr(dW), _stream(stream)))


def sp24_masked_decay(grad, W, idx, lam: float, stream=None):
    """grad[R, C] (fp32, in place) <- grad + lam * W on pruned entries."""
    import torch
    _need_rowmajor(grad, W, idx)
    R, C = _shape2(W, "W")
    _dtype_code(W)
    _expect(grad, "grad", torch.float32, R * C)
    _expect(idx, "idx", torch.uint8, (R // 4) * (C // 4))
    _need_device(grad, W, idx)
    _check("sp24_masked_decay",
           _lib.sp24_masked_decay(_ptr(grad), _ptr(W), _dtype_code(W), R, C, _ptr(idx), float(lam),
                                  _stream(stream)))


def sp24_flip_rate(idx_prev, idx_cur, count, stream=None):
    """count[0] (int64 CUDA tensor, read as uint64) <- number of mask entries that differ."""
    import torch
    _need_rowmajor(idx_prev, idx_cur, count)
    _expect(idx_cur, "idx_cur", torch.uint8, idx_cur.numel())
    _expect(idx_prev, "idx_prev", torch.uint8, idx_cur.numel())
    _expect(count, "count", torch.int64, 1)
    _need_device(idx_prev, idx_cur, count)
    _check("sp24_flip_rate",
           _lib.sp24_flip_rate(_ptr(idx_prev), _ptr(idx_cur), idx_cur.numel(), _ptr(count), _stream(stream)))


def sp24_device_status(stream=None) -> int:
    """Synchronizes the stream and returns (and clears) the device error status code."""
    return int(_lib.sp24_device_status(_stream(stream)))


def sp24_set_wait_budget(cycles: int):
    _check("sp24_set_wait_budget", _lib.sp24_set_wait_budget(int(cycles)))


# ------------------------------------------------------------ conveniences

def alloc_compressed(rows: int, cols: int, dtype, device="cuda"):
    """Allocates (vals_row, meta_row, vals_col, meta_col) for W [rows x cols] with torch."""
    import torch
    vr, mr = sp24_compressed_size(rows, cols)
    vc, mc = sp24_compressed_size(cols, rows)
    return (torch.empty(rows, cols // 2, dtype=dtype, device=device),
            torch.empty(mr, dtype=torch.uint8, device=device),
            torch.empty(cols, rows // 2, dtype=dtype, device=device),
            torch.empty(mc, dtype=torch.uint8, device=device))
