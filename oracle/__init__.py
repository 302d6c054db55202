"""CPU oracle for the 2:4 transposable-mask FFN path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It shares no code, table or helper with the CUDA
library; both sides only consume the seeded tensors of ``synthetic_inputs``.

What it computes, and where the pages define it ("Accelerating Transformer
Pre-training with 2:4 Sparsity"):

* ``patterns`` / ``mask_search`` -- Algorithm 1 of the reproducibility table's
  Pseudocode row: |W| convolved at stride 4 with the candidate 4x4 patterns,
  argmax per block.  Brute force over all patterns with exact integer sums
  (plain C, ``sp24_oracle.c``); ties go to the lowest pattern index.
* ``compress_rows`` / ``decompress_rows`` -- keep the two mask-selected values
  of every group of four along a row, plus 2-bit positions.  The pages only
  name the semi-structured conversion routines (abstract page, code samples);
  the canonical layout below is this project's comparison contract.
* ``sparse_fwd`` / ``sparse_dgrad`` -- the FFN GEMMs with the pruned weight,
  ``Y = X (W*m)^T`` and ``dX = dY (W*m)``, in fp64 (software dependencies row:
  2:4 sparse matrix multiplications; abstract: transposable masks make the
  backward product 2:4 as well).
* ``gelu`` / ``gelu_grad`` -- the exact erf form of GELU between the two FFN
  layers, in fp64.
* ``masked_decay`` -- abstract: the masked decay term applied on gradients,
  ``g + lambda * (not m) * W`` as one fp32 fused multiply-add (plain C).
* ``flip_count`` -- abstract: the flip rate monitoring mask stability, read as
  the number of mask entries that differ between two masks.

Every function here is pinned by ``tests/test_oracle_*.py`` against exhaustive
search, closed forms, invariants or exact rational arithmetic.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sp24_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_sp24.so")
_lib = None

DT = {"f16": 0, "bf16": 1}


def build(force: bool = False) -> str:
    """Compile the C half of the oracle with gcc (OpenMP over block rows)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I64, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        lib.oracle_mask_search.argtypes = [P, I32, I64, I64, I64, P]
        lib.oracle_masked_decay.argtypes = [P, I64, P, I32, I64, I64, I64, P, ctypes.c_float]
        lib.oracle_patterns.argtypes = [P]
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------- patterns

def pattern_bits() -> np.ndarray:
    """The candidate patterns as uint16 bit sets (bit 4*i+j: row i, column j kept)."""
    out = np.zeros(128, dtype=np.uint16)
    n = _load().oracle_patterns(_ptr(out))
    return out[:n].copy()


def patterns() -> np.ndarray:
    """The candidate patterns as a (P, 4, 4) uint8 0/1 array, in index order."""
    b = pattern_bits().astype(np.uint32)
    cells = (b[:, None] >> np.arange(16, dtype=np.uint32)[None, :]) & 1
    return cells.reshape(-1, 4, 4).astype(np.uint8)


# ------------------------------------------------------------ conversions

def to_f64(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 values of fp16/bf16 storage given as uint16 bits."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    if dtype == "f16":
        return bits.view(np.float16).astype(np.float64)
    if dtype == "bf16":
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    raise ValueError(dtype)


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to the storage dtype, returned as float64."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))
    tdt = {"f16": torch.float16, "bf16": torch.bfloat16}[dtype]
    return t.to(tdt).to(torch.float64).numpy()


# ------------------------------------------------------------ Algorithm 1

def mask_search(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Pattern index per 4x4 block of W (uint16 storage bits, [R, C] with R, C % 4 == 0).

    Returns uint8 [R/4, C/4]: the lowest-index pattern whose exact kept |W| sum
    is maximal.  Raises on non-finite weights or unsupported shapes.
    """
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    R, C = bits.shape
    idx = np.zeros((R // 4, C // 4), dtype=np.uint8)
    st = _load().oracle_mask_search(_ptr(bits), DT[dtype], R, C, C, _ptr(idx))
    if st != 0:
        raise ValueError(f"oracle_mask_search failed with status {st}")
    return idx


def dense_mask(idx: np.ndarray) -> np.ndarray:
    """Expand pattern indices [R/4, C/4] to the 0/1 keep-mask [R, C] (bool)."""
    pats = patterns().astype(bool)[idx]            # [R/4, C/4, 4, 4]
    br, bc = idx.shape
    return pats.transpose(0, 2, 1, 3).reshape(4 * br, 4 * bc)


def prune(bits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """W * m on the storage bits: pruned entries become +0."""
    return np.where(dense_mask(idx), bits, np.uint16(0)).astype(np.uint16)


# -------------------------------------------- canonical compressed layout

NIBBLE_CODES = (0x4, 0x8, 0xC, 0x9, 0xD, 0xE)  # (i0, i1) -> i0 | i1 << 2 for i0 < i1


def compress_rows(bits: np.ndarray, keep: np.ndarray):
    """Row-wise 2:4 compression in the canonical layout.

    For row r and group g (columns 4g..4g+3) with kept offsets i0 < i1:
    ``vals[r, 2g + k] = W[r, 4g + i_k]`` and the nibble ``i0 | i1 << 2`` sits at
    bits ``4*(g % 4)`` of ``meta[r, g // 4]`` (uint16).  The kept positions come
    from the mask, so a kept weight equal to zero still occupies its slot.
    """
    R, C = bits.shape
    assert C % 16 == 0 or C % 4 == 0
    keep = keep.astype(bool)
    groups = keep.reshape(R, C // 4, 4)
    if not np.all(groups.sum(-1) == 2):
        raise ValueError("mask is not 2:4 along rows")
    pos = np.argsort(~groups, axis=-1, kind="stable")[..., :2]      # kept offsets, ascending
    vals = np.take_along_axis(bits.reshape(R, C // 4, 4), pos, axis=-1).reshape(R, C // 2)
    nib = (pos[..., 0] | (pos[..., 1] << 2)).astype(np.uint16)       # [R, C/4]
    ng = C // 4
    pad = (-ng) % 4
    nib = np.concatenate([nib, np.full((R, pad), 0x4, np.uint16)], axis=1) if pad else nib
    nib = nib.reshape(R, -1, 4)
    meta = (nib[..., 0] | nib[..., 1] << 4 | nib[..., 2] << 8 | nib[..., 3] << 12).astype(np.uint16)
    return vals.astype(np.uint16), meta


def decompress_rows(vals: np.ndarray, meta: np.ndarray, cols: int) -> np.ndarray:
    """Inverse of ``compress_rows``: dense storage bits with zeros at pruned entries."""
    R = vals.shape[0]
    ng = cols // 4
    nib = np.stack([(meta >> (4 * k)) & 0xF for k in range(4)], axis=-1).reshape(R, -1)[:, :ng]
    i0, i1 = nib & 3, (nib >> 2) & 3
    out = np.zeros((R, ng, 4), dtype=np.uint16)
    v = vals.reshape(R, ng, 2)
    rr, gg = np.meshgrid(np.arange(R), np.arange(ng), indexing="ij")
    out[rr, gg, i0] = v[..., 0]
    out[rr, gg, i1] = v[..., 1]
    return out.reshape(R, cols)


def compress_both(bits: np.ndarray, idx: np.ndarray):
    """Canonical (vals, meta) of W along rows (forward operand) and of W^T along rows
    (input-gradient operand, i.e. W compressed along its columns)."""
    keep = dense_mask(idx)
    row = compress_rows(bits, keep)
    col = compress_rows(np.ascontiguousarray(bits.T), np.ascontiguousarray(keep.T))
    return row, col


# ------------------------------------------------------------------ GEMMs

def sparse_fwd(x: np.ndarray, w: np.ndarray, keep: np.ndarray) -> np.ndarray:
    """fp64 ``Y = X (W*m)^T`` for X [T, K] and W [N, K] (float64 inputs)."""
    return np.asarray(x, np.float64) @ np.where(keep, w, 0.0).T


def sparse_dgrad(dy: np.ndarray, w: np.ndarray, keep: np.ndarray) -> np.ndarray:
    """fp64 ``dX = dY (W*m)`` for dY [T, N] and W [N, K]."""
    return np.asarray(dy, np.float64) @ np.where(keep, w, 0.0)


GEGLU_GROUP = 16  # rows of W_gate, then of W_up, alternating in the stacked gated weight


def interleave_gate_up(w_gate: np.ndarray, w_up: np.ndarray, group: int = GEGLU_GROUP) -> np.ndarray:
    """The gated FFN's two input projections as one weight [2 ff, d]: groups of
    `group` rows of W_gate and of W_up alternate ("Accelerating Transformer
    Pre-training with 2:4 Sparsity", abstract: accelerating gated activation
    functions by reducing L2 cache misses -- the product of the two halves is
    taken where both are produced, so neither is re-read from memory)."""
    ff, d = w_gate.shape
    assert w_up.shape == (ff, d) and ff % group == 0
    out = np.empty((2 * ff, d), dtype=w_gate.dtype)
    g = out.reshape(ff // group, 2, group, d)
    g[:, 0] = w_gate.reshape(ff // group, group, d)
    g[:, 1] = w_up.reshape(ff // group, group, d)
    return out


def split_gate_up(a: np.ndarray, group: int = GEGLU_GROUP):
    """Columns of a [T, 2 ff] interleaved result -> (gate part, up part), each [T, ff]."""
    T, n2 = a.shape
    g = a.reshape(T, n2 // (2 * group), 2, group)
    return g[:, :, 0].reshape(T, n2 // 2), g[:, :, 1].reshape(T, n2 // 2)


def geglu(gate: np.ndarray, up: np.ndarray) -> np.ndarray:
    """Gated GELU unit, fp64: ``gelu(gate) * up``."""
    return gelu(gate) * np.asarray(up, np.float64)


def geglu_grad(dh: np.ndarray, gate: np.ndarray, up: np.ndarray):
    """Input gradients of ``h = gelu(gate) * up`` for the upstream gradient dh:
    ``(dh * up * gelu'(gate), dh * gelu(gate))``, fp64."""
    dh = np.asarray(dh, np.float64)
    return dh * np.asarray(up, np.float64) * gelu_grad(gate), dh * gelu(gate)


def dense_fwd(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """fp64 ``Y = X W^T`` for X [T, K] and W [N, K]: the FFN forward product of
    the dense fine-tuning phase ("Accelerating Transformer Pre-training with 2:4
    Sparsity", abstract: dense fine-tuning near the end of pre-training;
    Experiment Setup row: the last 1/6 of the total steps), where no mask applies."""
    return np.asarray(x, np.float64) @ np.asarray(w, np.float64).T


def dense_dgrad(dy: np.ndarray, w: np.ndarray) -> np.ndarray:
    """fp64 ``dX = dY W`` for dY [T, N] and W [N, K] (dense fine-tuning phase)."""
    return np.asarray(dy, np.float64) @ np.asarray(w, np.float64)


def gelu(x: np.ndarray) -> np.ndarray:
    """GELU, exact erf form ``0.5 x (1 + erf(x / sqrt 2))``, fp64."""
    from scipy.special import erf
    x = np.asarray(x, np.float64)
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def gelu_grad(x: np.ndarray) -> np.ndarray:
    """d gelu / dx = Phi(x) + x phi(x), fp64."""
    from scipy.special import erf
    x = np.asarray(x, np.float64)
    return 0.5 * (1.0 + erf(x / np.sqrt(2.0))) + x * np.exp(-0.5 * x * x) / np.sqrt(2.0 * np.pi)


# ----------------------------------------------------------- masked decay

def masked_decay(grad: np.ndarray, bits: np.ndarray, dtype: str, idx: np.ndarray,
                 lam: float) -> np.ndarray:
    """fp32 ``g + lambda * (not m) * W`` with one rounding (fmaf); returns a new array."""
    g = np.array(grad, dtype=np.float32, copy=True, order="C")
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    idx = np.ascontiguousarray(idx, dtype=np.uint8)
    R, C = bits.shape
    st = _load().oracle_masked_decay(_ptr(g), C, _ptr(bits), DT[dtype], R, C, C, _ptr(idx),
                                     ctypes.c_float(lam))
    if st != 0:
        raise ValueError(f"oracle_masked_decay failed with status {st}")
    return g


# -------------------------------------------------------------- flip rate

def flip_count(idx_prev: np.ndarray, idx_cur: np.ndarray) -> int:
    """Number of mask entries that differ between two masks given as pattern indices."""
    return int(np.count_nonzero(dense_mask(idx_prev) != dense_mask(idx_cur)))


def flip_rate(idx_prev: np.ndarray, idx_cur: np.ndarray) -> float:
    """``flip_count / (R*C)``: the fraction of weights whose mask bit changed."""
    return flip_count(idx_prev, idx_cur) / (16.0 * idx_cur.size)
