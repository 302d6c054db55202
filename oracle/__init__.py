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
* ``mvue_sparsify_t`` / ``weight_grad`` -- the weight gradient ``dW = Yhat X``
  with Yhat the minimum-variance unbiased 2:4 estimate of dY^T along tokens (the
  MVUE kernel of the Software Dependencies row; the estimator is this project's
  reading, see ``mvue_select``), drawn with ``philox4x64_10`` (Salmon et al.,
  SC 2011) so that both sides use the same random numbers.

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


def dense_weight_grad(dy: np.ndarray, x: np.ndarray) -> np.ndarray:
    """fp64 ``dW = dY^T X`` for dY [T, N] and X [T, K]: the weight gradient of the dense
    fine-tuning phase, [N, K] in the layout of W."""
    return np.asarray(dy, np.float64).T @ np.asarray(x, np.float64)


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


# --------------------------------------- weight gradient with the MVUE of dY

# Philox4x64-10 (Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as
# easy as 1, 2, 3", SC 2011): the round multipliers and the key increments
# (golden ratio and sqrt(3) - 1 in 0.64 fixed point) of the published definition.
PHILOX_M = (0xD2E7470EE14C6C93, 0xCA5A826395121157)
PHILOX_W = (0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B)
_U64 = (1 << 64) - 1


def _mulhilo64(m: int, a: np.ndarray):
    """(high, low) 64-bit halves of the 128-bit product m * a, from 32-bit pieces."""
    a = np.asarray(a, np.uint64)
    lo32 = np.uint64(0xFFFFFFFF)
    s32 = np.uint64(32)
    mlo, mhi = np.uint64(m & 0xFFFFFFFF), np.uint64(m >> 32)
    alo, ahi = a & lo32, a >> s32
    ll, lh, hl, hh = alo * mlo, alo * mhi, ahi * mlo, ahi * mhi
    cross = (ll >> s32) + (lh & lo32) + (hl & lo32)
    lo = (ll & lo32) | (cross << s32)
    hi = hh + (lh >> s32) + (hl >> s32) + (cross >> s32)
    return hi, lo


def philox4x64_10(ctr: np.ndarray, key) -> np.ndarray:
    """Philox4x64 with 10 rounds: uint64 counters [..., 4] and a two-word key -> uint64 [..., 4].

    Round: (c0, c1, c2, c3) -> (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0));
    the key grows by the Weyl increments before every round but the first."""
    ctr = np.asarray(ctr, np.uint64)
    c = [ctr[..., i] for i in range(4)]
    k0, k1 = int(key[0]) & _U64, int(key[1]) & _U64
    for r in range(10):
        if r:
            k0, k1 = (k0 + PHILOX_W[0]) & _U64, (k1 + PHILOX_W[1]) & _U64
        hi0, lo0 = _mulhilo64(PHILOX_M[0], c[0])
        hi1, lo1 = _mulhilo64(PHILOX_M[1], c[2])
        c = [hi1 ^ c[1] ^ np.uint64(k0), lo1, hi0 ^ c[3] ^ np.uint64(k1), lo0]
    return np.stack(c, axis=-1)


def mvue_uniforms(rows: int, groups: int, seed: int, offset: int, row0: int = 0) -> np.ndarray:
    """The uniform draw of every group of four of the sparsified operand, float64 [rows, groups],
    for rows row0 .. row0 + rows - 1 of it.

    Group g of row n takes 32 bits of philox4x64_10(counter (g // 8, n, 0, 0), key (seed, offset)):
    word (g % 8) // 2, low half for even g, high half for odd g.  The top 24 of those bits,
    times 2^-24, give u in [0, 1 - 2^-24] (exact in fp32 and fp64)."""
    n = np.arange(row0, row0 + rows, dtype=np.uint64)[:, None]
    blk = np.arange((groups + 7) // 8, dtype=np.uint64)[None, :]
    ctr = np.zeros((rows, blk.shape[1], 4), np.uint64)
    ctr[..., 0] = blk
    ctr[..., 1] = n
    words = philox4x64_10(ctr, (seed, offset))                   # [rows, blocks, 4]
    g = np.arange(groups)
    w = words[:, g // 8, (g % 8) // 2]                           # [rows, groups]
    u32 = np.where((g % 2) == 0, w & np.uint64(0xFFFFFFFF), w >> np.uint64(32))
    return (u32 >> np.uint64(8)).astype(np.float64) * 2.0 ** -24


def _check_two_entries(i1: np.ndarray, i2: np.ndarray, a: np.ndarray, capped: np.ndarray) -> None:
    """Raises unless, in every uncapped group, the systematic-sampling points select two
    different entries in increasing order, both with a nonzero magnitude (see mvue_select)."""
    free = ~np.asarray(capped, bool)
    if not np.any(free):
        return
    j1, j2 = np.asarray(i1)[free], np.asarray(i2)[free]
    af = np.asarray(a)[free]
    nz1 = np.take_along_axis(af, j1[..., None], axis=-1)[..., 0] > 0
    nz2 = np.take_along_axis(af, j2[..., None], axis=-1)[..., 0] > 0
    if not (np.all(j1 < j2) and np.all(nz1) and np.all(nz2)):
        raise ArithmeticError("MVUE systematic sampling selected one entry twice or a zero entry")


def mvue_select(v: np.ndarray, u: np.ndarray):
    """Minimum-variance unbiased 2:4 estimate of each group of four values.

    ``v`` float64 [..., 4] (exact fp16/bf16 values), ``u`` float64 [...] uniform draws.
    Returns (pos [..., 2] kept positions ascending, est [..., 2] float64 estimates there).

    Reading of the "MVUE kernel" the pages name (reproducibility table, Software
    Dependencies row): an unbiased estimate with exactly two of four kept whose summed
    variance sum_i v_i^2 (1/p_i - 1) is least.  That fixes the keep probabilities at
    p_i = min(1, c |v_i|) with sum p_i = 2, and the estimate at v_i / p_i where kept.
    Two kept values are drawn by systematic sampling with one uniform u:
      * no |v_i| reaches half the group's sum S: points u S/2 and u S/2 + S/2 on the
        cumulative sums of |v| in index order select two distinct entries, each with
        probability 2 |v_i| / S, kept as sign(v_i) S/2;
      * otherwise the largest |v_m| (lowest index among equal) is kept as is, and one
        point u R on the cumulative sums of the other three (R their sum) selects the
        second, kept as sign(v_k) R; if R = 0 the lowest other position is kept as +0.
    Every step is an fp64 operation in the order written (each sum is exact for fp16
    groups); an entry is selected by counting the cumulative sums at or below the point.

    The two points always select two different nonzero entries, although the cumulative
    sums c1 <= c2 <= c3 and the total s are rounded (fp64 round-to-nearest-even is
    monotone).  With h = s/2 and no |v_i| reaching h, let the first point p1 = fl(u h)
    select entry j, i.e. c_j <= p1 < c_(j+1) (c_0 = 0):
      * j < 3: c_(j+1) = fl(c_j + a_j) <= fl(p1 + h) = p2, so p2 selects an entry after j;
      * j = 3 would need c3 <= p1 <= h and a3 < h with s = fl(c3 + a3) = 2h, so the sum
        rounds up by at least h - a3 and at most half an ulp of s, i.e. ulp(h): then a3 is
        h - ulp(h) (h not a power of two; a format of at most 51 significant bits has no
        value in [2^k - 2^(k-52), 2^k)), c3 = h, and c3 + a3 is halfway between 2a3 and 2h.
        2a3 has the even significand (a3 has trailing zeros), so s = 2a3 and the group is
        capped after all.
    An entry j < 3 is selected only if c_(j+1) > c_j, so a_j > 0; the second point selects
    the last entry only if a3 > 0 (else s = c3, and p2 < 2h = c3 since u <= 1 - 2^-24).
    Hence `_check_two_entries` never raises; it is kept so that a slip in this function
    cannot pass unnoticed.
    """
    v = np.asarray(v, np.float64)
    u = np.asarray(u, np.float64)
    a = np.abs(v)
    a0, a1, a2, a3 = a[..., 0], a[..., 1], a[..., 2], a[..., 3]
    c1 = a0
    c2 = c1 + a1
    c3 = c2 + a2
    s = c3 + a3
    m = np.argmax(a, axis=-1)
    am = np.take_along_axis(a, m[..., None], axis=-1)[..., 0]
    capped = (am + am) >= s

    # systematic sampling with two points half the total apart
    h = s * 0.5
    p1 = u * h
    p2 = p1 + h
    i1 = (c1 <= p1).astype(np.int64) + (c2 <= p1) + (c3 <= p1)
    i2 = (c1 <= p2).astype(np.int64) + (c2 <= p2) + (c3 <= p2)
    _check_two_entries(i1, i2, a, capped)

    # the largest entry kept, one point over the other three
    b = np.where(np.arange(4) == m[..., None], 0.0, a)
    e1 = b[..., 0]
    e2 = e1 + b[..., 1]
    e3 = e2 + b[..., 2]
    r = e3 + b[..., 3]
    p = u * r
    k = (e1 <= p).astype(np.int64) + (e2 <= p) + (e3 <= p)
    k = np.where(r > 0, k, np.where(m == 0, 1, 0))

    vm = np.take_along_axis(v, m[..., None], axis=-1)[..., 0]
    vk = np.take_along_axis(v, k[..., None], axis=-1)[..., 0]
    v1 = np.take_along_axis(v, i1[..., None], axis=-1)[..., 0]
    v2 = np.take_along_axis(v, i2[..., None], axis=-1)[..., 0]
    xk = np.where(r > 0, np.copysign(r, vk), 0.0)

    pa = np.where(capped, m, i1)
    pb = np.where(capped, k, i2)
    xa = np.where(capped, vm, np.copysign(h, v1))
    xb = np.where(capped, xk, np.copysign(h, v2))
    swap = pa > pb
    pos = np.stack([np.where(swap, pb, pa), np.where(swap, pa, pb)], axis=-1)
    est = np.stack([np.where(swap, xb, xa), np.where(swap, xa, xb)], axis=-1)
    return pos, est


def _f64_to_bits_via_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    """Storage bits of RNE_dtype(RNE_fp32(x))."""
    x32 = np.asarray(x, np.float64).astype(np.float32)
    if dtype == "f16":
        return x32.astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        import torch
        return torch.from_numpy(np.ascontiguousarray(x32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    raise ValueError(dtype)


def mvue_sparsify_t(dy_bits: np.ndarray, dtype: str, seed: int, offset: int, col0: int = 0):
    """MVUE 2:4 sparsification of dY^T along the token axis.

    ``dy_bits`` uint16 [T, N] (T % 4 == 0): columns col0 .. col0 + N - 1 of dY (the draws
    depend on the column's index in the full dY).  Row n of the result is column n of dY,
    with every group of four consecutive tokens reduced to two kept estimates
    (``mvue_select`` with the draws of ``mvue_uniforms(N, T/4, seed, offset)``),
    each stored as RNE_dtype(RNE_fp32(estimate)).
    Returns (bits [N, T] dense storage bits with +0 at dropped tokens, keep [N, T] bool,
    est [N, T] float64 unrounded estimates with 0 at dropped tokens)."""
    dy_bits = np.ascontiguousarray(dy_bits, dtype=np.uint16)
    T, N = dy_bits.shape
    if T % 4:
        raise ValueError("token count must be a multiple of 4")
    v = to_f64(np.ascontiguousarray(dy_bits.T), dtype).reshape(N, T // 4, 4)
    u = mvue_uniforms(N, T // 4, seed, offset, col0)
    pos, est = mvue_select(v, u)
    keep = np.zeros((N, T // 4, 4), bool)
    dense = np.zeros((N, T // 4, 4), np.float64)
    nn, gg = np.meshgrid(np.arange(N), np.arange(T // 4), indexing="ij")
    for j in range(2):
        keep[nn, gg, pos[..., j]] = True
        dense[nn, gg, pos[..., j]] = est[..., j]
    bits = np.where(keep, _f64_to_bits_via_f32(dense, dtype), np.uint16(0)).astype(np.uint16)
    return bits.reshape(N, T), keep.reshape(N, T), dense.reshape(N, T)


def weight_grad(yhat: np.ndarray, x: np.ndarray) -> np.ndarray:
    """fp64 ``dW = Yhat X`` for the sparsified dY^T, Yhat [N, T], and the layer input X [T, K]
    (the FFN weight gradient, dW [N, K] in the layout of W)."""
    return np.asarray(yhat, np.float64) @ np.asarray(x, np.float64)
