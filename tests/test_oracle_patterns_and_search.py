"""Pins of the oracle's pattern table and exact mask search (Algorithm 1).

"Accelerating Transformer Pre-training with 2:4 Sparsity", reproducibility
table, Pseudocode row (Algorithm 1): |W| convolved at stride 4 with the
candidate patterns, argmax per block.  The checks here do not reuse the
oracle's arithmetic: they enumerate 8-subsets of a 4x4 block independently,
score them with exact rationals, and test invariants and symmetries.
"""
import itertools
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mask_blocks.txt")
PAIR_RANK = {p: i for i, p in enumerate(itertools.combinations(range(4), 2))}


def _doubly_two_subsets():
    """All 8-subsets of the 16 cells with two cells in every row and column."""
    out = []
    for cells in itertools.combinations(range(16), 8):
        rows = [0] * 4
        cols = [0] * 4
        for c in cells:
            rows[c // 4] += 1
            cols[c % 4] += 1
        if rows == [2] * 4 and cols == [2] * 4:
            out.append(frozenset(cells))
    return out


SUBSETS = _doubly_two_subsets()


def _lex_key(cells):
    """Rank key: the per-row column pairs, row 0 most significant."""
    key = []
    for i in range(4):
        pair = tuple(sorted(c % 4 for c in cells if c // 4 == i))
        key.append(PAIR_RANK[pair])
    return tuple(key)


def _cells_of_bits(b):
    return frozenset(c for c in range(16) if (int(b) >> c) & 1)


def _brute_force_block(vals):
    """Exact argmax over the independent enumeration, ties to the lexicographically first."""
    mags = [abs(Fraction(float(v))) for v in vals]
    best = None
    for cells in SUBSETS:
        s = sum(mags[c] for c in cells)
        key = (-s, _lex_key(cells))
        if best is None or key < best[0]:
            best = (key, cells)
    return best[1]


def _to_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    t = torch.from_numpy(np.asarray(x, dtype=np.float32)).to(si.DTYPES[dtype])
    return si.bits16(t)


# ------------------------------------------------------------------ patterns

def test_pattern_count_is_90():
    # Number of 4x4 0/1 matrices with all row and column sums 2 (OEIS A001499, n=4).
    assert len(SUBSETS) == 90
    assert oracle.patterns().shape == (90, 4, 4)


def test_pattern_table_equals_independent_enumeration():
    table = [_cells_of_bits(b) for b in oracle.pattern_bits()]
    assert len(set(table)) == 90
    assert set(table) == set(SUBSETS)


def test_pattern_table_is_lexicographic_on_row_pairs():
    keys = [_lex_key(_cells_of_bits(b)) for b in oracle.pattern_bits()]
    assert keys == sorted(keys)
    assert len(set(keys)) == len(keys)


def test_pattern_set_closed_under_transpose_and_complement():
    pats = oracle.patterns()
    as_set = {p.tobytes() for p in pats}
    for p in pats:
        assert p.sum(0).tolist() == [2] * 4 and p.sum(1).tolist() == [2] * 4
        assert np.ascontiguousarray(p.T).tobytes() in as_set
        assert (1 - p).astype(np.uint8).tobytes() in as_set


# ------------------------------------------------------------ golden blocks

def _load_golden():
    lines = [l.split() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    cases = []
    for i in range(0, len(lines), 9):
        name = lines[i][0]
        block = np.array([[float(v) for v in r] for r in lines[i + 1:i + 5]])
        keep = np.array([[int(v) for v in r] for r in lines[i + 5:i + 9]], dtype=np.uint8)
        cases.append((name, block, keep))
    return cases


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_golden_blocks(dtype):
    cases = _load_golden()
    assert len(cases) >= 8
    for name, block, keep in cases:
        bits = _to_bits(block, dtype)
        assert np.array_equal(oracle.to_f64(bits, dtype), block), name  # exact in both dtypes
        idx = oracle.mask_search(bits, dtype)
        got = oracle.patterns()[idx[0, 0]]
        assert np.array_equal(got, keep), (name, got)


# ----------------------------------------------------- exhaustive, exact

def _random_blocks(rng, n, dtype):
    """Blocks that stress exactness: gaussian, tie-heavy, wide exponent spread,
    subnormals, signed zeros, and repeated values."""
    blocks = []
    for k in range(n):
        kind = k % 6
        if kind == 0:
            v = rng.normal(0, 0.02, 16)
        elif kind == 1:
            v = np.clip(np.round(rng.normal(0, 0.02, 16) / 2**-6), -4, 3) * 2**-6
        elif kind == 2:
            lo, hi = (-24, 15) if dtype == "f16" else (-130, 120)
            v = rng.choice([-1, 1], 16) * 2.0 ** rng.integers(lo, hi, 16) * rng.uniform(1, 2, 16)
        elif kind == 3:
            v = rng.choice([0.0, -0.0, 2**-24 if dtype == "f16" else 2**-133, 1.0, 3.0], 16)
        elif kind == 4:
            v = rng.choice([0.25, -0.25, 0.5], 16)
        else:
            big = 2.0 ** (14 if dtype == "f16" else 100)
            v = rng.normal(0, 1, 16)
            v[rng.integers(0, 16)] = big
        blocks.append(np.asarray(v, dtype=np.float64).reshape(4, 4))
    return blocks


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_mask_search_matches_exhaustive_exact_search(dtype):
    rng = np.random.default_rng(1234 if dtype == "f16" else 4321)
    blocks = _random_blocks(rng, 120, dtype)
    W = np.concatenate([np.concatenate(blocks[i:i + 12], axis=1) for i in range(0, 120, 12)], axis=0)
    bits = _to_bits(W, dtype)
    idx = oracle.mask_search(bits, dtype)
    vals = oracle.to_f64(bits, dtype)
    table = [_cells_of_bits(b) for b in oracle.pattern_bits()]
    for br in range(idx.shape[0]):
        for bc in range(idx.shape[1]):
            blk = vals[4 * br:4 * br + 4, 4 * bc:4 * bc + 4].reshape(-1)
            assert table[idx[br, bc]] == _brute_force_block(blk), (br, bc, blk)


# --------------------------------------------------------------- invariants

def _scores_f64(vals):
    """Per-block scores of every pattern; exact for fp16 (sums of 8 multiples of 2^-24 < 2^19)."""
    R, C = vals.shape
    blocks = np.abs(vals).reshape(R // 4, 4, C // 4, 4).transpose(0, 2, 1, 3).reshape(-1, 16)
    pm = np.array([[1.0 if c in cells else 0.0 for c in range(16)] for cells in SUBSETS]).T
    keys = [_lex_key(c) for c in SUBSETS]
    order = np.argsort([k for k in map(lambda k: k[0] * 216 + k[1] * 36 + k[2] * 6 + k[3], keys)])
    return blocks @ pm[:, order]


def test_mask_is_maximal_and_first_on_gaussian_fp16():
    w = si.normal((256, 512), 0.02, seed=7, dtype="f16")
    bits = si.bits16(w)
    idx = oracle.mask_search(bits, "f16").reshape(-1)
    scores = _scores_f64(oracle.to_f64(bits, "f16"))
    best = scores.max(axis=1)
    assert np.all(scores[np.arange(len(idx)), idx] == best)
    assert np.all(np.argmax(scores, axis=1) == idx)


def test_mask_is_transposable_and_two_per_row_col():
    w = si.normal((128, 128), 0.02, seed=3, dtype="bf16")
    idx = oracle.mask_search(si.bits16(w), "bf16")
    keep = oracle.dense_mask(idx).astype(int)
    blocks = keep.reshape(32, 4, 32, 4)
    assert np.all(blocks.sum(axis=3) == 2)   # every row of every block keeps two
    assert np.all(blocks.sum(axis=1) == 2)   # every column of every block keeps two
    kt = keep.T.reshape(32, 4, 32, 4)
    assert np.all(kt.sum(axis=3) == 2)       # the transposed mask is 2:4 along its rows


# --------------------------------------------------------------- symmetries

def _unique_optimum(vals):
    s = _scores_f64(vals)
    top = np.sort(s, axis=1)
    return top[:, -1] > top[:, -2]


def test_metamorphic_sign_and_scale():
    w = si.normal((64, 128), 0.02, seed=11, dtype="f16")
    bits = si.bits16(w)
    idx = oracle.mask_search(bits, "f16")
    assert np.array_equal(oracle.mask_search(bits ^ np.uint16(0x8000), "f16"), idx)
    doubled = si.bits16((w.float() * 4).to(torch.float16))   # exact: no overflow at this scale
    assert np.array_equal(oracle.to_f64(doubled, "f16"), 4 * oracle.to_f64(bits, "f16"))
    assert np.array_equal(oracle.mask_search(doubled, "f16"), idx)


def test_metamorphic_transpose_and_permutation_when_unique():
    w = si.normal((64, 64), 0.02, seed=12, dtype="f16")
    bits = si.bits16(w)
    vals = oracle.to_f64(bits, "f16")
    uniq = _unique_optimum(vals).reshape(16, 16)
    assert uniq.mean() > 0.9
    pats = oracle.patterns()
    idx = oracle.mask_search(bits, "f16")
    idx_t = oracle.mask_search(np.ascontiguousarray(bits.T), "f16")
    perm = np.array([2, 0, 3, 1])
    rows = (np.arange(64) // 4) * 4 + perm[np.arange(64) % 4]
    idx_p = oracle.mask_search(np.ascontiguousarray(bits[rows]), "f16")
    for i in range(16):
        for j in range(16):
            if not uniq[i, j]:
                continue
            assert np.array_equal(pats[idx_t[j, i]], pats[idx[i, j]].T)
            assert np.array_equal(pats[idx_p[i, j]], pats[idx[i, j]][perm])


def test_rejects_non_finite_and_bad_shapes():
    bits = si.bits16(si.normal((8, 8), 0.02, 0))
    bad = bits.copy()
    bad[3, 5] = 0x7C00  # +inf in fp16
    with pytest.raises(ValueError):
        oracle.mask_search(bad, "f16")
    with pytest.raises(ValueError):
        oracle.mask_search(bits[:6, :8], "f16")
