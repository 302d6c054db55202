"""Pins of the oracle's masked decay and flip count.

"Accelerating Transformer Pre-training with 2:4 Sparsity", abstract: the masked
decay term is applied on gradients, and a flip rate monitors how stable the
2:4 mask is.  Decay is pinned against exact rational arithmetic (the fp32
result must be the correctly rounded g + lambda*W), flips against the
combinatorics of the pattern set.
"""
from fractions import Fraction

import numpy as np
import torch

import oracle
import synthetic_inputs as si


def _is_correctly_rounded_f32(exact: Fraction, r: np.float32) -> bool:
    """r is the fp32 nearest to ``exact`` (ties to even)."""
    up = np.nextafter(r, np.float32(np.inf))
    dn = np.nextafter(r, np.float32(-np.inf))
    d = abs(Fraction(float(r)) - exact)
    if d > abs(Fraction(float(up)) - exact) or d > abs(Fraction(float(dn)) - exact):
        return False
    for nb in (up, dn):
        if d == abs(Fraction(float(nb)) - exact):   # a tie: r must have an even significand
            return int(np.array(r).view(np.uint32)) % 2 == 0
    return True


def test_decay_lambda_zero_is_identity_and_kept_entries_untouched():
    w = si.normal((32, 64), 0.02, seed=0, dtype="f16")
    g = si.normal((32, 64), 1e-2, seed=4, dtype="f32").numpy()
    bits = si.bits16(w)
    idx = oracle.mask_search(bits, "f16")
    keep = oracle.dense_mask(idx)
    assert np.array_equal(oracle.masked_decay(g, bits, "f16", idx, 0.0).view(np.uint32),
                          g.view(np.uint32))
    out = oracle.masked_decay(g, bits, "f16", idx, 6e-5)
    assert np.array_equal(out.view(np.uint32)[keep], g.view(np.uint32)[keep])
    assert np.any(out[~keep] != g[~keep])


def test_decay_closed_form_on_constants():
    w = np.ones((4, 4), np.float32)
    bits = si.bits16(torch.from_numpy(w).half())
    idx = np.zeros((1, 1), np.uint8)  # pattern 0 keeps rows (0,1),(0,1),(2,3),(2,3)
    out = oracle.masked_decay(np.ones((4, 4), np.float32), bits, "f16", idx, 0.5)
    expect = np.array([[1, 1, 1.5, 1.5]] * 2 + [[1.5, 1.5, 1, 1]] * 2, np.float32)
    assert np.array_equal(out, expect)


def test_decay_is_single_rounding_of_the_exact_value():
    rng = np.random.default_rng(7)
    for dtype in ("f16", "bf16"):
        w = si.normal((16, 32), 0.02, seed=1, dtype=dtype)
        bits = si.bits16(w)
        wf = oracle.to_f64(bits, dtype)
        g = (rng.normal(0, 1e-2, (16, 32)) * 2.0 ** rng.integers(-20, 4, (16, 32))).astype(np.float32)
        lam = np.float32(6e-5)
        idx = oracle.mask_search(bits, dtype)
        keep = oracle.dense_mask(idx)
        out = oracle.masked_decay(g, bits, dtype, idx, float(lam))
        for r, c in zip(*np.nonzero(~keep)):
            exact = Fraction(float(g[r, c])) + Fraction(float(lam)) * Fraction(float(wf[r, c]))
            assert _is_correctly_rounded_f32(exact, out[r, c]), (dtype, r, c)


def test_decay_fused_rounding_differs_from_two_roundings_somewhere():
    # With lambda*w near g's ulp, fmaf and (g + round(lambda*w)) disagree on some
    # inputs; the oracle must side with the single rounding.
    rng = np.random.default_rng(3)
    w = si.normal((64, 64), 0.02, seed=9, dtype="f16")
    bits = si.bits16(w)
    idx = oracle.mask_search(bits, "f16")
    g = rng.normal(0, 1e-6, (64, 64)).astype(np.float32)
    lam = np.float32(1e-3)
    out = oracle.masked_decay(g, bits, "f16", idx, float(lam))
    two = (g + (lam * oracle.to_f64(bits, "f16").astype(np.float32))).astype(np.float32)
    keep = oracle.dense_mask(idx)
    assert np.any(out[~keep] != two[~keep])


def test_flip_count_invariants():
    pats = oracle.patterns()
    bits = oracle.pattern_bits().astype(np.uint32)
    complement = {p.tobytes(): i for i, p in enumerate(pats)}
    rng = np.random.default_rng(5)
    a = rng.integers(0, 90, (8, 16)).astype(np.uint8)
    b = rng.integers(0, 90, (8, 16)).astype(np.uint8)
    assert oracle.flip_count(a, a) == 0
    assert oracle.flip_count(a, b) == oracle.flip_count(b, a)
    per_block = [bin(int(bits[x] ^ bits[y])).count("1") for x, y in zip(a.ravel(), b.ravel())]
    assert all(c % 2 == 0 and c <= 16 for c in per_block)
    assert oracle.flip_count(a, b) == sum(per_block)
    comp = np.vectorize(lambda i: complement[(1 - pats[i]).astype(np.uint8).tobytes()])(a).astype(np.uint8)
    assert oracle.flip_count(a, comp) == 16 * a.size
    assert abs(oracle.flip_rate(a, comp) - 1.0) < 1e-15


def test_flip_after_small_perturbation_is_small():
    w = si.normal((256, 256), 0.02, seed=0, dtype="f16")
    w2 = si.perturb(w, seed=100)
    i1 = oracle.mask_search(si.bits16(w), "f16")
    i2 = oracle.mask_search(si.bits16(w2), "f16")
    rate = oracle.flip_rate(i1, i2)
    assert 0.0 < rate < 0.1
