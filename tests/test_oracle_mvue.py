"""Pins of the oracle's MVUE sparsification of dY^T and of the weight gradient.

"Accelerating Transformer Pre-training with 2:4 Sparsity" names an MVUE kernel
(reproducibility table, Software Dependencies row) without defining it; the
oracle reads it as the minimum-variance unbiased estimate that keeps exactly
two of every four consecutive tokens.  What pins it here, independently of the
oracle's own code:

* the counter-based generator against numpy's Philox4x64-10 (a separate
  implementation of the same published definition), including the layout of
  the draws per group;
* unbiasedness, exactly: the expectation over every value the 24-bit uniform can
  take (a 2^22-point sub-grid) equals the input group;
* minimum variance: the keep frequencies equal the water-filling solution found
  by bisection, and random feasible alternatives all have a larger variance;
* invariants and special cases (two kept per group, zero groups, groups with one
  or two nonzeros reproduced exactly);
* the weight-gradient product's orientation with one-hot inputs.
"""

import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si


# ----------------------------------------------------------- Philox draws

@pytest.mark.parametrize("key", [(0, 0), (123, 456), (2**64 - 1, 2**63 + 5)])
@pytest.mark.parametrize("c0", [0, 5, 2**64 - 3])
def test_philox_matches_numpy(key, c0):
    # numpy's Philox increments its 256-bit counter before each block of four words.
    g = np.random.Philox(key=np.array(key, np.uint64), counter=np.array([c0, 7, 0, 0], np.uint64))
    raw = g.random_raw(8).reshape(2, 4)
    for blk in range(2):
        c = c0 + 1 + blk
        ctr = np.array([[c % 2**64, 7 + c // 2**64, 0, 0]], np.uint64)
        assert np.array_equal(oracle.philox4x64_10(ctr, key)[0], raw[blk])


def test_uniform_layout_against_numpy_stream():
    rows, groups, seed, offset = 3, 40, 11, 7
    u = oracle.mvue_uniforms(rows, groups, seed, offset)
    for n in range(rows):
        # numpy stream starting at counter (-1, n - 1) yields blocks (0, n), (1, n), ...
        c0 = (0 - 1) % 2**64
        c1 = (n - 1) % 2**64
        g = np.random.Philox(key=np.array([seed, offset], np.uint64), counter=np.array([c0, c1, 0, 0], np.uint64))
        if n == 0:
            c1 = 2**64 - 1   # (-1, -1) + 1 carries through into word 2
            g = np.random.Philox(key=np.array([seed, offset], np.uint64),
                                 counter=np.array([2**64 - 1, 2**64 - 1, 2**64 - 1, 2**64 - 1], np.uint64))
        words = g.random_raw(4 * ((groups + 7) // 8)).reshape(-1, 4)
        for gi in range(groups):
            w = int(words[gi // 8, (gi % 8) // 2])
            u32 = (w >> (32 * (gi % 2))) & 0xFFFFFFFF
            assert u[n, gi] == (u32 >> 8) * 2.0**-24
    assert u.min() >= 0.0 and u.max() <= 1.0 - 2.0**-24


def test_uniform_first_row_counter_is_zero():
    # (block 0, row 0) is counter (0, 0, 0, 0); numpy reaches it from (-1, -1, -1, -1).
    g = np.random.Philox(key=np.array([3, 4], np.uint64), counter=np.full(4, 2**64 - 1, np.uint64))
    assert np.array_equal(oracle.philox4x64_10(np.zeros((1, 4), np.uint64), (3, 4))[0], g.random_raw(4))


# ------------------------------------------------- the estimator's moments

def _water_filling(a):
    """Keep probabilities p_i = min(1, c a_i) with sum 2, c found by bisection."""
    a = np.asarray(a, np.float64)
    if np.count_nonzero(a) <= 2:
        return (a > 0).astype(np.float64)
    lo, hi = 0.0, 2.0 / a[a > 0].min() + 1.0
    for _ in range(200):
        c = 0.5 * (lo + hi)
        if np.minimum(1.0, c * a).sum() < 2.0:
            lo = c
        else:
            hi = c
    return np.minimum(1.0, hi * a)


GROUPS = [
    [1.0, 2.0, 3.0, 4.0],
    [0.5, -0.25, 0.125, -1.0],       # largest below half the sum? 1.0 < 0.9375: no -> capped
    [-3.0, 1.0, 1.0, 1.0],           # capped exactly at half the sum
    [0.2, 0.3, -0.1, 0.4],
    [1.0, 1.0, 1.0, 0.0],
    [7.0, 0.0, 0.0, -2.0],           # two nonzeros: both kept exactly
]


def _all_draws(v, grid_bits=22):
    """est and keep of group v for every u on a 2^grid_bits sub-grid of the 24-bit draws."""
    n = 1 << grid_bits
    u = np.arange(n, dtype=np.float64) * 2.0**-grid_bits + (2.0**-grid_bits - 2.0**-24)
    mean = np.zeros(4)
    freq = np.zeros(4)
    sq = np.zeros(4)
    for lo in range(0, n, 1 << 20):
        uu = u[lo:lo + (1 << 20)]
        vv = np.broadcast_to(np.asarray(v, np.float64), (uu.size, 4))
        pos, est = oracle.mvue_select(vv, uu)
        for j in range(2):
            np.add.at(mean, pos[:, j], est[:, j])
            np.add.at(sq, pos[:, j], est[:, j] ** 2)
            np.add.at(freq, pos[:, j], 1.0)
    return mean / n, freq / n, sq / n


@pytest.mark.parametrize("v", GROUPS)
def test_unbiased_and_minimum_variance_marginals(v):
    v = np.asarray(v, np.float64)
    mean, freq, sq = _all_draws(v)
    s = np.abs(v).sum()
    # E[estimate] == v up to the draw grid (each selection probability is a multiple of 2^-22)
    assert np.allclose(mean, v, rtol=0, atol=8 * s * 2.0**-22), (mean, v)
    p = _water_filling(np.abs(v))
    keep_freq = np.where(np.abs(v) > 0, freq, 0.0)
    assert np.allclose(keep_freq, p, rtol=0, atol=8 * 2.0**-22), (keep_freq, p)
    # E[estimate^2] = v^2 / p: the variance that the water-filling marginals give
    nz = np.abs(v) > 0
    assert np.allclose(sq[nz], v[nz] ** 2 / p[nz], rtol=1e-5)


def test_water_filling_is_the_least_variance():
    rng = np.random.default_rng(5)
    for _ in range(200):
        a = np.abs(rng.normal(size=4)) * rng.choice([1.0, 10.0], size=4)
        p = _water_filling(a)
        best = (a**2 * (1 / p - 1)).sum()
        for _ in range(50):
            q = np.clip(p + rng.normal(scale=0.05, size=4), 1e-6, 1.0)
            q = q / q.sum() * 2.0
            if np.any(q > 1.0):
                continue
            assert (a**2 * (1 / q - 1)).sum() >= best - 1e-12


def test_special_groups():
    v = np.array([[0.0, 0.0, 0.0, 0.0],
                  [0.0, -5.0, 0.0, 0.0],
                  [0.0, 3.0, 0.0, -0.5],
                  [2.0, 2.0, 2.0, 2.0]])
    for u in (0.0, 0.37, 1.0 - 2.0**-24):
        pos, est = oracle.mvue_select(v, np.full(4, u))
        assert pos[0].tolist() == [0, 1] and est[0].tolist() == [0.0, 0.0]
        assert pos[1].tolist() == [0, 1] and est[1].tolist() == [0.0, -5.0]
        assert pos[2].tolist() == [1, 3] and est[2].tolist() == [3.0, -0.5]
        assert est[3].tolist() == [4.0, 4.0]
    # four equal magnitudes: each pair of neighbours half the total apart (0,2) or (1,3)
    pos, _ = oracle.mvue_select(np.tile(v[3], (4, 1)), np.array([0.0, 0.49, 0.5, 0.99]))
    assert pos.tolist() == [[0, 2], [0, 2], [1, 3], [1, 3]]


def test_golden_groups():
    """Hand-derived cases (tests/golden/mvue_groups.txt, derivations in the file)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "mvue_groups.txt")
    cases = [line.split("|") for line in open(path) if line.strip() and not line.startswith("#")]
    assert len(cases) == 10

    def num(x):
        return float.fromhex(x) if "0x" in x else float(x)

    for v, u, pos, est in cases:
        v = np.array([num(x) for x in v.split()])
        p, e = oracle.mvue_select(v[None], np.array([num(u)]))
        assert p[0].tolist() == [int(x) for x in pos.split()], (v, u)
        assert e[0].tolist() == [num(x) for x in est.split()], (v, u)


def _bf16_values(rng, shape, emin, emax):
    """Random bf16 values (as float64) with exponents uniform in [emin, emax], random signs."""
    e = rng.integers(emin, emax + 1, size=shape)
    m = rng.integers(0, 128, size=shape)
    v = np.ldexp(1.0 + m / 128.0, e) * rng.choice([-1.0, 1.0], size=shape)
    return v


def test_systematic_points_always_select_two_nonzero_entries():
    """The two sampling points of an uncapped group select two different nonzero entries for
    every input, although the fp64 cumulative sums round (the proof is in mvue_select's
    docstring); the oracle raises otherwise.  Groups here are built to stress the rounding:
    bf16 magnitudes spread over up to 250 binades, entries just below half the group's sum,
    tiny entries at rounding distance of the running sums, and the extreme draws."""
    rng = np.random.default_rng(7)
    us = np.array([0.0, 2.0**-24, 0.5, 1 - 2.0**-24])
    groups = [_bf16_values(rng, (40000, 4), -126, 124),
              _bf16_values(rng, (40000, 4), -10, 10)]
    # one entry just below half of the sum: x + y ~ z, plus a tiny entry t at or near the
    # rounding boundary of the running sums
    x = _bf16_values(rng, (40000,), -2, 2)
    y = _bf16_values(rng, (40000,), -2, 2)
    z = torch.from_numpy(np.abs(x) + np.abs(y)).to(torch.bfloat16).double().numpy()
    t = np.ldexp(1.0 + rng.integers(0, 128, 40000) / 128.0, rng.integers(-60, -45, 40000))
    for perm in ([0, 1, 2, 3], [3, 2, 1, 0], [1, 3, 0, 2]):
        groups.append(np.stack([t, x, y, z], axis=-1)[:, perm])
    checked = 0
    for g in groups:
        for u in us:
            pos, est = oracle.mvue_select(g, np.full(len(g), u))
            assert np.all(pos[:, 0] < pos[:, 1])
            kept = np.take_along_axis(g, pos, axis=-1)
            a = np.abs(g)
            capped = 2 * a.max(-1) >= a[:, 0] + a[:, 1] + a[:, 2] + a[:, 3]
            assert np.all(kept[~capped] != 0)
            checked += int((~capped).sum())
    assert checked > 100000


def test_two_entry_check_rejects_a_planted_slip():
    a = np.array([[1.0, 1.0, 1.0, 0.0]])
    capped = np.array([False])
    oracle._check_two_entries(np.array([0]), np.array([2]), a, capped)
    with pytest.raises(ArithmeticError):
        oracle._check_two_entries(np.array([1]), np.array([1]), a, capped)     # one entry twice
    with pytest.raises(ArithmeticError):
        oracle._check_two_entries(np.array([0]), np.array([3]), a, capped)     # a zero entry
    oracle._check_two_entries(np.array([1]), np.array([1]), a, np.array([True]))  # capped: not checked


def test_sparsify_invariants():
    t, n = 256, 64
    dy = si.normal((t, n), 1.0, 3, "f16")
    bits, keep, est = oracle.mvue_sparsify_t(si.bits16(dy), "f16", seed=9, offset=1)
    assert bits.shape == (n, t) and keep.shape == (n, t)
    assert np.all(keep.reshape(n, t // 4, 4).sum(-1) == 2)
    assert np.all(bits[~keep] == 0)
    # the stored value is the estimate rounded to fp32 then fp16
    assert np.array_equal(oracle.to_f64(bits, "f16")[keep],
                          est[keep].astype(np.float32).astype(np.float16).astype(np.float64))
    # an estimate is at least as large as the entry it replaces (p <= 1)
    dyt = dy.float().numpy().T
    assert np.all(np.abs(est[keep]) >= np.abs(dyt[keep]) * (1 - 1e-12))
    assert np.all(np.sign(est[keep]) * np.sign(dyt[keep]) >= 0)
    # canonical compression of the result: two codes per group, round trip exact
    vals, meta = oracle.compress_rows(bits, keep)
    assert np.array_equal(oracle.decompress_rows(vals, meta, t), bits)
    # the same seed and offset reproduce, another offset draws anew
    bits2, _, _ = oracle.mvue_sparsify_t(si.bits16(dy), "f16", seed=9, offset=1)
    bits3, _, _ = oracle.mvue_sparsify_t(si.bits16(dy), "f16", seed=9, offset=2)
    assert np.array_equal(bits, bits2) and not np.array_equal(bits, bits3)


def test_column_sample_matches_the_full_matrix():
    t, n = 64, 40
    dy = si.normal((t, n), 1.0, 12, "bf16")
    full, _, _ = oracle.mvue_sparsify_t(si.bits16(dy), "bf16", 4, 9)
    part, _, _ = oracle.mvue_sparsify_t(si.bits16(dy[:, 17:29].contiguous()), "bf16", 4, 9, col0=17)
    assert np.array_equal(part, full[17:29])


def test_sparsify_bf16_exact_keeps():
    # Groups with at most two nonzeros are reproduced exactly in any dtype.
    t, n = 16, 8
    x = torch.zeros(t, n)
    x[0, :] = torch.linspace(-3, 3, n)
    x[5, :] = 1e-30
    x[10, :] = 2.0**100
    bits, keep, est = oracle.mvue_sparsify_t(si.bits16(x.to(torch.bfloat16)), "bf16", seed=1, offset=0)
    assert np.array_equal(oracle.to_f64(bits, "bf16"), x.to(torch.bfloat16).double().numpy().T)


def test_sparsify_statistics_on_a_matrix():
    # Averaged over independent offsets the sparsified operand approaches dY^T.
    t, n, draws = 64, 16, 400
    dy = si.normal((t, n), 1.0, 4, "f16")
    acc = np.zeros((n, t))
    for off in range(draws):
        acc += oracle.mvue_sparsify_t(si.bits16(dy), "f16", seed=2, offset=off)[2]
    dyt = dy.double().numpy().T
    # per-entry standard deviation of one draw is below the group's |sum| / 2 * sqrt(2)
    err = np.abs(acc / draws - dyt)
    bound = 5 * np.abs(dyt).reshape(n, t // 4, 4).sum(-1).repeat(4, -1).reshape(n, t) / np.sqrt(draws)
    assert np.all(err <= bound)


# ------------------------------------------------------- weight gradient

def test_weight_grad_orientation_one_hot():
    t, n, k = 32, 8, 5
    dy = si.normal((t, n), 1.0, 6, "f16")
    bits, _, _ = oracle.mvue_sparsify_t(si.bits16(dy), "f16", seed=0, offset=0)
    yhat = oracle.to_f64(bits, "f16")                         # [n, t]
    col = np.arange(t) % k
    x = np.zeros((t, k))
    x[np.arange(t), col] = 1.0
    dw = oracle.weight_grad(yhat, x)
    assert dw.shape == (n, k)
    for j in range(k):
        assert np.array_equal(dw[:, j], yhat[:, col == j].sum(axis=1))


def test_weight_grad_expectation_is_dense():
    # E[Yhat] = dY^T entrywise, so for a fixed X the expected gradient is dY^T X.
    t, n, k, draws = 32, 4, 3, 600
    dy = si.normal((t, n), 1.0, 7, "f16")
    x = si.normal((t, k), 1.0, 8, "f16").double().numpy()
    acc = np.zeros((n, k))
    for off in range(draws):
        acc += oracle.weight_grad(oracle.mvue_sparsify_t(si.bits16(dy), "f16", seed=3, offset=off)[2], x)
    dense = dy.double().numpy().T @ x
    assert np.allclose(acc / draws, dense, atol=0.25 * np.abs(dense).max() + 0.5)
