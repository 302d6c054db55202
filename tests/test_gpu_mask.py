"""GPU parity of the mask path against the CPU oracle, through the C ABI.

Mask search (Algorithm 1 of "Accelerating Transformer Pre-training with 2:4
Sparsity", reproducibility table, Pseudocode row), compression, flip count
(abstract) and masked decay (abstract) must all be bit-exact.  Shapes cover
the PR1 weight and the GPT-2 355M/774M/1.5B FFN weights in full, ragged edges,
tie-heavy and wide-range inputs, and the large sweep sizes on sampled block
rows (blocks are independent, so a row slice of W has the same mask rows).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
import structured_sparse_transformer_b200 as sp
from gpu_util import bits_of

pytestmark = pytest.mark.gpu


def _search(w_cpu, ldw_pad=0):
    R, C = w_cpu.shape
    if ldw_pad:
        base = torch.zeros(R, C + ldw_pad, dtype=w_cpu.dtype, device="cuda")
        base[:, :C] = w_cpu.cuda()
        wd = base[:, :C]
    else:
        wd = w_cpu.cuda()
    idx = torch.full((R // 4, C // 4), 255, dtype=torch.uint8, device="cuda")
    sp.sp24_mask_search(wd, idx)
    torch.cuda.synchronize()
    return idx.cpu().numpy()


def _dt(t):
    return "bf16" if t.dtype == torch.bfloat16 else "f16"


def _wide_range_bf16(R, C, seed):
    rng = np.random.default_rng(seed)
    v = rng.choice([-1, 1], (R, C)) * 2.0 ** rng.integers(-130, 120, (R, C)) * rng.uniform(1, 2, (R, C))
    v[rng.random((R, C)) < 0.1] = 0.0
    return torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)


def _specials_f16(R, C, seed):
    rng = np.random.default_rng(seed)
    pool = np.array([0.0, -0.0, 2.0**-24, 3 * 2.0**-24, 2.0**-14, 0.5, 1.0, 65504.0, -65504.0, 1024.0],
                    dtype=np.float32)
    v = pool[rng.integers(0, len(pool), (R, C))]
    return torch.from_numpy(v).to(torch.float16)


CASES = [
    ("tiny-4x4", lambda: si.normal((4, 4), 0.02, 0)),
    ("ragged-36x44", lambda: si.normal((36, 44), 0.02, 1)),
    ("ragged-132x260-bf16", lambda: si.normal((132, 260), 0.02, 2, "bf16")),
    ("pr1-3072x768", lambda: si.normal((3072, 768), 0.02, 0)),
    ("355m-W1-4096x1024", lambda: si.GPT2_355M.weights()[0]),
    ("355m-W2-1024x4096", lambda: si.GPT2_355M.weights()[1]),
    ("774m-W1-5120x1280-bf16", lambda: si.GPT2_774M.weights()[0]),
    ("774m-W2-1280x5120-bf16", lambda: si.GPT2_774M.weights()[1]),
    ("1.5b-W1-6400x1600", lambda: si.GPT2_1P5B.weights()[0]),
    ("1.5b-W2-1600x6400", lambda: si.GPT2_1P5B.weights()[1]),
    ("tie-heavy-1024x4096-f16", lambda: si.tie_heavy((1024, 4096), 5, "f16")),
    ("tie-heavy-1024x4096-bf16", lambda: si.tie_heavy((1024, 4096), 6, "bf16")),
    ("wide-range-256x256-bf16", lambda: _wide_range_bf16(256, 256, 7)),
    ("specials-256x256-f16", lambda: _specials_f16(256, 256, 8)),
    ("sweep-1024x1024", lambda: si.normal((1024, 1024), 0.02, 10)),
    ("sweep-4096x4096", lambda: si.normal((4096, 4096), 0.02, 12)),
]


@pytest.mark.parametrize("name,make", CASES, ids=[c[0] for c in CASES])
def test_mask_search_bit_exact(name, make):
    w = make()
    got = _search(w)
    assert np.array_equal(got, oracle.mask_search(si.bits16(w), _dt(w))), name


def test_mask_search_strided_rows():
    w = si.normal((64, 96), 0.02, 3)
    assert np.array_equal(_search(w, ldw_pad=32), oracle.mask_search(si.bits16(w), "f16"))


def test_mask_search_empty_is_ok():
    idx = torch.empty(0, dtype=torch.uint8, device="cuda")
    w = torch.empty(0, 8, dtype=torch.float16, device="cuda")
    sp.sp24_mask_search(w, idx)
    torch.cuda.synchronize()


@pytest.mark.parametrize("shape,seed,kind", [((4096, 16384), 13, "normal"), ((16384, 16384), 14, "normal"),
                                             ((16384, 16384), 15, "tie"), ((16384, 65536), 16, "normal")])
def test_mask_search_sweep_sampled_rows(shape, seed, kind):
    w = si.normal(shape, 0.02, seed) if kind == "normal" else si.tie_heavy(shape, seed)
    got = _search(w)
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(shape[0] // 4, 24, replace=False))
    bits = si.bits16(w)
    for br in rows:
        exp = oracle.mask_search(np.ascontiguousarray(bits[4 * br:4 * br + 4]), "f16")
        assert np.array_equal(got[br:br + 1], exp), br


def _device_weights(R, C, seed, kind, update_seed=None):
    """fp16 [R, C] drawn on the device in row slabs: N(0, 0.02) (or its 8-level tie-heavy
    rounding), optionally followed by one N(0, 1e-4) update."""
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    w = torch.empty(R, C, dtype=torch.float16, device="cuda")
    for r0 in range(0, R, 1024):
        x = torch.randn(min(1024, R - r0), C, device="cuda", generator=g) * 0.02
        if kind == "tie":
            x = torch.clamp(torch.round(x / 2.0**-6), -4, 3) * 2.0**-6
        w[r0:r0 + x.shape[0]] = x.half()
    if update_seed is not None:
        g.manual_seed(update_seed)
        for r0 in range(0, R, 1024):
            sl = w[r0:r0 + 1024]
            sl.copy_((sl.float() + torch.randn(sl.shape, device="cuda", generator=g) * 1e-4).half())
    return w


@pytest.mark.parametrize("kind,seed", [("normal", 31), ("tie", 32)])
def test_mask_step_at_the_sweep_size(kind, seed):
    """The fused mask step on a 2 GiB fp16 weight (16384 x 65536, the sweep's largest size):
    the mask and the flip count equal the separate search and flip kernels in full, and 12
    sampled 16-row strips of the mask and of both compressed orientations equal the oracle."""
    R, C = 16384, 65536
    w0 = _device_weights(R, C, seed, kind)
    prev = torch.empty(R // 4, C // 4, dtype=torch.uint8, device="cuda")
    sp.sp24_mask_search(w0, prev)
    del w0
    w1 = _device_weights(R, C, seed, kind, update_seed=seed + 100)
    idx = torch.empty_like(prev)
    count = torch.zeros(1, dtype=torch.int64, device="cuda")
    bufs = sp.alloc_compressed(R, C, torch.float16)
    sp.sp24_mask_step(w1, idx, prev, count, *bufs)
    sep = torch.empty_like(prev)
    sp.sp24_mask_search(w1, sep)
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    sp.sp24_flip_rate(prev, sep, cnt)
    torch.cuda.synchronize()
    assert sp.sp24_device_status() == 0
    assert torch.equal(idx, sep)
    assert int(count.item()) == int(cnt.item()) > 0
    mr = sp.sp24_meta_to_canonical(bufs[1].cpu().numpy().tobytes(), R, C)
    mc = sp.sp24_meta_to_canonical(bufs[3].cpu().numpy().tobytes(), C, R)
    vr, vc = bufs[0], bufs[2]
    idx_h = idx.cpu().numpy()
    rng = np.random.default_rng(seed)
    for s16 in np.sort(rng.choice(R // 16, 12, replace=False)):
        r0 = 16 * int(s16)
        bits = si.bits16(w1[r0:r0 + 16].cpu())
        i_o = oracle.mask_search(bits, "f16")
        assert np.array_equal(idx_h[r0 // 4:r0 // 4 + 4], i_o), r0
        (vr_o, mr_o), (vc_o, mc_o) = oracle.compress_both(bits, i_o)
        assert np.array_equal(bits_of(vr[r0:r0 + 16]), vr_o), r0
        assert np.array_equal(mr[r0:r0 + 16], mr_o), r0
        assert np.array_equal(bits_of(vc[:, r0 // 2:r0 // 2 + 8].contiguous()), vc_o), r0
        assert np.array_equal(mc[:, r0 // 16:r0 // 16 + 1], mc_o), r0


# -------------------------------------------------------------- compression

def _compress_gpu(w_cpu, idx_np):
    R, C = w_cpu.shape
    bufs = sp.alloc_compressed(R, C, w_cpu.dtype)
    sp.sp24_prune_compress(w_cpu.cuda(), torch.from_numpy(idx_np).cuda(), *bufs)
    torch.cuda.synchronize()
    return bufs


@pytest.mark.parametrize("R,C,dtype,seed", [(16, 16, "f16", 0), (48, 80, "bf16", 1), (144, 400, "f16", 2),
                                            (3072, 768, "f16", 0), (6400, 1600, "f16", 3),
                                            (1280, 5120, "bf16", 4)])
def test_prune_compress_bit_exact(R, C, dtype, seed):
    w = si.normal((R, C), 0.02, seed, dtype)
    bits = si.bits16(w)
    idx = oracle.mask_search(bits, dtype)
    vr, mr, vc, mc = _compress_gpu(w, idx)
    (vr_o, mr_o), (vc_o, mc_o) = oracle.compress_both(bits, idx)
    assert np.array_equal(bits_of(vr), vr_o)
    assert np.array_equal(bits_of(vc), vc_o)
    mr_h, mc_h = mr.cpu().numpy(), mc.cpu().numpy()
    assert np.array_equal(sp.sp24_meta_to_canonical(mr_h.tobytes(), R, C), mr_o)
    assert np.array_equal(sp.sp24_meta_to_canonical(mc_h.tobytes(), C, R), mc_o)
    # the whole buffer is defined: padding is exactly what the host layout map writes
    assert np.array_equal(mr_h, sp.sp24_meta_from_canonical(mr_o, R, C))
    assert np.array_equal(mc_h, sp.sp24_meta_from_canonical(mc_o, C, R))


def test_prune_compress_one_orientation():
    w = si.normal((64, 128), 0.02, 9)
    bits = si.bits16(w)
    idx = oracle.mask_search(bits, "f16")
    vr, mr, _, _ = sp.alloc_compressed(64, 128, torch.float16)
    sp.sp24_prune_compress(w.cuda(), torch.from_numpy(idx).cuda(), vr, mr, None, None)
    torch.cuda.synchronize()
    (vr_o, mr_o), _ = oracle.compress_both(bits, idx)
    assert np.array_equal(bits_of(vr), vr_o)


# -------------------------------------------------- fused mask step + flip

@pytest.mark.parametrize("wl", [si.GPT2_774M, si.GPT2_1P5B], ids=lambda w: w.name)
def test_mask_step_fused_matches_separate_ops(wl):
    w0 = wl.weights()[0]
    w1 = si.perturb(w0, wl.perturb_seed(0, 0))
    dt = _dt(w0)
    R, C = w0.shape
    i0 = oracle.mask_search(si.bits16(w0), dt)
    i1 = oracle.mask_search(si.bits16(w1), dt)
    prev = torch.from_numpy(i0).cuda()
    idx = torch.empty_like(prev)
    count = torch.zeros(1, dtype=torch.int64, device="cuda")
    bufs = sp.alloc_compressed(R, C, w0.dtype)
    sp.sp24_mask_step(w1.cuda(), idx, prev, count, *bufs)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), i1)
    assert int(count.item()) == oracle.flip_count(i0, i1)
    (vr_o, mr_o), (vc_o, mc_o) = oracle.compress_both(si.bits16(w1), i1)
    assert np.array_equal(bits_of(bufs[0]), vr_o)
    assert np.array_equal(bits_of(bufs[2]), vc_o)
    assert np.array_equal(sp.sp24_meta_to_canonical(bufs[1].cpu().numpy().tobytes(), R, C), mr_o)
    assert np.array_equal(sp.sp24_meta_to_canonical(bufs[3].cpu().numpy().tobytes(), C, R), mc_o)


@pytest.mark.parametrize("n", [0, 1, 15, 16, 17, 640000, 640003])
def test_flip_rate_bit_exact(n):
    rng = np.random.default_rng(n)
    a = rng.integers(0, 90, n).astype(np.uint8)
    b = a.copy()
    ch = rng.random(n) < 0.3
    b[ch] = rng.integers(0, 90, int(ch.sum())).astype(np.uint8)
    count = torch.full((1,), 12345, dtype=torch.int64, device="cuda")
    da, db = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    sp.sp24_flip_rate(da, db, count)
    torch.cuda.synchronize()
    expect = oracle.flip_count(a.reshape(1, -1), b.reshape(1, -1)) if n else 0
    assert int(count.item()) == expect
    if n > 1:   # unaligned start: the vector path must not be taken
        sp.sp24_flip_rate(da[1:], db[1:], count)
        torch.cuda.synchronize()
        assert int(count.item()) == oracle.flip_count(a[1:].reshape(1, -1), b[1:].reshape(1, -1))


# ----------------------------------------------------------- masked decay

@pytest.mark.parametrize("R,C,dtype,lam", [(4, 4, "f16", 0.5), (36, 44, "bf16", 6e-5), (4096, 1024, "f16", 6e-5),
                                           (1280, 5120, "bf16", 6e-5), (64, 64, "f16", 0.0)])
def test_masked_decay_bit_exact(R, C, dtype, lam):
    w = si.normal((R, C), 0.02, R + C, dtype)
    g = si.normal((R, C), 1e-2, 4, "f32")
    bits = si.bits16(w)
    idx = oracle.mask_search(bits, dtype)
    gd = g.cuda()
    sp.sp24_masked_decay(gd, w.cuda(), torch.from_numpy(idx).cuda(), lam)
    torch.cuda.synchronize()
    exp = oracle.masked_decay(g.numpy(), bits, dtype, idx, lam)
    assert np.array_equal(gd.cpu().numpy().view(np.uint32), exp.view(np.uint32))
