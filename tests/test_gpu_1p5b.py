"""GPU parity of the GPT-2 1.5B FFN configuration at full size, as simulated training steps.

"Accelerating Transformer Pre-training with 2:4 Sparsity": reproducibility table,
Pseudocode row (Algorithm 1: the mask is searched again at every step) and Hardware
Specification row (GPT-2 sizes); abstract (flip rate as the monitor of mask stability;
masked decay on gradients; transposable masks for the input gradient).

d = 1600, ff = 6400, 32768 tokens, fp16.  Eight steps W_(t+1) = round(W_t + N(0, 1e-4)) of
both weights, each through the calls the benchmark times: the fused mask step (search, flip
count against the previous step's mask, both compressions), the forward and input-gradient
GEMMs of both layers with GELU between (the forward storing gelu' of its pre-activation, the
input gradient multiplying by it), and the masked decay of both gradients.  Per step:
masks, flip counts, compressed values and metadata, and decayed gradients bit for bit against
the oracle; the four GEMMs at the stated tolerance on sampled token rows, each on the GPU's
own inputs.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
import structured_sparse_transformer_b200 as sp
from gpu_util import assert_gemm_close, bits_of, f64_of

pytestmark = pytest.mark.gpu


def test_gpt2_1p5b_eight_steps():
    wl = si.GPT2_1P5B
    dt, tdt = wl.dtype, si.DTYPES[wl.dtype]
    T, d, ff = wl.tokens, wl.d, wl.ff
    W1, W2 = wl.weights()
    seq = wl.weight_sequence(W1, W2)
    assert len(seq[0]) == 9
    X, dY = wl.activations()
    G1, G2 = wl.grads()
    shapes = [(ff, d), (d, ff)]
    Xd, dYd = X.cuda(), dY.cuda()
    comp = [sp.alloc_compressed(*shapes[li], tdt) for li in range(2)]
    idx_prev = [torch.empty(r // 4, c // 4, dtype=torch.uint8, device="cuda") for r, c in shapes]
    idx_cur = [torch.empty_like(i) for i in idx_prev]
    count = torch.zeros(2, dtype=torch.int64, device="cuda")
    H, Gp, dH = (torch.empty(T, ff, dtype=tdt, device="cuda") for _ in range(3))
    Y, dX = (torch.empty(T, d, dtype=tdt, device="cuda") for _ in range(2))
    o_prev = []
    for li in range(2):
        sp.sp24_mask_search(seq[li][0].cuda(), idx_prev[li])
        o_prev.append(oracle.mask_search(si.bits16(seq[li][0]), dt))
        assert np.array_equal(idx_prev[li].cpu().numpy(), o_prev[li])
    flips = []
    for t in range(8):
        Wd, o_cur = [], []
        for li in range(2):
            w = seq[li][t + 1]
            Wd.append(w.cuda())
            sp.sp24_mask_step(Wd[li], idx_cur[li], idx_prev[li], count[li:li + 1], *comp[li])
        vr1, mr1, vc1, mc1 = comp[0]
        vr2, mr2, vc2, mc2 = comp[1]
        sp.sp24_gemm_fwd(Xd, vr1, mr1, ff, H, "gelu_deriv", Gp)
        sp.sp24_gemm_fwd(H, vr2, mr2, d, Y)
        sp.sp24_gemm_dgrad(dYd, vc2, mc2, ff, dH, "mul_aux", Gp)
        sp.sp24_gemm_dgrad(dH, vc1, mc1, d, dX)
        Gd = [G1.cuda(), G2.cuda()]
        for li in range(2):
            sp.sp24_masked_decay(Gd[li], Wd[li], idx_cur[li], wl.lam)
        assert sp.sp24_device_status() == 0
        # mask step: search, flip count and both compressions, bit for bit
        for li in range(2):
            R, C = shapes[li]
            b = si.bits16(seq[li][t + 1])
            o_cur.append(oracle.mask_search(b, dt))
            assert np.array_equal(idx_cur[li].cpu().numpy(), o_cur[li]), (t, li, "mask")
            assert int(count[li].item()) == oracle.flip_count(o_prev[li], o_cur[li]), (t, li, "flips")
            (ovr, omr), (ovc, omc) = oracle.compress_both(b, o_cur[li])
            vr, mr, vc, mc = comp[li]
            assert np.array_equal(bits_of(vr).reshape(ovr.shape), ovr), (t, li, "row values")
            assert np.array_equal(bits_of(vc).reshape(ovc.shape), ovc), (t, li, "column values")
            assert np.array_equal(sp.sp24_meta_to_canonical(mr.cpu().numpy().tobytes(), R, C), omr), (t, li)
            assert np.array_equal(sp.sp24_meta_to_canonical(mc.cpu().numpy().tobytes(), C, R), omc), (t, li)
            g = (G1, G2)[li].numpy()
            ref = oracle.masked_decay(g, b, dt, o_cur[li], wl.lam)
            assert np.array_equal(Gd[li].cpu().numpy().view(np.uint32), ref.view(np.uint32)), (t, li, "decay")
        flips.append([int(c) for c in count.cpu().tolist()])
        # the four GEMMs on sampled token rows (a different sample each step)
        rows = np.arange(t * 61 % 512, T, 512)
        w1f, w2f = oracle.to_f64(si.bits16(seq[0][t + 1]), dt), oracle.to_f64(si.bits16(seq[1][t + 1]), dt)
        k1, k2 = oracle.dense_mask(o_cur[0]), oracle.dense_mask(o_cur[1])
        xs = oracle.to_f64(si.bits16(X)[rows], dt)
        pre = oracle.sparse_fwd(xs, w1f, k1)
        gp_gpu = f64_of(Gp, dt)[rows]
        assert_gemm_close(gp_gpu, oracle.gelu_grad(pre), dt, f"step {t} fwd1 gelu'")
        assert_gemm_close(f64_of(H, dt)[rows], oracle.gelu(pre), dt, f"step {t} fwd1 gelu")
        assert_gemm_close(f64_of(Y, dt)[rows], oracle.sparse_fwd(f64_of(H, dt)[rows], w2f, k2), dt, f"step {t} fwd2")
        dys = oracle.to_f64(si.bits16(dY)[rows], dt)
        assert_gemm_close(f64_of(dH, dt)[rows], oracle.sparse_dgrad(dys, w2f, k2) * gp_gpu, dt,
                          f"step {t} dgrad2 times gelu'")
        assert_gemm_close(f64_of(dX, dt)[rows], oracle.sparse_dgrad(f64_of(dH, dt)[rows], w1f, k1), dt,
                          f"step {t} dgrad1")
        o_prev = o_cur
        idx_prev, idx_cur = idx_cur, idx_prev
    # every step flips some of the mask, and none flips much of it
    n = np.array(flips, np.float64) / (d * ff)
    assert np.all(n > 0) and np.all(n < 0.05), flips
