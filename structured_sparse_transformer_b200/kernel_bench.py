"""Single-kernel benchmark of libsp24 on one GPU (also the target of ncu captures).

    python -m structured_sparse_transformer_b200.kernel_bench --kernel mask_search --rows 16384 --cols 16384
    python -m structured_sparse_transformer_b200.kernel_bench --kernel gemm_fwd --rows 4096 --cols 1024 \
        --tokens 8192 --epi gelu

W is [rows x cols] (N(0, 0.02), or the 8-level tie-heavy variant with
--dist tie), drawn on the device from a seeded generator.  GEMMs use
T = --tokens rows of N(0, 1) activations: gemm_fwd computes [T x rows] from
[T x cols], gemm_dgrad [T x cols] from [T x rows], gemm_wgrad the fp32
[rows x cols] weight gradient from dY [T x rows] (MVUE-sparsified) and
X [T x cols] (gemm_wgrad_decay: with the masked decay of W's mask in its epilogue;
gemm_wgrad_dense: dY dense, read as stored); mvue sparsifies dY [T x rows] (bytes per dY
element).  Each timed launch follows an
L2 flush (256 MiB write) and is timed alone with CUDA events on the current
stream.  Prints one JSON line: average microseconds per launch and the
algorithmic throughput (bytes for the memory-bound kernels, dense-equivalent
FLOPs 2*T*rows*cols for the GEMMs).
"""
from __future__ import annotations

import argparse
import json

import torch

import structured_sparse_transformer_b200 as sp

# Algorithmic bytes per weight element.
BYTES_PER_ELEMENT = {
    "mask_search": 2 + 1 / 16,                       # read W, write the index
    "mask_step": 2 + 1 / 16 + 1 / 16 + 2 + 0.25,     # + previous index, both compressed orientations
    "prune_compress": 2 + 1 / 16 + 2 + 0.25,         # read W and index, write both orientations
    "masked_decay": 4 + 2 + 1 / 16 + 4,              # read g, W, index; write g
    "flip": 2 / 16,                                  # read two indices
    "transpose": 4,                                  # read W, write W^T
    "mvue": 2 + 1 + 1 / 8,                           # read dY; write kept values and metadata
}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--kernel", required=True,
                    choices=sorted(BYTES_PER_ELEMENT) + ["gemm_fwd", "gemm_dgrad", "gemm_dense_fwd", "gemm_dense_dgrad",
                                                         "gemm_wgrad", "gemm_wgrad_decay", "gemm_wgrad_dense"])
    ap.add_argument("--rows", type=int, required=True)
    ap.add_argument("--cols", type=int, required=True)
    ap.add_argument("--tokens", type=int, default=8192)
    ap.add_argument("--dtype", choices=["f16", "bf16"], default="f16")
    ap.add_argument("--via-transpose", action="store_true",
                    help="gemm_dense_dgrad: multiply by W^T formed with sp24_transpose")
    ap.add_argument("--dist", choices=["normal", "tie"], default="normal")
    ap.add_argument("--epi", choices=["none", "gelu", "dgelu", "gelu_deriv", "mul_aux", "geglu", "dgeglu",
                                      "gelu_deriv_packed", "mul_aux_packed"],
                    default="none")
    ap.add_argument("--iters", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--seed", type=int, default=0)
    args = ap.parse_args(argv)

    dev = torch.device("cuda", torch.cuda.current_device())
    tdt = torch.float16 if args.dtype == "f16" else torch.bfloat16
    gen = torch.Generator(device=dev)
    gen.manual_seed(args.seed)
    R, C, T = args.rows, args.cols, args.tokens
    w = torch.randn(R, C, device=dev, generator=gen) * 0.02
    if args.dist == "tie":
        w = torch.clamp(torch.round(w / 2.0**-6), -4, 3) * 2.0**-6
    w = w.to(tdt)
    idx = torch.empty(R // 4, C // 4, dtype=torch.uint8, device=dev)
    prev = torch.empty_like(idx)
    count = torch.zeros(1, dtype=torch.int64, device=dev)
    bufs = sp.alloc_compressed(R, C, tdt, device=dev)
    sp.sp24_mask_step(w, prev, None, None, *bufs)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    k = args.kernel
    if k == "mask_search":
        fn = lambda: sp.sp24_mask_search(w, idx)
    elif k == "mask_step":
        fn = lambda: sp.sp24_mask_step(w, idx, prev, count, *bufs)
    elif k == "prune_compress":
        fn = lambda: sp.sp24_prune_compress(w, prev, *bufs)
    elif k == "masked_decay":
        g = torch.randn(R, C, device=dev, generator=gen) * 1e-2
        fn = lambda: sp.sp24_masked_decay(g, w, prev, 6e-5)
    elif k == "flip":
        fn = lambda: sp.sp24_flip_rate(prev, idx, count)
        sp.sp24_mask_search(w, idx)
    elif k == "gemm_fwd":
        x = torch.randn(T, C, device=dev, generator=gen).to(tdt)
        epi = args.epi if args.epi in ("gelu", "gelu_deriv", "geglu", "gelu_deriv_packed") else None
        # geglu: W is the stacked gate/up weight [rows = 2 ff, cols]; out [T, ff], aux [T, 2 ff]
        y = torch.empty(T, R // 2 if epi == "geglu" else R, dtype=tdt, device=dev)
        aux = torch.empty(sp.aux_elements(T, R, epi), dtype=tdt, device=dev) if epi else None
        fn = lambda: sp.sp24_gemm_fwd(x, bufs[0], bufs[1], R, y, epi, aux)
    elif k in ("mvue", "gemm_wgrad", "gemm_wgrad_decay"):
        dy = torch.randn(T, R, device=dev, generator=gen).to(tdt)
        yv = torch.empty(R, T // 2, dtype=tdt, device=dev)
        ym = torch.empty(sp.sp24_compressed_size(R, T)[1], dtype=torch.uint8, device=dev)
        sp.sp24_mvue_sparsify(dy, 200, 0, yv, ym)
        if k == "mvue":
            fn = lambda: sp.sp24_mvue_sparsify(dy, 200, 1, yv, ym)
        else:
            x = torch.randn(T, C, device=dev, generator=gen).to(tdt)
            dw = torch.empty(R, C, dtype=torch.float32, device=dev)
            if k == "gemm_wgrad":
                fn = lambda: sp.sp24_gemm_wgrad(x, yv, ym, R, dw)
            else:   # dW of W [rows x cols] with the masked decay in the epilogue
                fn = lambda: sp.sp24_gemm_wgrad_decay(x, yv, ym, R, w, prev, 6e-5, dw)
    elif k == "gemm_wgrad_dense":
        # dW [rows x cols] fp32 = dY^T X, dY [T x rows] and X [T x cols] read as stored
        dy = torch.randn(T, R, device=dev, generator=gen).to(tdt)
        x = torch.randn(T, C, device=dev, generator=gen).to(tdt)
        dw = torch.empty(R, C, dtype=torch.float32, device=dev)
        fn = lambda: sp.sp24_gemm_wgrad_dense(x, dy, dw)
    elif k == "transpose":
        wt = torch.empty(C, R, dtype=tdt, device=dev)
        fn = lambda: sp.sp24_transpose(w, wt)
    elif k == "gemm_dense_fwd":
        x = torch.randn(T, C, device=dev, generator=gen).to(tdt)
        y = torch.empty(T, R, dtype=tdt, device=dev)
        aux = torch.empty(T, R, dtype=tdt, device=dev) if args.epi == "gelu" else None
        epi = "gelu" if args.epi == "gelu" else None
        fn = lambda: sp.sp24_gemm_dense(x, w, y, epi, aux)
    elif k == "gemm_dense_dgrad":
        # dX = dY W with W read as stored (--via-transpose: sp24_gemm_dense on W^T)
        dy = torch.randn(T, R, device=dev, generator=gen).to(tdt)
        dx = torch.empty(T, C, dtype=tdt, device=dev)
        epi = args.epi if args.epi in ("dgelu", "mul_aux") else None
        aux = torch.randn(T, C, device=dev, generator=gen).to(tdt) if epi else None
        if args.via_transpose:
            wt = torch.empty(C, R, dtype=tdt, device=dev)
            sp.sp24_transpose(w, wt)
            fn = lambda: sp.sp24_gemm_dense(dy, wt, dx, epi, aux)
        else:
            fn = lambda: sp.sp24_gemm_dgrad_dense(dy, w, dx, epi, aux)
    else:
        dy = torch.randn(T, R, device=dev, generator=gen).to(tdt)
        epi = args.epi if args.epi in ("dgelu", "mul_aux", "dgeglu", "mul_aux_packed") else None
        # dgeglu: W is the down projection [rows = d, cols = ff]; aux and dX are [T, 2 ff]
        width = 2 * C if epi == "dgeglu" else C
        dx = torch.empty(T, width, dtype=tdt, device=dev)
        aux = torch.randn(sp.aux_elements(T, width, epi), device=dev, generator=gen).to(tdt) if epi else None
        fn = lambda: sp.sp24_gemm_dgrad(dy, bufs[2], bufs[3], C, dx, epi, aux)

    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    total = 0.0
    for _ in range(args.iters):
        flush.fill_(1.0)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        fn()
        e.record()
        torch.cuda.synchronize()
        total += s.elapsed_time(e)
    status = sp.sp24_device_status()
    avg_s = total / args.iters * 1e-3
    if k.startswith("gemm"):
        amount, unit = 2.0 * T * R * C / avg_s / 1e12, "TFLOP/s"
    elif k == "mvue":
        amount, unit = T * R * BYTES_PER_ELEMENT[k] / avg_s / 1e9, "GB/s"
    else:
        amount, unit = R * C * BYTES_PER_ELEMENT[k] / avg_s / 1e9, "GB/s"
    print(json.dumps({"kernel": k, "rows": R, "cols": C, "tokens": T if k.startswith("gemm") else None,
                      "dtype": args.dtype, "dist": args.dist, "epi": args.epi, "avg_us": round(avg_s * 1e6, 2),
                      "achieved": round(amount, 1), "unit": unit, "status": sp.sp24_status_string(status)}))
    return 0 if status == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())
