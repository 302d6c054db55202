"""Benchmark of the 2:4 sparse FFN hot path on B200.

One step = the whole path on one GPT-2 FFN (default: the 1.5B shape, d = 1600,
ff = 6400, fp16, 32768 tokens), as simulated training steps: the weights
W_0 .. W_S of both layers follow W_(t+1) = round(W_t + N(0, 1e-4)) (S = 8 for
the 1.5B shape), and step t runs
  mask step on W1 and W2 at W_(t+1) (transposable 2:4 search, flip count against
  the mask of W_t, compression of both orientations), forward GEMMs
  (X -> gelu(X W1m^T) -> H W2m^T, the first also storing gelu' of its
  pre-activation), input-gradient GEMMs (dY -> dH = (dY W2m) * gelu' -> dX),
  masked decay on both weights' gradients (lambda = 6e-5).
Timed steps cycle through t = 0 .. S-1.  The metric is the dense-equivalent
FLOPs of the four GEMMs divided by the step time (TFLOP/s); per-kernel times
give the roofline.  The same JSON line carries the mask-search bandwidth sweep
(fused mask step and search alone on fp16 16384 x 16384 and 16384 x 65536,
Gaussian and 8-level tie-heavy), the GPT-2 355M step, and, on the headline
workload, the training step with the weight gradients (MVUE 2:4 sparsification
of dY^T and dH^T, then dW2 = MVUE(dY^T) H and dW1 = MVUE(dH^T) X in fp32,
decayed in place), the dense fine-tuning step and the gated (GEGLU) FFN step.

Multi-GPU: one process per GPU (torchrun), data-parallel replicas with their
own token batch; masks are computed redundantly and bit-identically, so no
collective runs on the data path (weak scaling).  Timing: W untimed warm-up
steps, then exactly K steps between barrier + synchronize; L2 is flushed
(256 MiB write) before every timed step outside the step's events; the step
time is the sum of CUDA-event step times, max over ranks.

--impl reference times the CPU oracle (the only other implementation this
project has) on a bounded token sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synthetic_inputs as si  # noqa: E402

METRIC = "2:4 FFN GEMM TFLOP/s (% sparse TC peak); mask-search GB/s (% HBM) on 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------ distributed

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def rank_seeds(wl: si.FFNWorkload, rank: int) -> dict:
    """Per-rank seeds: every replica holds the same weights and its own token batch."""
    seeds = dict(wl.seeds)
    seeds["X"] = wl.seeds["X"] + 1000 * rank
    seeds["dY"] = wl.seeds["dY"] + 1000 * rank
    return seeds


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def kernel_source_hash(*names: str) -> str:
    """Short hash of the CUDA sources a profile was taken from (stale profiles report null)."""
    import hashlib
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "structured_sparse_transformer_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(kernel: str, workload: str):
    """DRAM bytes per launch measured by ncu for `kernel` on `workload`
    (profiles/traffic.json), or None if absent or taken from other sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    entry = json.load(open(p)).get(kernel, {}).get(workload)
    if not entry:
        return None
    if entry.get("source_hash") != kernel_source_hash(*entry.get("sources", [])):
        return None
    return entry.get("dram_bytes_per_launch")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons of the GPU the
    process runs on from a background thread: through NVML in-process every
    ~5 ms (read-only queries), else with nvidia-smi every ~200 ms."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    NVML_BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
                 "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int, period_s: float = 0.2):
        import threading
        self.gpu, self.period = gpu_index, period_s
        self.samples = []   # (monotonic time, SM MHz, max SM MHz, active reasons)
        self.marks = []     # (phase name, monotonic time at its start)
        self.error = None
        self.source = None
        self._nvml = self._open_nvml()
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._run, daemon=True)

    def _open_nvml(self):
        """NVML handle of the torch device (by UUID, then PCI bus id), or None."""
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(self.gpu)
            handle = None
            for uid in (f"GPU-{props.uuid}", str(props.uuid)):
                try:
                    handle = pynvml.nvmlDeviceGetHandleByUUID(uid)
                    break
                except Exception:
                    continue
            if handle is None:
                bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
                handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            return pynvml, handle
        except Exception as e:  # no NVML binding or no match: fall back to nvidia-smi
            self.error = f"nvml: {str(e)[:120]}"
            return None

    def _query_nvml(self):
        pynvml, h = self._nvml
        sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
        smax = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        bits = int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))
        return sm, smax, {n for n, b in self.NVML_BITS.items() if bits & b}

    def _query_smi(self):
        r = subprocess.run(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                            "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=10)
        if r.returncode != 0:
            raise RuntimeError(r.stderr.strip() or f"nvidia-smi exit {r.returncode}")
        f = [x.strip() for x in r.stdout.strip().splitlines()[0].split(",")]
        reasons = {n for n, v in zip(self.NAMES, f[5:9]) if v.lower().startswith("active")}
        return float(f[1]), float(f[2]), reasons

    def _run(self):
        query, period = ((self._query_nvml, 0.005) if self._nvml else (self._query_smi, self.period))
        self.source = "nvml" if self._nvml else "nvidia-smi"
        while not self._stop.is_set():
            try:
                self.samples.append((time.monotonic(), *query()))
            except Exception as e:  # a field unsupported: stop sampling, keep what was read
                self.error = str(e)[:200]
                return
            self._stop.wait(period)

    def __enter__(self):
        self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._thread.join(timeout=15)

    def mark(self, phase: str):
        """Start of a named phase of the run (the previous one ends here)."""
        self.marks.append((phase, time.monotonic()))

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.error or "no samples"]}
        sm = [x[1] for x in self.samples]
        reasons = sorted(set().union(*[x[3] for x in self.samples]))
        period = "~5 ms" if self.source == "nvml" else "~200 ms"
        phases = {}
        for i, (name, t0) in enumerate(self.marks):
            t1 = self.marks[i + 1][1] if i + 1 < len(self.marks) else float("inf")
            v = [x[1] for x in self.samples if t0 <= x[0] < t1]
            if v:
                phases[name] = {"sm_mhz_median": statistics.median(v), "sm_mhz_min": min(v), "samples": len(v)}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(x[2] for x in self.samples),
                "sm_min_mhz": min(sm), "samples": len(sm), "reasons": reasons, "source": self.source,
                "window": f"warm-up of the headline step through the mask-search sweep, one query per {period} "
                          "(fewer while the host is busy)",
                "phases": phases}


# ------------------------------------------------------------------ our arm

class FFNStep:
    """Device buffers and the launch sequence of one step (kernel launches only)."""

    GEMMS = ("gemm_fwd1_gelu", "gemm_fwd2", "gemm_dgrad2_dgelu", "gemm_dgrad1")
    KERNELS = ("mask_step",) + GEMMS + ("masked_decay",)
    WGRAD_KERNELS = ("mvue_dy", "mvue_dh", "gemm_wgrad2", "gemm_wgrad1")

    def __init__(self, wl: si.FFNWorkload, rank: int, with_host=True):
        import torch
        import structured_sparse_transformer_b200 as sp
        self.sp, self.torch, self.wl = sp, torch, wl
        tdt = si.DTYPES[wl.dtype]
        T, d, ff = wl.tokens, wl.d, wl.ff
        seeds = rank_seeds(wl, rank)
        wl_r = si.FFNWorkload(wl.name, wl.d, wl.ff, wl.tokens, wl.dtype, wl.steps, wl.lam, seeds)
        W1, W2 = wl_r.weights()
        X, dY = wl_r.activations()
        G1, G2 = wl_r.grads()
        dev = "cuda"
        # The simulated training steps: W_(t+1) = round(W_t + N(0, 1e-4)), t = 0 .. S-1.
        self.S = max(1, wl.steps)
        hostW = wl.weight_sequence(W1, W2)
        self.host = {"W": hostW, "X": X, "dY": dY, "G1": G1, "G2": G2} if with_host else None
        self.W = [[w.to(dev) for w in hostW[li]] for li in range(2)]
        self.X, self.dY = X.to(dev), dY.to(dev)
        self.G = [G1.to(dev), G2.to(dev)]
        shapes = ((ff // 4, d // 4), (d // 4, ff // 4))
        self.idx = [[torch.zeros(*shapes[li], dtype=torch.uint8, device=dev) for _ in range(self.S + 1)]
                    for li in range(2)]
        self.flips = torch.zeros(self.S, 2, dtype=torch.int64, device=dev)
        self.c = [sp.alloc_compressed(ff, d, tdt), sp.alloc_compressed(d, ff, tdt)]
        for li in range(2):   # the mask of W_0, against which step 0 counts its flips
            sp.sp24_mask_search(self.W[li][0], self.idx[li][0])
        self.H = torch.empty(T, ff, dtype=tdt, device=dev)
        # gelu' of the pre-activation, sized for either layout: the 2:4 step keeps it in the
        # layout choose_aux_layout() measured faster, the dense step row-major
        self.Gp = torch.empty(sp.aux_elements(T, ff, "gelu_deriv_packed"), dtype=tdt, device=dev)
        self.aux_pair = ("gelu_deriv_packed", "mul_aux_packed")
        self.dH = torch.empty(T, ff, dtype=tdt, device=dev)
        self.Y = torch.empty(T, d, dtype=tdt, device=dev)
        self.dX = torch.empty(T, d, dtype=tdt, device=dev)
        # MVUE-sparsified dY^T [d x T] and dH^T [ff x T] (compressed along tokens)
        self.yh = [(torch.empty(n, T // 2, dtype=tdt, device=dev),
                    torch.empty(sp.sp24_compressed_size(n, T)[1], dtype=torch.uint8, device=dev)) for n in (d, ff)]
        self.step_no = 0
        self.launches_per_step = 8

    def run(self, events=None, wgrad=False):
        """Enqueue one step; if `events` is a dict, record (start, end) CUDA events per kernel.
        The two layers' mask steps, and their decays, are independent: the second of each
        pair runs on a side stream, concurrently with the first (the step forks before the
        mask steps and joins before the second layer's forward GEMM and after the decays);
        with `events` everything runs on one stream.  With `wgrad` the step also computes
        both weight gradients into the gradient buffers (MVUE + weight-gradient GEMM)
        before they are decayed."""
        sp, torch, wl = self.sp, self.torch, self.wl
        d, ff = wl.d, wl.ff
        t = self.step_no % self.S
        cur, prev = t + 1, t
        main = torch.cuda.current_stream()
        if not hasattr(self, "side"):
            self.side = torch.cuda.Stream()
        # The instrumented pass serialises everything on one stream, so that each
        # kernel's events time that kernel alone.
        side = self.side if events is None else main

        def timed(name, fn, stream):
            with torch.cuda.stream(stream):
                if events is None:
                    fn()
                    return
                s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                s.record(stream)
                fn()
                e.record(stream)
                events.setdefault(name, []).append((s, e))

        def fork():
            ev = torch.cuda.Event()
            ev.record(main)
            side.wait_event(ev)

        def join():
            ev = torch.cuda.Event()
            ev.record(side)
            main.wait_event(ev)

        fork()
        for li, stream in ((0, main), (1, side)):
            c = self.c[li]
            timed("mask_step", lambda li=li, c=c: sp.sp24_mask_step(
                self.W[li][cur], self.idx[li][cur], self.idx[li][prev], self.flips[t, li:li + 1], *c), stream)
        c1, c2 = self.c
        timed("gemm_fwd1_gelu", lambda: sp.sp24_gemm_fwd(self.X, c1[0], c1[1], ff, self.H, self.aux_pair[0],
                                                         self.Gp),
              main)
        join()
        timed("gemm_fwd2", lambda: sp.sp24_gemm_fwd(self.H, c2[0], c2[1], d, self.Y), main)
        timed("gemm_dgrad2_dgelu",
              lambda: sp.sp24_gemm_dgrad(self.dY, c2[2], c2[3], ff, self.dH, self.aux_pair[1], self.Gp), main)
        if wgrad:
            # Weight gradients into the gradient buffers, decayed in the same kernels:
            # dW2 = MVUE(dY^T) H, dW1 = MVUE(dH^T) X, then + lambda W where pruned;
            # fresh draws every step and layer (offset 2 * step + layer).
            seed = wl.seeds["mvue"]
            (y2v, y2m), (y1v, y1m) = self.yh
            timed("mvue_dy", lambda: sp.sp24_mvue_sparsify(self.dY, seed, 2 * self.step_no + 1, y2v, y2m), main)
            timed("gemm_wgrad2", lambda: sp.sp24_gemm_wgrad_decay(self.H, y2v, y2m, d, self.W[1][cur],
                                                                    self.idx[1][cur], wl.lam, self.G[1]), main)
            timed("mvue_dh", lambda: sp.sp24_mvue_sparsify(self.dH, seed, 2 * self.step_no, y1v, y1m), main)
            timed("gemm_wgrad1", lambda: sp.sp24_gemm_wgrad_decay(self.X, y1v, y1m, ff, self.W[0][cur],
                                                                    self.idx[0][cur], wl.lam, self.G[0]), main)
        timed("gemm_dgrad1", lambda: sp.sp24_gemm_dgrad(self.dH, c1[2], c1[3], d, self.dX), main)
        if not wgrad:
            # the gradients come from elsewhere: the masked decay as its own pass
            fork()
            for li, stream in ((0, main), (1, side)):
                timed("masked_decay", lambda li=li: sp.sp24_masked_decay(self.G[li], self.W[li][cur],
                                                                          self.idx[li][cur], wl.lam), stream)
            join()
        self.step_no += 1

    def choose_aux_layout(self, reps: int = 3, force: str = "auto"):
        """Times the derivative-saving pair (forward 1 storing GELU', input gradient 2 multiplying
        by it) with the derivative row-major and packed, on the step's own operands, and keeps
        the faster for the 2:4 step.  The packed layout lets the input gradient take wider
        tiles at some shapes and costs a little at others.  Needs one step run first (the
        compressed weights).  `force` ("packed" or "row-major") skips the timing, for runs under
        a profiler, whose serialised launches make the events meaningless."""
        sp, torch, wl = self.sp, self.torch, self.wl
        if force != "auto":
            self.aux_pair = (("gelu_deriv_packed", "mul_aux_packed") if force == "packed"
                             else ("gelu_deriv", "mul_aux"))
            return {"aux_layout": force}
        c1, c2 = self.c
        best = None
        for pair in (("gelu_deriv", "mul_aux"), ("gelu_deriv_packed", "mul_aux_packed")):
            times = []
            for _ in range(reps):
                s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                s.record()
                sp.sp24_gemm_fwd(self.X, c1[0], c1[1], wl.ff, self.H, pair[0], self.Gp)
                sp.sp24_gemm_dgrad(self.dY, c2[2], c2[3], wl.ff, self.dH, pair[1], self.Gp)
                e.record()
                torch.cuda.synchronize()
                times.append(s.elapsed_time(e))
            t = min(times)
            if best is None or t < best[0]:
                best = (t, pair)
        self.aux_pair = best[1]
        return {"aux_layout": "packed" if "packed" in best[1][0] else "row-major"}

    def run_dense(self, events=None):
        """One step of the dense fine-tuning phase (the last 1/6 of the steps):
        the six FFN products on the dense tensor-core path, every operand read
        as stored (the input gradients load W MN-major, the weight gradients dY
        and dH); no mask, compression or decay."""
        sp, torch = self.sp, self.torch
        cur = self.step_no % self.S + 1

        def timed(name, fn):
            if events is None:
                fn()
                return
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            fn()
            e.record()
            events.setdefault(name, []).append((s, e))

        W1, W2 = self.W[0][cur], self.W[1][cur]
        timed("gemm_fwd1_gelu", lambda: sp.sp24_gemm_dense(self.X, W1, self.H, "gelu_deriv", self.Gp))
        timed("gemm_fwd2", lambda: sp.sp24_gemm_dense(self.H, W2, self.Y))
        timed("gemm_dgrad2_dgelu", lambda: sp.sp24_gemm_dgrad_dense(self.dY, W2, self.dH, "mul_aux", self.Gp))
        timed("gemm_wgrad2", lambda: sp.sp24_gemm_wgrad_dense(self.H, self.dY, self.G[1]))
        timed("gemm_wgrad1", lambda: sp.sp24_gemm_wgrad_dense(self.X, self.dH, self.G[0]))
        timed("gemm_dgrad1", lambda: sp.sp24_gemm_dgrad_dense(self.dH, W1, self.dX))
        self.step_no += 1

    # algorithmic bytes / flops per launch of each kernel
    def work(self):
        wl = self.wl
        n_el = wl.d * wl.ff
        gemm = ("TFLOP/s", 2.0 * wl.tokens * wl.d * wl.ff)
        w = {
            # read W (2 B/el), idx_prev (1/16), write idx (1/16), values of both orientations (2 B/el),
            # metadata of both orientations (2 x 1/8 B/el)
            "mask_step": ("GB/s", n_el * (2 + 1 / 16 + 1 / 16 + 2 + 0.25)),
            # read dY (2 B/el), write the kept values (1 B/el) and their metadata (1/8 B/el)
            "mvue_dy": ("GB/s", wl.tokens * wl.d * (2 + 1 + 1 / 8)),
            "mvue_dh": ("GB/s", wl.tokens * wl.ff * (2 + 1 + 1 / 8)),
            # read g (4), W (2), idx (1/16), write g (4)
            "masked_decay": ("GB/s", n_el * (10 + 1 / 16)),
        }
        for g in self.GEMMS + ("gemm_wgrad2", "gemm_wgrad1"):
            w[g] = gemm
        return w


def kernel_table(events, work, peaks, names):
    """Per-kernel launches, average duration and roofline fraction from the instrumented pass."""
    sparse_peak = 2.0 * peaks["bf16_tflops"]
    out = {}
    for name in names:
        if name not in events:
            continue
        unit, amount = work[name]
        times = [s.elapsed_time(e) * 1e-3 for s, e in events[name]]
        avg = sum(times) / len(times)
        achieved = amount / avg / (1e12 if unit == "TFLOP/s" else 1e9)
        peak = sparse_peak if unit == "TFLOP/s" else peaks["hbm_gbs"]
        out[name] = {"launches": len(times), "avg_us": round(avg * 1e6, 2), "achieved": round(achieved, 1),
                     "unit": unit, "peak": peak, "frac": round(achieved / peak, 4)}
    return out


def timed_steps(step_fn, steps, flush, barrier):
    """Runs `steps` steps back to back, each bracketed by CUDA events after an L2 flush;
    returns the summed step time in ms."""
    import torch
    ev = []
    barrier()
    for _ in range(steps):
        flush.fill_(1.0)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        step_fn()
        e.record()
        ev.append((s, e))
    barrier()
    return sum(s.elapsed_time(e) for s, e in ev)


def run_ours(args, wl, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import structured_sparse_transformer_b200 as sp
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    step = FFNStep(wl, rank)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def status(where):
        st = sp.sp24_device_status()
        if st != 0:
            raise RuntimeError(f"device status {where}: {sp.sp24_status_string(st)}")

    clk = ClockSampler(torch.cuda.current_device()).__enter__()
    try:
        clk.mark("headline warm-up and timed steps")
        for _ in range(args.warmup):
            step.run()
        aux_choice = step.choose_aux_layout(force=args.aux_layout)
        torch.cuda.synchronize()
        status("after warm-up")
        # Timed region: the step's launches back to back (each kernel may start
        # while its predecessor drains: programmatic dependent launch).
        step_ms = timed_steps(step.run, args.steps, flush, barrier)
        status("after timing")
        flips = step.flips.cpu().tolist()
        # Per-kernel durations: a second pass of the same steps with events around
        # every launch (an event between two launches serialises them).
        events = {}
        barrier()
        clk.mark("headline event pass")
        for _ in range(args.steps):
            flush.fill_(1.0)
            step.run(events)
        barrier()
        peaks, peak_kind = load_peaks()
        kernels = kernel_table(events, step.work(), peaks, FFNStep.KERNELS)
        clk.mark("weight-gradient step")
        wgrad = run_wgrad_phase(args, step, wl, world, dev, flush, barrier, peaks)
        clk.mark("dense step")
        dense = run_dense_phase(args, step, wl, world, dev, flush, barrier, peaks)
        clk.mark("gated step")
        geglu = run_geglu_phase(args, step, wl, world, dev, flush, barrier)
        clk.mark("end to end")
        e2e = run_e2e(args, step, wl, world, dev, barrier)
        del step
        torch.cuda.empty_cache()
        clk.mark("gpt2-355m")
        secondary = run_secondary(args, si.GPT2_355M, rank, world, dev, flush, barrier, peaks)
        clk.mark("mask-search sweep")
        sweep = None if args.no_sweep else run_sweep(args, dev, flush, barrier, peaks)
        clk.mark("end")
    finally:
        clk.__exit__()
    total_ms = max_over_ranks(step_ms, world, dev)
    ms_per_step = total_ms / args.steps
    value = wl.gemm_flops() * world * args.steps / (total_ms * 1e-3) / 1e12

    sparse_peak = 2.0 * peaks["bf16_tflops"]
    g = [kernels[k] for k in FFNStep.GEMMS]
    g_avg = sum(v["avg_us"] * v["launches"] for v in g) / sum(v["launches"] for v in g) * 1e-6
    g_ach = 2.0 * wl.tokens * wl.d * wl.ff / g_avg / 1e12
    roofline = {"bound": "tensor", "achieved": round(g_ach, 1), "peak": sparse_peak, "unit": "TFLOP/s",
                "frac": round(g_ach / sparse_peak, 4),
                "traffic": args.gemm_traffic or load_traffic("gemm", wl.name),
                "kernel": "sp24_gemm_pair_kernel (the four forward and input-gradient launches)",
                "peak_source": f"2 x {peak_kind} dense bf16 burst ({peaks['bf16_tflops']} TFLOP/s), "
                               "the nominal 2:4 sparse ratio"}
    # 2:4 over dense, per product, from the two instrumented passes on the same workload
    ratio = {k: round(dense["kernels"][k]["avg_us"] / kernels[k]["avg_us"], 3) for k in FFNStep.GEMMS}
    for k in ("gemm_wgrad2", "gemm_wgrad1"):
        ratio[k] = round(dense["kernels"][k]["avg_us"] / wgrad["kernels"][k]["avg_us"], 3)
    mask = kernels["mask_step"]
    gate = sweep["16384x65536"]["normal"]["mask_step"] if sweep else None
    clocks = clk.summary()
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic (seeded N(0,0.02) weights, N(0,1) tokens)",
        "config": {"workload": wl.name, "d_model": wl.d, "d_ff": wl.ff, "tokens_per_gpu": wl.tokens,
                   "global_tokens": wl.tokens * world, "simulated_steps": max(1, wl.steps),
                   "perturbation": "W_(t+1) = round(W_t + N(0, 1e-4)) per weight; timed steps cycle t = 0..S-1",
                   "parallelism": f"dp{world} replicas, no collective",
                   "l2": "flushed before every timed step (256 MiB write, outside the step events)",
                   "gelu_derivative": aux_choice["aux_layout"] + (" (the faster of the two layouts, timed on "
                                                                  "the step's own operands after warm-up)"
                                                                  if args.aux_layout == "auto" else " (as asked)"),
                   "kernel_times": "second pass of the same steps with events around each launch, all on "
                                   "one stream (the timed steps run the second layer's mask step and "
                                   "decay concurrently on a side stream)"},
        "roofline": roofline,
        "mask_search_roofline": (
            {"bound": "hbm", "achieved": gate["achieved"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
             "frac": gate["frac"], "traffic": args.mask_traffic or load_traffic("mask_step", "sweep-16384x65536"),
             "kernel": "mask_tile_kernel (search + flip + both compressions), fp16 16384 x 65536 N(0, 0.02) "
                       "(2 GiB of weights, beyond L2)"} if gate else None),
        "kernels": kernels,
        "sparse_over_dense": ratio,
        "flip_counts_per_step": flips,
        "flip_rate_per_step": [[round(c / (wl.d * wl.ff), 6) for c in row] for row in flips],
        "mask_search_sweep": sweep,
        "ffn_step_with_weight_gradients": wgrad,
        "dense_finetune_step": dense,
        "geglu_ffn_step": geglu,
        "gpt2_355m": secondary,
        "e2e": e2e,
        "gpu_launches": 8 * args.steps,
        "clocks": clocks,
        "peaks": peak_kind,
    }
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_tokens)
    return line


def run_secondary(args, wl, rank, world, dev, flush, barrier, peaks):
    """The headline step on a second workload (timed the same way), with its kernels."""
    import torch
    import structured_sparse_transformer_b200 as sp
    step = FFNStep(wl, rank, with_host=False)
    for _ in range(args.warmup):
        step.run()
    aux_choice = step.choose_aux_layout(force=args.aux_layout)
    ms = max_over_ranks(timed_steps(step.run, args.steps, flush, barrier), world, dev) / args.steps
    events = {}
    for _ in range(args.steps):
        flush.fill_(1.0)
        step.run(events)
    barrier()
    st = sp.sp24_device_status()
    if st != 0:
        raise RuntimeError(f"device status after the {wl.name} step: {sp.sp24_status_string(st)}")
    kernels = kernel_table(events, step.work(), peaks, FFNStep.KERNELS)
    del step
    torch.cuda.empty_cache()
    return {"workload": wl.name, "d_model": wl.d, "d_ff": wl.ff, "tokens_per_gpu": wl.tokens, **aux_choice,
            "ms_per_step": round(ms, 4), "value": round(wl.gemm_flops() * world / (ms * 1e-3) / 1e12, 2),
            "unit": "TFLOP/s", "kernels": kernels}


def run_sweep(args, dev, flush, barrier, peaks):
    """Mask-search bandwidth sweep at the sizes beyond L2: the fused mask step (search + flip
    count against the mask before an N(0, 1e-4) update + both compressions) and the search
    alone, on fp16 Gaussian N(0, 0.02) and 8-level tie-heavy weights.  Inputs are drawn on
    the device from seeded generators; each launch follows an L2 flush and is timed alone."""
    import torch
    import structured_sparse_transformer_b200 as sp
    out = {}
    per_el = {"mask_step": 2 + 1 / 16 + 1 / 16 + 2 + 0.25, "search": 2 + 1 / 16}
    for R, C in args.sweep_shapes:
        key = f"{R}x{C}"
        out[key] = {}
        idx = torch.empty(R // 4, C // 4, dtype=torch.uint8, device=dev)
        prev = torch.empty_like(idx)
        count = torch.zeros(1, dtype=torch.int64, device=dev)
        bufs = sp.alloc_compressed(R, C, torch.float16, device=dev)
        for dist_name in ("normal", "tie"):
            g = torch.Generator(device=dev)
            g.manual_seed(400 + (dist_name == "tie"))
            w = torch.empty(R, C, dtype=torch.float16, device=dev)
            for r0 in range(0, R, 1024):   # fp32 draws in row slabs (bounded temporaries)
                x = torch.randn(min(1024, R - r0), C, device=dev, generator=g) * 0.02
                if dist_name == "tie":
                    x = torch.clamp(torch.round(x / 2.0**-6), -4, 3) * 2.0**-6
                w[r0:r0 + x.shape[0]] = x.to(torch.float16)
            sp.sp24_mask_search(w, prev)
            for r0 in range(0, R, 1024):   # one simulated update, so that the flip count is live
                sl = w[r0:r0 + 1024]
                sl.copy_((sl.float() + torch.randn(sl.shape, device=dev, generator=g) * 1e-4).to(torch.float16))
            fns = {"mask_step": lambda: sp.sp24_mask_step(w, idx, prev, count, *bufs),
                   "search": lambda: sp.sp24_mask_search(w, idx)}
            res = {}
            for name, fn in fns.items():
                for _ in range(2):
                    fn()
                barrier()
                ev = []
                for _ in range(args.sweep_iters):
                    flush.fill_(1.0)
                    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    s.record()
                    fn()
                    e.record()
                    ev.append((s, e))
                barrier()
                avg = sum(s.elapsed_time(e) for s, e in ev) / len(ev) * 1e-3
                gbs = R * C * per_el[name] / avg / 1e9
                res[name] = {"avg_us": round(avg * 1e6, 2), "achieved": round(gbs, 1), "unit": "GB/s",
                             "peak": peaks["hbm_gbs"], "frac": round(gbs / peaks["hbm_gbs"], 4),
                             "bytes_per_element": round(per_el[name], 4)}
            res["flips"] = int(count.item())
            st = sp.sp24_device_status()
            if st != 0:
                raise RuntimeError(f"device status after the sweep at {key}: {sp.sp24_status_string(st)}")
            out[key][dist_name] = res
            del w
        del idx, prev, bufs
        torch.cuda.empty_cache()
    return out


def run_wgrad_phase(args, step, wl, world, dev, flush, barrier, peaks):
    """The 2:4 training step with both weight gradients (MVUE + weight-gradient GEMM, then the
    decay of the computed gradients), timed like the headline step, and its MVUE and
    weight-gradient kernels from an instrumented pass."""
    import structured_sparse_transformer_b200 as sp
    for _ in range(args.warmup):
        step.run(wgrad=True)
    ms = max_over_ranks(timed_steps(lambda: step.run(wgrad=True), args.steps, flush, barrier), world, dev)
    ms /= args.steps
    events = {}
    for _ in range(args.steps):
        flush.fill_(1.0)
        step.run(events, wgrad=True)
    barrier()
    st = sp.sp24_device_status()
    if st != 0:
        raise RuntimeError(f"device status after the weight-gradient step: {sp.sp24_status_string(st)}")
    kernels = kernel_table(events, step.work(), peaks, FFNStep.WGRAD_KERNELS)
    flops = 6 * 2.0 * wl.tokens * wl.d * wl.ff
    return {"ms_per_step": round(ms, 4), "value": round(flops * world / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "launches_per_step": 10, "kernels": kernels,
            "note": "the headline step with both weight gradients: MVUE 2:4 sparsification of dY^T and dH^T "
                    "(Philox4x64-10 draws), dW2 = MVUE(dY^T) H and dW1 = MVUE(dH^T) X on the sparse tensor "
                    "cores in fp32 with the masked decay applied in the same kernels' epilogues (no separate "
                    "decay pass); FLOPs 6 x 2 T d ff"}


def run_dense_phase(args, step, wl, world, dev, flush, barrier, peaks):
    """The dense fine-tuning step, timed like the 2:4 step (back to back, L2
    flushed outside the step events), and its kernels from an instrumented pass."""
    import structured_sparse_transformer_b200 as sp
    for _ in range(args.warmup):
        step.run_dense()
    ms = max_over_ranks(timed_steps(step.run_dense, args.steps, flush, barrier), world, dev) / args.steps
    events = {}
    for _ in range(args.steps):
        flush.fill_(1.0)
        step.run_dense(events)
    barrier()
    st = sp.sp24_device_status()
    if st != 0:
        raise RuntimeError(f"device status after the dense phase: {sp.sp24_status_string(st)}")
    work = {k: ("TFLOP/s", 2.0 * wl.tokens * wl.d * wl.ff) for k in FFNStep.GEMMS + ("gemm_wgrad2", "gemm_wgrad1")}
    dense_peaks = dict(peaks)
    dense_peaks["bf16_tflops"] = peaks["bf16_tflops"] / 2.0   # kernel_table doubles it for the 2:4 peak
    kernels = kernel_table(events, work, dense_peaks, list(work))
    return {"ms_per_step": round(ms, 4),
            "value": round(6 * 2.0 * wl.tokens * wl.d * wl.ff * world / (ms * 1e-3) / 1e12, 2),
            "unit": "TFLOP/s", "kernels": kernels,
            "note": "dense fine-tuning phase (last 1/6 of the steps): the six FFN products (forward, input "
                    "gradient reading W as stored, weight gradient reading dY and dH as stored) on the dense "
                    "tcgen05 path, same workload; FLOPs 6 x 2 T d ff; GEMM peak = the dense bf16 burst"}


class GegluStep:
    """The gated FFN of the same width on the 2:4 path: stacked gate/up weight
    [2 ff, d] (16-row groups alternate), down projection [d, ff]; per step the
    two mask steps, the GEGLU forward, the down projection, its input gradient
    with the gated-gradient epilogue, the stacked input gradient, the weight
    gradients of both weights on the MVUE sparsification of dY and of the stacked
    gate/up gradient (which is already in the stacked weight's row order), and
    the decays of those gradients."""

    def __init__(self, step):
        import torch
        import structured_sparse_transformer_b200 as sp
        self.sp, self.torch, self.step = sp, torch, step
        wl = step.wl
        tdt = si.DTYPES[wl.dtype]
        T, d, ff = wl.tokens, wl.d, wl.ff
        g = torch.Generator().manual_seed(300)
        mk = lambda shape, std, dt: (torch.randn(*shape, generator=g) * std).to(dt).cuda()
        self.Wgu, self.Wd = mk((2 * ff, d), 0.02, tdt), mk((d, ff), 0.02, tdt)
        self.Ggu, self.Gd = mk((2 * ff, d), 1e-2, torch.float32), mk((d, ff), 1e-2, torch.float32)
        self.idx = [torch.zeros(2 * ff // 4, d // 4, dtype=torch.uint8, device="cuda"),
                    torch.zeros(d // 4, ff // 4, dtype=torch.uint8, device="cuda")]
        self.c = [sp.alloc_compressed(2 * ff, d, tdt), sp.alloc_compressed(d, ff, tdt)]
        self.H = torch.empty(T, ff, dtype=tdt, device="cuda")
        self.GU = torch.empty(T, 2 * ff, dtype=tdt, device="cuda")
        self.dGU = torch.empty(T, 2 * ff, dtype=tdt, device="cuda")
        self.Y = torch.empty(T, d, dtype=tdt, device="cuda")
        self.dX = torch.empty(T, d, dtype=tdt, device="cuda")
        # MVUE-sparsified dY^T [d x T] and dGU^T [2 ff x T]
        self.yh = [(torch.empty(n, T // 2, dtype=tdt, device="cuda"),
                    torch.empty(sp.sp24_compressed_size(n, T)[1], dtype=torch.uint8, device="cuda")) for n in (d, 2 * ff)]
        self.step_no = 0
        self.flops = 9 * 2.0 * T * d * ff

    def run(self):
        sp, st, wl = self.sp, self.step, self.step.wl
        d, ff = wl.d, wl.ff
        for w, i, c in ((self.Wgu, self.idx[0], self.c[0]), (self.Wd, self.idx[1], self.c[1])):
            sp.sp24_mask_step(w, i, None, None, *c)
        (vr_gu, mr_gu, vc_gu, mc_gu), (vr_d, mr_d, vc_d, mc_d) = self.c
        sp.sp24_gemm_fwd(st.X, vr_gu, mr_gu, 2 * ff, self.H, "geglu", self.GU)
        sp.sp24_gemm_fwd(self.H, vr_d, mr_d, d, self.Y)
        sp.sp24_gemm_dgrad(st.dY, vc_d, mc_d, ff, self.dGU, "dgeglu", self.GU)
        seed = wl.seeds["mvue"] + 1
        (ydv, ydm), (ygv, ygm) = self.yh
        sp.sp24_mvue_sparsify(st.dY, seed, 2 * self.step_no + 1, ydv, ydm)
        sp.sp24_gemm_wgrad(self.H, ydv, ydm, d, self.Gd)
        sp.sp24_mvue_sparsify(self.dGU, seed, 2 * self.step_no, ygv, ygm)
        sp.sp24_gemm_wgrad(st.X, ygv, ygm, 2 * ff, self.Ggu)
        sp.sp24_gemm_dgrad(self.dGU, vc_gu, mc_gu, d, self.dX)
        sp.sp24_masked_decay(self.Ggu, self.Wgu, self.idx[0], wl.lam)
        sp.sp24_masked_decay(self.Gd, self.Wd, self.idx[1], wl.lam)
        self.step_no += 1


def run_geglu_phase(args, step, wl, world, dev, flush, barrier):
    """The gated FFN step, timed like the 2:4 step."""
    import torch
    import structured_sparse_transformer_b200 as sp
    g = GegluStep(step)
    for _ in range(args.warmup):
        g.run()
    ev = []
    barrier()
    for _ in range(args.steps):
        flush.fill_(1.0)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        g.run()
        e.record()
        ev.append((s, e))
    barrier()
    st = sp.sp24_device_status()
    if st != 0:
        raise RuntimeError(f"device status after the gated step: {sp.sp24_status_string(st)}")
    ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in ev), world, dev) / args.steps
    return {"ms_per_step": round(ms, 4), "value": round(g.flops * world / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "note": "gated FFN (GEGLU) of the same d and ff on the 2:4 path: stacked gate/up weight [2 ff, d], "
                    "down projection [d, ff]; mask steps, the forward and input-gradient GEMMs with the gated "
                    "epilogues, both weight gradients on the MVUE sparsification of dY and of the stacked "
                    "gate/up gradient, both decays; FLOPs 9 x 2 T d ff dense-equivalent"}


def run_e2e(args, step, wl, world, dev, barrier):
    """Same metric through the C ABI with host buffers: H2D of the step's inputs (both weights,
    X, dY, both gradients) from pinned memory and D2H of its results (Y, dX, both decayed
    gradients, the flip counts) inside the timed region.  Copies run on their own streams
    and overlap the neighbouring steps' kernels: step k's inputs land in slot k % 2 while
    step k-1 computes, and its results leave while step k+1 computes."""
    import torch
    h = {k: step.host[k].pin_memory() for k in ("X", "dY", "G1", "G2")}
    # The weights a host sends change every step: step t sends W_(t+1) of both layers
    # (the simulated updates), so the masks flip as in training.
    hw = [[w.pin_memory() for w in step.host["W"][li]] for li in range(2)]
    out_y = torch.empty(step.Y.shape, dtype=step.Y.dtype).pin_memory()
    out_dx = torch.empty(step.dX.shape, dtype=step.dX.dtype).pin_memory()
    out_g = [torch.empty(g.shape, dtype=g.dtype).pin_memory() for g in step.G]
    out_f = torch.empty(step.flips.shape, dtype=torch.int64).pin_memory()
    slots = [{"X": step.X, "dY": step.dY, "G": step.G, "Y": step.Y, "dX": step.dX, "flips": step.flips}]
    slots.append({k: ([t.clone() for t in v] if isinstance(v, list) else v.clone()) for k, v in slots[0].items()})
    cs = torch.cuda.current_stream()
    hs, ds = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    d2h_done = [None, None]

    def one():
        k = step.step_no
        sl, b = slots[k % 2], k % 2
        with torch.cuda.stream(hs):
            if d2h_done[b] is not None:
                hs.wait_event(d2h_done[b])     # slot b's previous results have left
            cur = k % step.S + 1
            step.W[0][cur].copy_(hw[0][cur], non_blocking=True)
            step.W[1][cur].copy_(hw[1][cur], non_blocking=True)
            sl["X"].copy_(h["X"], non_blocking=True)
            sl["dY"].copy_(h["dY"], non_blocking=True)
            sl["G"][0].copy_(h["G1"], non_blocking=True)
            sl["G"][1].copy_(h["G2"], non_blocking=True)
            landed = ev()
            landed.record(hs)
        cs.wait_event(landed)
        step.X, step.dY, step.G, step.Y, step.dX, step.flips = (sl["X"], sl["dY"], sl["G"], sl["Y"], sl["dX"],
                                                                sl["flips"])
        step.run()
        done = ev()
        done.record(cs)
        with torch.cuda.stream(ds):
            ds.wait_event(done)
            out_y.copy_(sl["Y"], non_blocking=True)
            out_dx.copy_(sl["dX"], non_blocking=True)
            out_g[0].copy_(sl["G"][0], non_blocking=True)
            out_g[1].copy_(sl["G"][1], non_blocking=True)
            out_f.copy_(sl["flips"], non_blocking=True)
            d2h_done[b] = ev()
            d2h_done[b].record(ds)

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    barrier()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(cs)
    hs.wait_event(s)
    ds.wait_event(s)
    for _ in range(args.steps):
        one()
    for b in range(2):
        cs.wait_event(d2h_done[b])
    e.record(cs)
    barrier()
    ms = max_over_ranks(s.elapsed_time(e), world, dev)
    h2d = sum(v.numel() * v.element_size() for v in (hw[0][1], hw[1][1], h["X"], h["dY"], h["G1"], h["G2"]))
    d2h = sum(t.numel() * t.element_size() for t in (out_y, out_dx, *out_g, out_f))
    return {"value": round(wl.gemm_flops() * world * args.steps / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms / args.steps, 4),
            "copies": "host-to-device and device-to-host copies on their own streams, double-buffered, "
                      "overlapping the neighbouring steps' kernels"}


# ---------------------------------------------------------- oracle (CPU) arm

def oracle_host(wl):
    """Host inputs of the oracle arm: the weight sequence, activations, gradients, and the
    masks of W_0 (step 0 counts its flips against them)."""
    import oracle
    W1, W2 = wl.weights()
    X, dY = wl.activations()
    G1, G2 = wl.grads()
    seq = wl.weight_sequence(W1, W2)
    masks = [[oracle.mask_search(si.bits16(seq[li][0]), wl.dtype)] + [None] * max(1, wl.steps) for li in range(2)]
    return {"W": seq, "X": X, "dY": dY, "G1": G1, "G2": G2, "masks": masks}


def oracle_step(wl, host, rows, t):
    """Simulated step t of the CPU oracle on a token sample: both mask searches on W_(t+1),
    both compressions, the flip counts against the masks of W_t, the four GEMMs on `rows`
    token rows with GELU between, masked decay on both gradients.  Returns the GEMM FLOPs
    it processed."""
    import oracle
    dt = wl.dtype
    cur = t % max(1, wl.steps) + 1
    b = [si.bits16(host["W"][li][cur]) for li in range(2)]
    idx = [oracle.mask_search(b[li], dt) for li in range(2)]
    for li in range(2):
        oracle.compress_both(b[li], idx[li])
        prev = host["masks"][li][cur - 1]
        if prev is None:   # an earlier step's mask the sample has not computed yet
            prev = host["masks"][li][cur - 1] = oracle.mask_search(si.bits16(host["W"][li][cur - 1]), dt)
        oracle.flip_count(prev, idx[li])
        host["masks"][li][cur] = idx[li]
    k1, k2 = oracle.dense_mask(idx[0]), oracle.dense_mask(idx[1])
    w1, w2 = oracle.to_f64(b[0], dt), oracle.to_f64(b[1], dt)
    x = oracle.to_f64(si.bits16(host["X"])[:rows], dt)
    dy = oracle.to_f64(si.bits16(host["dY"])[:rows], dt)
    pre = oracle.sparse_fwd(x, w1, k1)
    h = oracle.gelu(pre)
    oracle.sparse_fwd(h, w2, k2)
    dh = oracle.sparse_dgrad(dy, w2, k2) * oracle.gelu_grad(pre)
    oracle.sparse_dgrad(dh, w1, k1)
    oracle.masked_decay(host["G1"].numpy(), b[0], dt, idx[0], wl.lam)
    oracle.masked_decay(host["G2"].numpy(), b[1], dt, idx[1], wl.lam)
    return 4 * 2.0 * rows * wl.d * wl.ff


def cpu_baseline(wl, rows):
    import oracle
    oracle.build()
    host = oracle_host(wl)
    t0 = time.perf_counter()
    flops = oracle_step(wl, host, rows, 0)
    dt = time.perf_counter() - t0
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle", "seconds": round(dt, 2),
            "sample": f"one simulated step of {wl.name} on the oracle with the four GEMMs on the first {rows} "
                      f"of {wl.tokens} token rows (both mask searches, compressions, flip counts and decays "
                      f"in full)"}


def run_reference(args, wl):
    import oracle
    oracle.build()
    host = oracle_host(wl)
    rows = args.cpu_tokens
    for k in range(args.warmup):
        oracle_step(wl, host, rows, k)
    t0 = time.perf_counter()
    flops = 0.0
    for k in range(args.steps):
        flops += oracle_step(wl, host, rows, args.warmup + k)
    sec = time.perf_counter() - t0
    value = flops / sec / 1e12
    sample = (f"each step: one simulated step of {wl.name} on the oracle with the four GEMMs on the first "
              f"{rows} of {wl.tokens} token rows (mask searches, compressions, flips, decays in full)")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": wl.name, "d_model": wl.d, "d_ff": wl.ff,
                                            "tokens_per_gpu": wl.tokens, "parallelism": "host cores"},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=si.GPT2_1P5B.name, choices=sorted(si.FFN_WORKLOADS))
    ap.add_argument("--no-sweep", action="store_true", help="skip the mask-search bandwidth sweep")
    ap.add_argument("--sweep-iters", type=int, default=5)
    ap.add_argument("--cpu-tokens", type=int, default=256, help="token rows of the oracle's GEMM sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--aux-layout", choices=["auto", "packed", "row-major"], default="auto",
                    help="layout of the stored GELU' in the 2:4 step (auto: the faster, timed after warm-up)")
    ap.add_argument("--gemm-traffic", type=float, default=None, help="ncu DRAM bytes per GEMM launch")
    ap.add_argument("--mask-traffic", type=float, default=None, help="ncu DRAM bytes per mask-step launch")
    args = ap.parse_args(argv)
    args.sweep_shapes = [(16384, 16384), (16384, 65536)]
    wl = si.FFN_WORKLOADS[args.workload]
    rank, world, local_rank = dist_env()

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, wl)), flush=True)
        return 0

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, wl, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
