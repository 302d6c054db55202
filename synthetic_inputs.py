"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check.

This module only draws random numbers and names workload shapes.  It holds none
of the method's arithmetic (no mask search, no pruning, no GEMM, no decay), so
the CUDA path and the CPU oracle can both consume its tensors without sharing
any computation.

Every tensor is produced on the host with a ``torch.Generator`` seeded per
tensor, as fp32 ``randn`` scaled by the stated standard deviation and then cast
round-to-nearest-even to the storage dtype.  ``N(0, s)`` means standard
deviation ``s`` (GPT-2's weight init is N(0, 0.02)).

Workloads stand in for the GPT-2 pre-training runs of "Accelerating Transformer
Pre-training with 2:4 Sparsity" (reproducibility table, Open Datasets and
Hardware Specification rows): only the FFN shapes are used; no dataset or
trained weight is involved.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal(shape, std: float, seed: int, dtype: str = "f16") -> torch.Tensor:
    """fp32 N(0, std) drawn with ``seed`` and cast RNE to ``dtype`` (CPU tensor)."""
    x = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32) * float(std)
    return x.to(DTYPES[dtype]).contiguous()


def tie_heavy(shape, seed: int, dtype: str = "f16") -> torch.Tensor:
    """8-level weights ``clamp(round(w / 2^-6), -4, 3) * 2^-6`` with w ~ N(0, 0.02).

    Every level is exact in fp16 and bf16, so most 4x4 blocks hold many equal
    magnitudes and the pattern argmax is decided by the tie-break alone.
    """
    w = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32) * 0.02
    q = torch.clamp(torch.round(w / 2.0**-6), -4, 3) * 2.0**-6
    return q.to(DTYPES[dtype]).contiguous()


def perturb(w: torch.Tensor, seed: int, std: float = 1e-4) -> torch.Tensor:
    """``round_dtype(float(w) + eps)`` with eps ~ N(0, std): one simulated update step."""
    eps = torch.randn(*w.shape, generator=_gen(seed), dtype=torch.float32) * float(std)
    return (w.float() + eps).to(w.dtype).contiguous()


def bits16(t: torch.Tensor):
    """Raw 16-bit storage of an fp16/bf16 CPU tensor as a numpy uint16 array."""
    assert t.dtype in (torch.float16, torch.bfloat16)
    return t.contiguous().view(torch.int16).numpy().view("uint16")


@dataclass
class FFNWorkload:
    """A GPT-2-shaped FFN: W1 [ff x d], W2 [d x ff], T tokens."""

    name: str
    d: int
    ff: int
    tokens: int
    dtype: str
    steps: int = 1
    lam: float = 6e-5
    seeds: dict = field(default_factory=lambda: {
        "W1": 0, "W2": 1, "X": 2, "dY": 3, "G1": 4, "G2": 5, "H": 6, "dH": 7, "perturb": 100,
        "mvue": 200})

    def weights(self):
        return (normal((self.ff, self.d), 0.02, self.seeds["W1"], self.dtype),
                normal((self.d, self.ff), 0.02, self.seeds["W2"], self.dtype))

    def activations(self):
        return (normal((self.tokens, self.d), 1.0, self.seeds["X"], self.dtype),
                normal((self.tokens, self.d), 1.0, self.seeds["dY"], self.dtype))

    def hidden(self):
        """Stand-ins for the hidden activation H and its gradient dH [T x ff], N(0, 1): the
        operands of the weight-gradient products when they are tested on their own."""
        return (normal((self.tokens, self.ff), 1.0, self.seeds["H"], self.dtype),
                normal((self.tokens, self.ff), 1.0, self.seeds["dH"], self.dtype))

    def grads(self):
        return (normal((self.ff, self.d), 1e-2, self.seeds["G1"], "f32"),
                normal((self.d, self.ff), 1e-2, self.seeds["G2"], "f32"))

    def perturb_seed(self, step: int, which: int) -> int:
        """Seed of the N(0, 1e-4) update of weight ``which`` (0: W1, 1: W2) at ``step``."""
        return self.seeds["perturb"] + 2 * step + which

    def weight_sequence(self, W1, W2):
        """[[W1_0 .. W1_S], [W2_0 .. W2_S]] with W_(t+1) = perturb(W_t): the weights of the
        simulated training steps (S = max(1, steps)), seeds ``perturb_seed(t, layer)``."""
        seq = [[W1], [W2]]
        for t in range(max(1, self.steps)):
            for li in range(2):
                seq[li].append(perturb(seq[li][-1], self.perturb_seed(t, li)))
        return seq

    def gemm_flops(self) -> int:
        """Dense-equivalent FLOPs of the four FFN GEMMs (fwd and dX for both layers)."""
        return 4 * 2 * self.tokens * self.d * self.ff


# The workloads: PR1 (one weight, fwd only) and three GPT-2 FFN shapes.
PR1 = dict(name="pr1-3072x768-f16", R=3072, C=768, tokens=1024, dtype="f16", w_seed=0, x_seed=1)
GPT2_355M = FFNWorkload("gpt2-355m-ffn-f16", d=1024, ff=4096, tokens=8192, dtype="f16")
GPT2_774M = FFNWorkload("gpt2-774m-ffn-bf16", d=1280, ff=5120, tokens=16384, dtype="bf16")
GPT2_1P5B = FFNWorkload("gpt2-1.5b-ffn-f16", d=1600, ff=6400, tokens=32768, dtype="f16", steps=8)
FFN_WORKLOADS = {w.name: w for w in (GPT2_355M, GPT2_774M, GPT2_1P5B)}

# Mask-search bandwidth sweep: x4 elements per step, alternating dimensions.
SWEEP_SHAPES = [(1024, 1024), (1024, 4096), (4096, 4096), (4096, 16384),
                (16384, 16384), (16384, 65536)]
