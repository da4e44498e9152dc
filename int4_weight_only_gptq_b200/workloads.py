"""Seeded synthetic inputs for the symmetric INT4 GPTQ W4A16 linear layer.

This module only draws random numbers and shapes them into arrays. It holds
none of the layer's arithmetic (no unpacking, no zero point, no scaling, no
rounding of products), so the CPU oracle and the CUDA path can both take their
inputs from here without sharing any step of the computation.

Layouts (GPTQ-Pro README, "Runtime contract"; GPTQModel wiki "Installation and
Quickstart", "Defaults and compatibility decisions" table, pack_dtype int32):
  x       float16 [M, K]          activations, row-major
  qweight int32   [K // 8, N]     eight 4-bit codes per int32 along K
  scales  float16 [n_groups, N]   one scale per (group, output column)

Codes are uniform in {0..15} and independent, so an int32 word holding eight
of them is uniform over all 2**32 bit patterns; the generator draws the words
directly.  Which nibble holds which k is therefore a property of the reader
(oracle and kernels), not of this generator.

Generator: numpy PCG64 with the given seed (0 by default); sub-streams are
drawn in the fixed order x, qweight words, scales, outlier channel indices.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

GROUP_SIZES = (-1, 16, 32, 64, 128, 256, 512, 1024)


def num_groups(K: int, group: int) -> int:
    """Number of scale rows: one when group == -1, else ceil(K / group)."""
    if group == -1 or group >= K:
        return 1
    return -(-K // group)


@dataclasses.dataclass
class Problem:
    name: str
    M: int
    K: int
    N: int
    group: int
    x: np.ndarray        # float16 [M, K]
    qweight: np.ndarray  # int32 [K//8, N]
    scales: np.ndarray   # float16 [n_groups, N]

    @property
    def algorithmic_bytes(self) -> int:
        """Bytes the layer must move once: packed weights, scales, X and Y."""
        return (self.K * self.N // 2 + self.scales.size * 2
                + self.M * self.K * 2 + self.M * self.N * 2)

    @property
    def flops(self) -> int:
        return 2 * self.M * self.K * self.N


def _scales_uniform(rng, shape, lo, hi):
    return rng.uniform(lo, hi, size=shape).astype(np.float16)


def _scales_log_uniform(rng, shape, lo, hi):
    return np.exp(rng.uniform(math.log(lo), math.log(hi), size=shape)).astype(np.float16)


def make_problem(M: int, K: int, N: int, group: int, *, seed: int = 0,
                 scale_dist: str = "uniform", scale_range=(1e-3, 2e-2),
                 outlier_frac: float = 0.0, outlier_gain: float = 20.0,
                 name: str = "") -> Problem:
    """Draw one seeded problem.

    x ~ N(0, 1) in float64, then rounded to float16.  With outlier_frac > 0, a
    set of floor(outlier_frac * K) input channels (the same channels in every
    row) is multiplied by outlier_gain in float64 before the float16 rounding.
    """
    if K % 8:
        raise ValueError("K must be a multiple of 8 to pack eight codes per int32")
    rng = np.random.Generator(np.random.PCG64(seed))
    x64 = rng.standard_normal(size=(M, K))
    words = rng.integers(0, 2 ** 32, size=(K // 8, N), dtype=np.uint64).astype(np.uint32)
    ng = num_groups(K, group)
    if scale_dist == "uniform":
        scales = _scales_uniform(rng, (ng, N), *scale_range)
    elif scale_dist == "log_uniform":
        scales = _scales_log_uniform(rng, (ng, N), *scale_range)
    else:
        raise ValueError(scale_dist)
    n_out = int(math.floor(outlier_frac * K))
    if n_out:
        cols = rng.choice(K, size=n_out, replace=False)
        x64[:, cols] *= outlier_gain
    return Problem(name=name or f"M{M}_K{K}_N{N}_g{group}", M=M, K=K, N=N, group=group,
                   x=x64.astype(np.float16), qweight=words.view(np.int32),
                   scales=scales)


@dataclasses.dataclass
class Adapter:
    """A LoRA adapter for a K -> N linear (PEFT's layouts)."""
    rank: int
    lora_a: np.ndarray   # float16 [rank, K]
    lora_b: np.ndarray   # float16 [N, rank], the adapter's scaling applied

    def extra_bytes(self, M: int) -> int:
        """Bytes the adapter adds to the layer: lora_a, lora_b, and T [M, rank]
        written once and read once."""
        return self.lora_a.size * 2 + self.lora_b.size * 2 + 2 * M * self.rank * 2

    def extra_flops(self, M: int) -> int:
        K, N = self.lora_a.shape[1], self.lora_b.shape[0]
        return 2 * M * K * self.rank + 2 * M * self.rank * N


def make_adapter(K: int, N: int, rank: int, *, seed: int = 0, b_std: float = 0.05) -> Adapter:
    """Draw one seeded adapter: lora_a ~ N(0, 1/K) (so that T = x . lora_a^T
    has unit variance for unit-variance x) and lora_b ~ N(0, b_std^2), both
    drawn in float64 and rounded to float16.  The pages give no adapter
    statistics; these keep the adapter's term a tenth or so of the layer's.
    Its own stream: PCG64 seeded with (seed, 1), lora_a drawn before lora_b."""
    rng = np.random.Generator(np.random.PCG64([seed, 1]))
    a = rng.standard_normal(size=(rank, K)) / math.sqrt(K)
    b = rng.standard_normal(size=(N, rank)) * b_std
    return Adapter(rank=rank, lora_a=a.astype(np.float16), lora_b=b.astype(np.float16))


def make_qzeros(n_groups: int, N: int, *, seed: int = 0) -> np.ndarray:
    """Packed zero points int32 [n_groups, N/8] for the asymmetric layer,
    drawn as whole words (uniform over all bit patterns, so every 4-bit zero
    is uniform in 0..15 and independent), from their own stream: PCG64
    seeded with (seed, 2)."""
    if N % 8:
        raise ValueError("N must be a multiple of 8")
    rng = np.random.Generator(np.random.PCG64([seed, 2]))
    words = rng.integers(0, 2 ** 32, size=(n_groups, N // 8), dtype=np.uint64).astype(np.uint32)
    return words.view(np.int32)


def make_gidx(K: int, group: int, *, seed: int = 0, kind: str = "perm") -> np.ndarray:
    """Group index per input channel, int32 [K], for act-order weights.
    kind "perm": GPTQ's act order, the channels taken in a seeded random
    order and the i-th of that order put in group i // group (every group
    holds `group` channels, the last the rest); "random": each channel in a
    uniformly drawn group of the ceil(K / group) (group sizes unequal);
    "consecutive": k // group (the plain layer).  Own stream: PCG64 seeded
    with (seed, 3)."""
    rng = np.random.Generator(np.random.PCG64([seed, 3]))
    ng = num_groups(K, group)
    G = K if group == -1 or group >= K else group
    if kind == "consecutive":
        return (np.arange(K) // G).astype(np.int32)
    if kind == "perm":
        order = rng.permutation(K)
        g = np.empty(K, dtype=np.int32)
        g[order] = np.arange(K) // G
        return g
    if kind == "random":
        return rng.integers(0, ng, size=K).astype(np.int32)
    raise ValueError(kind)


# The five synthetic workloads, restated from their prose descriptions.
def tiny(M: int = 1, seed: int = 0) -> Problem:
    """W4A16 GEMM, M in {1, 4}, K=512, N=256, group=128, scales U[1e-3, 2e-2]."""
    return make_problem(M, 512, 256, 128, seed=seed, name=f"tiny_M{M}")


def decode_up(seed: int = 0) -> Problem:
    """Decode GEMV, FFN up-projection shape: M=1, K=5120, N=17408, group=128."""
    return make_problem(1, 5120, 17408, 128, seed=seed, name="decode_up_M1")


def decode_down(M: int = 1, seed: int = 0) -> Problem:
    """Small-batch decode, FFN down-projection: M in {1,2,4,8,16}, K=17408,
    N=5120, group=32; 1 % of input channels scaled x20; scales log-U[5e-4, 5e-2]."""
    return make_problem(M, 17408, 5120, 32, seed=seed, scale_dist="log_uniform",
                        scale_range=(5e-4, 5e-2), outlier_frac=0.01,
                        name=f"decode_down_M{M}")


def prefill(M: int = 2048, seed: int = 0) -> Problem:
    """Prefill GEMM: M in {512, 2048, 8192}, K=5120, N=17408, group=128."""
    return make_problem(M, 5120, 17408, 128, seed=seed, name=f"prefill_M{M}")


def group_sweep(group: int, M: int = 1, seed: int = 0) -> Problem:
    """Square K=N=5120 at each group size, M in {1, 16, 4096}."""
    return make_problem(M, 5120, 5120, group, seed=seed, name=f"square_g{group}_M{M}")


# One hidden-5120 decoder layer's linears: (name, K, N, count).
LAYER_LINEARS = (("attn_proj", 5120, 5120, 4), ("gate_up", 5120, 17408, 2),
                 ("down", 17408, 5120, 1))


def layer_linear(which: str, M: int = 1, seed: int = 0) -> Problem:
    for name, K, N, _ in LAYER_LINEARS:
        if name == which:
            return make_problem(M, K, N, 128, seed=seed, name=f"layer_{name}_M{M}")
    raise KeyError(which)
