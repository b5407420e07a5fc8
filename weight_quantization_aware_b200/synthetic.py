"""Seeded synthetic inputs for the fake-quantized linear layer.

This module only draws random numbers and casts them to the storage dtype.  It
holds none of the quantizer's arithmetic, so the CPU oracle (tests) and the CUDA
path (library, tests, bench) can both take their inputs from it.

Recipe (stated once, used everywhere):

* generator: NumPy PCG64 ``default_rng``; one independent stream per linear layer,
  spawned from ``SeedSequence([1000 + config_index, linear_index])``;
* X ~ N(0, 1) [M, K], dY ~ N(0, 1) [M, N], W ~ N(0, sigma) [N, K], all drawn in
  fp32;
* outliers: floor(0.001 * N * K) distinct entries of W, drawn uniformly without
  replacement from the same stream, are multiplied by 10;
* cast to the layer dtype (bf16 by round-to-nearest-even, or kept fp32).

Shapes are those of the Llama-2 linears the EfficientQAT pages quantize (only the
linear layers inside transformer blocks are quantized; paperlayer summary,
section D), with the token counts of the Block-AP (2048-token samples) and E2E-QP
(4096-token samples) recipes (modelfoundations note, "The recipe in numbers").
The pages' datasets (RedPajama, C4, ...) and checkpoints stand behind these
shapes; the values here are synthetic.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Linear:
    name: str
    n: int  # out-features (rows of W)
    k: int  # in-features (columns of W, the grouped dimension)


@dataclass(frozen=True)
class Workload:
    index: int  # 1-based; seeds are 1000 + index
    name: str
    mode: str  # "block_ap" (fake-quant W, s, z trainable) or "e2e_qp" (frozen packed codes)
    m: int  # tokens
    linears: tuple
    bits: int
    group: int
    sigma: float
    dtype: str  # "f32" or "bf16"
    outliers: bool = True
    extra: dict = field(default_factory=dict)

    def flops_per_step(self) -> int:
        """fwd + dX + dW-hat contractions: 6*M*N*K per linear."""
        return sum(6 * self.m * l.n * l.k for l in self.linears)


WORKLOADS = {
    1: Workload(1, "single-linear-fp32-m128-n512-k256-w2g64", "block_ap", 128,
                (Linear("linear", 512, 256),), 2, 64, 0.02, "f32"),
    2: Workload(2, "llama2-7b-q_proj-blockap-w2g64-m4096", "block_ap", 4096,
                (Linear("q_proj", 4096, 4096),), 2, 64, 0.02, "bf16"),
    3: Workload(3, "llama2-7b-mlp-blockap-w3g128-m8192", "block_ap", 8192,
                (Linear("gate_proj", 11008, 4096), Linear("up_proj", 11008, 4096),
                 Linear("down_proj", 4096, 11008)), 3, 128, 0.02, "bf16"),
    4: Workload(4, "llama2-13b-e2eqp-w2g64-m4096", "e2e_qp", 4096,
                (Linear("q_proj", 5120, 5120), Linear("o_proj", 5120, 5120),
                 Linear("gate_proj", 13824, 5120), Linear("up_proj", 13824, 5120),
                 Linear("down_proj", 5120, 13824)), 2, 64, 0.02, "bf16", outliers=False),
    5: Workload(5, "llama2-70b-block-blockap-w2g64-m2048", "block_ap", 2048,
                (Linear("q_proj", 8192, 8192), Linear("k_proj", 1024, 8192),
                 Linear("v_proj", 1024, 8192), Linear("o_proj", 8192, 8192),
                 Linear("gate_proj", 28672, 8192), Linear("up_proj", 28672, 8192),
                 Linear("down_proj", 8192, 28672)), 2, 64, 0.015, "bf16"),
}


def rng_for(seed_index: int, linear_index: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([1000 + seed_index, linear_index]))


def to_dtype(a: np.ndarray, dtype: str) -> torch.Tensor:
    """fp32 numpy -> CPU torch tensor of the storage dtype (bf16: round-to-nearest-even)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t
    raise ValueError(dtype)


def draw_linear(rng: np.random.Generator, m: int, n: int, k: int, sigma: float,
                dtype: str, outliers: bool = True) -> dict:
    """Draw X [m,k], W [n,k], dY [m,n] as CPU torch tensors of `dtype`."""
    w = rng.standard_normal((n, k), dtype=np.float32) * np.float32(sigma)
    if outliers and n * k > 0:
        cnt = (n * k) // 1000
        if cnt:
            idx = rng.choice(n * k, size=cnt, replace=False)
            w.reshape(-1)[idx] *= np.float32(10.0)
    x = rng.standard_normal((m, k), dtype=np.float32)
    dy = rng.standard_normal((m, n), dtype=np.float32)
    return {"X": to_dtype(x, dtype), "W": to_dtype(w, dtype), "dY": to_dtype(dy, dtype)}


def workload_linear(wl: Workload, li: int, m: int | None = None) -> dict:
    lin = wl.linears[li]
    rng = rng_for(wl.index, li)
    return draw_linear(rng, wl.m if m is None else m, lin.n, lin.k, wl.sigma, wl.dtype, wl.outliers)


def perturb_quant_params(s: np.ndarray, z: np.ndarray, seed: int) -> tuple:
    """"Trained-state" quantization parameters: s *= U(0.6, 1.0), z += U{-1, 0, 1}.

    Min-max init clamps (almost) nothing, which leaves the clamped branch of the
    straight-through backward untested; shrinking s and shifting z by random
    amounts puts a few percent of the weights outside the grid.  Pure random draws:
    the inputs s, z are passed in, whoever computed them.
    """
    rng = np.random.default_rng(np.random.SeedSequence([7000 + seed]))
    f = rng.uniform(0.6, 1.0, size=s.shape).astype(np.float32)
    dz = rng.integers(-1, 2, size=z.shape).astype(np.float32)
    return (s.astype(np.float32) * f).astype(np.float32), (z.astype(np.float32) + dz).astype(np.float32)


def random_quant_params(n: int, g_count: int, bits: int, seed: int, s_lo=1e-3, s_hi=5e-2) -> tuple:
    """Independent random s > 0 and float (non-integer) z spanning beyond [0, 2^bits - 1]."""
    rng = np.random.default_rng(np.random.SeedSequence([8000 + seed]))
    s = rng.uniform(s_lo, s_hi, size=(n, g_count)).astype(np.float32)
    q = (1 << bits) - 1
    z = rng.uniform(-1.5, q + 1.5, size=(n, g_count)).astype(np.float32)
    return s, z


def as_f32_numpy(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16/fp32 CPU tensor to fp32 numpy (bf16 -> fp32 is exact)."""
    return t.detach().to("cpu").float().contiguous().numpy()
