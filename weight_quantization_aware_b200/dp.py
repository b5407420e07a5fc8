"""Data parallelism over tokens for the fake-quantized linear layer.

Every rank holds the same W, s, z (or frozen codes) and its own batch of tokens.
The forward and the input gradient are rank-local; the weight-side gradients
dW, ds, dz (Block-AP) and ds (E2E-QP) are sums over tokens, hence over ranks, and
are the layer's one exchange: an all-reduce (sum) after the backward.
"""
from __future__ import annotations

from . import synthetic


def rank_batch(wl: synthetic.Workload, li: int, rank: int, m: int | None = None) -> dict:
    """X, W, dY for `rank`: W is the workload's (shared); X and dY come from a
    rank-specific stream (rank 0 sees the workload's own tokens)."""
    d = synthetic.workload_linear(wl, li, m)
    if rank:
        lin = wl.linears[li]
        other = synthetic.draw_linear(synthetic.rng_for(wl.index, 1000 * (li + 1) + rank),
                                      wl.m if m is None else m, lin.n, lin.k, wl.sigma, wl.dtype, wl.outliers)
        d["X"], d["dY"] = other["X"], other["dY"]
    return d


def allreduce_weight_grads(tensors, dist, group=None) -> None:
    """Sums the weight-side gradients over ranks in place (None entries skipped)."""
    for t in tensors:
        if t is not None:
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
