"""Data parallelism over tokens for the fake-quantized linear layer.

Every rank holds the same W, s, z (or frozen codes) and its own batch of tokens.
The forward and the input gradient are rank-local; the weight-side gradients
dW, ds, dz (Block-AP) and ds (E2E-QP) are sums over tokens, hence over ranks, and
are the layer's one exchange: an all-reduce after the backward.

The two helpers scale differently, on purpose:

* allreduce_weight_grads(..., op="sum") SUMS over ranks (the default): the
  gradient of a loss that is a sum over every rank's tokens (the bench step's
  dY is a per-token gradient, so the sum is the full-batch gradient).
* OverlappedGradReducer AVERAGES over ranks: the Block-AP loss is a mean over
  tokens, and each rank's dY already carries 1 / (its own tokens), so the mean of
  the ranks' gradients is the gradient of the mean over all tokens.

allreduce_weight_grads(..., op="mean") gives the reducer's scaling in one call.
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


def allreduce_weight_grads(tensors, dist, group=None, op: str = "sum") -> None:
    """All-reduces the weight-side gradients over ranks in place (None entries
    skipped): op="sum" adds them, op="mean" adds them and divides by the number
    of ranks (the scaling of OverlappedGradReducer)."""
    if op not in ("sum", "mean"):
        raise ValueError(f"op must be 'sum' or 'mean', got {op!r}")
    world = dist.get_world_size(group)
    for t in tensors:
        if t is not None:
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
            if op == "mean" and world > 1:
                t.mul_(1.0 / world)


class OverlappedGradReducer:
    """Averages the weight-side gradients over ranks while later work runs.

    submit(tensors) starts the exchange of one layer's gradients as soon as the
    kernels that produced them are done: on CUDA it records an event on the
    compute stream, and a communication stream waits on it and all-reduces there,
    so the next layer's forward and backward proceed meanwhile.  wait() makes the
    compute stream wait for every exchange submitted (call it before the optimizer
    step).  The Block-AP loss is a mean over tokens, so the exchange is a mean
    over ranks (NCCL's AVG; SUM then a scale where the backend has no AVG).
    On CPU tensors (gloo) the exchange runs at submit time."""

    def __init__(self, dist, group=None, device=None):
        import torch
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.cuda = device is not None and torch.device(device).type == "cuda"
        self.stream = torch.cuda.Stream(device=device) if self.cuda else None
        self.has_avg = dist.get_backend(group) == "nccl"
        self.order = []  # submission order, for checks

    def _reduce(self, tensors):
        d = self.dist
        for t in tensors:
            if t is None:
                continue
            if self.has_avg:
                d.all_reduce(t, op=d.ReduceOp.AVG, group=self.group)
            else:
                d.all_reduce(t, op=d.ReduceOp.SUM, group=self.group)
                t.mul_(1.0 / self.world)

    def submit(self, tensors, tag=None):
        import torch
        self.order.append(tag)
        if not self.cuda:
            self._reduce(tensors)
            return
        ev = torch.cuda.Event()
        ev.record(torch.cuda.current_stream(self.stream.device))
        with torch.cuda.stream(self.stream):
            self.stream.wait_event(ev)
            self._reduce(tensors)
        for t in tensors:  # in use on the communication stream until wait()
            if t is not None:
                t.record_stream(self.stream)

    def wait(self):
        import torch
        if self.cuda:
            torch.cuda.current_stream(self.stream.device).wait_stream(self.stream)
