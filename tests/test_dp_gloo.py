"""Data parallelism over tokens, two gloo ranks on CPU with the oracle standing in
for the kernels: the sum over ranks of each rank's weight-side gradients equals the
gradients of the concatenated batch, and the forward and input gradient need no
exchange.  This is the exchange bench.py performs with NCCL under torchrun."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from weight_quantization_aware_b200 import dp, synthetic

WL = synthetic.Workload(90, "dp-test-linear", "block_ap", 48, (synthetic.Linear("linear", 40, 128),),
                        2, 32, 0.02, "bf16")


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, out):
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        d = dp.rank_batch(WL, 0, rank)
        X, W, dY = (synthetic.as_f32_numpy(d[k]) for k in ("X", "W", "dY"))
        s, z = oracle.minmax_init(W, WL.bits, WL.group)
        s, z = synthetic.perturb_quant_params(s, z, 5)
        dX, dW, ds, dz = oracle.fq_linear_bwd(X, W, s, z, dY, WL.bits, WL.group)
        packed, zq = oracle.pack(W, s, z, WL.bits, WL.group)
        _, ds2 = oracle.dq_linear_bwd_s(X, packed, zq, s, dY, WL.bits, WL.group)
        grads = [torch.from_numpy(np.ascontiguousarray(a)) for a in (dW, ds, dz, ds2)]
        dp.allreduce_weight_grads(grads, dist)
        out[rank] = [g.numpy() for g in grads] + [dX]
    finally:
        dist.destroy_process_group()


def test_allreduced_weight_grads_equal_full_batch_grads(orc):
    world = 2
    out = mp.Manager().dict()
    mp.spawn(worker, args=(world, free_port(), out), nprocs=world, join=True)
    batches = [dp.rank_batch(WL, 0, r) for r in range(world)]
    X = np.concatenate([synthetic.as_f32_numpy(b["X"]) for b in batches])
    dY = np.concatenate([synthetic.as_f32_numpy(b["dY"]) for b in batches])
    W = synthetic.as_f32_numpy(batches[0]["W"])
    assert np.array_equal(W, synthetic.as_f32_numpy(batches[1]["W"]))  # W is shared
    assert not np.array_equal(synthetic.as_f32_numpy(batches[0]["X"]), synthetic.as_f32_numpy(batches[1]["X"]))
    s, z = orc.minmax_init(W, WL.bits, WL.group)
    s, z = synthetic.perturb_quant_params(s, z, 5)
    dX, dW, ds, dz = orc.fq_linear_bwd(X, W, s, z, dY, WL.bits, WL.group)
    packed, zq = orc.pack(W, s, z, WL.bits, WL.group)
    _, ds2 = orc.dq_linear_bwd_s(X, packed, zq, s, dY, WL.bits, WL.group)
    for r in range(world):
        got = out[r]
        np.testing.assert_allclose(got[0], dW, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(got[1], ds, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(got[2], dz, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(got[3], ds2, rtol=1e-12, atol=1e-12)
        # the input gradient is rank-local: rows r*M .. (r+1)*M of the full batch
        np.testing.assert_allclose(got[4], dX[r * WL.m:(r + 1) * WL.m], rtol=1e-12, atol=1e-12)


def reducer_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        red = dp.OverlappedGradReducer(dist)
        rng = np.random.default_rng(100 + rank)
        layers = [[torch.from_numpy(rng.standard_normal(sh).astype(np.float32)) for sh in ((8, 16), (8, 2), (8, 2))]
                  for _ in range(3)]
        before = [[t.clone() for t in ts] for ts in layers]
        for i, ts in enumerate(layers):
            red.submit(ts + [None], tag=i)
        red.wait()
        # the helper with op="mean" scales the same way as the reducer
        meaned = [t.clone() for t in before[0]]
        dp.allreduce_weight_grads(meaned + [None], dist, op="mean")
        out[rank] = ([[t.numpy() for t in ts] for ts in before], [[t.numpy() for t in ts] for ts in layers], red.order,
                     [t.numpy() for t in meaned])
    finally:
        dist.destroy_process_group()


def test_overlapped_reducer_averages_each_layer_in_order():
    """The Block-AP step's exchange: each linear's (dW, ds, dz) averaged over ranks, in
    submission order; None entries skipped."""
    world = 2
    out = mp.Manager().dict()
    mp.spawn(reducer_worker, args=(world, free_port(), out), nprocs=world, join=True)
    before = [out[r][0] for r in range(world)]
    for r in range(world):
        _, after, order, meaned = out[r]
        assert order == [0, 1, 2]
        for j in range(3):
            np.testing.assert_array_equal(meaned[j], after[0][j])
        for i in range(3):
            for j in range(3):
                mean = (before[0][i][j] + before[1][i][j]) / 2
                np.testing.assert_allclose(after[i][j], mean, rtol=1e-6, atol=1e-7)
