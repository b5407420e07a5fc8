"""Comparison helpers shared by the GPU parity tests.

Tolerances (stated once): contractions with bf16 operands and fp32 accumulation
(Y, dX, dW) must satisfy max|gpu - ref| / max|ref| <= 2e-2; the fp32 per-group
reductions ds and dz must satisfy the same ratio <= 1e-3.  When the reference is
identically zero (dz after min-max init: nothing is clamped) the CUDA result must
be exactly zero too.  Integer outputs (codes, masks, packed bytes, zero points)
and the fp32 init outputs s, z must match bit for bit.
"""
import numpy as np
import torch

TOL_GEMM = 2e-2
TOL_RED = 1e-3


def to_np(t):
    if t is None:
        return None
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.numpy()


def rel_err(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    if gpu.size == 0:
        return 0.0
    assert np.isfinite(gpu).all(), "non-finite values in the CUDA result"
    den = np.abs(ref).max()
    num = np.abs(gpu - ref).max()
    if den == 0:
        return float("inf") if num > 0 else 0.0
    return float(num / den)


def assert_close(gpu, ref, tol, name):
    e = rel_err(gpu, ref)
    assert e <= tol, f"{name}: max|diff|/max|ref| = {e:.3e} > {tol:.1e}"
    return e


def assert_bits_equal(gpu, ref, name):
    gpu = np.ascontiguousarray(gpu)
    ref = np.ascontiguousarray(ref)
    assert gpu.shape == ref.shape, (name, gpu.shape, ref.shape)
    if gpu.dtype == np.float32:
        same = gpu.view(np.uint32) == ref.astype(np.float32).view(np.uint32)
        # +0.0 and -0.0 are the same value
        same |= (gpu == 0) & (ref == 0)
    else:
        same = gpu == ref
    bad = np.argwhere(~same)
    assert bad.size == 0, f"{name}: {len(bad)} mismatches, first at {bad[0].tolist()}: gpu={gpu[tuple(bad[0])]} ref={ref[tuple(bad[0])]}"


def bf16_round(a):
    """fp32 -> bf16 (round to nearest even) -> fp32, as the CUDA path rounds W-hat."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).float().numpy()
