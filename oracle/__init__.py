"""CPU oracle for the EfficientQAT fake-quantized linear layer (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import this package.  The library's product path never does: it has no CPU
fallback.  The arithmetic lives in ``eqat_oracle.c`` (plain C, fp32 element math,
fp64 accumulation); this module builds it with gcc, loads it with ctypes and
strings its steps together in the pages' order:

* Block-AP (zhaoyang97 ACL2025 notes, Eq. 1 / Eq. 2; paperlayer appendix A):
  min-max init -> fake-quant (codes, mask, W-hat) -> Y = X W-hat^T ->
  dX = dY W-hat, dW-hat = dY^T X -> straight-through dW, ds, dz.
* E2E-QP (modelfoundations note, Phase 2): pack -> W-hat = (W_q - z) s ->
  Y, dX, ds = sum dW-hat (W_q - z).

Every function here that calls the C library checks its arguments and returns
NumPy arrays; float outputs of the contractions are fp64.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "eqat_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

CFLAGS = ["-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
          "-fPIC", "-shared", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile eqat_oracle.c into liboracle.so (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        # EQAT_ORACLE_LIB points the wrapper at another build of eqat_oracle.c (the
        # mutation test builds copies with a planted mistake and checks that the pins
        # reject each of them).
        path = os.environ.get("EQAT_ORACLE_LIB")
        if not path:
            path = build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        D = ctypes.c_double
        sig = {
            "orc_minmax_init": [P, I64, I64, I, I, P, P],
            "orc_fake_quant": [P, P, P, I64, I64, I, I, P, P, P, P],
            "orc_pack": [P, P, P, I64, I64, I, I, P, P],
            "orc_dequant_packed": [P, P, P, I64, I64, I, I, P],
            "orc_linear_fwd": [P, P, I64, I64, I64, P, I64, P],
            "orc_linear_dx": [P, P, I64, I64, I64, P, I64, P],
            "orc_linear_dwhat": [P, P, I64, I64, I64, P, I64, P],
            "orc_ste_grads": [P, P, P, P, P, I64, I64, I64, I, I, P, P, P],
            "orc_e2e_ds": [P, P, P, P, I64, I64, I64, I, I, P],
            "orc_ste_grads_clamp_pass": [P, P, P, P, P, I64, I64, I64, I, I, P, P, P],
            "orc_e2e_dz": [P, P, P, I64, I64, I64, I, P],
            "orc_adamw": [P, P, P, P, I64, D, D, D, D, D, I64],
        }
        for name, args in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = None
        lib.orc_num_threads.restype = I
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().orc_num_threads())


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return a


def _rows(rows):
    if rows is None:
        return None, 0
    r = np.ascontiguousarray(rows, dtype=np.int64)
    return r, int(r.size)


def _check(N, K, bits, group):
    if bits not in (2, 3, 4):
        raise ValueError("bits must be 2, 3 or 4")
    if group <= 0 or K % group:
        raise ValueError("K must be a multiple of group")


def packed_row_bytes(K: int, bits: int) -> int:
    return K // 4 if bits == 2 else K // 2 if bits == 4 else K


def minmax_init(W, bits, group):
    W = _f32(W)
    N, K = W.shape
    _check(N, K, bits, group)
    s = np.empty((N, K // group), np.float32)
    z = np.empty((N, K // group), np.float32)
    _load().orc_minmax_init(_p(W), N, K, bits, group, _p(s), _p(z))
    return s, z


def fake_quant(W, s, z, bits, group):
    """Returns (W_hat fp32, code uint8, mask uint8, u = W/s fp32)."""
    W, s, z = _f32(W), _f32(s), _f32(z)
    N, K = W.shape
    _check(N, K, bits, group)
    assert s.shape == z.shape == (N, K // group)
    wh = np.empty((N, K), np.float32)
    code = np.empty((N, K), np.uint8)
    mask = np.empty((N, K), np.uint8)
    u = np.empty((N, K), np.float32)
    _load().orc_fake_quant(_p(W), _p(s), _p(z), N, K, bits, group, _p(wh), _p(code), _p(mask), _p(u))
    return wh, code, mask, u


def pack(W, s, z, bits, group):
    """Returns (packed codes uint8 [N, row_bytes], zq uint8 [N, G])."""
    W, s, z = _f32(W), _f32(s), _f32(z)
    N, K = W.shape
    _check(N, K, bits, group)
    packed = np.empty((N, packed_row_bytes(K, bits)), np.uint8)
    zq = np.empty((N, K // group), np.uint8)
    _load().orc_pack(_p(W), _p(s), _p(z), N, K, bits, group, _p(packed), _p(zq))
    return packed, zq


def dequant_packed(packed, zq, s, K, bits, group):
    """W-hat = (W_q - zq) s in fp32.  s may be float16 (the pages' fp16 step-size
    storage); widening it to fp32 is exact."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    zq = np.ascontiguousarray(zq, dtype=np.uint8)
    s = _f32(s)
    N = packed.shape[0]
    _check(N, K, bits, group)
    wh = np.empty((N, K), np.float32)
    _load().orc_dequant_packed(_p(packed), _p(zq), _p(s), N, K, bits, group, _p(wh))
    return wh


def linear_fwd(X, W_hat, rows=None):
    X, W_hat = _f32(X), _f32(W_hat)
    M, K = X.shape
    N = W_hat.shape[0]
    r, nr = _rows(rows)
    Y = np.empty((M if r is None else nr, N), np.float64)
    _load().orc_linear_fwd(_p(X), _p(W_hat), M, N, K, _p(r), nr, _p(Y))
    return Y


def linear_dx(dY, W_hat, rows=None):
    dY, W_hat = _f32(dY), _f32(W_hat)
    M, N = dY.shape
    K = W_hat.shape[1]
    r, nr = _rows(rows)
    dX = np.empty((M if r is None else nr, K), np.float64)
    _load().orc_linear_dx(_p(dY), _p(W_hat), M, N, K, _p(r), nr, _p(dX))
    return dX


def linear_dwhat(dY, X, wrows=None):
    dY, X = _f32(dY), _f32(X)
    M, N = dY.shape
    K = X.shape[1]
    r, nr = _rows(wrows)
    out = np.empty((N if r is None else nr, K), np.float64)
    _load().orc_linear_dwhat(_p(dY), _p(X), M, N, K, _p(r), nr, _p(out))
    return out


def ste_grads(W, s, z, dWhat, bits, group, wrows=None, clamp_pass=False):
    """Block-AP straight-through grads for the weight rows `wrows` (rows of dWhat).
    clamp_pass=True: the clamp is straight-through as well (all-pass variant)."""
    W, s, z = _f32(W), _f32(s), _f32(z)
    dWhat = np.ascontiguousarray(dWhat, dtype=np.float64)
    N, K = W.shape
    _check(N, K, bits, group)
    r, nr = _rows(wrows)
    n_out = N if r is None else nr
    assert dWhat.shape == (n_out, K)
    G = K // group
    dW = np.empty((n_out, K), np.float64)
    ds = np.empty((n_out, G), np.float64)
    dz = np.empty((n_out, G), np.float64)
    fn = _load().orc_ste_grads_clamp_pass if clamp_pass else _load().orc_ste_grads
    fn(_p(W), _p(s), _p(z), _p(dWhat), _p(r), nr, N, K, bits, group, _p(dW), _p(ds), _p(dz))
    return dW, ds, dz


def e2e_ds(packed, zq, dWhat, K, bits, group, wrows=None):
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    zq = np.ascontiguousarray(zq, dtype=np.uint8)
    dWhat = np.ascontiguousarray(dWhat, dtype=np.float64)
    N = packed.shape[0]
    _check(N, K, bits, group)
    r, nr = _rows(wrows)
    n_out = N if r is None else nr
    assert dWhat.shape == (n_out, K)
    ds = np.empty((n_out, K // group), np.float64)
    _load().orc_e2e_ds(_p(packed), _p(zq), _p(dWhat), _p(r), nr, N, K, bits, group, _p(ds))
    return ds


def e2e_dz(s, dWhat, K, group, wrows=None):
    """E2E-QP zero-point gradient dz = -s * sum_group dW-hat (z trained as a float)."""
    s = _f32(s)
    dWhat = np.ascontiguousarray(dWhat, dtype=np.float64)
    N = s.shape[0]
    _check(N, K, 2, group)
    r, nr = _rows(wrows)
    n_out = N if r is None else nr
    assert dWhat.shape == (n_out, K)
    dz = np.empty((n_out, K // group), np.float64)
    _load().orc_e2e_dz(_p(s), _p(dWhat), _p(r), nr, N, K, group, _p(dz))
    return dz


def adamw(p, g, m, v, lr, b1, b2, eps, wd, t):
    """One AdamW step (decoupled weight decay) on fp32 state; returns new (p, m, v)."""
    p, m, v = (np.array(a, dtype=np.float32, copy=True) for a in (p, m, v))
    g = _f32(g)
    assert p.shape == g.shape == m.shape == v.shape and t >= 1
    _load().orc_adamw(_p(p), _p(g), _p(m), _p(v), p.size, float(lr), float(b1), float(b2), float(eps),
                      float(wd), int(t))
    return p, m, v


def cosine_lr(lr0, lr_min, t, total):
    """Cosine annealing of the learning rate at step t of `total` ([MF] Phase 1: weights and
    quantization parameters on separate cosine schedules): lr_min + (lr0 - lr_min)(1 + cos(pi t / total)) / 2."""
    return lr_min + (lr0 - lr_min) * (1.0 + math.cos(math.pi * t / total)) / 2.0


def mse_grad(Y, T):
    """Reconstruction loss of Block-AP against the full-precision output ([MF] "Both phases": MSE
    to FP block outputs), mean over all elements, and its gradient dL/dY = 2 (Y - T) / numel."""
    Y = np.asarray(Y, dtype=np.float64)
    T = np.asarray(T, dtype=np.float64)
    R = Y - T
    return float(np.sum(R * R) / R.size), 2.0 * R / R.size


# ----------------------------------------------------------------------------
# The layer, step by step in the pages' order.
# ----------------------------------------------------------------------------

def fq_linear_fwd(X, W, s, z, bits, group, rows=None):
    """Block-AP forward: W-hat from Eq. 1-2, then Y = X W-hat^T (rows of Y listed)."""
    wh = fake_quant(W, s, z, bits, group)[0]
    return linear_fwd(X, wh, rows)


def fq_linear_bwd(X, W, s, z, dY, bits, group, rows=None, wrows=None, clamp_pass=False):
    """Block-AP backward: dX (token rows `rows`), dW, ds, dz (weight rows `wrows`)."""
    wh = fake_quant(W, s, z, bits, group)[0]
    dX = linear_dx(dY, wh, rows)
    dwh = linear_dwhat(dY, X, wrows)
    dW, ds, dz = ste_grads(W, s, z, dwh, bits, group, wrows, clamp_pass=clamp_pass)
    return dX, dW, ds, dz


def dq_linear_fwd(X, packed, zq, s, bits, group, rows=None):
    K = np.asarray(X).shape[1]
    wh = dequant_packed(packed, zq, s, K, bits, group)
    return linear_fwd(X, wh, rows)


def dq_linear_bwd_s(X, packed, zq, s, dY, bits, group, rows=None, wrows=None):
    """E2E-QP backward: dX (token rows `rows`) and ds (weight rows `wrows`)."""
    dX, ds, _ = dq_linear_bwd(X, packed, zq, s, dY, bits, group, rows, wrows)
    return dX, ds


def dq_linear_bwd(X, packed, zq, s, dY, bits, group, rows=None, wrows=None):
    """E2E-QP backward with the zero-point gradient: dX (token rows `rows`), ds and
    dz (weight rows `wrows`).  s may be float16 (fp16 step-size storage); widening
    it to fp32 is exact."""
    K = np.asarray(X).shape[1]
    wh = dequant_packed(packed, zq, s, K, bits, group)
    dX = linear_dx(dY, wh, rows)
    dwh = linear_dwhat(dY, X, wrows)
    ds = e2e_ds(packed, zq, dwh, K, bits, group, wrows)
    dz = e2e_dz(s, dwh, K, group, wrows)
    return dX, ds, dz
