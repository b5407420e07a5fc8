"""eqat_fq_linear_fwd_noalloc: the Block-AP forward for callers that cannot
allocate device memory or pass a workspace (an operator interface that hands the
library only its inputs and outputs, a process that must not call cudaMalloc while
it runs, memory owned by an allocator the library cannot reach).  It keeps W-hat in
the library's own 32 MiB static device array instead of a caller workspace.

Called here through the C ABI (ctypes) several times in a row and compared with the
workspace entry point eqat_fq_linear_fwd (the same two kernels, so the results must
be identical bit for bit) and with the CPU oracle (within the GEMM tolerance of the
other parity tests).  The first call fills the whole static array with NaN (s = NaN
makes every W-hat element NaN), so a later call that failed to write part of its
W-hat would read NaN and show it in Y.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import weight_quantization_aware_b200 as eqat
from weight_quantization_aware_b200 import synthetic
from parity import TOL_GEMM, TOL_RED, assert_close, to_np

pytestmark = pytest.mark.gpu

EQAT_OK, EQAT_ERR_WORKSPACE = 0, 6
SCRATCH_BYTES = 32 << 20


def noalloc_call(X, W, s, z, Y, bits, group):
    lib = eqat.load_library()
    M, K = X.shape
    N = W.shape[0]
    dt = eqat.EQAT_BF16 if X.dtype == torch.bfloat16 else eqat.EQAT_F32
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.eqat_fq_linear_fwd_noalloc(p(X), p(W), dt, p(s), p(z), p(Y), M, N, K, bits, group, stream)


def layer(M, N, K, bits, group, seed, dtype="bf16"):
    d = synthetic.draw_linear(np.random.default_rng(seed), M, N, K, 0.02, dtype)
    X, W = d["X"].cuda(), d["W"].cuda()
    s, z = eqat.minmax_init(W, bits, group)
    return X, W, s, z


def oracle_rows(orc, X, W, s, z, bits, group, rows):
    Xn, Wn = to_np(X).astype(np.float32), to_np(W).astype(np.float32)
    return orc.fq_linear_fwd(Xn, Wn, to_np(s), to_np(z), bits, group, rows=rows)


def test_noalloc_forward_matches_workspace_forward_and_oracle_on_calls_in_a_row(orc):
    from weight_quantization_aware_b200 import build
    build.build()
    # 1: fill the whole 32 MiB array with NaN W-hat (4096 x 4096 bf16, s = NaN).
    X, W, s, z = layer(64, 4096, 4096, 2, 64, 11)
    Y = torch.zeros((64, 4096), dtype=torch.bfloat16, device="cuda")
    assert noalloc_call(X, W, torch.full_like(s, float("nan")), z, Y, 2, 64) == EQAT_OK
    torch.cuda.synchronize()
    assert torch.isnan(Y).all()
    # 2, 3: a small layer on the poisoned array, then a full-size one; each must equal
    # the workspace forward bit for bit and the oracle within the GEMM tolerance.
    rng = np.random.default_rng(3)
    for M, N, K, bits, group, seed in [(300, 392, 384, 2, 64, 1), (256, 4096, 4096, 3, 128, 2)]:
        X, W, s, z = layer(M, N, K, bits, group, seed)
        Y_ref = eqat.fq_linear_fwd(X, W, s, z, bits, group)
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert noalloc_call(X, W, s, z, Y, bits, group) == EQAT_OK
        torch.cuda.synchronize()
        assert torch.isfinite(Y).all()
        assert torch.equal(Y, Y_ref), "no-alloc and workspace forward differ"
        rows = np.sort(rng.choice(M, min(M, 48), replace=False))
        want = oracle_rows(orc, X, W, s, z, bits, group, rows)
        assert_close(to_np(Y)[rows], want, TOL_GEMM, "Y (no-alloc vs oracle)")
    assert eqat.device_error() == 0


def test_noalloc_fp32_layer_through_the_binding(orc):
    """The fp32 branch (CUDA-core GEMM on the static array) through the Python binding."""
    X, W, s, z = layer(96, 136, 256, 4, 32, 5, dtype="f32")
    Y_ref = eqat.fq_linear_fwd(X, W, s, z, 4, 32)
    for _ in range(2):
        Y = torch.full((96, 136), float("nan"), dtype=torch.float32, device="cuda")
        eqat.fq_linear_fwd_noalloc(X, W, s, z, 4, 32, Y=Y)
        torch.cuda.synchronize()
        assert torch.equal(Y, Y_ref)
    want = oracle_rows(orc, X, W, s, z, 4, 32, None)
    assert_close(to_np(Y), want, TOL_RED, "Y fp32 (no-alloc vs oracle)")
    assert eqat.device_error() == 0


def test_noalloc_rejects_layers_beyond_the_scratch():
    lib = eqat.load_library()
    X = torch.empty(8, 4096 + 64, dtype=torch.bfloat16, device="cuda")
    W = torch.empty(4096, 4096 + 64, dtype=torch.bfloat16, device="cuda")  # 4096*4160*2 B > 32 MiB
    s = torch.empty(4096, (4096 + 64) // 64, dtype=torch.float32, device="cuda")
    Y = torch.empty(8, 4096, dtype=torch.bfloat16, device="cuda")
    assert 4096 * (4096 + 64) * 2 > SCRATCH_BYTES
    assert noalloc_call(X, W, s, s, Y, 2, 64) == EQAT_ERR_WORKSPACE
    assert b"32 MiB" in lib.eqat_last_error_detail()
