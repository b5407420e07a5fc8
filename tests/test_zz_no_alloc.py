"""eqat_fq_linear_fwd_noalloc: the Block-AP forward for callers that cannot
allocate device memory or pass a workspace (an operator interface that hands the
library only its inputs and outputs, a process that must not call cudaMalloc while
it runs, memory owned by an allocator the library cannot reach).  It keeps W-hat in
the library's own 32 MiB static device array instead of a caller workspace.

Called here through the C ABI (ctypes) twice in a row, on two different layers, and
compared with the workspace entry point eqat_fq_linear_fwd within the tolerance of
the other parity tests.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import weight_quantization_aware_b200 as eqat
from weight_quantization_aware_b200 import synthetic
from parity import TOL_GEMM, assert_close, to_np

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


def layer(M, N, K, bits, group, seed):
    d = synthetic.draw_linear(np.random.default_rng(seed), M, N, K, 0.02, "bf16")
    X, W = d["X"].cuda(), d["W"].cuda()
    s, z = eqat.minmax_init(W, bits, group)
    return X, W, s, z


def test_noalloc_forward_matches_workspace_forward_on_two_calls_in_a_row():
    from weight_quantization_aware_b200 import build
    build.build()
    # Second layer fills the whole 32 MiB scratch (4096 x 4096 bf16), so stale
    # contents of the first call cannot hide behind a smaller footprint.
    for M, N, K, bits, group, seed in [(300, 392, 384, 2, 64, 1), (256, 4096, 4096, 3, 128, 2)]:
        X, W, s, z = layer(M, N, K, bits, group, seed)
        Y_ref = eqat.fq_linear_fwd(X, W, s, z, bits, group)
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert noalloc_call(X, W, s, z, Y, bits, group) == EQAT_OK
        torch.cuda.synchronize()
        assert_close(to_np(Y), to_np(Y_ref).astype(np.float64), TOL_GEMM, "Y (no-alloc vs workspace)")
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
