"""GPU parity of the decode-size path of eqat_dq_linear_fwd (M <= 8, group 64 or 128:
the codes are streamed once and never dequantized to memory) against the CPU oracle's
E2E-QP forward, over 2/3/4-bit codes, fp32 and fp16 step sizes, ragged N and K, one
and several K chunks, and the Llama-2 shapes the pages train."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import weight_quantization_aware_b200 as eqat
from weight_quantization_aware_b200 import synthetic
from parity import TOL_GEMM, assert_close, to_np

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from weight_quantization_aware_b200 import build
    build.build()
    eqat.load_library()
    assert torch.cuda.is_available()
    yield
    assert eqat.device_error() == 0


def run_case(orc, M, N, K, bits, g, s16, seed, trained=True):
    d = synthetic.draw_linear(np.random.default_rng(seed), M, N, K, 0.02, "bf16")
    Xn, Wn = synthetic.as_f32_numpy(d["X"]), synthetic.as_f32_numpy(d["W"])
    s, z = orc.minmax_init(Wn, bits, g)
    packed, zq = orc.pack(Wn, s, z, bits, g)
    if trained:
        s, _ = synthetic.perturb_quant_params(s, z, seed)
    if s16:
        s = s.astype(np.float16)
    Y = eqat.dq_linear_fwd(d["X"].cuda(), torch.from_numpy(packed).cuda(), torch.from_numpy(zq).cuda(),
                           torch.from_numpy(s).cuda(), bits, g)
    Y_ref = orc.dq_linear_fwd(Xn, packed, zq, s, bits, g)
    assert_close(to_np(Y), Y_ref, TOL_GEMM, f"Y M={M} N={N} K={K} b={bits} g={g}")
    return to_np(Y), Y_ref


CASES = [  # (M, N, K, bits, group)
    (1, 8, 64, 2, 64),          # one set, one partial row tile
    (1, 264, 960, 2, 64),       # ragged N (2 tiles + 8 rows), K not a multiple of the stage
    (3, 136, 4096, 2, 128),     # several K chunks (split-K partials)
    (8, 392, 2304, 4, 64),
    (5, 200, 1152, 4, 128),
    (8, 520, 1600, 3, 64),
    (2, 96, 768, 3, 128),
    (7, 1024, 8192, 2, 64),
    # groups of a stage sharing the mma columns: every (bits, group, slots) layout
    (1, 200, 1664, 2, 128),     # 4 slots, 2 token columns (one empty)
    (2, 136, 1088, 2, 64),      # 4 slots x 2 tokens
    (4, 264, 2048, 2, 64),      # 2 slots x 4 tokens
    (1, 392, 1344, 4, 64),      # 4 slots
    (2, 136, 2304, 4, 128),     # 2 slots x 4 columns (two empty)
    (4, 128, 512, 4, 64),       # 2 slots x 4 tokens
    (1, 72, 704, 3, 64),        # 2 slots
    (1, 136, 384, 3, 128),      # 1 slot, 7 empty columns
]


@pytest.mark.parametrize("s16", [False, True], ids=["s32", "s16"])
@pytest.mark.parametrize("case", CASES, ids=["x".join(map(str, c)) for c in CASES])
def test_gemv_parity(orc, case, s16):
    M, N, K, bits, g = case
    run_case(orc, M, N, K, bits, g, s16, 900 + M + N + K)


def test_gemv_tokens_are_independent(orc):
    """Each token row of Y depends only on its own row of X: M=8 equals eight M=1 calls."""
    M, N, K, bits, g = 8, 264, 1536, 2, 64
    d = synthetic.draw_linear(np.random.default_rng(5), M, N, K, 0.02, "bf16")
    Wn = synthetic.as_f32_numpy(d["W"])
    s, z = orc.minmax_init(Wn, bits, g)
    packed, zq = orc.pack(Wn, s, z, bits, g)
    c, q, sd = (torch.from_numpy(a).cuda() for a in (packed, zq, s))
    X = d["X"].cuda()
    Y8 = eqat.dq_linear_fwd(X, c, q, sd, bits, g)
    for m in range(M):
        Y1 = eqat.dq_linear_fwd(X[m:m + 1].contiguous(), c, q, sd, bits, g)
        # the K split may differ with M, so allow the bf16 rounding of the output
        assert_close(to_np(Y1[0]), to_np(Y8[m]), 8e-3, f"token {m}")


@pytest.mark.parametrize("shape", [(4096, 4096), (11008, 4096), (4096, 11008), (1024, 8192)],
                         ids=lambda s: f"{s[0]}x{s[1]}")
def test_gemv_llama_shapes(orc, shape):
    N, K = shape
    run_case(orc, 1, N, K, 2, 64, False, 77 + N)


def test_gemv_matches_dequant_gemm_path(orc):
    """The same call with the decode path switched off (EQAT_DQ_GEMV=0, dequant + GEMM)
    agrees with it within the bf16 output rounding."""
    code = (
        "import numpy as np, torch, weight_quantization_aware_b200 as e\n"
        "from weight_quantization_aware_b200 import synthetic\n"
        "import oracle as o\n"
        "d = synthetic.draw_linear(np.random.default_rng(3), 4, 392, 2048, 0.02, 'bf16')\n"
        "W = synthetic.as_f32_numpy(d['W'])\n"
        "s, z = o.minmax_init(W, 2, 64)\n"
        "p, q = o.pack(W, s, z, 2, 64)\n"
        "Y = e.dq_linear_fwd(d['X'].cuda(), torch.from_numpy(p).cuda(), torch.from_numpy(q).cuda(),"
        " torch.from_numpy(s).cuda(), 2, 64)\n"
        "np.save(__import__('sys').argv[1], Y.float().cpu().numpy())\n")
    import tempfile
    outs = []
    tmp = tempfile.mkdtemp()
    for flag in ("1", "0"):
        path = os.path.join(tmp, f"gemv_path_{flag}.npy")
        env = dict(os.environ, EQAT_DQ_GEMV=flag, PYTHONPATH=ROOT)
        r = subprocess.run([sys.executable, "-c", code, path], cwd=ROOT, env=env, capture_output=True,
                           text=True, timeout=600)
        assert r.returncode == 0, r.stderr[-2000:]
        outs.append(np.load(path))
    ref = np.abs(outs[1]).max()
    assert np.abs(outs[0] - outs[1]).max() <= 1e-2 * ref


@pytest.mark.parametrize("shape", [(1, 8, 64), (8, 392, 2304)], ids=lambda s: "x".join(map(str, s)))
def test_gemv_with_w_hat_sized_workspace(orc, shape):
    """The smallest workspace the call accepts, N K bf16 elements, holds the decode
    path's partial sums (at most M N K / 128 bytes) and gives the right result."""
    M, N, K = shape
    bits, g = 2, 64
    d = synthetic.draw_linear(np.random.default_rng(11), M, N, K, 0.02, "bf16")
    Xn, Wn = synthetic.as_f32_numpy(d["X"]), synthetic.as_f32_numpy(d["W"])
    s, z = orc.minmax_init(Wn, bits, g)
    packed, zq = orc.pack(Wn, s, z, bits, g)
    assert eqat.workspace_bytes(M, N, K, bits, g, torch.bfloat16) >= N * K * 2
    ws = torch.empty(N * K * 2, dtype=torch.uint8, device="cuda")
    Y = eqat.dq_linear_fwd(d["X"].cuda(), torch.from_numpy(packed).cuda(), torch.from_numpy(zq).cuda(),
                           torch.from_numpy(s).cuda(), bits, g, ws=ws)
    assert_close(to_np(Y), orc.dq_linear_fwd(Xn, packed, zq, s, bits, g), TOL_GEMM, "Y")


@pytest.mark.parametrize("M", [1, 2])
def test_gemv_large_layer_fragment_mode(orc, M):
    """A layer above the build-mode size (44 MB of codes, s and zq, so the fragments
    come from the separate X kernel at M = 1 and 2, with eight and four group slots),
    checked on sampled row tiles: the first, two inner ones and the ragged last.
    The frozen codes, zq and s are drawn directly (any bytes are valid codes)."""
    N, K, bits, g = 16392, 8192, 2, 64
    rng = np.random.default_rng(4100 + M)
    packed = rng.integers(0, 256, size=(N, K // 4), dtype=np.uint8)
    zq = rng.integers(0, 4, size=(N, K // g), dtype=np.uint8)
    s = (rng.random((N, K // g), dtype=np.float32) * 0.01 + 1e-3).astype(np.float32)
    X = torch.randn(M, K, generator=torch.Generator().manual_seed(M)).to(torch.bfloat16)
    Y = eqat.dq_linear_fwd(X.cuda(), torch.from_numpy(packed).cuda(), torch.from_numpy(zq).cuda(),
                           torch.from_numpy(s).cuda(), bits, g)
    rows = np.r_[0:128, 7040:7168, 12800:12928, 16384:N]
    Xn = synthetic.as_f32_numpy(X)
    Y_ref = orc.dq_linear_fwd(Xn, packed[rows], zq[rows], s[rows], bits, g)
    assert_close(to_np(Y)[:, rows], Y_ref, TOL_GEMM, f"Y sampled rows M={M}")
