"""GPU parity of the quantizer variants against the CPU oracle:
- the all-pass clamp gradient of the Block-AP backward (EQAT_GRAD_CLAMP_PASS);
- the E2E-QP backward with the zero-point gradient dz;
- fp16 step-size storage in the E2E-QP dequant, forward and backward.
Inputs are the seeded generators of the main parity suite; the trained quantizer
state clamps a few percent of the weights, where the variants differ."""
import numpy as np
import pytest
import torch

import weight_quantization_aware_b200 as eqat
from weight_quantization_aware_b200 import synthetic
from parity import TOL_GEMM, TOL_RED, assert_bits_equal, assert_close, bf16_round, to_np

pytestmark = pytest.mark.gpu

SHAPES = [  # (M, N, K, bits, group, dtype)
    (300, 392, 384, 2, 64, "bf16"),
    (200, 136, 160, 4, 32, "bf16"),
    (257, 520, 640, 3, 128, "bf16"),
    (77, 24, 96, 3, 32, "f32"),
    (128, 512, 256, 2, 64, "f32"),
]
IDS = ["x".join(map(str, s)) for s in SHAPES]


@pytest.fixture(scope="module", autouse=True)
def built():
    from weight_quantization_aware_b200 import build
    build.build()
    eqat.load_library()
    assert torch.cuda.is_available()
    yield
    assert eqat.device_error() == 0


def draw(M, N, K, dtype, seed):
    d = synthetic.draw_linear(np.random.default_rng(seed), M, N, K, 0.02, dtype)
    return d, {k: synthetic.as_f32_numpy(v) for k, v in d.items()}


@pytest.mark.parametrize("shape", SHAPES, ids=IDS)
def test_clamp_pass_backward(orc, shape):
    M, N, K, bits, g, dtype = shape
    d, h = draw(M, N, K, dtype, 700 + M)
    s, z = orc.minmax_init(h["W"], bits, g)
    s, z = synthetic.perturb_quant_params(s, z, 700 + M)
    z = z + np.float32(0.375)
    _, _, mask, _ = orc.fake_quant(h["W"], s, z, bits, g)
    assert 0 < mask.mean() < 1
    X, W, dY = d["X"].cuda(), d["W"].cuda(), d["dY"].cuda()
    sd, zd = torch.from_numpy(s).cuda(), torch.from_numpy(z).cuda()
    dX, dW, ds, dz = eqat.fq_linear_bwd(X, W, sd, zd, dY, bits, g, clamp_pass=True)
    dX_r, dW_r, ds_r, dz_r = orc.fq_linear_bwd(h["X"], h["W"], s, z, h["dY"], bits, g, clamp_pass=True)
    assert_close(to_np(dX), dX_r, TOL_GEMM, "dX")
    assert_close(to_np(dW), dW_r, TOL_GEMM, "dW")
    assert_close(to_np(ds), ds_r, TOL_RED, "ds")
    assert (to_np(dz) == 0).all()
    # clamped weights now carry their gradient: dW there is dW-hat, not 0
    dwh = orc.linear_dwhat(h["dY"], h["X"])
    assert_close(to_np(dW)[mask == 0], dwh[mask == 0], TOL_GEMM, "dW on clamped weights")
    # the default convention on the same inputs still masks them
    _, dW0, ds0, _ = eqat.fq_linear_bwd(X, W, sd, zd, dY, bits, g)
    assert (to_np(dW0)[mask == 0] == 0).all()


@pytest.mark.parametrize("s16", [False, True], ids=["s32", "s16"])
@pytest.mark.parametrize("shape", SHAPES, ids=IDS)
def test_e2e_backward_with_dz_and_step_storage(orc, shape, s16):
    M, N, K, bits, g, dtype = shape
    d, h = draw(M, N, K, dtype, 800 + M)
    s, z = orc.minmax_init(h["W"], bits, g)
    p_ref, zq_ref = orc.pack(h["W"], s, z, bits, g)
    s2, _ = synthetic.perturb_quant_params(s, z, 800 + M)
    if s16:
        s2 = s2.astype(np.float16)
    codes, zq = torch.from_numpy(p_ref).cuda(), torch.from_numpy(zq_ref).cuda()
    sd = torch.from_numpy(s2).cuda()
    X, dY = d["X"].cuda(), d["dY"].cuda()
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    ws = eqat.workspace(M, N, K, bits, g, tdt)
    Y = eqat.dq_linear_fwd(X, codes, zq, sd, bits, g, ws=ws)
    dX, ds, dz = eqat.dq_linear_bwd(X, codes, zq, sd, dY, bits, g, ws=ws, w_hat_in_ws=True)
    Y_r = orc.dq_linear_fwd(h["X"], p_ref, zq_ref, s2, bits, g)
    dX_r, ds_r, dz_r = orc.dq_linear_bwd(h["X"], p_ref, zq_ref, s2, h["dY"], bits, g)
    assert_close(to_np(Y), Y_r, TOL_GEMM, "Y")
    assert_close(to_np(dX), dX_r, TOL_GEMM, "dX")
    assert_close(to_np(ds), ds_r, TOL_RED, "ds")
    assert_close(to_np(dz), dz_r, TOL_RED, "dz")
    # dz alone (no dX, no ds) runs the weight-side contraction by itself
    _, ds1, dz1 = eqat.dq_linear_bwd(X, codes, zq, sd, dY, bits, g, need_dx=False, need_ds=False)
    assert ds1 is None
    assert_close(to_np(dz1), dz_r, TOL_RED, "dz alone")


@pytest.mark.parametrize("bits,g", [(2, 64), (3, 128), (4, 32)])
def test_fp16_step_dequant_bit_exact(orc, bits, g):
    N, K = 136, 384
    W = synthetic.as_f32_numpy(synthetic.draw_linear(np.random.default_rng(bits), 1, N, K, 0.02, "bf16")["W"])
    s, z = orc.minmax_init(W, bits, g)
    p_ref, zq_ref = orc.pack(W, s, z, bits, g)
    s16 = s.astype(np.float16)
    ref = orc.dequant_packed(p_ref, zq_ref, s16, K, bits, g)
    codes, zq = torch.from_numpy(p_ref).cuda(), torch.from_numpy(zq_ref).cuda()
    sd = torch.from_numpy(s16).cuda()
    assert_bits_equal(to_np(eqat.dequant_codes(codes, zq, sd, K, bits, g, dtype=torch.float32)), ref, "W-hat f32")
    assert_bits_equal(to_np(eqat.dequant_codes(codes, zq, sd, K, bits, g, dtype=torch.bfloat16)),
                      bf16_round(ref), "W-hat bf16")
