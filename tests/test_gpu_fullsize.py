"""Parity at the full sizes of the five workloads (Llama-2 7B/13B/70B shapes), through
the same entry points and launch configuration bench.py times.

Integer outputs (codes, masks, packed bytes, zero points) and the fp32 min-max init
are compared bit for bit over every weight.  The contractions are compared on
sampled outputs the oracle computes one by one: token rows of Y and dX, and whole
weight rows of dW, ds, dz (including the rows that hold the most outliers)."""
import numpy as np
import pytest
import torch

import weight_quantization_aware_b200 as eqat
from weight_quantization_aware_b200 import synthetic
from parity import TOL_GEMM, TOL_RED, assert_bits_equal, assert_close, bf16_round, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from weight_quantization_aware_b200 import build
    build.build()
    eqat.load_library()
    yield
    assert eqat.device_error() == 0


def sample_rows(n, count, seed, must=()):
    rng = np.random.default_rng(seed)
    rows = set(int(r) for r in must)
    rows |= {0, n - 1}
    rows |= set(int(r) for r in rng.choice(n, size=min(n, count), replace=False))
    return np.array(sorted(rows), dtype=np.int64)


def outlier_rows(Wn, count):
    big = (np.abs(Wn) > 8 * np.abs(Wn).std()).sum(1)
    return np.argsort(-big, kind="stable")[:count]


def check_blockap_linear(orc, wl, li, trained, nrows):
    d = synthetic.workload_linear(wl, li)
    Xn, Wn, dYn = (synthetic.as_f32_numpy(d[k]) for k in ("X", "W", "dY"))
    X, W, dY = (d[k].cuda() for k in ("X", "W", "dY"))
    bits, g = wl.bits, wl.group
    M, K = Xn.shape
    N = Wn.shape[0]

    s_ref, z_ref = orc.minmax_init(Wn, bits, g)
    s, z = eqat.minmax_init(W, bits, g)
    assert_bits_equal(to_np(s), s_ref, "s")
    assert_bits_equal(to_np(z), z_ref, "z")
    if trained:
        s_ref, z_ref = synthetic.perturb_quant_params(s_ref, z_ref, 1000 + li)
        s, z = torch.from_numpy(s_ref).cuda(), torch.from_numpy(z_ref).cuda()

    wh_ref, c_ref, m_ref, _ = orc.fake_quant(Wn, s_ref, z_ref, bits, g)
    wh, c, m = eqat.fake_quant(W, s, z, bits, g)
    assert_bits_equal(to_np(c), c_ref, "codes")
    assert_bits_equal(to_np(m), m_ref, "mask")
    assert_bits_equal(to_np(wh), bf16_round(wh_ref) if wl.dtype == "bf16" else wh_ref, "W_hat")
    del wh, c, m

    p_ref, zq_ref = orc.pack(Wn, s_ref, z_ref, bits, g)
    p, zq = eqat.pack_codes(W, s, z, bits, g)
    assert_bits_equal(to_np(p), p_ref, "packed")
    assert_bits_equal(to_np(zq), zq_ref, "zq")
    del p, zq

    Y = eqat.fq_linear_fwd(X, W, s, z, bits, g)
    rows = sample_rows(M, nrows, 1 + li)
    assert_close(to_np(Y)[rows], orc.linear_fwd(Xn, wh_ref, rows), TOL_GEMM, "Y rows")
    del Y
    dX, dW, ds, dz = eqat.fq_linear_bwd(X, W, s, z, dY, bits, g)
    assert_close(to_np(dX)[rows], orc.linear_dx(dYn, wh_ref, rows), TOL_GEMM, "dX rows")
    wrows = sample_rows(N, nrows, 2 + li, must=outlier_rows(Wn, 4))
    dwh = orc.linear_dwhat(dYn, Xn, wrows)
    dW_ref, ds_ref, dz_ref = orc.ste_grads(Wn, s_ref, z_ref, dwh, bits, g, wrows)
    dW_s = to_np(dW[torch.from_numpy(wrows).cuda()])
    assert_close(dW_s, dW_ref, TOL_GEMM, "dW rows")
    assert (dW_s[m_ref[wrows] == 0] == 0).all()
    assert_close(to_np(ds)[wrows], ds_ref, TOL_RED, "ds rows")
    if np.abs(dz_ref).max() == 0:
        assert (to_np(dz)[wrows] == 0).all()
    else:
        assert_close(to_np(dz)[wrows], dz_ref, TOL_RED, "dz rows")
    if trained:
        assert (m_ref == 0).mean() > 0.01


def check_e2e_linear(orc, wl, li, nrows):
    d = synthetic.workload_linear(wl, li)
    Xn, Wn, dYn = (synthetic.as_f32_numpy(d[k]) for k in ("X", "W", "dY"))
    X, W, dY = (d[k].cuda() for k in ("X", "W", "dY"))
    bits, g = wl.bits, wl.group
    M, K = Xn.shape
    N = Wn.shape[0]
    # frozen codes from min-max init and pack of W (the oracle's; the GPU pack must agree)
    s_ref, z_ref = orc.minmax_init(Wn, bits, g)
    p_ref, zq_ref = orc.pack(Wn, s_ref, z_ref, bits, g)
    p, zq = eqat.pack_codes(W, torch.from_numpy(s_ref).cuda(), torch.from_numpy(z_ref).cuda(), bits, g)
    assert_bits_equal(to_np(p), p_ref, "packed")
    assert_bits_equal(to_np(zq), zq_ref, "zq")
    s2, _ = synthetic.perturb_quant_params(s_ref, z_ref, 2000 + li)  # steps moved by E2E-QP
    s2d = torch.from_numpy(s2).cuda()
    wh_ref = orc.dequant_packed(p_ref, zq_ref, s2, K, bits, g)
    Y = eqat.dq_linear_fwd(X, p, zq, s2d, bits, g)
    rows = sample_rows(M, nrows, 3 + li)
    assert_close(to_np(Y)[rows], orc.linear_fwd(Xn, wh_ref, rows), TOL_GEMM, "Y rows")
    del Y
    dX, ds = eqat.dq_linear_bwd_s(X, p, zq, s2d, dY, bits, g)
    assert_close(to_np(dX)[rows], orc.linear_dx(dYn, wh_ref, rows), TOL_GEMM, "dX rows")
    wrows = sample_rows(N, nrows, 4 + li)
    dwh = orc.linear_dwhat(dYn, Xn, wrows)
    ds_ref = orc.e2e_ds(p_ref, zq_ref, dwh, K, bits, g, wrows)
    assert_close(to_np(ds)[wrows], ds_ref, TOL_RED, "ds rows")


@pytest.mark.parametrize("trained", [False, True])
def test_cfg1_single_linear_fp32_full(orc, trained):
    wl = synthetic.WORKLOADS[1]
    check_blockap_linear(orc, wl, 0, trained, nrows=wl.m)


@pytest.mark.parametrize("trained", [False, True])
def test_cfg2_llama2_7b_q_proj_w2g64(orc, trained):
    wl = synthetic.WORKLOADS[2]
    check_blockap_linear(orc, wl, 0, trained, nrows=48)
    check_e2e_linear(orc, wl, 0, nrows=48)  # bench.py's step also runs E2E-QP on this layer


@pytest.mark.parametrize("li", [0, 1, 2])
def test_cfg3_llama2_7b_mlp_w3g128(orc, li):
    wl = synthetic.WORKLOADS[3]
    check_blockap_linear(orc, wl, li, trained=(li == 0), nrows=24)


@pytest.mark.parametrize("li", [0, 1, 2, 3, 4])
def test_cfg4_llama2_13b_e2e_w2g64(orc, li):
    wl = synthetic.WORKLOADS[4]
    check_e2e_linear(orc, wl, li, nrows=24)


@pytest.mark.parametrize("li", [0, 1, 2, 3, 4, 5, 6])
def test_cfg5_llama2_70b_block_w2g64(orc, li):
    wl = synthetic.WORKLOADS[5]
    check_blockap_linear(orc, wl, li, trained=(li == 1), nrows=12)
