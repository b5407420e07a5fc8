"""GPU parity: the CUDA path (through the Python binding and the C ABI) against the
CPU oracle on the same seeded inputs, at sizes that span several tiles and end in
ragged tails, in both quantizer states (min-max init, where nothing is clamped,
and a "trained" state with shrunk steps and shifted zero points, where a few
percent of the weights are clamped)."""
import numpy as np
import pytest
import torch

import weight_quantization_aware_b200 as eqat
from weight_quantization_aware_b200 import synthetic
from parity import TOL_GEMM, TOL_RED, assert_bits_equal, assert_close, bf16_round, to_np

pytestmark = pytest.mark.gpu

BF16_SHAPES = [  # (M, N, K, bits, group)
    (300, 392, 384, 2, 64),
    (128, 256, 256, 3, 128),
    (200, 136, 160, 4, 32),
    (1, 8, 32, 2, 32),
    (257, 520, 640, 2, 128),
]


@pytest.fixture(scope="module", autouse=True)
def built():
    from weight_quantization_aware_b200 import build
    build.build()
    eqat.load_library()
    assert torch.cuda.is_available()
    yield
    assert eqat.device_error() == 0


def inputs(M, N, K, bits, g, dtype, seed, trained, orc):
    d = synthetic.draw_linear(np.random.default_rng(seed), M, N, K, 0.02, dtype)
    Xn, Wn, dYn = (synthetic.as_f32_numpy(d[k]) for k in ("X", "W", "dY"))
    s, z = orc.minmax_init(Wn, bits, g)
    if trained:
        s, z = synthetic.perturb_quant_params(s, z, seed)
        z = z + np.float32(0.375)  # non-integer zero points: round(z) in every forward
    dev = {k: v.cuda() for k, v in d.items()}
    dev["s"] = torch.from_numpy(s).cuda()
    dev["z"] = torch.from_numpy(z).cuda()
    return dev, Xn, Wn, dYn, s, z


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("bits,g", [(2, 32), (2, 64), (2, 128), (3, 128), (3, 64), (4, 32)])
def test_minmax_init_bit_exact(orc, dtype, bits, g):
    rng = np.random.default_rng(bits * 1000 + g)
    d = synthetic.draw_linear(rng, 1, 264, 1024, 0.02, dtype)
    Wn = synthetic.as_f32_numpy(d["W"])
    s_ref, z_ref = orc.minmax_init(Wn, bits, g)
    s, z = eqat.minmax_init(d["W"].cuda(), bits, g)
    assert_bits_equal(to_np(s), s_ref, "s")
    assert_bits_equal(to_np(z), z_ref, "z")


def test_minmax_init_degenerate_groups(orc):
    W = np.zeros((8, 128), np.float32)
    W[0, :64] = 0.25          # constant group: step floor
    W[1, :64] = -0.5          # all negative
    W[1, 64:] = np.linspace(0.1, 0.9, 64)  # all positive
    W[2, :] = np.linspace(-1, 1, 128)
    W[3, ::2] = 1e-3
    Wt = torch.from_numpy(W)
    for dtype in (torch.float32, torch.bfloat16):
        Wd = Wt.to(dtype)
        Wn = Wd.float().numpy()
        s_ref, z_ref = orc.minmax_init(Wn, 2, 64)
        s, z = eqat.minmax_init(Wd.cuda(), 2, 64)
        assert_bits_equal(to_np(s), s_ref, "s")
        assert_bits_equal(to_np(z), z_ref, "z")
        wh_ref, c_ref, m_ref, _ = orc.fake_quant(Wn, s_ref, z_ref, 2, 64)
        wh, c, m = eqat.fake_quant(Wd.cuda(), s, z, 2, 64)
        assert_bits_equal(to_np(c), c_ref, "code")
        assert_bits_equal(to_np(m), m_ref, "mask")


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_codes_for_extreme_step_sizes_bit_exact(orc, bits):
    """Groups whose W/s leaves every fp32 shortcut range: u = W/s between -2.5e7 and
    -1.26e7 (where M + zr + u is negative but its bits, read as an integer and
    reduced by those of M, would wrap around), below -2^31, above 2^22, and plain
    ones beside them.  Codes clamp to 0 or Q exactly as the definition says, in the
    prepass (code, mask, W-hat) and in pack."""
    g = 64
    rng = np.random.default_rng(600 + bits)
    W = rng.standard_normal((8, 8 * g)).astype(np.float32)
    W = torch.from_numpy(W).to(torch.bfloat16).float().numpy()
    Q = (1 << bits) - 1
    steps = np.array([1 / 1.5e7, 1 / 1.9e7, 1e-9, 1e-30, 3e-8, 0.4, 1 / 1.3e7, 2.0], np.float32)
    s = np.tile(steps, (8, 1))
    s = np.roll(s, 3, axis=1) * np.float32(1)
    z = rng.uniform(0, Q, (8, 8)).astype(np.float32)
    Wd, sd, zd = torch.from_numpy(W).to(torch.bfloat16).cuda(), torch.from_numpy(s).cuda(), torch.from_numpy(z).cuda()
    u = W.reshape(8, 8, g) / s[:, :, None]
    assert ((u > -2.5e7) & (u < -1.26e7)).sum() > 100 and (u < -2.0 ** 31).any() and (u > 2.0 ** 22).any()
    wh_ref, c_ref, m_ref, _ = orc.fake_quant(W, s, z, bits, g)
    wh, c, m = eqat.fake_quant(Wd, sd, zd, bits, g)
    assert_bits_equal(to_np(c), c_ref, "code")
    assert_bits_equal(to_np(m), m_ref, "mask")
    assert_bits_equal(to_np(wh), bf16_round(wh_ref), "W_hat")
    p_ref, zq_ref = orc.pack(W, s, z, bits, g)
    p, zq = eqat.pack_codes(Wd, sd, zd, bits, g)
    assert_bits_equal(to_np(zq), zq_ref, "zq")
    assert_bits_equal(to_np(p), p_ref, "packed codes")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("trained", [False, True])
@pytest.mark.parametrize("bits,g", [(2, 64), (3, 128), (4, 32)])
def test_fake_quant_and_pack_bit_exact(orc, dtype, trained, bits, g):
    dev, Xn, Wn, dYn, s, z = inputs(4, 136, 512, bits, g, dtype, 31 + bits, trained, orc)
    wh_ref, c_ref, m_ref, _ = orc.fake_quant(Wn, s, z, bits, g)
    wh, c, m = eqat.fake_quant(dev["W"], dev["s"], dev["z"], bits, g)
    assert_bits_equal(to_np(c), c_ref, "code")
    assert_bits_equal(to_np(m), m_ref, "mask")
    exp_wh = wh_ref if dtype == "f32" else bf16_round(wh_ref)
    assert_bits_equal(to_np(wh), exp_wh, "W_hat")
    if trained:
        assert 0 < m_ref.mean() < 1
    p_ref, zq_ref = orc.pack(Wn, s, z, bits, g)
    p, zq = eqat.pack_codes(dev["W"], dev["s"], dev["z"], bits, g)
    assert_bits_equal(to_np(p), p_ref, "packed codes")
    assert_bits_equal(to_np(zq), zq_ref, "zq")
    dq_ref = orc.dequant_packed(p_ref, zq_ref, s, 512, bits, g)
    for odt in (torch.float32, torch.bfloat16):
        dq = eqat.dequant_codes(p, zq, dev["s"], 512, bits, g, odt)
        assert_bits_equal(to_np(dq), dq_ref if odt == torch.float32 else bf16_round(dq_ref), "dequant")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("N,K,bits,g", [(8, 96, 2, 32), (8, 640, 3, 128), (40, 1152, 4, 64), (40, 1184, 2, 32),
                                        (72, 4160, 2, 64)])
def test_quantizer_ragged_tiles_bit_exact(orc, dtype, N, K, bits, g):
    """Prepass, pack and dequant where the weight count is not a whole number of the
    kernels' tiles (and one layer below a single tile), in both quantizer states."""
    for trained in (False, True):
        d = synthetic.draw_linear(np.random.default_rng(N * K + bits), 1, N, K, 0.02, dtype)
        Wn = synthetic.as_f32_numpy(d["W"])
        s, z = orc.minmax_init(Wn, bits, g)
        if trained:
            s, z = synthetic.perturb_quant_params(s, z, N + K)
        W, sd, zd = d["W"].cuda(), torch.from_numpy(s).cuda(), torch.from_numpy(z).cuda()
        wh_ref, c_ref, m_ref, _ = orc.fake_quant(Wn, s, z, bits, g)
        wh, c, m = eqat.fake_quant(W, sd, zd, bits, g)
        assert_bits_equal(to_np(c), c_ref, "code")
        assert_bits_equal(to_np(m), m_ref, "mask")
        assert_bits_equal(to_np(wh), wh_ref if dtype == "f32" else bf16_round(wh_ref), "W_hat")
        wh_only, _, _ = eqat.fake_quant(W, sd, zd, bits, g, want_code=False, want_mask=False)
        assert_bits_equal(to_np(wh_only), to_np(wh), "W_hat without codes")
        p_ref, zq_ref = orc.pack(Wn, s, z, bits, g)
        p, zq = eqat.pack_codes(W, sd, zd, bits, g)
        assert_bits_equal(to_np(p), p_ref, "packed codes")
        assert_bits_equal(to_np(zq), zq_ref, "zq")
        dq = eqat.dequant_codes(p, zq, sd, K, bits, g, torch.float32)
        assert_bits_equal(to_np(dq), orc.dequant_packed(p_ref, zq_ref, s, K, bits, g), "dequant")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("bits,g", [(2, 64), (3, 128), (4, 32)])
def test_multi_layer_init_and_pack_bit_exact(orc, dtype, bits, g):
    """min-max init and pack of several layers in one call (tiles and units
    numbered through the layers, one launch per eight layers): the results of
    every layer equal the oracle's, bit for bit.  Eleven layers (two launches),
    of unlike shapes: one below a single warp tile, ragged tile counts, an empty
    layer in the middle, and one whose rows are the concatenation of two others."""
    shapes = [(8, 256), (40, 1152), (72, 4224), (16, 128), (0, 512), (264, 1024), (8, 128 * 5),
              (136, 512), (48, 2048), (24, 384), (16, 1024)]
    rng = np.random.default_rng(800 + bits + g)
    Ws, Wns = [], []
    for i, (N, K) in enumerate(shapes):
        d = synthetic.draw_linear(rng, 1, N, K, 0.02, dtype)
        Ws.append(d["W"].cuda())
        Wns.append(synthetic.as_f32_numpy(d["W"]))
    ss, zs = eqat.minmax_init_multi(Ws, bits, g)
    refs = [orc.minmax_init(Wn, bits, g) if Wn.size else (np.zeros((0, Wn.shape[1] // g), np.float32),) * 2
            for Wn in Wns]
    for i, (s_ref, z_ref) in enumerate(refs):
        assert_bits_equal(to_np(ss[i]), s_ref, f"s[{i}]")
        assert_bits_equal(to_np(zs[i]), z_ref, f"z[{i}]")
    # trained-state steps on every other layer, so clamped codes occur too
    sp, zp = [], []
    for i, (s_ref, z_ref) in enumerate(refs):
        if i % 2 and s_ref.size:
            s_ref, z_ref = synthetic.perturb_quant_params(s_ref, z_ref, i)
        sp.append(s_ref)
        zp.append(z_ref)
    codes, zqs = eqat.pack_codes_multi(Ws, [torch.from_numpy(a).cuda() for a in sp],
                                       [torch.from_numpy(a).cuda() for a in zp], bits, g)
    for i, Wn in enumerate(Wns):
        if not Wn.size:
            assert codes[i].numel() == 0
            continue
        p_ref, zq_ref = orc.pack(Wn, sp[i], zp[i], bits, g)
        assert_bits_equal(to_np(codes[i]), p_ref, f"codes[{i}]")
        assert_bits_equal(to_np(zqs[i]), zq_ref, f"zq[{i}]")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_w_hat_outputs_aligned_to_16_bytes_only(orc, dtype):
    """W-hat written into a buffer that starts 16 bytes past a 32-byte boundary (the
    ABI asks for 16): the prepass and the dequantize kernel then store each 16-weight
    chunk as two 16-byte halves instead of one 32-byte store.  Both give the oracle's
    values, bit for bit, and leave the bytes around the view untouched."""
    N, K, bits, g = 40, 1152, 2, 64
    d = synthetic.draw_linear(np.random.default_rng(77), 1, N, K, 0.02, dtype)
    Wn = synthetic.as_f32_numpy(d["W"])
    s, z = synthetic.perturb_quant_params(*orc.minmax_init(Wn, bits, g), 5)
    W, sd, zd = d["W"].cuda(), torch.from_numpy(s).cuda(), torch.from_numpy(z).cuda()
    wh_ref = orc.fake_quant(Wn, s, z, bits, g)[0]
    p_ref, zq_ref = orc.pack(Wn, s, z, bits, g)
    p, zq = eqat.pack_codes(W, sd, zd, bits, g)
    tdt = W.dtype
    shift = 16 // W.element_size()
    for which in ("fake_quant", "dequant"):
        buf = torch.full((N * K + 2 * shift,), 7.0, dtype=tdt, device="cuda")
        view = buf[shift:shift + N * K].view(N, K)
        assert view.data_ptr() % 32 == 16
        if which == "fake_quant":
            eqat.fake_quant(W, sd, zd, bits, g, want_code=False, want_mask=False, W_hat=view)
            ref = wh_ref
        else:
            eqat.dequant_codes(p, zq, sd, K, bits, g, out=view)
            ref = orc.dequant_packed(p_ref, zq_ref, s, K, bits, g)
        assert_bits_equal(to_np(view), ref if dtype == "f32" else bf16_round(ref), which)
        edge = to_np(buf)
        assert (edge[:shift] == 7.0).all() and (edge[shift + N * K:] == 7.0).all(), f"{which} wrote outside its view"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_codes_at_and_around_rounding_boundaries_bit_exact(orc, dtype, bits):
    """Weights on, and one or two ulps either side of, half-integer multiples of s:
    the cases where the kernels' reciprocal-multiply decision must hand over to the
    exact one (a residual test against the half-integer, the IEEE division where that
    cannot decide) to reproduce round(W/s)."""
    Q = (1 << bits) - 1
    rng = np.random.default_rng(4321 + bits)
    N, K, g = 64, 512, 32
    z = rng.integers(-1, Q + 2, size=(N, K // g)).astype(np.float32)
    j = rng.integers(-Q - 3, Q + 3, size=(N, K)).astype(np.float32)
    off = rng.integers(-2, 3, size=(N, K))
    if dtype == "f32":
        s = rng.uniform(1e-3, 0.1, size=(N, K // g)).astype(np.float32)
        W = ((j + np.float32(0.5)) * np.repeat(s, g, 1)).astype(np.float32)
        for step in (1, 2):
            W = np.where(off >= step, np.nextafter(W, np.float32(np.inf)), W)
            W = np.where(off <= -step, np.nextafter(W, np.float32(-np.inf)), W)
        Wt = torch.from_numpy(W.astype(np.float32))
    else:
        # s with at most two significant bits keeps (j + 1/2) s exact in bf16; the
        # offsets then step the bf16 bit pattern by one or two units.
        s = (rng.choice([1.0, 3.0], size=(N, K // g)) * 2.0 ** rng.integers(-12, -4, size=(N, K // g))).astype(np.float32)
        W = ((j + np.float32(0.5)) * np.repeat(s, g, 1)).astype(np.float32)
        Wb = torch.from_numpy(W).to(torch.bfloat16)
        assert np.array_equal(Wb.float().numpy(), W)
        pattern = Wb.view(torch.int16).numpy().astype(np.int32) + off
        Wt = torch.from_numpy(pattern.astype(np.int16)).view(torch.bfloat16)
    Wn = Wt.float().numpy()
    _, c_ref, m_ref, u_ref = orc.fake_quant(Wn, s, z, bits, g)
    frac = np.abs(u_ref - np.floor(u_ref) - 0.5)
    assert (frac == 0).sum() > 50  # exact ties present
    sd, zd = torch.from_numpy(s).cuda(), torch.from_numpy(z).cuda()
    _, c, m = eqat.fake_quant(Wt.cuda(), sd, zd, bits, g, want_w_hat=False)
    assert_bits_equal(to_np(c), c_ref, "codes")
    assert_bits_equal(to_np(m), m_ref, "mask")
    p_ref, zq_ref = orc.pack(Wn, s, z, bits, g)
    p, zq = eqat.pack_codes(Wt.cuda(), sd, zd, bits, g)
    assert_bits_equal(to_np(p), p_ref, "packed")
    if dtype == "bf16":
        X = torch.randn(64, K).to(torch.bfloat16)
        dY = torch.randn(64, N).to(torch.bfloat16)
        dX, dW, ds, dz = eqat.fq_linear_bwd(X.cuda(), Wt.cuda(), sd, zd, dY.cuda(), bits, g)
        dX_r, dW_r, ds_r, dz_r = orc.fq_linear_bwd(X.float().numpy(), Wn, s, z, dY.float().numpy(), bits, g)
        assert (to_np(dW)[m_ref == 0] == 0).all() and (dW_r[m_ref == 0] == 0).all()
        assert ((to_np(dW) != 0) == (dW_r != 0)).mean() > 0.999
        assert_close(to_np(ds), ds_r, TOL_RED, "ds")
        assert_close(to_np(dz), dz_r, TOL_RED, "dz")


def check_fq(orc, M, N, K, bits, g, dtype, seed, trained, reuse=False):
    dev, Xn, Wn, dYn, s, z = inputs(M, N, K, bits, g, dtype, seed, trained, orc)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    ws = eqat.workspace(M, N, K, bits, g, tdt) if reuse else None
    Y = eqat.fq_linear_fwd(dev["X"], dev["W"], dev["s"], dev["z"], bits, g, ws=ws)
    dX, dW, ds, dz = eqat.fq_linear_bwd(dev["X"], dev["W"], dev["s"], dev["z"], dev["dY"], bits, g,
                                        ws=ws, w_hat_in_ws=reuse)
    Y_ref = orc.fq_linear_fwd(Xn, Wn, s, z, bits, g)
    dX_ref, dW_ref, ds_ref, dz_ref = orc.fq_linear_bwd(Xn, Wn, s, z, dYn, bits, g)
    assert_close(to_np(Y), Y_ref, TOL_GEMM, "Y")
    assert_close(to_np(dX), dX_ref, TOL_GEMM, "dX")
    assert_close(to_np(dW), dW_ref, TOL_GEMM, "dW")
    # the straight-through mask is an integer decision: clamped weights get exactly 0
    _, _, m_ref, _ = orc.fake_quant(Wn, s, z, bits, g)
    assert (to_np(dW)[m_ref == 0] == 0).all()
    assert_close(to_np(ds), ds_ref, TOL_RED, "ds")
    if np.abs(dz_ref).max() == 0:
        assert (to_np(dz) == 0).all()
    else:
        assert_close(to_np(dz), dz_ref, TOL_RED, "dz")
    return m_ref


@pytest.mark.parametrize("trained", [False, True])
@pytest.mark.parametrize("shape", BF16_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_fq_linear_bf16_tensor_core(orc, shape, trained):
    M, N, K, bits, g = shape
    check_fq(orc, M, N, K, bits, g, "bf16", 100 + M + K, trained)


@pytest.mark.parametrize("trained", [False, True])
@pytest.mark.parametrize("shape", [(128, 512, 256, 2, 64), (77, 24, 96, 3, 32), (5, 64, 128, 4, 128)],
                         ids=lambda s: "x".join(map(str, s)))
def test_fq_linear_f32(orc, shape, trained):
    M, N, K, bits, g = shape
    check_fq(orc, M, N, K, bits, g, "f32", 200 + M, trained)


def check_dq(orc, M, N, K, bits, g, dtype, seed, reuse=False):
    dev, Xn, Wn, dYn, s, z = inputs(M, N, K, bits, g, dtype, seed, False, orc)
    p_ref, zq_ref = orc.pack(Wn, s, z, bits, g)
    s2, _ = synthetic.perturb_quant_params(s, z, seed)  # E2E-QP has moved the steps
    codes = torch.from_numpy(p_ref).cuda()
    zq = torch.from_numpy(zq_ref).cuda()
    s2d = torch.from_numpy(s2).cuda()
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    ws = eqat.workspace(M, N, K, bits, g, tdt) if reuse else None
    Y = eqat.dq_linear_fwd(dev["X"], codes, zq, s2d, bits, g, ws=ws)
    dX, ds = eqat.dq_linear_bwd_s(dev["X"], codes, zq, s2d, dev["dY"], bits, g, ws=ws, w_hat_in_ws=reuse)
    Y_ref = orc.dq_linear_fwd(Xn, p_ref, zq_ref, s2, bits, g)
    dX_ref, ds_ref = orc.dq_linear_bwd_s(Xn, p_ref, zq_ref, s2, dYn, bits, g)
    assert_close(to_np(Y), Y_ref, TOL_GEMM, "Y")
    assert_close(to_np(dX), dX_ref, TOL_GEMM, "dX")
    assert_close(to_np(ds), ds_ref, TOL_RED, "ds")


@pytest.mark.parametrize("shape", BF16_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_dq_linear_bf16_tensor_core(orc, shape):
    M, N, K, bits, g = shape
    check_dq(orc, M, N, K, bits, g, "bf16", 300 + M)


@pytest.mark.parametrize("shape", [(128, 512, 256, 2, 64), (33, 40, 96, 3, 32)], ids=lambda s: "x".join(map(str, s)))
def test_dq_linear_f32(orc, shape):
    M, N, K, bits, g = shape
    check_dq(orc, M, N, K, bits, g, "f32", 400 + M)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [(300, 392, 384, 2, 64), (96, 136, 256, 3, 128)], ids=lambda s: "x".join(map(str, s)))
def test_backward_reuses_forward_w_hat(orc, shape, dtype):
    """Training flow: the backward skips its prepass and reads the W-hat the forward
    left in the shared workspace."""
    M, N, K, bits, g = shape
    check_fq(orc, M, N, K, bits, g, dtype, 500 + M, True, reuse=True)
    check_dq(orc, M, N, K, bits, g, dtype, 600 + M, reuse=True)


def test_backward_single_contraction_paths(orc):
    """dX alone and the weight side alone each launch one contraction."""
    M, N, K, bits, g = 200, 264, 320, 2, 64
    dev, Xn, Wn, dYn, s, z = inputs(M, N, K, bits, g, "bf16", 9, True, orc)
    dX_ref, dW_ref, ds_ref, dz_ref = orc.fq_linear_bwd(Xn, Wn, s, z, dYn, bits, g)
    dX, dW, ds, dz = eqat.fq_linear_bwd(dev["X"], dev["W"], dev["s"], dev["z"], dev["dY"], bits, g,
                                        need_dw=False, need_ds=False, need_dz=False)
    assert dW is None and ds is None and dz is None
    assert_close(to_np(dX), dX_ref, TOL_GEMM, "dX only")
    dX, dW, ds, dz = eqat.fq_linear_bwd(dev["X"], dev["W"], dev["s"], dev["z"], dev["dY"], bits, g,
                                        need_dx=False, need_dw=False)
    assert dX is None and dW is None
    assert_close(to_np(ds), ds_ref, TOL_RED, "ds only")
    assert_close(to_np(dz), dz_ref, TOL_RED, "dz only")
    p_ref, zq_ref = orc.pack(Wn, s, z, bits, g)
    codes, zq = torch.from_numpy(p_ref).cuda(), torch.from_numpy(zq_ref).cuda()
    dX2_ref, ds2_ref = orc.dq_linear_bwd_s(Xn, p_ref, zq_ref, s, dYn, bits, g)
    dX2, ds2 = eqat.dq_linear_bwd_s(dev["X"], codes, zq, dev["s"], dev["dY"], bits, g, need_ds=False)
    assert ds2 is None
    assert_close(to_np(dX2), dX2_ref, TOL_GEMM, "E2E dX only")
    dX2, ds2 = eqat.dq_linear_bwd_s(dev["X"], codes, zq, dev["s"], dev["dY"], bits, g, need_dx=False)
    assert dX2 is None
    assert_close(to_np(ds2), ds2_ref, TOL_RED, "E2E ds only")


@pytest.mark.parametrize("shape", [
    (1024, 520, 2048, 2, 64),    # fewer tiles than SMs, long K
    (1024, 1024, 1024, 3, 128),  # grouped backward with one partial wave
    (520, 256, 1536, 2, 32),     # ragged M and N tails, long K
    (256, 4096, 2048, 2, 64),    # grouped backward whose dX tiles are 16x deeper than its dW-hat tiles
    (4096, 256, 1024, 2, 64),    # and the other way round
], ids=lambda s: "x".join(map(str, s)))
def test_long_k_partial_wave_launches(orc, shape):
    """Launches of fewer tiles than SMs with long reductions, twice in a row on one
    workspace (store, straight-through and E2E-QP ds epilogues)."""
    M, N, K, bits, g = shape
    check_fq(orc, M, N, K, bits, g, "bf16", 700 + M, True)
    check_dq(orc, M, N, K, bits, g, "bf16", 800 + M)
    dev, Xn, Wn, dYn, s, z = inputs(M, N, K, bits, g, "bf16", 900 + M, True, orc)
    ws = eqat.workspace(M, N, K, bits, g, torch.bfloat16)
    ref = orc.fq_linear_fwd(Xn, Wn, s, z, bits, g)
    for _ in range(2):
        Y = eqat.fq_linear_fwd(dev["X"], dev["W"], dev["s"], dev["z"], bits, g, ws=ws)
        assert_close(to_np(Y), ref, TOL_GEMM, "Y (repeat)")


def test_persistent_tiles_wrap_accumulator_ring(orc):
    """More than two output tiles per CTA (the double-buffered accumulator ring wraps
    several times), checked on sampled rows."""
    M, N, K, bits, g = 4864, 4096, 256, 2, 64  # fwd: 38 x 16 = 608 tiles on 148 SMs
    dev, Xn, Wn, dYn, s, z = inputs(M, N, K, bits, g, "bf16", 77, True, orc)
    Y = eqat.fq_linear_fwd(dev["X"], dev["W"], dev["s"], dev["z"], bits, g)
    dX, dW, ds, dz = eqat.fq_linear_bwd(dev["X"], dev["W"], dev["s"], dev["z"], dev["dY"], bits, g)
    rows = np.r_[0, 1, 127, 128, 2047, 2048, np.random.default_rng(0).integers(0, M, 40), M - 1]
    wrows = np.r_[0, 255, 256, 1000, N - 1, np.random.default_rng(1).integers(0, N, 27)]
    wh = orc.fake_quant(Wn, s, z, bits, g)[0]
    assert_close(to_np(Y)[rows], orc.linear_fwd(Xn, wh, rows), TOL_GEMM, "Y rows")
    assert_close(to_np(dX)[rows], orc.linear_dx(dYn, wh, rows), TOL_GEMM, "dX rows")
    dwh = orc.linear_dwhat(dYn, Xn, wrows)
    dW_ref, ds_ref, dz_ref = orc.ste_grads(Wn, s, z, dwh, bits, g, wrows)
    assert_close(to_np(dW)[wrows], dW_ref, TOL_GEMM, "dW rows")
    assert_close(to_np(ds)[wrows], ds_ref, TOL_RED, "ds rows")
    assert_close(to_np(dz)[wrows], dz_ref, TOL_RED, "dz rows")


def test_empty_and_degenerate_problems(orc):
    dev = "cuda"
    bf = torch.bfloat16
    # M == 0: Y and dX are empty; the weight gradients are exact zeros
    X = torch.empty(0, 64, dtype=bf, device=dev)
    W = torch.randn(16, 64, device=dev).to(bf)
    s, z = eqat.minmax_init(W, 2, 64)
    dY = torch.empty(0, 16, dtype=bf, device=dev)
    assert eqat.fq_linear_fwd(X, W, s, z, 2, 64).shape == (0, 16)
    dX, dW, ds, dz = eqat.fq_linear_bwd(X, W, s, z, dY, 2, 64)
    assert dX.shape == (0, 64)
    assert (dW == 0).all() and (ds == 0).all() and (dz == 0).all()
    dX2, ds2 = eqat.dq_linear_bwd_s(X, *eqat.pack_codes(W, s, z, 2, 64), s, dY, 2, 64)
    assert (ds2 == 0).all()
    # N == 0: Y empty, dX exact zeros
    X = torch.randn(8, 64, device=dev).to(bf)
    W0 = torch.empty(0, 64, dtype=bf, device=dev)
    s0, z0 = eqat.minmax_init(W0, 2, 64)
    dY0 = torch.empty(8, 0, dtype=bf, device=dev)
    assert eqat.fq_linear_fwd(X, W0, s0, z0, 2, 64).shape == (8, 0)
    dX, dW, ds, dz = eqat.fq_linear_bwd(X, W0, s0, z0, dY0, 2, 64)
    assert (dX == 0).all()
    # optional outputs skipped
    dX, dW, ds, dz = eqat.fq_linear_bwd(X, W, s, z, torch.randn(8, 16, device=dev).to(bf), 2, 64,
                                        need_dx=False, need_dw=False, need_dz=False)
    assert dX is None and dW is None and dz is None and ds is not None
    torch.cuda.synchronize()


def test_bounded_wait_reports_timeout_and_context_survives():
    assert eqat.device_error() == 0
    eqat.selftest_bounded_wait(50_000_000)  # 50 ms
    with pytest.raises(eqat.EqatError) as ei:
        eqat.device_error()
    assert ei.value.status == eqat.EQAT_ERR_TIMEOUT
    assert eqat.device_error() == 0  # read-and-clear
    W = torch.randn(8, 64, device="cuda").to(torch.bfloat16)
    s, z = eqat.minmax_init(W, 2, 64)
    torch.cuda.synchronize()
    assert torch.isfinite(s).all()
