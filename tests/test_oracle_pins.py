"""Pins for the CPU oracle, independent of the oracle itself (CPU only).

Each test checks the oracle against something the pages or the mathematics fix:
hand-derived worked cases of the closed forms (tests/golden), invariants the
pages state (group endpoints on the first and last codes, 2^N affine levels with
0 representable, exact dW-hat/ds = W_q - z), textbook routines (NumPy matmul for
the three contractions), an independent autograd re-derivation of the
straight-through backward, finite differences, and brute force on tiny shapes.
"""
import json
import os

import numpy as np
import pytest
import torch

from weight_quantization_aware_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def unpack_codes(packed, K, bits):
    """Independent reader of the packed layout: 2-bit = 4 codes/byte (code k at bits
    2*(k%4)), 4-bit = 2 codes/byte (bits 4*(k%2)), 3-bit = one code per byte."""
    packed = np.asarray(packed, dtype=np.uint8)
    if bits == 3:
        return packed.copy()
    per = 8 // bits
    out = np.zeros((packed.shape[0], K), np.uint8)
    for k in range(K):
        out[:, k] = (packed[:, k // per] >> (bits * (k % per))) & ((1 << bits) - 1)
    return out


def rand_w(n, k, seed, sigma=0.02):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((n, k)) * sigma).astype(np.float32)
    return w


# ---------------------------------------------------------------- golden cases

def golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", golden_cases(), ids=lambda c: c["name"])
def test_golden_worked_examples(orc, case):
    bits, g = case["bits"], case["group"]
    if "W" in case:
        W = np.array(case["W"], np.float32)
        if "init" in case:
            s, z = orc.minmax_init(W, bits, g)
            np.testing.assert_array_equal(s, np.array(case["init"]["s"], np.float32))
            np.testing.assert_array_equal(z, np.array(case["init"]["z"], np.float32))
        else:
            s, z = np.array(case["s"], np.float32), np.array(case["z"], np.float32)
        wh, code, mask, _ = orc.fake_quant(W, s, z, bits, g)
        np.testing.assert_array_equal(code, np.array(case["codes"], np.uint8))
        np.testing.assert_array_equal(mask, np.array(case["mask"], np.uint8))
        np.testing.assert_array_equal(wh, np.array(case["W_hat"], np.float32))
        for key in ("packed_w2", "packed_w3"):
            if key in case:
                packed, zq = orc.pack(W, s, z, bits, g)
                np.testing.assert_array_equal(packed, np.array(case[key], np.uint8))
                np.testing.assert_array_equal(zq, np.array(case["zq"], np.uint8))
        if "layer" in case:
            L = case["layer"]
            X = np.array(L["X"], np.float32)
            dY = np.array(L["dY"], np.float32)
            np.testing.assert_array_equal(orc.fq_linear_fwd(X, W, s, z, bits, g), np.array(L["Y"]))
            dX, dW, ds, dz = orc.fq_linear_bwd(X, W, s, z, dY, bits, g)
            np.testing.assert_array_equal(dX, np.array(L["dX"]))
            np.testing.assert_array_equal(orc.linear_dwhat(dY, X), np.array(L["dW_hat"]))
            np.testing.assert_array_equal(dW, np.array(L["dW"]))
            np.testing.assert_array_equal(ds, np.array(L["ds"]))
            np.testing.assert_array_equal(dz, np.array(L["dz"]))
    else:  # E2E case on frozen packed codes
        packed = np.array(case["packed_w2"], np.uint8)
        zq = np.array(case["zq"], np.uint8)
        s = np.array(case["s"], np.float32)
        K = case["K"]
        np.testing.assert_array_equal(orc.dequant_packed(packed, zq, s, K, bits, g),
                                      np.array(case["W_hat"], np.float32))
        L = case["layer"]
        X = np.array(L["X"], np.float32)
        dY = np.array(L["dY"], np.float32)
        np.testing.assert_array_equal(orc.dq_linear_fwd(X, packed, zq, s, bits, g), np.array(L["Y"]))
        dX, ds = orc.dq_linear_bwd_s(X, packed, zq, s, dY, bits, g)
        np.testing.assert_array_equal(dX, np.array(L["dX"]))
        np.testing.assert_array_equal(ds, np.array(L["ds"]))


# ---------------------------------------------------------------- init invariants

@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("bits,g", [(2, 32), (2, 64), (2, 128), (3, 128), (3, 64), (4, 64)])
def test_minmax_endpoints_land_on_first_and_last_codes(orc, bits, g, bf16):
    """Phase 1 init: group min lands on code 0, group max on code 2^N-1 (or Q-1 at an
    exact half-way tie), both within s/2 of the grid.  bf16 weights sit on a coarse
    grid, so exact ties of W/s at .5 are common there."""
    Q = (1 << bits) - 1
    W = rand_w(96, 512, 11 + bits + g)
    if bf16:
        W = synthetic.as_f32_numpy(synthetic.to_dtype(W, "bf16"))
    s, z = orc.minmax_init(W, bits, g)
    wh, code, mask, u = orc.fake_quant(W, s, z, bits, g)
    G = 512 // g
    Wg = W.reshape(96, G, g)
    ci = code.reshape(96, G, g)
    ui = u.reshape(96, G, g)
    whg = wh.reshape(96, G, g)
    imin = Wg.argmin(-1)
    imax = Wg.argmax(-1)
    take = lambda a, i: np.take_along_axis(a, i[..., None], -1)[..., 0]
    assert (take(ci, imin) == 0).all()
    cmax = take(ci, imax)
    umax = take(ui, imax)
    tie = np.abs(umax - np.floor(umax) - 0.5) == 0
    assert ((cmax == Q) | (tie & (cmax == Q - 1))).all()
    assert (s > 0).all()
    # s/2, plus Q times the one rounding of s = (xmax - xmin)/Q (relative 2^-24), doubled
    tol = s * (0.5 + Q * 2.0 ** -23)
    assert (np.abs(take(whg, imin) - Wg.min(-1)) <= tol).all()
    assert (np.abs(take(whg, imax) - Wg.max(-1)) <= tol).all()
    # With xmin < 0 < xmax, min-max init clamps nothing except, at a half-way tie, the
    # group maximum: xmax/s - xmin/s is Q up to one rounding of s, and when one of the
    # two quotients sits exactly on .5 and rounds up (to even) while the other also
    # rounds up, round(xmax/s) + round(-xmin/s) reaches Q + 1.
    mixed = (Wg.min(-1) < 0) & (Wg.max(-1) > 0)
    assert ((z >= 0) & (z <= Q))[mixed].all()
    q = np.rint(ui) + z[..., None]
    clamped = (mask.reshape(96, G, g) == 0) & mixed[..., None]
    assert (q[clamped] == Q + 1).all()
    assert (Wg[clamped] == np.broadcast_to(Wg.max(-1, keepdims=True), Wg.shape)[clamped]).all()
    assert clamped.sum() <= mixed.sum()


def test_init_matches_numpy_fp32_brute_force(orc):
    W = rand_w(40, 256, 3)
    for bits, g in [(2, 64), (3, 128), (4, 32)]:
        s, z = orc.minmax_init(W, bits, g)
        Wg = W.reshape(40, -1, g)
        rng_ = (Wg.max(-1) - Wg.min(-1)).astype(np.float32)
        s_ref = np.maximum(np.float32(rng_) / np.float32((1 << bits) - 1), np.float32(1e-5)).astype(np.float32)
        z_ref = np.rint((-Wg.min(-1)).astype(np.float32) / s_ref).astype(np.float32)
        np.testing.assert_array_equal(s, s_ref)
        np.testing.assert_array_equal(z, z_ref)


# ---------------------------------------------------------------- quantizer invariants

@pytest.mark.parametrize("bits", [2, 3, 4])
def test_grid_has_2N_affine_levels_with_exact_zero(orc, bits):
    """Eq. 1-2: every W-hat of a group lies on {(c - zr) s : c = 0..Q}; the 2^N levels
    are distinct and affine; W = 0 maps to 0.0 exactly when zr is in [0, Q]."""
    Q = (1 << bits) - 1
    g = 64
    W = rand_w(32, 256, 5 + bits)
    W[:, ::17] = 0.0
    s, z = orc.minmax_init(W, bits, g)
    s, z = synthetic.perturb_quant_params(s, z, seed=bits)
    wh, code, mask, _ = orc.fake_quant(W, s, z, bits, g)
    G = 256 // g
    zr = np.rint(z)
    for n in range(32):
        for j in range(G):
            levels = ((np.arange(Q + 1, dtype=np.float32) - zr[n, j]).astype(np.float32) * s[n, j]).astype(np.float32)
            assert len(np.unique(levels)) == Q + 1
            d = np.diff(levels.astype(np.float64))
            np.testing.assert_allclose(d, d[0], rtol=1e-6)
            seg = wh[n, j * g:(j + 1) * g]
            assert np.isin(seg, levels).all()
            np.testing.assert_array_equal(seg, levels[code[n, j * g:(j + 1) * g]])
            zeros = W[n, j * g:(j + 1) * g] == 0
            if 0 <= zr[n, j] <= Q:
                assert (seg[zeros] == 0).all()


def test_fake_quant_matches_numpy_fp32_brute_force(orc):
    """Codes, mask and W-hat against a NumPy fp32 restatement (IEEE division, rint),
    on random weights plus constructed near-ties W = fp32((j + 0.5) s), where a
    reciprocal multiply instead of the division would flip the rounding."""
    bits, g, Q = 2, 32, 3
    rng = np.random.default_rng(77)
    N, K = 64, 256
    s = rng.uniform(0.003, 0.05, size=(N, K // g)).astype(np.float32)
    z = rng.uniform(-1.4, 4.4, size=(N, K // g)).astype(np.float32)
    srep = np.repeat(s, g, 1)
    j = rng.integers(-3, 5, size=(N, K)).astype(np.float32)
    W = ((j + np.float32(0.5)) * srep).astype(np.float32)
    W[:, ::3] = rng.standard_normal((N, (K + 2) // 3)).astype(np.float32) * np.float32(0.03)
    u = (W / srep).astype(np.float32)
    zr = np.repeat(np.rint(z), g, 1).astype(np.float32)
    q = (np.rint(u) + zr).astype(np.float32)
    c = np.clip(q, 0, Q).astype(np.float32)
    wh = ((c - zr).astype(np.float32) * srep).astype(np.float32)
    wh_o, code_o, mask_o, u_o = orc.fake_quant(W, s, z, bits, g)
    np.testing.assert_array_equal(u_o, u)
    np.testing.assert_array_equal(code_o, c.astype(np.uint8))
    np.testing.assert_array_equal(mask_o, ((q >= 0) & (q <= Q)).astype(np.uint8))
    np.testing.assert_array_equal(wh_o, wh)
    recip = (W * (np.float32(1.0) / srep)).astype(np.float32)
    assert (np.rint(recip) != np.rint(u)).any(), "the case must separate W/s from W*(1/s)"


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_dequant_round_trips_codes(orc, bits):
    """quant(dequant(c)) == c for every code c of every group."""
    Q = (1 << bits) - 1
    g = 32
    N, G = 16, 8
    s, z = synthetic.random_quant_params(N, G, bits, seed=bits)
    z = np.clip(np.rint(z), 0, Q).astype(np.float32)
    rng = np.random.default_rng(bits)
    c = rng.integers(0, Q + 1, size=(N, G * g)).astype(np.uint8)
    c[:, :Q + 1] = np.arange(Q + 1)
    srep = np.repeat(s, g, axis=1)
    zrep = np.repeat(z, g, axis=1)
    Wd = ((c.astype(np.float32) - zrep).astype(np.float32) * srep).astype(np.float32)
    _, code, mask, _ = orc.fake_quant(Wd, s, z, bits, g)
    np.testing.assert_array_equal(code, c)
    assert mask.all()


@pytest.mark.parametrize("bits,g", [(2, 64), (3, 128), (4, 32), (2, 32)])
def test_pack_layout_and_e2e_dequant(orc, bits, g):
    """Packed bytes decode (independent reader) to the fake-quant codes with zr := zq,
    zq = clamp(rint(z), 0, Q), and Eq. 2 on the frozen codes equals (c - zq) s."""
    Q = (1 << bits) - 1
    N, K = 24, 512
    W = rand_w(N, K, 99 + bits)
    s, z = orc.minmax_init(W, bits, g)
    s, z = synthetic.perturb_quant_params(s, z, seed=3 * bits + g)
    z = z + np.float32(0.3)  # non-integer zero points exercise round(z)
    packed, zq = orc.pack(W, s, z, bits, g)
    np.testing.assert_array_equal(zq, np.clip(np.rint(z), 0, Q).astype(np.uint8))
    zint = zq.astype(np.float32)
    _, code, _, _ = orc.fake_quant(W, s, zint, bits, g)
    np.testing.assert_array_equal(unpack_codes(packed, K, bits), code)
    exp_bytes = {2: K // 4, 3: K, 4: K // 2}[bits]
    assert packed.shape == (N, exp_bytes)
    wh = orc.dequant_packed(packed, zq, s, K, bits, g)
    ref = ((code.astype(np.float32) - np.repeat(zint, g, 1)).astype(np.float32) * np.repeat(s, g, 1)).astype(np.float32)
    np.testing.assert_array_equal(wh, ref)


def test_rounding_is_half_to_even(orc):
    W = np.array([[0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5, 0.0]], np.float32)
    s = np.ones((1, 1), np.float32)
    z = np.full((1, 1), 4.0, np.float32)
    _, code, _, _ = orc.fake_quant(W, s, z, 4, 8)
    np.testing.assert_array_equal(code[0], [4, 6, 6, 4, 2, 2, 8, 4])
    # round(z) is half-to-even too: z = 2.5 -> 2, 3.5 -> 4
    _, c2, _, _ = orc.fake_quant(np.zeros((1, 8), np.float32), s, np.full((1, 1), 2.5, np.float32), 4, 8)
    _, c3, _, _ = orc.fake_quant(np.zeros((1, 8), np.float32), s, np.full((1, 1), 3.5, np.float32), 4, 8)
    assert (c2 == 2).all() and (c3 == 4).all()


# ---------------------------------------------------------------- contractions vs NumPy

def test_contractions_match_numpy_matmul(orc):
    rng = np.random.default_rng(5)
    M, N, K = 37, 24, 96
    X = rng.standard_normal((M, K)).astype(np.float32)
    Wh = rng.standard_normal((N, K)).astype(np.float32)
    dY = rng.standard_normal((M, N)).astype(np.float32)
    X64, W64, d64 = X.astype(np.float64), Wh.astype(np.float64), dY.astype(np.float64)
    np.testing.assert_allclose(orc.linear_fwd(X, Wh), X64 @ W64.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(orc.linear_dx(dY, Wh), d64 @ W64, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(orc.linear_dwhat(dY, X), d64.T @ X64, rtol=1e-12, atol=1e-12)
    rows = np.array([36, 0, 5])
    wrows = np.array([23, 2])
    np.testing.assert_allclose(orc.linear_fwd(X, Wh, rows), (X64 @ W64.T)[rows], rtol=1e-12)
    np.testing.assert_allclose(orc.linear_dx(dY, Wh, rows), (d64 @ W64)[rows], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(orc.linear_dwhat(dY, X, wrows), (d64.T @ X64)[wrows], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- straight-through backward

class _RoundSTE(torch.autograd.Function):
    """round_ste: the value of round (decided in fp32, like the quantizer), the
    gradient of the identity."""

    @staticmethod
    def forward(ctx, x, rounded):
        return rounded.clone()

    @staticmethod
    def backward(ctx, grad):
        return grad, None


class _ClampSTE(torch.autograd.Function):
    """clamp_ste: the value of clamp, the gradient of the identity."""

    @staticmethod
    def forward(ctx, x, lo, hi):
        return torch.clamp(x, lo, hi)

    @staticmethod
    def backward(ctx, grad):
        return grad, None, None


def _surrogate_torch(X, W, s, z, dY, bits, g, clamp_pass=False):
    """Independent autograd re-derivation of Eq. 1-2 with round_ste on both round(W/s)
    and round(z), and torch.clamp (whose own backward passes the gradient only inside
    [0, Q], bounds included), in fp64.  The rounded values come from fp32 arithmetic
    so that the integer decisions match the fp32 quantizer."""
    Q = (1 << bits) - 1
    u32 = (W / np.repeat(s, g, 1)).astype(np.float32)
    r = torch.from_numpy(np.rint(u32).astype(np.float64))
    zr_val = torch.from_numpy(np.rint(z).astype(np.float64))
    Wt = torch.tensor(W, dtype=torch.float64, requires_grad=True)
    st = torch.tensor(s, dtype=torch.float64, requires_grad=True)
    zt = torch.tensor(z, dtype=torch.float64, requires_grad=True)
    srep = st.repeat_interleave(g, dim=1)
    zr = _RoundSTE.apply(zt, zr_val).repeat_interleave(g, dim=1)
    q = _RoundSTE.apply(Wt / srep, r) + zr
    c = _ClampSTE.apply(q, 0, Q) if clamp_pass else torch.clamp(q, 0, Q)
    wh = (c - zr) * srep
    Xt = torch.tensor(X, dtype=torch.float64, requires_grad=True)
    Y = Xt @ wh.T
    dYt = torch.tensor(dY, dtype=torch.float64)
    (Y * dYt).sum().backward()
    return Y.detach().numpy(), Xt.grad.numpy(), Wt.grad.numpy(), st.grad.numpy(), zt.grad.numpy()


def test_torch_clamp_gradient_bounds_are_inclusive():
    x = torch.tensor([-1.0, 0.0, 1.5, 3.0, 4.0], dtype=torch.float64, requires_grad=True)
    torch.clamp(x, 0, 3).sum().backward()
    assert x.grad.tolist() == [0.0, 1.0, 1.0, 1.0, 0.0]


@pytest.mark.parametrize("bits,g", [(2, 4), (3, 8), (2, 32)])
def test_ste_backward_matches_autograd_rederivation(orc, bits, g):
    rng = np.random.default_rng(17 + bits)
    M, N, K = 3, 5, 4 * g
    X = rng.standard_normal((M, K)).astype(np.float32)
    dY = rng.standard_normal((M, N)).astype(np.float32)
    W = rand_w(N, K, 23 + g)
    s, z = orc.minmax_init(W, bits, g)
    s, z = synthetic.perturb_quant_params(s, z, seed=g)
    z = z + np.float32(0.25)
    _, _, mask, _ = orc.fake_quant(W, s, z, bits, g)
    assert 0 < mask.mean() < 1, "the case must clamp some weights"
    Y_ref, dX_ref, dW_ref, ds_ref, dz_ref = _surrogate_torch(X, W, s, z, dY, bits, g)
    Y = orc.fq_linear_fwd(X, W, s, z, bits, g)
    dX, dW, ds, dz = orc.fq_linear_bwd(X, W, s, z, dY, bits, g)
    # the surrogate evaluates W-hat in fp64; the oracle's W-hat is fp32 (Block-AP math)
    np.testing.assert_allclose(Y, Y_ref, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(dX, dX_ref, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(dW, dW_ref, rtol=1e-12, atol=1e-12)
    # ds uses u = W/s rounded to fp32 (the quantizer's precision); autograd uses fp64:
    # the two differ by at most 2^-24 |u| per term.
    _, _, _, u = orc.fake_quant(W, s, z, bits, g)
    dwh = dY.astype(np.float64).T @ X.astype(np.float64)
    bound = (np.abs(dwh) * np.abs(u.astype(np.float64)) * 2.0 ** -23).reshape(N, -1, g).sum(-1)
    assert (np.abs(ds - ds_ref) <= bound + 1e-12).all()
    np.testing.assert_allclose(dz, dz_ref, rtol=1e-12, atol=1e-12)
    assert np.abs(dz).max() > 0


def test_ste_backward_matches_finite_differences_of_frozen_offset_surrogate(orc):
    """Central differences of W-hat = (clamp(W/s + delta + zr, 0, Q) - zr) s with the
    rounding offsets delta, zr frozen at the base point (what round_ste differentiates).
    At the base point q is an integer, so elements with q = 0 or q = Q sit on the clamp
    kink, where a central difference averages the two sides; only weights (for dW) and
    groups (for ds, dz) off the kinks are compared.  The inclusive-bound convention at
    the kink is pinned by the autograd test above."""
    bits, g = 2, 4
    Q = 3
    rng = np.random.default_rng(8)
    M, N, K = 2, 24, 16
    X = rng.standard_normal((M, K)).astype(np.float32)
    dY = rng.standard_normal((M, N)).astype(np.float32)
    W = rand_w(N, K, 41)
    s, z = orc.minmax_init(W, bits, g)
    s, z = synthetic.perturb_quant_params(s, z, seed=41)
    u32 = (W / np.repeat(s, g, 1)).astype(np.float32)
    delta = (np.rint(u32) - u32).astype(np.float64)
    zr0 = np.rint(z).astype(np.float64)
    X64, dY64 = X.astype(np.float64), dY.astype(np.float64)

    def loss(Wv, sv, zv):
        srep = np.repeat(sv, g, 1)
        zr = np.repeat(zv - z.astype(np.float64) + zr0, g, 1)
        q = Wv / srep + delta + zr
        wh = (np.clip(q, 0, Q) - zr) * srep
        return float(np.sum(dY64 * (X64 @ wh.T)))

    q0 = np.rint(u32).astype(np.float64) + np.repeat(zr0, g, 1)
    off_kink = (q0 != 0) & (q0 != Q)
    _, dW, ds, dz = orc.fq_linear_bwd(X, W, s, z, dY, bits, g)
    W64, s64, z64 = W.astype(np.float64), s.astype(np.float64), z.astype(np.float64)
    h = 1e-7
    elems = np.argwhere(off_kink)
    assert len(elems) > 20
    for n, k in elems[:: max(1, len(elems) // 24)]:
        e = np.zeros_like(W64); e[n, k] = h
        fd = (loss(W64 + e, s64, z64) - loss(W64 - e, s64, z64)) / (2 * h)
        assert abs(fd - dW[n, k]) <= 1e-6 * max(1.0, abs(fd))
    groups = np.argwhere(off_kink.reshape(N, -1, g).all(-1))
    clamped_groups = [tuple(t) for t in groups if (q0.reshape(N, -1, g)[t[0], t[1]] < 0).any()
                      or (q0.reshape(N, -1, g)[t[0], t[1]] > Q).any()]
    assert len(groups) >= 4 and len(clamped_groups) >= 1
    for n, j in [tuple(t) for t in groups[:8]] + clamped_groups[:4]:
        hs = 1e-7 * s64[n, j]
        e = np.zeros_like(s64); e[n, j] = hs
        fd = (loss(W64, s64 + e, z64) - loss(W64, s64 - e, z64)) / (2 * hs)
        assert abs(fd - ds[n, j]) <= 1e-5 * max(1.0, abs(fd))
        e = np.zeros_like(z64); e[n, j] = h
        fd = (loss(W64, s64, z64 + e) - loss(W64, s64, z64 - e)) / (2 * h)
        assert abs(fd - dz[n, j]) <= 1e-6 * max(1.0, abs(fd))
    assert any(abs(dz[n, j]) > 0 for n, j in clamped_groups)


def test_ste_no_clamping_special_case(orc):
    """With nothing clamped (min-max init, mixed-sign groups): dW == dW-hat, dz == 0 and
    ds == sum dW-hat (round(u) - u)."""
    rng = np.random.default_rng(4)
    M, N, K, g, bits = 7, 12, 128, 64, 2
    X = rng.standard_normal((M, K)).astype(np.float32)
    dY = rng.standard_normal((M, N)).astype(np.float32)
    W = rand_w(N, K, 4)
    s, z = orc.minmax_init(W, bits, g)
    _, _, mask, u = orc.fake_quant(W, s, z, bits, g)
    assert mask.all()
    dX, dW, ds, dz = orc.fq_linear_bwd(X, W, s, z, dY, bits, g)
    dwh = dY.astype(np.float64).T @ X.astype(np.float64)
    np.testing.assert_allclose(dW, dwh, rtol=1e-12, atol=1e-12)
    assert (dz == 0).all()
    ref = (dwh * (np.rint(u).astype(np.float64) - u.astype(np.float64))).reshape(N, -1, g).sum(-1)
    np.testing.assert_allclose(ds, ref, rtol=1e-9, atol=1e-12)


# ---------------------------------------------------------------- all-pass clamp variant

@pytest.mark.parametrize("bits,g", [(2, 4), (3, 8), (4, 16)])
def test_clamp_pass_backward_matches_autograd_rederivation(orc, bits, g):
    """With the clamp straight-through too (clamp_ste), autograd of Eq. 1-2 gives
    dW = dW-hat everywhere, dz = 0, ds = sum dW-hat ((c - zr) - u)."""
    rng = np.random.default_rng(31 + bits)
    M, N, K = 3, 6, 4 * g
    X = rng.standard_normal((M, K)).astype(np.float32)
    dY = rng.standard_normal((M, N)).astype(np.float32)
    W = rand_w(N, K, 37 + g)
    s, z = orc.minmax_init(W, bits, g)
    s, z = synthetic.perturb_quant_params(s, z, seed=g + 1)
    _, _, mask, u = orc.fake_quant(W, s, z, bits, g)
    assert 0 < mask.mean() < 1, "the case must clamp some weights"
    _, dX_ref, dW_ref, ds_ref, dz_ref = _surrogate_torch(X, W, s, z, dY, bits, g, clamp_pass=True)
    dX, dW, ds, dz = orc.fq_linear_bwd(X, W, s, z, dY, bits, g, clamp_pass=True)
    np.testing.assert_allclose(dX, dX_ref, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(dW, dW_ref, rtol=1e-12, atol=1e-12)
    dwh = dY.astype(np.float64).T @ X.astype(np.float64)
    bound = (np.abs(dwh) * np.abs(u.astype(np.float64)) * 2.0 ** -23).reshape(N, -1, g).sum(-1)
    assert (np.abs(ds - ds_ref) <= bound + 1e-12).all()
    np.testing.assert_allclose(dz_ref, 0.0, atol=1e-12)
    assert (dz == 0).all()
    # the variant differs from the default convention exactly on the clamped weights
    _, dW0, ds0, _ = orc.fq_linear_bwd(X, W, s, z, dY, bits, g)
    assert (dW0[mask == 1] == dW[mask == 1]).all() and (dW0[mask == 0] == 0).all()
    assert np.abs(ds - ds0).max() > 0


def test_clamp_pass_matches_finite_differences_of_frozen_offset_surrogate(orc):
    """What the all-pass variant differentiates: W-hat = (W/s + delta + zr + eps - zr) s
    with the rounding offset delta and the clamp offset eps = clamp(q0) - q0 frozen at
    the base point.  The surrogate is linear in W and z and smooth in s, so central
    differences pin every weight and every group, on the clamp kinks too."""
    bits, g, Q = 2, 4, 3
    rng = np.random.default_rng(9)
    M, N, K = 2, 16, 16
    X = rng.standard_normal((M, K)).astype(np.float32)
    dY = rng.standard_normal((M, N)).astype(np.float32)
    W = rand_w(N, K, 43)
    s, z = orc.minmax_init(W, bits, g)
    s, z = synthetic.perturb_quant_params(s, z, seed=43)
    u32 = (W / np.repeat(s, g, 1)).astype(np.float32)
    delta = (np.rint(u32) - u32).astype(np.float64)
    zr0 = np.rint(z).astype(np.float64)
    q0 = np.rint(u32).astype(np.float64) + np.repeat(zr0, g, 1)
    eps = np.clip(q0, 0, Q) - q0
    assert (eps != 0).any()
    X64, dY64 = X.astype(np.float64), dY.astype(np.float64)

    def loss(Wv, sv, zv):
        srep = np.repeat(sv, g, 1)
        zr = np.repeat(zv - z.astype(np.float64) + zr0, g, 1)
        wh = (Wv / srep + delta + zr + eps - zr) * srep
        return float(np.sum(dY64 * (X64 @ wh.T)))

    _, dW, ds, dz = orc.fq_linear_bwd(X, W, s, z, dY, bits, g, clamp_pass=True)
    W64, s64, z64 = W.astype(np.float64), s.astype(np.float64), z.astype(np.float64)
    h = 1e-7
    for n, k in [(n, k) for n in range(N) for k in range(0, K, 3)]:
        e = np.zeros_like(W64); e[n, k] = h
        fd = (loss(W64 + e, s64, z64) - loss(W64 - e, s64, z64)) / (2 * h)
        assert abs(fd - dW[n, k]) <= 1e-6 * max(1.0, abs(fd))
    for n in range(N):
        for j in range(K // g):
            hs = 1e-7 * s64[n, j]
            e = np.zeros_like(s64); e[n, j] = hs
            fd = (loss(W64, s64 + e, z64) - loss(W64, s64 - e, z64)) / (2 * hs)
            assert abs(fd - ds[n, j]) <= 1e-5 * max(1.0, abs(fd))
            e = np.zeros_like(z64); e[n, j] = h
            fd = (loss(W64, s64, z64 + e) - loss(W64, s64, z64 - e)) / (2 * h)
            assert abs(fd - dz[n, j]) <= 1e-6


def test_clamp_pass_equals_default_when_nothing_is_clamped(orc):
    rng = np.random.default_rng(5)
    M, N, K, g, bits = 4, 8, 128, 32, 3
    X = rng.standard_normal((M, K)).astype(np.float32)
    dY = rng.standard_normal((M, N)).astype(np.float32)
    W = rand_w(N, K, 5)
    s, z = orc.minmax_init(W, bits, g)
    assert orc.fake_quant(W, s, z, bits, g)[2].all()
    a = orc.fq_linear_bwd(X, W, s, z, dY, bits, g)
    b = orc.fq_linear_bwd(X, W, s, z, dY, bits, g, clamp_pass=True)
    for x, y in zip(a, b):
        assert (x == y).all()


# ---------------------------------------------------------------- E2E-QP

def test_e2e_ds_is_exact_gradient_finite_differences(orc):
    """Phase 2: W-hat is linear in s, so central differences of
    L(s) = sum dY * (X W-hat(s)^T) equal ds = sum dW-hat (W_q - z) to ~1e-10."""
    bits, g = 2, 16
    rng = np.random.default_rng(12)
    M, N, K = 6, 5, 64
    X = rng.standard_normal((M, K)).astype(np.float32)
    dY = rng.standard_normal((M, N)).astype(np.float32)
    W = rand_w(N, K, 12)
    s, z = orc.minmax_init(W, bits, g)
    packed, zq = orc.pack(W, s, z, bits, g)
    codes = unpack_codes(packed, K, bits).astype(np.float64)
    X64, dY64 = X.astype(np.float64), dY.astype(np.float64)

    def loss(sv):
        wh = (codes - np.repeat(zq.astype(np.float64), g, 1)) * np.repeat(sv, g, 1)
        return float(np.sum(dY64 * (X64 @ wh.T)))

    dX, ds = orc.dq_linear_bwd_s(X, packed, zq, s, dY, bits, g)
    s64 = s.astype(np.float64)
    for n in range(N):
        for j in range(K // g):
            h = 1e-3 * s64[n, j]
            e = np.zeros_like(s64); e[n, j] = h
            fd = (loss(s64 + e) - loss(s64 - e)) / (2 * h)
            assert abs(fd - ds[n, j]) <= 1e-10 * max(1.0, abs(ds).max())
    wh = orc.dequant_packed(packed, zq, s, K, bits, g).astype(np.float64)
    np.testing.assert_allclose(dX, dY64 @ wh, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(orc.dq_linear_fwd(X, packed, zq, s, bits, g), X64 @ wh.T, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("s_dtype", [np.float32, np.float16])
def test_e2e_dz_is_exact_gradient_finite_differences(orc, s_dtype):
    """With z trained as a float at the frozen codes, W-hat = (W_q - z) s is linear in z:
    central differences of L(z) equal dz = -s sum dW-hat to ~1e-10.  With fp16 step
    storage the oracle widens s exactly, so the same holds with s = float(s16)."""
    bits, g = 3, 8
    rng = np.random.default_rng(14)
    M, N, K = 5, 4, 32
    X = rng.standard_normal((M, K)).astype(np.float32)
    dY = rng.standard_normal((M, N)).astype(np.float32)
    W = rand_w(N, K, 14)
    s, z = orc.minmax_init(W, bits, g)
    packed, zq = orc.pack(W, s, z, bits, g)
    s = s.astype(s_dtype)
    codes = unpack_codes(packed, K, bits).astype(np.float64)
    X64, dY64 = X.astype(np.float64), dY.astype(np.float64)
    s64 = s.astype(np.float64)

    def loss(zv):
        wh = (codes - np.repeat(zv, g, 1)) * np.repeat(s64, g, 1)
        return float(np.sum(dY64 * (X64 @ wh.T)))

    dX, ds, dz = orc.dq_linear_bwd(X, packed, zq, s, dY, bits, g)
    z64 = zq.astype(np.float64)
    for n in range(N):
        for j in range(K // g):
            e = np.zeros_like(z64); e[n, j] = 0.5
            fd = (loss(z64 + e) - loss(z64 - e)) / 1.0
            assert abs(fd - dz[n, j]) <= 1e-10 * max(1.0, abs(dz).max())
    _, ds_s = orc.dq_linear_bwd_s(X, packed, zq, s, dY, bits, g)
    assert (ds == ds_s).all()


def test_fp16_step_storage_dequant_is_exact(orc):
    """(W_q - zq) is an integer of at most 5 bits and an fp16 s has an 11-bit
    significand, so with fp16 step storage W-hat = (W_q - zq) s is exact in fp32: it
    equals the fp64 product with the fp16 value of s (numpy's float16 conversion)."""
    bits, g = 4, 16
    W = rand_w(8, 64, 15)
    s, z = orc.minmax_init(W, bits, g)
    packed, zq = orc.pack(W, s, z, bits, g)
    s16 = s.astype(np.float16)
    wh = orc.dequant_packed(packed, zq, s16, 64, bits, g)
    codes = unpack_codes(packed, 64, bits).astype(np.float64)
    ref = (codes - np.repeat(zq.astype(np.float64), g, 1)) * np.repeat(s16.astype(np.float64), g, 1)
    assert (wh.astype(np.float64) == ref).all()
    assert not (s16.astype(np.float32) == s).all()


def test_effective_bits_closed_form():
    """Group-wise bookkeeping (paperlayer appendix D; modelfoundations 'Limitations'):
    an fp16 step and an N-bit zero point per g weights add (16 + N)/g bits; at g = 64,
    N = 2 that is ~0.28 bits, and the step sizes are 1/64 ~ 1.6% of the weight count."""
    for bits, g in [(2, 64), (3, 128)]:
        extra = (16 + bits) / g
        assert 0.1 < extra < 0.3
    assert abs(1 / 64 - 0.0156) < 1e-3


# ---------------------------------------------------------------- Block-AP optimizer step

@pytest.mark.parametrize("wd", [0.0, 0.01])
def test_adamw_matches_torch_optim_adamw(orc, wd):
    """The oracle's AdamW against torch.optim.AdamW (fp64, CPU) with the two learning-rate
    groups of Block-AP (weights 2e-5, quantization parameters 1e-4) over five steps."""
    rng = np.random.default_rng(21)
    shapes = {"W": (6, 16), "s": (6, 4)}
    lrs = {"W": 2e-5, "s": 1e-4}
    p0 = {k: (rng.standard_normal(sh) * (0.02 if k == "W" else 0.005) + (0 if k == "W" else 0.01)).astype(np.float32)
          for k, sh in shapes.items()}
    tp = {k: torch.tensor(p0[k].astype(np.float64), requires_grad=True) for k in shapes}
    opt = torch.optim.AdamW([{"params": [tp["W"]], "lr": lrs["W"]}, {"params": [tp["s"]], "lr": lrs["s"]}],
                            betas=(0.9, 0.999), eps=1e-8, weight_decay=wd)
    st = {k: (p0[k].copy(), np.zeros_like(p0[k]), np.zeros_like(p0[k])) for k in shapes}
    for t in range(1, 6):
        grads = {k: (rng.standard_normal(sh) * 0.1).astype(np.float32) for k, sh in shapes.items()}
        for k in shapes:
            tp[k].grad = torch.tensor(grads[k].astype(np.float64))
        opt.step()
        for k in shapes:
            p, m, v = st[k]
            st[k] = orc.adamw(p, grads[k], m, v, lrs[k], 0.9, 0.999, 1e-8, wd, t)
        for k in shapes:
            ref = tp[k].detach().numpy()
            got = st[k][0].astype(np.float64)
            # fp32 storage of p, m and v: within a few ulps of p per step
            assert np.abs(got - ref).max() <= 4 * t * np.spacing(np.abs(ref).max().astype(np.float32))
            state = opt.state[tp[k]]
            # m is a signed running sum: compare against its scale, not element-wise
            m_ref, v_ref = state["exp_avg"].numpy(), state["exp_avg_sq"].numpy()
            assert np.abs(st[k][1] - m_ref).max() <= 1e-6 * np.abs(m_ref).max()
            np.testing.assert_allclose(st[k][2], v_ref, rtol=2e-6, atol=1e-16)
        assert np.abs(st["W"][0] - p0["W"]).max() > 0


def test_cosine_schedule_matches_torch_scheduler(orc):
    """Closed form of cosine annealing against torch.optim.lr_scheduler.CosineAnnealingLR."""
    T, lr0, lr_min = 37, 1e-4, 1e-6
    p = torch.nn.Parameter(torch.zeros(1))
    opt = torch.optim.AdamW([p], lr=lr0)
    sch = torch.optim.lr_scheduler.CosineAnnealingLR(opt, T_max=T, eta_min=lr_min)
    for t in range(T + 1):
        assert abs(opt.param_groups[0]["lr"] - orc.cosine_lr(lr0, lr_min, t, T)) <= 1e-12 * lr0
        opt.step()
        sch.step()


def test_mse_gradient_matches_autograd(orc):
    rng = np.random.default_rng(3)
    Y = rng.standard_normal((5, 7))
    T = rng.standard_normal((5, 7))
    Yt = torch.tensor(Y, requires_grad=True)
    loss = ((Yt - torch.tensor(T)) ** 2).mean()
    loss.backward()
    l, dY = orc.mse_grad(Y, T)
    assert abs(l - loss.item()) <= 1e-14
    np.testing.assert_allclose(dY, Yt.grad.numpy(), rtol=1e-14, atol=1e-16)
