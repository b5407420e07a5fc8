"""The rule the prepass and pack kernels use to decide round(RN(W/s)) near a
half-integer h without a division, restated in numpy and checked against numpy's
IEEE fp32 division on the inputs where it matters: weights on, and a few ulps either
side of, h s, and every near-tie weight of min-max-initialised bf16 layers (where
ties of W/s are common).

The rule (fp32 throughout): u = RN(W RN(1/s)); if u is at least 2^-7 from every
half-integer, round(u) is the answer.  Otherwise, with h that half-integer,
e = RN(W - h s) (one rounding, as fma gives) and T = s sp / 2 (sp the fp32 spacing
next to h on the side of e): |e| < T means RN(W/s) = h (then half to even);
|e| > T means RN(W/s) is on the side of e; |e| = T is left to the division.
"""
import numpy as np
import torch

f32 = np.float32
M = f32(12582912.0)  # 1.5 * 2^23


def rint_small(u):
    return ((u + M).astype(f32) - M).astype(f32)


def fma32(a, b, c):
    # RN32(a b + c): a b is exact in fp64 (24 x 24 bits) and, near a tie, so is the
    # sum (it cancels), so one rounding to fp32 is the fused result.
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(f32)


def rule(w, s):
    """Returns round(RN(w/s)) by the rule, and masks of the entries it decided as
    RN(w/s) = h and of those it left to the division."""
    u = (w * (f32(1) / s).astype(f32)).astype(f32)
    v = rint_small(u)
    r = (u - v).astype(f32)
    small = np.abs(u) < f32(2 ** 14)
    far = small & (np.abs(r) < f32(0.5 - 2 ** -7))
    h = (v + np.copysign(f32(0.5), r)).astype(f32)
    e = fma32(-h, s, w)
    p = ((h.view(np.int32) & 0x7F800000) - (24 << 23)).astype(np.int32).view(f32)
    T = (s * p).astype(f32)
    toward_zero = (np.abs(h) == f32(0.5)) & ((e > 0) != (h > 0))
    T = np.where(toward_zero, (f32(0.5) * T).astype(f32), T)
    ok = small & ~far & (T >= f32(2 ** -100))
    inside = ok & (np.abs(e) < T)
    outside = ok & (np.abs(e) > T)
    out = np.full(w.shape, np.nan, f32)
    out[far] = v[far]
    out[inside] = rint_small(h)[inside]
    side = np.where(e > 0, (h + f32(0.5)).astype(f32), (h - f32(0.5)).astype(f32))
    out[outside] = side[outside]
    return out, inside, ~(far | inside | outside)


def ieee_round(w, s):
    return np.rint((w / s).astype(f32))


def test_rule_on_and_around_half_integer_multiples_of_s():
    rng = np.random.default_rng(11)
    n = 300_000
    s = rng.uniform(1e-4, 0.2, n).astype(f32)
    h = (rng.integers(-40, 40, n) + 0.5).astype(f32)
    w = (h.astype(np.float64) * s).astype(f32)
    w = (w.view(np.int32) + rng.integers(-3, 4, n).astype(np.int32)).view(f32)
    got, on_tie, undecided = rule(w, s)
    want = ieee_round(w, s)
    assert (got[~undecided] == want[~undecided]).all()
    assert undecided.mean() < 1e-3  # the division is the exception
    # both branches of the residual test occur: RN(w/s) = h, and RN(w/s) beside h
    assert 0.01 < on_tie.mean() < 0.99


def test_rule_on_min_max_initialised_bf16_layers():
    for bits, g, seed in [(2, 64, 0), (3, 128, 1), (4, 32, 2)]:
        Q = (1 << bits) - 1
        W = (torch.randn(128, 4096, generator=torch.Generator().manual_seed(seed)) * 0.015).to(torch.bfloat16)
        Wg = W.float().numpy().reshape(128, 4096 // g, g)
        xmin, xmax = Wg.min(-1), Wg.max(-1)
        s = np.maximum(((xmax - xmin) / f32(Q)).astype(f32), f32(1e-5))
        S = np.broadcast_to(s[..., None], Wg.shape).astype(f32)
        u = (Wg * (f32(1) / S).astype(f32)).astype(f32)
        near = np.abs(u - rint_small(u)) >= f32(0.5 - 2 ** -16)
        assert near.sum() > 50  # ties of W/s do occur with min-max steps
        got, _, undecided = rule(Wg[near], S[near])
        want = ieee_round(Wg[near], S[near])
        assert (got[~undecided] == want[~undecided]).all()
