"""The C-ABI library loads, exports every entry point its header declares, and
rejects bad arguments on the host before any CUDA call (CPU only: every call
here fails validation or has nothing to do, so no kernel is launched)."""
import ctypes
import os
import re

import pytest

import weight_quantization_aware_b200 as eqat

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "eqat.h")

OK, NULL, SHAPE, ALIGN, DTYPE, UNSUP, WS, CUDA, TIMEOUT = range(9)
FAKE = 0x10  # aligned, never dereferenced: each call below fails validation first


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(eqat_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from weight_quantization_aware_b200 import build
    build.build()
    return eqat.load_library()


def test_every_declared_entry_point_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), f"{n} declared in eqat.h but not exported"


def test_status_strings_and_version(lib):
    for code, name in [(OK, "EQAT_OK"), (NULL, "EQAT_ERR_NULL"), (SHAPE, "EQAT_ERR_SHAPE"),
                       (ALIGN, "EQAT_ERR_ALIGN"), (DTYPE, "EQAT_ERR_DTYPE"),
                       (UNSUP, "EQAT_ERR_UNSUPPORTED"), (WS, "EQAT_ERR_WORKSPACE"),
                       (CUDA, "EQAT_ERR_CUDA"), (TIMEOUT, "EQAT_ERR_TIMEOUT")]:
        assert eqat.status_name(code) == name
    assert eqat.status_name(99) == "EQAT_ERR_UNKNOWN"
    assert lib.eqat_version() == 1


def test_workspace_bytes(lib):
    assert lib.eqat_workspace_bytes(4096, 4096, 4096, 2, 64, 1) == 4096 * 4096 * 2
    assert lib.eqat_workspace_bytes(128, 512, 256, 2, 64, 0) == 512 * 256 * 8
    assert lib.eqat_workspace_bytes(1, 8, 32, 2, 32, 1) == 512  # rounded up to 256 B
    assert lib.eqat_workspace_bytes(1, 0, 32, 2, 32, 1) == 0
    assert lib.eqat_workspace_bytes(1, 8, 32, 2, 32, 7) == 0


def P(v):
    return ctypes.c_void_p(v)


def fwd(lib, X=FAKE, W=FAKE, dt=1, s=FAKE, z=FAKE, Y=FAKE, M=16, N=16, K=64, bits=2, group=64,
        ws=FAKE, ws_bytes=1 << 20):
    return lib.eqat_fq_linear_fwd(P(X), P(W), dt, P(s), P(z), P(Y), M, N, K, bits, group, P(ws), ws_bytes, None)


def test_fq_fwd_argument_errors(lib):
    assert fwd(lib, bits=5) == UNSUP
    assert fwd(lib, bits=1) == UNSUP
    assert fwd(lib, group=48, K=96) == UNSUP
    assert fwd(lib, K=96, group=64) == SHAPE
    assert fwd(lib, N=12) == SHAPE
    assert fwd(lib, M=-1) == SHAPE
    assert fwd(lib, M=1 << 31) == SHAPE
    assert fwd(lib, dt=3) == DTYPE
    assert fwd(lib, X=0) == NULL
    assert fwd(lib, W=0) == NULL
    assert fwd(lib, s=0) == NULL
    assert fwd(lib, Y=0) == NULL
    assert fwd(lib, X=FAKE + 4) == ALIGN
    assert fwd(lib, Y=FAKE + 8) == ALIGN
    assert fwd(lib, ws=0) == WS
    assert fwd(lib, ws_bytes=100) == WS
    assert fwd(lib, ws=FAKE + 16) == ALIGN  # 16-aligned but not 256-aligned
    assert b"256" in lib.eqat_last_error_detail()
    # empty problems have nothing to do and touch no device
    assert fwd(lib, M=0) == OK
    assert fwd(lib, N=0) == OK


def test_other_entry_points_argument_errors(lib):
    st = None
    assert lib.eqat_minmax_init(P(FAKE), 1, 16, 96, 2, 64, P(FAKE), P(FAKE), st) == SHAPE
    assert lib.eqat_minmax_init(P(FAKE), 1, 16, 64, 2, 64, P(0), P(FAKE), st) == NULL
    assert lib.eqat_minmax_init(P(FAKE), 1, 0, 64, 2, 64, P(0), P(0), st) == OK
    assert lib.eqat_fake_quant(P(FAKE), 1, P(FAKE), P(FAKE), 16, 64, 2, 64, P(FAKE + 2), P(0), P(0), st) == ALIGN
    assert lib.eqat_fake_quant(P(FAKE), 1, P(FAKE), P(FAKE), 16, 64, 2, 64, P(0), P(0), P(0), st) == OK
    assert lib.eqat_pack_codes(P(FAKE), 1, P(FAKE), P(FAKE), 16, 64, 2, 64, P(0), P(FAKE), st) == NULL
    assert lib.eqat_pack_codes(P(FAKE), 1, P(FAKE), P(FAKE), 16, 64, 6, 64, P(FAKE), P(FAKE), st) == UNSUP
    assert lib.eqat_dequant_codes(P(FAKE), P(FAKE), P(FAKE), 16, 64, 2, 64, P(FAKE), 2, st) == DTYPE
    assert lib.eqat_fq_linear_bwd(P(FAKE), P(FAKE), 1, P(FAKE), P(FAKE), P(0), P(FAKE), P(0), P(0), P(0),
                                  16, 16, 64, 2, 64, P(FAKE), 1 << 20, 0, st) == NULL
    # nothing requested -> nothing to do
    assert lib.eqat_fq_linear_bwd(P(FAKE), P(FAKE), 1, P(FAKE), P(FAKE), P(FAKE), P(0), P(0), P(0), P(0),
                                  16, 16, 64, 2, 64, P(0), 0, 0, st) == OK
    assert lib.eqat_fq_linear_bwd(P(FAKE), P(FAKE), 1, P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(0), P(0), P(0),
                                  16, 16, 64, 2, 64, P(FAKE), 10, 1, st) == WS
    assert lib.eqat_dq_linear_fwd(P(FAKE), 1, P(FAKE), P(FAKE), P(FAKE), P(FAKE), 16, 16, 64, 3, 128,
                                  P(FAKE), 1 << 20, st) == SHAPE
    assert lib.eqat_dq_linear_bwd_s(P(FAKE), 1, P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(0), P(0),
                                    16, 16, 64, 2, 64, P(0), 0, 0, st) == OK
    # no workspace: only a bf16 forward whose code rows are a multiple of 16 bytes may do without one
    assert lib.eqat_dq_linear_fwd(P(FAKE), 0, P(FAKE), P(FAKE), P(FAKE), P(FAKE), 16, 16, 64, 2, 64,
                                  P(0), 0, st) == WS
    assert lib.eqat_dq_linear_fwd(P(FAKE), 1, P(FAKE), P(FAKE), P(FAKE), P(FAKE), 16, 16, 32, 2, 32,
                                  P(0), 0, st) == WS
    assert lib.eqat_selftest_bounded_wait(10, st) == SHAPE


def test_variant_entry_points_argument_errors(lib):
    st = None
    U = ctypes.c_uint32
    # unknown gradient flag bits are refused; flags 0 and EQAT_GRAD_CLAMP_PASS pass validation
    assert lib.eqat_fq_linear_bwd_ex(P(FAKE), P(FAKE), 1, P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(0), P(0), P(0),
                                     16, 16, 64, 2, 64, U(2), P(FAKE), 1 << 20, 0, st) == UNSUP
    for flags in (0, 1):
        assert lib.eqat_fq_linear_bwd_ex(P(FAKE), P(FAKE), 1, P(FAKE), P(FAKE), P(FAKE), P(0), P(0), P(0), P(0),
                                         16, 16, 64, 2, 64, U(flags), P(0), 0, 0, st) == OK
    # step-size dtype: fp32 or fp16 only
    assert lib.eqat_dequant_codes_ex(P(FAKE), P(FAKE), P(FAKE), 1, 16, 64, 2, 64, P(FAKE), 1, st) == DTYPE
    assert lib.eqat_dequant_codes_ex(P(FAKE), P(FAKE), P(FAKE), 2, 0, 64, 2, 64, P(FAKE), 1, st) == OK
    assert lib.eqat_dq_linear_fwd_ex(P(FAKE), 1, P(FAKE), P(FAKE), P(FAKE), 3, P(FAKE), 16, 16, 64, 2, 64,
                                     P(FAKE), 1 << 20, st) == DTYPE
    assert lib.eqat_dq_linear_fwd_ex(P(FAKE), 2, P(FAKE), P(FAKE), P(FAKE), 2, P(FAKE), 16, 16, 64, 2, 64,
                                     P(FAKE), 1 << 20, st) == DTYPE
    assert lib.eqat_dq_linear_bwd(P(FAKE), 1, P(FAKE), P(FAKE), P(FAKE), 2, P(FAKE), P(0), P(0), P(FAKE + 4),
                                  16, 16, 64, 2, 64, P(FAKE), 1 << 20, 0, st) == ALIGN
    assert lib.eqat_dq_linear_bwd(P(FAKE), 1, P(FAKE), P(FAKE), P(0), 2, P(FAKE), P(0), P(0), P(FAKE),
                                  16, 16, 64, 2, 64, P(FAKE), 1 << 20, 0, st) == NULL
    assert lib.eqat_dq_linear_bwd(P(FAKE), 1, P(FAKE), P(FAKE), P(FAKE), 2, P(FAKE), P(0), P(0), P(0),
                                  16, 16, 64, 2, 64, P(0), 0, 0, st) == OK


def test_multi_layer_entry_points_argument_errors(lib):
    """Layer-by-layer validation of the block-wide init and pack: a bad layer
    anywhere refuses the whole call before any launch."""
    st = None
    VP, I64 = ctypes.c_void_p, ctypes.c_int64

    def arr(t, xs):
        return (t * len(xs))(*xs)

    def pack(n=2, W=(FAKE, FAKE), s=(FAKE, FAKE), z=(FAKE, FAKE), N=(16, 8), K=(64, 128), codes=(FAKE, FAKE),
             zq=(FAKE, FAKE), bits=2, group=64):
        return lib.eqat_pack_codes_multi(n, arr(VP, W), 1, arr(VP, s), arr(VP, z), arr(I64, N), arr(I64, K),
                                         bits, group, arr(VP, codes), arr(VP, zq), st)

    def init(n=2, W=(FAKE, FAKE), N=(16, 8), K=(64, 128), s=(FAKE, FAKE), z=(FAKE, FAKE), group=64):
        return lib.eqat_minmax_init_multi(n, arr(VP, W), 1, arr(I64, N), arr(I64, K), 2, group, arr(VP, s),
                                          arr(VP, z), st)

    assert pack(n=-1) == SHAPE
    assert pack(n=65) == SHAPE
    assert lib.eqat_pack_codes_multi(1, None, 1, None, None, None, None, 2, 64, None, None, st) == NULL
    assert pack(N=(16, 12)) == SHAPE            # second layer: N not a multiple of 8
    assert pack(K=(64, 96)) == SHAPE            # second layer: K not a multiple of g
    assert pack(codes=(FAKE, 0)) == NULL
    assert pack(zq=(FAKE + 4, FAKE)) == ALIGN
    assert pack(bits=5) == UNSUP
    assert pack(N=(0, 0)) == OK                 # nothing to pack, no device touched
    assert pack(n=0) == OK
    assert init(N=(16, 12)) == SHAPE
    assert init(s=(FAKE, 0)) == NULL
    assert init(W=(FAKE + 2, FAKE)) == ALIGN
    assert init(group=48) == UNSUP
    assert init(N=(0, 0)) == OK


def test_binding_refuses_cpu_tensors():
    import torch
    W = torch.zeros(16, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        eqat.minmax_init(W, 2, 64)


def test_blockap_entry_points_argument_errors(lib):
    st = None
    # loss must be 8-byte aligned and non-NULL; the rest as for the forward
    assert lib.eqat_fq_linear_fwd_mse(P(FAKE), P(FAKE), 1, P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(0),
                                      16, 16, 64, 2, 64, P(FAKE), 1 << 20, st) == NULL
    assert lib.eqat_fq_linear_fwd_mse(P(FAKE), P(FAKE), 1, P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE + 4),
                                      16, 16, 64, 2, 64, P(FAKE), 1 << 20, st) == ALIGN
    assert lib.eqat_fq_linear_fwd_mse(P(FAKE), P(FAKE), 1, P(FAKE), P(FAKE), P(0), P(FAKE), P(FAKE),
                                      16, 16, 64, 2, 64, P(FAKE), 1 << 20, st) == NULL
    T = eqat.AdamwTensor(FAKE, FAKE, 1, FAKE, FAKE, None, 0, 0, 64)
    G = eqat.AdamwGroup(1e-4, 0.9, 0.999, 1e-8, 0.0)
    args = lambda t, ng, g, step: (ctypes.byref(t), 1, ctypes.byref(g), ng, step, st)
    assert lib.eqat_adamw_step(*args(T, 1, G, 0)) == SHAPE          # step >= 1
    assert lib.eqat_adamw_step(*args(T, 0, G, 1)) == SHAPE          # no groups
    bad = eqat.AdamwGroup(1e-4, 1.0, 0.999, 1e-8, 0.0)
    assert lib.eqat_adamw_step(*args(T, 1, bad, 1)) == UNSUP        # beta1 = 1
    T2 = eqat.AdamwTensor(FAKE, FAKE, 7, FAKE, FAKE, None, 0, 0, 64)
    assert lib.eqat_adamw_step(*args(T2, 1, G, 1)) == DTYPE
    T3 = eqat.AdamwTensor(FAKE, FAKE, 1, FAKE, FAKE, None, 0, 3, 64)
    assert lib.eqat_adamw_step(*args(T3, 1, G, 1)) == SHAPE         # group index
    T4 = eqat.AdamwTensor(FAKE + 8, FAKE, 1, FAKE, FAKE, None, 0, 0, 64)
    assert lib.eqat_adamw_step(*args(T4, 1, G, 1)) == ALIGN
    T0 = eqat.AdamwTensor(FAKE, FAKE, 1, FAKE, FAKE, None, 0, 0, 0)
    assert lib.eqat_adamw_step(*args(T0, 1, G, 1)) == OK            # nothing to do
    assert abs(eqat.cosine_lr(1e-4, 0.0, 0, 10) - 1e-4) < 1e-18
    assert abs(eqat.cosine_lr(1e-4, 0.0, 10, 10)) < 1e-18
    assert abs(eqat.cosine_lr(1e-4, 1e-6, 5, 10) - (1e-6 + (1e-4 - 1e-6) / 2)) < 1e-15


def test_binding_refuses_wrong_shapes_before_the_library():
    """The C ABI sees only pointers and sizes, so the binding must refuse an
    undersized or mis-shaped buffer itself (it would be read or written out of
    bounds on the device).  The checks run before the device checks, so they are
    exercised here on CPU tensors."""
    import torch
    bf, f32, u8 = torch.bfloat16, torch.float32, torch.uint8
    M, N, K, g, b = 8, 16, 128, 64, 2
    X, W = torch.zeros(M, K, dtype=bf), torch.zeros(N, K, dtype=bf)
    s, z = torch.zeros(N, K // g, dtype=f32), torch.zeros(N, K // g, dtype=f32)
    codes, zq = torch.zeros(N, K // 4, dtype=u8), torch.zeros(N, K // g, dtype=u8)
    Y_bad = torch.zeros(M, N - 8, dtype=bf)
    cases = [
        lambda: eqat.fq_linear_fwd_noalloc(X, W, s, z, b, g, Y=Y_bad),
        lambda: eqat.fq_linear_fwd(X, W, s, z, b, g, Y=Y_bad),
        lambda: eqat.fq_linear_fwd(X, W, s[:, :1], z, b, g),
        lambda: eqat.fq_linear_fwd(X, torch.zeros(N, K - 64, dtype=bf), s, z, b, g),
        lambda: eqat.fq_linear_bwd(X, W, s, z, torch.zeros(M, N + 8, dtype=bf), b, g),
        lambda: eqat.fq_linear_bwd(X, W, s, z, torch.zeros(M, N, dtype=bf), b, g,
                                   out=(torch.zeros(M, K - 8, dtype=bf), None, None, None)),
        lambda: eqat.dq_linear_fwd(X, codes[:, :-1], zq, s, b, g),
        lambda: eqat.dq_linear_fwd(X, codes, zq[:-8], s, b, g),
        lambda: eqat.dq_linear_bwd_s(X, codes, zq, s, torch.zeros(M, N, dtype=bf), b, g,
                                     out=(None, torch.zeros(N, 1, dtype=f32))),
        lambda: eqat.dq_linear_bwd(X, codes, zq, s, Y_bad, b, g),
        lambda: eqat.fq_linear_fwd_mse(X, W, s, z, Y_bad, b, g),
        lambda: eqat.pack_codes(W, s, z, b, g, codes=torch.zeros(N, K // 8, dtype=u8)),
        lambda: eqat.minmax_init(W, b, g, s=torch.zeros(N, 1, dtype=f32)),
        lambda: eqat.fake_quant(W, s[:8], z, b, g),
        lambda: eqat.dequant_codes(codes, zq, s[:, :1], K, b, g),
    ]
    for i, call in enumerate(cases):
        with pytest.raises(ValueError, match="shape|in-features|2-D"):
            call()
