"""Python binding of libeqat, the B200 (sm_100a) fake-quantized linear layer of
EfficientQAT.

Argument marshalling only: every function checks tensor placement, dtype and
contiguity, allocates the outputs with PyTorch (the library itself allocates
nothing), passes raw pointers and the current CUDA stream to the C ABI
(``include/eqat.h``) and raises :class:`EqatError` on a non-zero status.  All the
arithmetic runs in the library's CUDA kernels; there is no CPU path.  If
``libeqat.so`` has not been built, loading fails loudly.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libeqat.so")

EQAT_F32 = 0
EQAT_BF16 = 1
EQAT_F16 = 2  # step sizes of the E2E-QP calls only
EQAT_GRAD_CLAMP_PASS = 1
EQAT_ERR_TIMEOUT = 8

_lib = None


class EqatError(RuntimeError):
    def __init__(self, fn, status, detail):
        self.status = status
        super().__init__(f"{fn}: {status_name(status)} ({status}): {detail}")


def load_library():
    """Loads libeqat.so (built in-tree by ``weight_quantization_aware_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m weight_quantization_aware_b200.build`"
            " (there is no fallback implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    U32 = ctypes.c_uint32
    sigs = {
        "eqat_minmax_init": [P, I, I64, I64, I, I, P, P, P],
        "eqat_fake_quant": [P, I, P, P, I64, I64, I, I, P, P, P, P],
        "eqat_pack_codes": [P, I, P, P, I64, I64, I, I, P, P, P],
        "eqat_minmax_init_multi": [I, P, I, P, P, I, I, P, P, P],
        "eqat_pack_codes_multi": [I, P, I, P, P, P, P, I, I, P, P, P],
        "eqat_dequant_codes": [P, P, P, I64, I64, I, I, P, I, P],
        "eqat_fq_linear_fwd": [P, P, I, P, P, P, I64, I64, I64, I, I, P, SZ, P],
        "eqat_fq_linear_bwd": [P, P, I, P, P, P, P, P, P, P, I64, I64, I64, I, I, P, SZ, I, P],
        "eqat_dq_linear_fwd": [P, I, P, P, P, P, I64, I64, I64, I, I, P, SZ, P],
        "eqat_dq_linear_bwd_s": [P, I, P, P, P, P, P, P, I64, I64, I64, I, I, P, SZ, I, P],
        "eqat_fq_linear_fwd_noalloc": [P, P, I, P, P, P, I64, I64, I64, I, I, P],
        "eqat_fq_linear_bwd_ex": [P, P, I, P, P, P, P, P, P, P, I64, I64, I64, I, I, U32, P, SZ, I, P],
        "eqat_dequant_codes_ex": [P, P, P, I, I64, I64, I, I, P, I, P],
        "eqat_dq_linear_fwd_ex": [P, I, P, P, P, I, P, I64, I64, I64, I, I, P, SZ, P],
        "eqat_dq_linear_bwd": [P, I, P, P, P, I, P, P, P, P, I64, I64, I64, I, I, P, SZ, I, P],
        "eqat_fq_linear_fwd_mse": [P, P, I, P, P, P, P, P, I64, I64, I64, I, I, P, SZ, P],
        "eqat_adamw_step": [P, I, P, I, I64, P],
        "eqat_device_error": [P, P],
        "eqat_selftest_bounded_wait": [I64, P],
    }
    for name, args in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = I
    lib.eqat_status_string.argtypes = [I]
    lib.eqat_status_string.restype = ctypes.c_char_p
    lib.eqat_last_error_detail.argtypes = []
    lib.eqat_last_error_detail.restype = ctypes.c_char_p
    lib.eqat_version.restype = I
    lib.eqat_cosine_lr.argtypes = [ctypes.c_double, ctypes.c_double, I64, I64]
    lib.eqat_cosine_lr.restype = ctypes.c_double
    lib.eqat_workspace_bytes.argtypes = [I64, I64, I64, I, I, I]
    lib.eqat_workspace_bytes.restype = SZ
    _lib = lib
    return lib


def status_name(status: int) -> str:
    return load_library().eqat_status_string(int(status)).decode()


def _call(name, *args):
    lib = load_library()
    st = getattr(lib, name)(*args)
    if st != 0:
        raise EqatError(name, st, lib.eqat_last_error_detail().decode())


def _p(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr()) if t.numel() > 0 else None


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return EQAT_BF16
    if t.dtype == torch.float32:
        return EQAT_F32
    raise TypeError(f"unsupported dtype {t.dtype}; use torch.bfloat16 or torch.float32")


def _sdt(s: torch.Tensor) -> int:
    """Step-size dtype of the E2E-QP calls: fp32, or fp16 storage."""
    if s.dtype == torch.float32:
        return EQAT_F32
    if s.dtype == torch.float16:
        return EQAT_F16
    raise TypeError(f"s must be torch.float32 or torch.float16, got {s.dtype}")


def _req(t, name, dtype=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def _shape(t, name, shape):
    """Refuses a tensor whose shape is not `shape` before any pointer reaches the
    library: the C ABI sees only pointers and sizes, so an undersized buffer would
    otherwise be read or written out of bounds on the device."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _linear_shapes(X, W_rows, K_w, group):
    """(M, N, K, G) of a linear layer; X is [M, K] and the weight side [N, K_w]."""
    if X.dim() != 2:
        raise ValueError(f"X must be 2-D [M, K], got shape {tuple(X.shape)}")
    M, K = X.shape
    if K_w != K:
        raise ValueError(f"the weight has {K_w} in-features, X has {K}")
    if group <= 0 or K % group:
        raise ValueError(f"K = {K} is not a multiple of group = {group}")
    return M, W_rows, K, K // group


def packed_row_bytes(K: int, bits: int) -> int:
    return K // 4 if bits == 2 else K // 2 if bits == 4 else K


def workspace_bytes(M: int, N: int, K: int, bits: int, group: int, dtype: torch.dtype) -> int:
    dt = EQAT_BF16 if dtype == torch.bfloat16 else EQAT_F32
    return int(load_library().eqat_workspace_bytes(M, N, K, bits, group, dt))


def workspace(M, N, K, bits, group, dtype, device=None) -> torch.Tensor:
    """A uint8 CUDA buffer of eqat_workspace_bytes() bytes (PyTorch blocks are 512-byte aligned)."""
    n = workspace_bytes(M, N, K, bits, group, dtype)
    return torch.empty(max(n, 1), dtype=torch.uint8, device=device or "cuda")


def _ws(ws, M, N, K, bits, group, dtype, device):
    if ws is None:
        ws = workspace(M, N, K, bits, group, dtype, device)
    _req(ws, "ws", torch.uint8)
    return ws


def minmax_init(W, bits, group, s=None, z=None):
    """Per-group min-max init: returns (s, z) fp32 [N, K/group]."""
    N, K = W.shape
    G = K // group if group else 0
    _shape(s, "s", (N, G)); _shape(z, "z", (N, G))
    _req(W, "W")
    s = torch.empty((N, G), dtype=torch.float32, device=W.device) if s is None else _req(s, "s", torch.float32)
    z = torch.empty((N, G), dtype=torch.float32, device=W.device) if z is None else _req(z, "z", torch.float32)
    _call("eqat_minmax_init", _p(W), _dt(W), N, K, bits, group, _p(s), _p(z), _stream())
    return s, z


def _ptr_array(ts):
    return (ctypes.c_void_p * max(1, len(ts)))(*[_p(t) for t in ts])


def _i64_array(xs):
    return (ctypes.c_int64 * max(1, len(xs)))(*xs)


def _same_kind(Ws):
    if not Ws:
        return None
    dt = Ws[0].dtype
    for i, W in enumerate(Ws):
        if W.dim() != 2:
            raise ValueError(f"W[{i}] must be 2-D")
        if W.dtype != dt:
            raise TypeError(f"W[{i}] is {W.dtype}, W[0] is {dt}: one dtype per call")
        _req(W, f"W[{i}]")
    return dt


def minmax_init_multi(Ws, bits, group, ss=None, zs=None):
    """min-max init of several weight matrices (the linears of a block) in one
    launch per eight layers: returns lists (s, z) as minmax_init gives per layer."""
    Ws = list(Ws)
    _same_kind(Ws)
    ss = [None] * len(Ws) if ss is None else list(ss)
    zs = [None] * len(Ws) if zs is None else list(zs)
    if len(ss) != len(Ws) or len(zs) != len(Ws):
        raise ValueError("one s and one z per W")
    for i, W in enumerate(Ws):
        N, K = W.shape
        G = K // group if group else 0
        _shape(ss[i], f"s[{i}]", (N, G)); _shape(zs[i], f"z[{i}]", (N, G))
        ss[i] = torch.empty((N, G), dtype=torch.float32, device=W.device) if ss[i] is None else \
            _req(ss[i], f"s[{i}]", torch.float32)
        zs[i] = torch.empty((N, G), dtype=torch.float32, device=W.device) if zs[i] is None else \
            _req(zs[i], f"z[{i}]", torch.float32)
    if Ws:
        _call("eqat_minmax_init_multi", len(Ws), _ptr_array(Ws), _dt(Ws[0]),
              _i64_array([W.shape[0] for W in Ws]), _i64_array([W.shape[1] for W in Ws]), bits, group,
              _ptr_array(ss), _ptr_array(zs), _stream())
    return ss, zs


def pack_codes_multi(Ws, ss, zs, bits, group, codes=None, zqs=None):
    """pack of several weight matrices (the linears of a block) in one launch per
    eight layers: returns lists (codes, zq) as pack_codes gives per layer."""
    Ws, ss, zs = list(Ws), list(ss), list(zs)
    _same_kind(Ws)
    codes = [None] * len(Ws) if codes is None else list(codes)
    zqs = [None] * len(Ws) if zqs is None else list(zqs)
    if not (len(ss) == len(zs) == len(codes) == len(zqs) == len(Ws)):
        raise ValueError("one s, z, codes and zq per W")
    for i, W in enumerate(Ws):
        N, K = W.shape
        G = K // group
        _shape(ss[i], f"s[{i}]", (N, G)); _shape(zs[i], f"z[{i}]", (N, G))
        _shape(codes[i], f"codes[{i}]", (N, packed_row_bytes(K, bits))); _shape(zqs[i], f"zq[{i}]", (N, G))
        _req(ss[i], f"s[{i}]", torch.float32); _req(zs[i], f"z[{i}]", torch.float32)
        if codes[i] is None:
            codes[i] = torch.empty((N, packed_row_bytes(K, bits)), dtype=torch.uint8, device=W.device)
        if zqs[i] is None:
            zqs[i] = torch.empty((N, G), dtype=torch.uint8, device=W.device)
        _req(codes[i], f"codes[{i}]", torch.uint8); _req(zqs[i], f"zq[{i}]", torch.uint8)
    if Ws:
        _call("eqat_pack_codes_multi", len(Ws), _ptr_array(Ws), _dt(Ws[0]), _ptr_array(ss), _ptr_array(zs),
              _i64_array([W.shape[0] for W in Ws]), _i64_array([W.shape[1] for W in Ws]), bits, group,
              _ptr_array(codes), _ptr_array(zqs), _stream())
    return codes, zqs


def fake_quant(W, s, z, bits, group, want_w_hat=True, want_code=True, want_mask=True, W_hat=None):
    """Quantizer prepass: returns (W_hat (W's dtype), code uint8, mask uint8), None where not wanted.
    W_hat, if given, receives the fake-quantized weight (it is then always written)."""
    N, K = W.shape
    _shape(s, "s", (N, K // group)); _shape(z, "z", (N, K // group)); _shape(W_hat, "W_hat", (N, K))
    _req(W, "W"); _req(s, "s", torch.float32); _req(z, "z", torch.float32)
    if W_hat is not None:
        wh = _req(W_hat, "W_hat", W.dtype)
    else:
        wh = torch.empty_like(W) if want_w_hat else None
    code = torch.empty((N, K), dtype=torch.uint8, device=W.device) if want_code else None
    mask = torch.empty((N, K), dtype=torch.uint8, device=W.device) if want_mask else None
    _call("eqat_fake_quant", _p(W), _dt(W), _p(s), _p(z), N, K, bits, group, _p(wh), _p(code), _p(mask),
          _stream())
    return wh, code, mask


def pack_codes(W, s, z, bits, group, codes=None, zq=None):
    """Pack to low-bit integers: returns (codes uint8 [N, row_bytes], zq uint8 [N, K/group])."""
    N, K = W.shape
    _shape(s, "s", (N, K // group)); _shape(z, "z", (N, K // group))
    _shape(codes, "codes", (N, packed_row_bytes(K, bits))); _shape(zq, "zq", (N, K // group))
    _req(W, "W"); _req(s, "s", torch.float32); _req(z, "z", torch.float32)
    if codes is None:
        codes = torch.empty((N, packed_row_bytes(K, bits)), dtype=torch.uint8, device=W.device)
    if zq is None:
        zq = torch.empty((N, K // group), dtype=torch.uint8, device=W.device)
    _req(codes, "codes", torch.uint8); _req(zq, "zq", torch.uint8)
    _call("eqat_pack_codes", _p(W), _dt(W), _p(s), _p(z), N, K, bits, group, _p(codes), _p(zq), _stream())
    return codes, zq


def dequant_codes(codes, zq, s, K, bits, group, dtype=torch.bfloat16, out=None):
    """E2E-QP dequant of frozen codes: W_hat = (W_q - zq) s, [N, K] of `dtype` (or into
    `out`, whose dtype then decides).  s is fp32 or fp16 (fp16 step-size storage)."""
    N = codes.shape[0]
    _shape(codes, "codes", (N, packed_row_bytes(K, bits))); _shape(zq, "zq", (N, K // group))
    _shape(s, "s", (N, K // group)); _shape(out, "out", (N, K))
    _req(codes, "codes", torch.uint8); _req(zq, "zq", torch.uint8); _req(s, "s")
    wh = torch.empty((N, K), dtype=dtype, device=codes.device) if out is None else _req(out, "out")
    _call("eqat_dequant_codes_ex", _p(codes), _p(zq), _p(s), _sdt(s), N, K, bits, group, _p(wh), _dt(wh),
          _stream())
    return wh


def _fq_shapes(X, W, s, z, group, **mn):
    """Shapes of a Block-AP call: W [N, K], s and z [N, K/group], and each [M, N]
    tensor of `mn` (Y, dY, T)."""
    if W.dim() != 2:
        raise ValueError(f"W must be 2-D [N, K], got shape {tuple(W.shape)}")
    M, N, K, G = _linear_shapes(X, W.shape[0], W.shape[1], group)
    _shape(s, "s", (N, G)); _shape(z, "z", (N, G))
    for name, t in mn.items():
        _shape(t, name, (M, N))
    return M, N, K, G


def _dq_shapes(X, codes, zq, s, bits, group, **mn):
    """Shapes of an E2E-QP call: codes [N, packed row bytes of K], zq and s
    [N, K/group], and each [M, N] tensor of `mn`."""
    if codes.dim() != 2:
        raise ValueError(f"codes must be 2-D [N, row bytes], got shape {tuple(codes.shape)}")
    if X.dim() != 2:
        raise ValueError(f"X must be 2-D [M, K], got shape {tuple(X.shape)}")
    M, N, K, G = _linear_shapes(X, codes.shape[0], X.shape[1], group)
    _shape(codes, "codes", (N, packed_row_bytes(K, bits)))
    _shape(zq, "zq", (N, G)); _shape(s, "s", (N, G))
    for name, t in mn.items():
        _shape(t, name, (M, N))
    return M, N, K, G


def fq_linear_fwd(X, W, s, z, bits, group, ws=None, Y=None):
    """Block-AP forward Y = X W_hat^T."""
    _fq_shapes(X, W, s, z, group, Y=Y)
    _req(X, "X"); _req(W, "W", X.dtype); _req(s, "s", torch.float32); _req(z, "z", torch.float32)
    M, K = X.shape
    N = W.shape[0]
    Y = torch.empty((M, N), dtype=X.dtype, device=X.device) if Y is None else _req(Y, "Y", X.dtype)
    ws = _ws(ws, M, N, K, bits, group, X.dtype, X.device)
    _call("eqat_fq_linear_fwd", _p(X), _p(W), _dt(X), _p(s), _p(z), _p(Y), M, N, K, bits, group,
          _p(ws), ws.numel(), _stream())
    return Y


def fq_linear_fwd_noalloc(X, W, s, z, bits, group, Y):
    """Block-AP forward for callers that cannot allocate: no workspace, W-hat lives in
    the library's static 32 MiB device scratch (N*K*sizeof(dtype) must fit).  The
    output Y is the caller's.  Calls that overlap on the GPU share that scratch and
    race; serialise them."""
    if Y is None:
        raise ValueError("Y is required: this entry point allocates nothing")
    _fq_shapes(X, W, s, z, group, Y=Y)
    _req(X, "X"); _req(W, "W", X.dtype); _req(s, "s", torch.float32); _req(z, "z", torch.float32)
    _req(Y, "Y", X.dtype)
    M, K = X.shape
    N = W.shape[0]
    _call("eqat_fq_linear_fwd_noalloc", _p(X), _p(W), _dt(X), _p(s), _p(z), _p(Y), M, N, K, bits, group,
          _stream())
    return Y


def fq_linear_bwd(X, W, s, z, dY, bits, group, need_dx=True, need_dw=True, need_ds=True, need_dz=True,
                  ws=None, out=None, w_hat_in_ws=False, clamp_pass=False):
    """Block-AP straight-through backward: returns (dX, dW, ds, dz), None where not requested.
    w_hat_in_ws=True reuses the W-hat that fq_linear_fwd left in `ws` (same W, s, z).
    clamp_pass=True lets the clamp pass the gradient too (EQAT_GRAD_CLAMP_PASS)."""
    M, N, K, G = _fq_shapes(X, W, s, z, group, dY=dY)
    if out is not None:
        _shape(out[0], "dX", (M, K)); _shape(out[1], "dW", (N, K))
        _shape(out[2], "ds", (N, G)); _shape(out[3], "dz", (N, G))
    _req(X, "X"); _req(W, "W", X.dtype); _req(s, "s", torch.float32); _req(z, "z", torch.float32)
    _req(dY, "dY", X.dtype)
    M, K = X.shape
    N = W.shape[0]
    G = K // group
    if out is None:
        dev = X.device
        dX = torch.empty((M, K), dtype=X.dtype, device=dev) if need_dx else None
        dW = torch.empty((N, K), dtype=X.dtype, device=dev) if need_dw else None
        ds = torch.empty((N, G), dtype=torch.float32, device=dev) if need_ds else None
        dz = torch.empty((N, G), dtype=torch.float32, device=dev) if need_dz else None
    else:
        dX, dW, ds, dz = out
    ws = _ws(ws, M, N, K, bits, group, X.dtype, X.device)
    if w_hat_in_ws and ws is None:
        raise ValueError("w_hat_in_ws needs the workspace of the forward call")
    flags = EQAT_GRAD_CLAMP_PASS if clamp_pass else 0
    _call("eqat_fq_linear_bwd_ex", _p(X), _p(W), _dt(X), _p(s), _p(z), _p(dY), _p(dX), _p(dW), _p(ds),
          _p(dz), M, N, K, bits, group, flags, _p(ws), ws.numel(), int(bool(w_hat_in_ws)), _stream())
    return dX, dW, ds, dz


def dq_linear_fwd(X, codes, zq, s, bits, group, ws=None, Y=None, keep_w_hat=True):
    """E2E-QP forward on frozen codes: Y = X ((W_q - zq) s)^T; s fp32 or fp16.
    keep_w_hat=False passes no workspace (ws must be None): W-hat is made from the
    codes inside the contraction and kept nowhere (forward-only use)."""
    _dq_shapes(X, codes, zq, s, bits, group, Y=Y)
    _req(X, "X"); _req(codes, "codes", torch.uint8); _req(zq, "zq", torch.uint8); _req(s, "s")
    M, K = X.shape
    N = codes.shape[0]
    Y = torch.empty((M, N), dtype=X.dtype, device=X.device) if Y is None else _req(Y, "Y", X.dtype)
    if keep_w_hat:
        ws = _ws(ws, M, N, K, bits, group, X.dtype, X.device)
        wsp, wsn = _p(ws), ws.numel()
    else:
        if ws is not None:
            raise ValueError("keep_w_hat=False takes no workspace")
        wsp, wsn = None, 0
    _call("eqat_dq_linear_fwd_ex", _p(X), _dt(X), _p(codes), _p(zq), _p(s), _sdt(s), _p(Y), M, N, K, bits,
          group, wsp, wsn, _stream())
    return Y


def dq_linear_bwd_s(X, codes, zq, s, dY, bits, group, need_dx=True, need_ds=True, ws=None, out=None,
                    w_hat_in_ws=False):
    """E2E-QP backward (scales only): returns (dX, ds).  w_hat_in_ws=True reuses the
    W-hat that dq_linear_fwd left in `ws`."""
    M, N, K, G = _dq_shapes(X, codes, zq, s, bits, group, dY=dY)
    if out is not None:
        _shape(out[0], "dX", (M, K)); _shape(out[1], "ds", (N, G))
    _req(X, "X"); _req(codes, "codes", torch.uint8); _req(zq, "zq", torch.uint8); _req(s, "s", torch.float32)
    _req(dY, "dY", X.dtype)
    M, K = X.shape
    N = codes.shape[0]
    if out is None:
        dX = torch.empty((M, K), dtype=X.dtype, device=X.device) if need_dx else None
        ds = torch.empty((N, K // group), dtype=torch.float32, device=X.device) if need_ds else None
    else:
        dX, ds = out
    ws = _ws(ws, M, N, K, bits, group, X.dtype, X.device)
    if w_hat_in_ws and ws is None:
        raise ValueError("w_hat_in_ws needs the workspace of the forward call")
    _call("eqat_dq_linear_bwd_s", _p(X), _dt(X), _p(codes), _p(zq), _p(s), _p(dY), _p(dX), _p(ds),
          M, N, K, bits, group, _p(ws), ws.numel(), int(bool(w_hat_in_ws)), _stream())
    return dX, ds


def dq_linear_bwd(X, codes, zq, s, dY, bits, group, need_dx=True, need_ds=True, need_dz=True, ws=None,
                  out=None, w_hat_in_ws=False):
    """E2E-QP backward with the zero-point gradient: returns (dX, ds, dz), None where not
    requested; dz = -s sum_group dY^T X.  s fp32 or fp16."""
    M, N, K, G = _dq_shapes(X, codes, zq, s, bits, group, dY=dY)
    if out is not None:
        _shape(out[0], "dX", (M, K)); _shape(out[1], "ds", (N, G)); _shape(out[2], "dz", (N, G))
    _req(X, "X"); _req(codes, "codes", torch.uint8); _req(zq, "zq", torch.uint8); _req(s, "s")
    _req(dY, "dY", X.dtype)
    M, K = X.shape
    N = codes.shape[0]
    G = K // group
    if out is None:
        dX = torch.empty((M, K), dtype=X.dtype, device=X.device) if need_dx else None
        ds = torch.empty((N, G), dtype=torch.float32, device=X.device) if need_ds else None
        dz = torch.empty((N, G), dtype=torch.float32, device=X.device) if need_dz else None
    else:
        dX, ds, dz = out
    ws = _ws(ws, M, N, K, bits, group, X.dtype, X.device)
    if w_hat_in_ws and ws is None:
        raise ValueError("w_hat_in_ws needs the workspace of the forward call")
    _call("eqat_dq_linear_bwd", _p(X), _dt(X), _p(codes), _p(zq), _p(s), _sdt(s), _p(dY), _p(dX), _p(ds),
          _p(dz), M, N, K, bits, group, _p(ws), ws.numel(), int(bool(w_hat_in_ws)), _stream())
    return dX, ds, dz


def fq_linear_fwd_mse(X, W, s, z, T, bits, group, ws=None, dY=None, loss=None):
    """Block-AP forward against the full-precision output T, Y not stored: returns
    (dY = 2 (Y - T) / (M N), loss = mean (Y - T)^2 as a 1-element fp64 CUDA tensor)."""
    M, N, K, G = _fq_shapes(X, W, s, z, group, T=T, dY=dY)
    _shape(loss, "loss", (1,))
    _req(X, "X"); _req(W, "W", X.dtype); _req(s, "s", torch.float32); _req(z, "z", torch.float32)
    _req(T, "T", X.dtype)
    M, K = X.shape
    N = W.shape[0]
    dY = torch.empty((M, N), dtype=X.dtype, device=X.device) if dY is None else _req(dY, "dY", X.dtype)
    loss = torch.empty(1, dtype=torch.float64, device=X.device) if loss is None else _req(loss, "loss", torch.float64)
    ws = _ws(ws, M, N, K, bits, group, X.dtype, X.device)
    _call("eqat_fq_linear_fwd_mse", _p(X), _p(W), _dt(X), _p(s), _p(z), _p(T), _p(dY), _p(loss), M, N, K, bits,
          group, _p(ws), ws.numel(), _stream())
    return dY, loss


class AdamwTensor(ctypes.Structure):
    _fields_ = [("param", ctypes.c_void_p), ("grad", ctypes.c_void_p), ("grad_dtype", ctypes.c_int),
                ("exp_avg", ctypes.c_void_p), ("exp_avg_sq", ctypes.c_void_p), ("param_copy", ctypes.c_void_p),
                ("copy_dtype", ctypes.c_int), ("group", ctypes.c_int), ("numel", ctypes.c_int64)]


class AdamwGroup(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_double), ("beta1", ctypes.c_double), ("beta2", ctypes.c_double),
                ("eps", ctypes.c_double), ("weight_decay", ctypes.c_double)]


def adamw_step(entries, groups, step):
    """One fused AdamW step.  entries: list of (param fp32, grad fp32|bf16, exp_avg, exp_avg_sq,
    param_copy or None, group index); groups: list of dicts lr, beta1, beta2, eps, weight_decay."""
    arr = (AdamwTensor * max(1, len(entries)))()
    for i, (p, g, m, v, c, gi) in enumerate(entries):
        _req(p, "param", torch.float32); _req(m, "exp_avg", torch.float32); _req(v, "exp_avg_sq", torch.float32)
        _req(g, "grad")
        if c is not None:
            _req(c, "param_copy")
        arr[i] = AdamwTensor(p.data_ptr(), g.data_ptr(), _dt(g), m.data_ptr(), v.data_ptr(),
                             c.data_ptr() if c is not None else None, _dt(c) if c is not None else EQAT_F32,
                             int(gi), p.numel())
    garr = (AdamwGroup * len(groups))()
    for i, gr in enumerate(groups):
        garr[i] = AdamwGroup(gr["lr"], gr.get("beta1", 0.9), gr.get("beta2", 0.999), gr.get("eps", 1e-8),
                             gr.get("weight_decay", 0.0))
    _call("eqat_adamw_step", ctypes.cast(arr, ctypes.c_void_p), len(entries), ctypes.cast(garr, ctypes.c_void_p),
          len(groups), int(step), _stream())


def cosine_lr(lr0, lr_min, step, total):
    """The learning rate at `step` of a cosine schedule of `total` steps."""
    return float(load_library().eqat_cosine_lr(lr0, lr_min, int(step), int(total)))


def device_error():
    """Synchronises the current stream and returns the raw device error word (0 when clean).
    Raises EqatError(EQAT_ERR_TIMEOUT) if a bounded on-chip wait ran out."""
    where = ctypes.c_int(0)
    lib = load_library()
    st = lib.eqat_device_error(ctypes.byref(where), _stream())
    if st != 0:
        raise EqatError("eqat_device_error", st, lib.eqat_last_error_detail().decode())
    return where.value


def selftest_bounded_wait(timeout_ns: int):
    _call("eqat_selftest_bounded_wait", int(timeout_ns), _stream())
