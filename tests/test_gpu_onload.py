"""Dequantize-on-load in the E2E-QP contractions (Eq. 2 inside the pair GEMM).

The forward Y = X ((W_q - zq) s)^T and the input gradient dX = dY W-hat can make
W-hat from the packed codes in shared memory instead of reading a W-hat that the
dequantize kernel wrote.  The converter is exact: each weight is the fp32 product
(W_q - zq) s rounded to bf16, the value the dequantize kernel writes.  So with the
same tile shapes the results must equal, bit for bit, those of the
dequantize-then-GEMM path, and match the oracle within the GEMM tolerance.

Both paths are forced in fresh processes (EQAT_DQ_ONLOAD=1 / 0, CTA-pair tiles) on
the same inputs.  Shapes cover 2-, 3- and 4-bit codes, groups of 32, 64 and 128 (a
2-bit group of 32 splits a 16-byte code unit), ragged M, N and K, fp16 step sizes,
and both N-tile widths the wave model picks.  A last case checks the default choice:
a forward without a workspace takes the on-load path, one with a workspace and
every backward the other."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import weight_quantization_aware_b200 as eqat
from weight_quantization_aware_b200 import synthetic
from parity import TOL_GEMM, TOL_RED, assert_close, to_np

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SHAPES = [  # (M, N, K, bits, group, s dtype)
    (300, 392, 384, 2, 64, "f32"),
    (128, 256, 256, 3, 128, "f32"),
    (200, 136, 160, 4, 32, "f32"),
    (257, 520, 640, 2, 128, "f16"),
    (384, 1032, 1024, 2, 32, "f32"),
    (513, 264, 2112, 4, 64, "f16"),
    (96, 2048, 512, 3, 64, "f32"),
]

RUN_SCRIPT = r'''
import sys, numpy as np, torch
import weight_quantization_aware_b200 as eqat
for inp in sys.argv[1:]:
    d = dict(np.load(inp))
    X, dY = (torch.from_numpy(d[k]).to(torch.bfloat16).cuda() for k in ("X", "dY"))
    codes, zq = torch.from_numpy(d["codes"]).cuda(), torch.from_numpy(d["zq"]).cuda()
    s = torch.from_numpy(d["s"]).cuda()
    b, g = int(d["bits"]), int(d["group"])
    Y = eqat.dq_linear_fwd(X, codes, zq, s, b, g)
    dX, ds, dz = eqat.dq_linear_bwd(X, codes, zq, s, dY, b, g)
    torch.cuda.synchronize()
    assert eqat.device_error() == 0
    np.savez(inp.replace(".npz", "_out.npz"), Y=Y.float().cpu().numpy(), dX=dX.float().cpu().numpy(),
             ds=ds.cpu().numpy(), dz=dz.cpu().numpy())
'''


def make_case(orc, M, N, K, bits, g, sdt, seed):
    d = synthetic.draw_linear(np.random.default_rng(seed), M, N, K, 0.02, "bf16")
    Xn, Wn, dYn = (synthetic.as_f32_numpy(d[k]) for k in ("X", "W", "dY"))
    s, z = orc.minmax_init(Wn, bits, g)
    s, z = synthetic.perturb_quant_params(s, z, seed)
    packed, zq = orc.pack(Wn, s, z, bits, g)
    s_t = s.astype(np.float16) if sdt == "f16" else s
    return Xn, dYn, packed, zq, s_t


def run_forced(mode, paths):
    """Runs forward and backward of every saved case in a fresh process with the path forced."""
    env = dict(os.environ, EQAT_DQ_ONLOAD=mode, EQAT_GEMM_PAIR="1", PYTHONPATH=ROOT)
    env.pop("EQAT_GEMM_BN", None)
    r = subprocess.run([sys.executable, "-c", RUN_SCRIPT, *map(str, paths)], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-3000:]
    outs = []
    for p in paths:
        o = str(p).replace(".npz", "_out.npz")
        outs.append(dict(np.load(o)))
        os.replace(o, o.replace("_out.npz", f"_out{mode}.npz"))
    return outs


@pytest.fixture(scope="module")
def forced(orc, tmp_path_factory):
    """The cases, and each path's results on them."""
    tmp = tmp_path_factory.mktemp("onload")
    cases, paths = [], []
    for i, (M, N, K, bits, g, sdt) in enumerate(SHAPES):
        Xn, dYn, packed, zq, s = make_case(orc, M, N, K, bits, g, sdt, 500 + M)
        p = tmp / f"case{i}.npz"
        np.savez(p, X=Xn, dY=dYn, codes=packed, zq=zq, s=s, bits=bits, group=g)
        cases.append((Xn, dYn, packed, zq, s))
        paths.append(p)
    return cases, run_forced("1", paths), run_forced("0", paths)


@pytest.mark.parametrize("i", range(len(SHAPES)), ids=lambda i: "x".join(map(str, SHAPES[i])))
def test_onload_equals_dequantize_path_and_oracle(orc, forced, i):
    M, N, K, bits, g, sdt = SHAPES[i]
    cases, on, off = forced
    Xn, dYn, packed, zq, s = cases[i]
    for name in ("Y", "dX", "ds", "dz"):
        a, b = on[i][name], off[i][name]
        assert np.array_equal(a, b), \
            f"{name}: on-load differs from the dequantize path at {np.argwhere(a != b)[:3].tolist()}"
    rng = np.random.default_rng(7)
    rows = np.sort(rng.choice(M, min(M, 64), replace=False))
    Y_ref = orc.dq_linear_fwd(Xn, packed, zq, s, bits, g, rows=rows)
    dX_ref, ds_ref, dz_ref = orc.dq_linear_bwd(Xn, packed, zq, s, dYn, bits, g, rows=rows)
    assert_close(on[i]["Y"][rows], Y_ref, TOL_GEMM, "Y")
    assert_close(on[i]["dX"][rows], dX_ref, TOL_GEMM, "dX")
    assert_close(on[i]["ds"], ds_ref, TOL_RED, "ds")
    assert_close(on[i]["dz"], dz_ref, TOL_RED, "dz")


def test_default_choice_by_workspace(orc, tmp_path):
    """By default the forward makes W-hat on load exactly when it gets no workspace
    (keep_w_hat=False): its results then equal, bit for bit, the forced on-load
    run's.  With a workspace it dequantizes into it, equal to the forced dequantize
    run, and a backward reusing that W-hat equals the forced dequantize backward;
    the backward never makes W-hat on load by default, also after a forward without
    a workspace (w_hat_in_ws=False).  Layer: 13824 x 5120 (Llama-2-13B gate_proj) at
    64 and 512 tokens; everything also matches the oracle."""
    N, K, bits, g = 13824, 5120, 2, 64
    for M in (64, 512):
        Xn, dYn, packed, zq, s = make_case(orc, M, N, K, bits, g, "f32", 900 + M)
        X = torch.from_numpy(Xn).to(torch.bfloat16).cuda()
        dY = torch.from_numpy(dYn).to(torch.bfloat16).cuda()
        codes_d, zq_d, s_d = (torch.from_numpy(a).cuda() for a in (packed, zq, s))
        ws = eqat.workspace(M, N, K, bits, g, torch.bfloat16)
        Y_nows = eqat.dq_linear_fwd(X, codes_d, zq_d, s_d, bits, g, keep_w_hat=False)
        dX_a, ds_a, dz_a = eqat.dq_linear_bwd(X, codes_d, zq_d, s_d, dY, bits, g, ws=ws, w_hat_in_ws=False)
        Y_ws = eqat.dq_linear_fwd(X, codes_d, zq_d, s_d, bits, g, ws=ws)
        dX_b, ds_b, dz_b = eqat.dq_linear_bwd(X, codes_d, zq_d, s_d, dY, bits, g, ws=ws, w_hat_in_ws=True)
        torch.cuda.synchronize()
        assert eqat.device_error() == 0
        p = tmp_path / f"m{M}.npz"
        np.savez(p, X=Xn, dY=dYn, codes=packed, zq=zq, s=s, bits=bits, group=g)
        on = run_forced("1", [p])[0]
        off = run_forced("0", [p])[0]
        assert np.array_equal(to_np(Y_nows), on["Y"]), f"M={M}: forward without a workspace is not the on-load one"
        assert np.array_equal(to_np(Y_ws), off["Y"]), f"M={M}: forward with a workspace is not the dequantize one"
        for name, a, b in (("dX", dX_a, dX_b), ("ds", ds_a, ds_b), ("dz", dz_a, dz_b)):
            assert np.array_equal(to_np(a), off[name]), f"M={M} {name}: backward after a workspace-free forward"
            assert np.array_equal(to_np(b), off[name]), f"M={M} {name}: backward reusing the forward's W-hat"
        rows = np.sort(np.random.default_rng(3).choice(M, min(M, 32), replace=False))
        wrows = np.sort(np.random.default_rng(4).choice(N, 256, replace=False))
        Y_ref = orc.dq_linear_fwd(Xn, packed, zq, s, bits, g, rows=rows)
        dX_ref, ds_ref, dz_ref = orc.dq_linear_bwd(Xn, packed, zq, s, dYn, bits, g, rows=rows, wrows=wrows)
        assert_close(to_np(Y_nows)[rows], Y_ref, TOL_GEMM, "Y")
        assert_close(to_np(dX_b)[rows], dX_ref, TOL_GEMM, "dX")
        assert_close(to_np(ds_b)[wrows], ds_ref, TOL_RED, "ds")
        assert_close(to_np(dz_b)[wrows], dz_ref, TOL_RED, "dz")
