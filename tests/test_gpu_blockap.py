"""GPU parity of the Block-AP step pieces against the CPU oracle: the forward with
the fused reconstruction-loss epilogue, the multi-tensor AdamW kernel, and a few
composed steps over several linears."""
import numpy as np
import pytest
import torch

import weight_quantization_aware_b200 as eqat
from weight_quantization_aware_b200 import synthetic
from weight_quantization_aware_b200.blockap import BlockAPConfig, QuantLinearState, blockap_step
from parity import TOL_GEMM, assert_close, bf16_round, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from weight_quantization_aware_b200 import build
    build.build()
    eqat.load_library()
    assert torch.cuda.is_available()
    yield
    assert eqat.device_error() == 0


def fp_target(Xn, Wn, dtype):
    """The full-precision output the quantized layer is trained to reproduce."""
    return synthetic.to_dtype((Xn.astype(np.float64) @ Wn.astype(np.float64).T).astype(np.float32), dtype)


@pytest.mark.parametrize("shape", [(300, 392, 384, 2, 64, "bf16"), (257, 136, 640, 3, 128, "bf16"),
                                   (64, 520, 256, 4, 32, "bf16"), (77, 24, 96, 2, 32, "f32"),
                                   (128, 64, 128, 3, 64, "f32")], ids=lambda s: "x".join(map(str, s)))
def test_fq_linear_fwd_mse(orc, shape):
    M, N, K, bits, g, dtype = shape
    d = synthetic.draw_linear(np.random.default_rng(40 + M), M, N, K, 0.02, dtype)
    Xn, Wn = synthetic.as_f32_numpy(d["X"]), synthetic.as_f32_numpy(d["W"])
    T = fp_target(Xn, Wn, dtype)
    Tn = synthetic.as_f32_numpy(T)
    s, z = orc.minmax_init(Wn, bits, g)
    s, z = synthetic.perturb_quant_params(s, z, M)
    dY, loss = eqat.fq_linear_fwd_mse(d["X"].cuda(), d["W"].cuda(), torch.from_numpy(s).cuda(),
                                      torch.from_numpy(z).cuda(), T.cuda(), bits, g)
    Y_ref = orc.fq_linear_fwd(Xn, Wn, s, z, bits, g)
    l_ref, dY_ref = orc.mse_grad(Y_ref, Tn)
    assert_close(to_np(dY), dY_ref, TOL_GEMM, "dY")
    assert abs(loss.item() - l_ref) <= TOL_GEMM * l_ref
    if dtype == "bf16":
        # with W-hat rounded to bf16 as the kernel's operand, the loss is the oracle's to fp32 sums
        wh = bf16_round(orc.fake_quant(Wn, s, z, bits, g)[0])
        l_b, _ = orc.mse_grad(orc.linear_fwd(Xn, wh), Tn)
        assert abs(loss.item() - l_b) <= 1e-4 * l_b


def test_fq_linear_fwd_mse_k_zero(orc):
    for dtype, tdt in (("bf16", torch.bfloat16), ("f32", torch.float32)):
        T = torch.randn(16, 8, dtype=torch.float32).to(tdt)
        X = torch.empty(16, 0, dtype=tdt)
        W = torch.empty(8, 0, dtype=tdt)
        s = torch.empty(8, 0, dtype=torch.float32)
        dY, loss = eqat.fq_linear_fwd_mse(X.cuda(), W.cuda(), s.cuda(), s.cuda(), T.cuda(), 2, 64)
        Tn = T.float().numpy()
        l_ref, dY_ref = orc.mse_grad(np.zeros_like(Tn), Tn)
        assert_close(to_np(dY), dY_ref, 1e-2, "dY")
        assert abs(loss.item() - l_ref) <= 1e-6 * l_ref


def test_adamw_kernel_matches_oracle(orc):
    rng = np.random.default_rng(8)
    sizes = [4096 * 3 + 5, 7, 4096, 13, 64 * 37]
    gdt = [torch.bfloat16, torch.float32, torch.bfloat16, torch.float32, torch.float32]
    groups = [dict(lr=2e-5, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01),
              dict(lr=1e-4, beta1=0.8, beta2=0.99, eps=1e-6, weight_decay=0.0)]
    gidx = [0, 1, 0, 1, 1]
    host = []
    dev = []
    for n, gd, gi in zip(sizes, gdt, gidx):
        p = (rng.standard_normal(n) * 0.02).astype(np.float32)
        host.append([p, np.zeros(n, np.float32), np.zeros(n, np.float32)])
        dev.append([torch.from_numpy(p).cuda(), torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda"),
                    torch.empty(n, dtype=torch.bfloat16, device="cuda") if gd == torch.bfloat16 else None])
    for t in range(1, 4):
        entries = []
        grads = []
        for i, (n, gd, gi) in enumerate(zip(sizes, gdt, gidx)):
            g = torch.from_numpy((rng.standard_normal(n) * 0.1).astype(np.float32)).to(gd)
            grads.append(g.float().numpy())
            p, m, v, c = dev[i]
            entries.append((p, g.cuda(), m, v, c, gi))
        eqat.adamw_step(entries, groups, t)
        for i, gi in enumerate(gidx):
            gr = groups[gi]
            host[i] = list(orc.adamw(*host[i][:1], grads[i], host[i][1], host[i][2], gr["lr"], gr["beta1"],
                                     gr["beta2"], gr["eps"], gr["weight_decay"], t))
    for i, gi in enumerate(gidx):
        p, m, v, c = (to_np(x) if x is not None else None for x in dev[i])
        pr, mr, vr = host[i]
        lr = groups[gi]["lr"]
        assert np.abs(p - pr).max() <= 4 * np.spacing(np.abs(pr).max()) + 1e-3 * lr
        assert np.abs(m - mr).max() <= 1e-6 * np.abs(mr).max()
        np.testing.assert_allclose(v, vr, rtol=1e-5, atol=1e-20)
        if c is not None:
            assert (c == bf16_round(p)).all()


def test_blockap_steps_match_oracle(orc):
    """Three composed steps over three linears (ragged shapes): losses, and the moves of
    W, s and z against the oracle running the same algorithm in fp64 on fp32 state."""
    cfg = BlockAPConfig(bits=2, group=64, total_steps=10, weight_decay=0.0)
    M = 192
    shapes = [(136, 256), (264, 384), (128, 640)]
    rng = np.random.default_rng(99)
    lin, Xs, Ts, ref = [], [], [], []
    for N, K in shapes:
        d = synthetic.draw_linear(rng, M, N, K, 0.02, "bf16")
        Xn, Wn = synthetic.as_f32_numpy(d["X"]), synthetic.as_f32_numpy(d["W"])
        T = fp_target(Xn, Wn, "bf16")
        L = QuantLinearState.from_weight(d["W"].float().cuda(), cfg.bits, cfg.group, M)
        lin.append(L)
        Xs.append(d["X"].cuda())
        Ts.append(T.cuda())
        s0, z0 = orc.minmax_init(Wn, cfg.bits, cfg.group)
        assert_close(to_np(L.s), s0, 0, "s init")
        ref.append({"X": Xn, "T": synthetic.as_f32_numpy(T), "W": Wn.copy(), "s": s0, "z": z0,
                    "mW": np.zeros_like(Wn), "vW": np.zeros_like(Wn), "ms": np.zeros_like(s0),
                    "vs": np.zeros_like(s0), "mz": np.zeros_like(z0), "vz": np.zeros_like(z0)})
    W0 = [r["W"].copy() for r in ref]
    s0 = [r["s"].copy() for r in ref]
    z0 = [r["z"].copy() for r in ref]
    for t in range(1, 4):
        losses = to_np(blockap_step(lin, Xs, Ts, cfg, t))
        lr_w = orc.cosine_lr(cfg.lr_w, cfg.lr_min, t - 1, cfg.total_steps)
        lr_q = orc.cosine_lr(cfg.lr_q, cfg.lr_min, t - 1, cfg.total_steps)
        for i, r in enumerate(ref):
            Wb = bf16_round(r["W"])  # the forward reads the bf16 copy of W
            Y = orc.fq_linear_fwd(r["X"], Wb, r["s"], r["z"], cfg.bits, cfg.group)
            l_ref, dY = orc.mse_grad(Y, r["T"])
            assert abs(losses[i] - l_ref) <= TOL_GEMM * l_ref
            dwh = orc.linear_dwhat(dY.astype(np.float32), r["X"])
            dW, ds, dz = orc.ste_grads(Wb, r["s"], r["z"], dwh, cfg.bits, cfg.group)
            r["W"], r["mW"], r["vW"] = orc.adamw(r["W"], dW, r["mW"], r["vW"], lr_w, 0.9, 0.999, 1e-8, 0.0, t)
            r["s"], r["ms"], r["vs"] = orc.adamw(r["s"], ds, r["ms"], r["vs"], lr_q, 0.9, 0.999, 1e-8, 0.0, t)
            r["z"], r["mz"], r["vz"] = orc.adamw(r["z"], dz, r["mz"], r["vz"], lr_q, 0.9, 0.999, 1e-8, 0.0, t)
    for i, (L, r) in enumerate(zip(lin, ref)):
        # Adam moves each parameter by about lr per step, with the sign of its gradient's
        # running mean: compare the moves; a tiny gradient may flip sign between the
        # bf16 kernel and the fp64 oracle, so allow that on a small fraction
        for got, want, start, lr, moves in ((to_np(L.W_master), r["W"], W0[i], cfg.lr_w, True),
                                            (to_np(L.s), r["s"], s0[i], cfg.lr_q, True),
                                            (to_np(L.z), r["z"], z0[i], cfg.lr_q, False)):
            move_g, move_r = got - start, want - start
            if moves:
                assert np.abs(move_r).max() > 0.5 * lr
            err = np.abs(move_g - move_r)
            assert err.max() <= 2.01 * 3 * lr
            assert np.mean(err <= 0.05 * 3 * lr) >= 0.95
        assert (to_np(L.W) == bf16_round(to_np(L.W_master))).all()


def test_blockap_steps_trained_state_match_oracle_per_element(orc):
    """Three composed steps from a trained-like state (s shrunk, z shifted: a few
    percent of the weights clamp, so dz != 0 and z must move), with a per-element
    bound on the moves of W, s and z against the oracle.

    Elements whose oracle gradient stays well away from zero at every step must move
    as the oracle's do to within a tenth of one learning-rate step per step; there the
    kernels' error cannot flip the sign of Adam's update.  "Well away" is measured
    against each tensor's own largest gradient at that step, at the scale of its
    tolerance: a tenth of it for dW (bf16 GEMM, 2e-2 of the largest), a hundredth for
    ds and dz (fp32 reductions, 1e-3 of the largest).  The rest (gradients within
    rounding of zero) keep the global bound of one flipped update per step."""
    cfg = BlockAPConfig(bits=2, group=64, total_steps=10, weight_decay=0.0)
    M = 192
    shapes = [(136, 256), (264, 384)]
    rng = np.random.default_rng(123)
    lin, Xs, Ts, ref = [], [], [], []
    for i, (N, K) in enumerate(shapes):
        d = synthetic.draw_linear(rng, M, N, K, 0.02, "bf16")
        Xn, Wn = synthetic.as_f32_numpy(d["X"]), synthetic.as_f32_numpy(d["W"])
        T = fp_target(Xn, Wn, "bf16")
        L = QuantLinearState.from_weight(d["W"].float().cuda(), cfg.bits, cfg.group, M)
        s0, z0 = orc.minmax_init(Wn, cfg.bits, cfg.group)
        s0, z0 = synthetic.perturb_quant_params(s0, z0, 31 + i)
        L.s.copy_(torch.from_numpy(s0))
        L.z.copy_(torch.from_numpy(z0))
        lin.append(L)
        Xs.append(d["X"].cuda())
        Ts.append(T.cuda())
        ref.append({"X": Xn, "T": synthetic.as_f32_numpy(T), "W": Wn.copy(), "s": s0.copy(), "z": z0.copy(),
                    "mW": np.zeros_like(Wn), "vW": np.zeros_like(Wn), "ms": np.zeros_like(s0),
                    "vs": np.zeros_like(s0), "mz": np.zeros_like(z0), "vz": np.zeros_like(z0),
                    "g": {"W": [], "s": [], "z": []}})
    start = [(r["W"].copy(), r["s"].copy(), r["z"].copy()) for r in ref]
    for t in range(1, 4):
        blockap_step(lin, Xs, Ts, cfg, t)
        lr_w = orc.cosine_lr(cfg.lr_w, cfg.lr_min, t - 1, cfg.total_steps)
        lr_q = orc.cosine_lr(cfg.lr_q, cfg.lr_min, t - 1, cfg.total_steps)
        for r in ref:
            Wb = bf16_round(r["W"])
            Y = orc.fq_linear_fwd(r["X"], Wb, r["s"], r["z"], cfg.bits, cfg.group)
            _, dY = orc.mse_grad(Y, r["T"])
            dwh = orc.linear_dwhat(dY.astype(np.float32), r["X"])
            dW, ds, dz = orc.ste_grads(Wb, r["s"], r["z"], dwh, cfg.bits, cfg.group)
            for name, g in (("W", dW), ("s", ds), ("z", dz)):
                r["g"][name].append(np.asarray(g, dtype=np.float64))
            r["W"], r["mW"], r["vW"] = orc.adamw(r["W"], dW, r["mW"], r["vW"], lr_w, 0.9, 0.999, 1e-8, 0.0, t)
            r["s"], r["ms"], r["vs"] = orc.adamw(r["s"], ds, r["ms"], r["vs"], lr_q, 0.9, 0.999, 1e-8, 0.0, t)
            r["z"], r["mz"], r["vz"] = orc.adamw(r["z"], dz, r["mz"], r["vz"], lr_q, 0.9, 0.999, 1e-8, 0.0, t)
    for i, (L, r) in enumerate(zip(lin, ref)):
        assert np.abs(np.stack(r["g"]["z"])).max() > 0, "the trained-state case must clamp"
        for name, got, lr, frac in (("W", to_np(L.W_master), cfg.lr_w, 0.1), ("s", to_np(L.s), cfg.lr_q, 0.01),
                                    ("z", to_np(L.z), cfg.lr_q, 0.01)):
            st = start[i][{"W": 0, "s": 1, "z": 2}[name]]
            move_g, move_r = got - st, r[name] - st
            gs = np.stack(r["g"][name])  # [steps, ...]
            scale = np.abs(gs).reshape(gs.shape[0], -1).max(axis=1).reshape((-1,) + (1,) * (gs.ndim - 1))
            firm = (np.abs(gs) >= frac * scale).all(axis=0)
            err = np.abs(move_g - move_r)
            assert firm.sum() >= 16, f"{name}: too few elements with firm gradients ({firm.sum()} of {firm.size})"
            assert err[firm].max() <= 0.1 * 3 * lr, \
                f"{name}: move error {err[firm].max():.3e} on firm elements > {0.3 * lr:.3e}"
            assert err.max() <= 2.01 * 3 * lr
            if name == "z":
                moved = firm & (np.abs(move_r) > 0.5 * lr)
                assert moved.any() and (np.abs(move_g[moved]) > 0.5 * lr).all(), "z must move where the oracle's does"
        assert (to_np(L.W) == bf16_round(to_np(L.W_master))).all()


def test_blockap_step_with_overlapped_reducer_single_rank():
    """The NCCL stream plumbing of the overlapped gradient exchange, on one rank (the mean
    over one rank is the identity): the step gives the same state as without it."""
    import os
    import subprocess
    import sys
    code = r'''
import os, torch, numpy as np, torch.distributed as dist
import weight_quantization_aware_b200 as eqat
from weight_quantization_aware_b200 import dp
from weight_quantization_aware_b200.blockap import BlockAPConfig, QuantLinearState, blockap_step
os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=os.environ["PORT"])
torch.cuda.set_device(0)
dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
cfg = BlockAPConfig(total_steps=10)
g = torch.Generator(device="cuda"); g.manual_seed(5)
def make():
    Ls, Xs, Ts = [], [], []
    for N, K in ((136, 256), (128, 384)):
        g.manual_seed(N * K)
        W = torch.randn(N, K, generator=g, device="cuda") * 0.02
        X = torch.randn(64, K, generator=g, device="cuda").to(torch.bfloat16)
        Ls.append(QuantLinearState.from_weight(W, 2, 64, 64)); Xs.append(X); Ts.append(X @ W.to(torch.bfloat16).t())
    return Ls, Xs, Ts
A = make(); B = make()
red = dp.OverlappedGradReducer(dist, device="cuda")
for t in range(1, 4):
    blockap_step(*A, cfg, t)
    blockap_step(*B, cfg, t, reducer=red)
torch.cuda.synchronize()
for a, b in zip(A[0], B[0]):
    assert torch.equal(a.W_master, b.W_master) and torch.equal(a.s, b.s) and torch.equal(a.z, b.z)
assert red.order == [0, 1] * 3
dist.destroy_process_group()
print("ok")
'''
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env=dict(os.environ, PORT=str(port), PYTHONPATH=root,
                                                                         NCCL_NVLS_ENABLE="0"),
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout[-2000:] + r.stderr[-3000:]
