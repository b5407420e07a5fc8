"""One Block-AP training step over the quantized linear layers of a block.

Block-AP trains every parameter of a block (the weights W, the step sizes s, the
zero points z) with AdamW against the full-precision block's outputs, under an
MSE loss; the weights and the quantization parameters have separate learning
rates on cosine schedules (modelfoundations note "EfficientQAT, low-bit training
on a single GPU": Phase 1, "Both phases", "Paper vs. code").

This module strings the library's calls together; every step runs in the CUDA
kernels behind the C ABI:

    for each linear:  dY, loss = fq_linear_fwd_mse(X, W_bf16, s, z, T)   (fused MSE epilogue)
                      dW, ds, dz = fq_linear_bwd(X, W_bf16, s, z, dY)     (straight-through)
    adamw_step over all W (fp32 master, bf16 copy for the next forward), s and z.

The block's other sublayers (norms, attention, the SwiGLU product) are not part of
the method and are not built: each linear is trained against the output of its
own full-precision copy on the same synthetic input, so the loss is the sum of the
per-linear MSEs.  X and T are inputs of the step.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

from . import adamw_step, cosine_lr, fq_linear_bwd, fq_linear_fwd_mse, minmax_init, workspace


@dataclass
class QuantLinearState:
    """Trainable state of one fake-quantized linear: fp32 master W, its bf16 copy (the
    GEMM operand), s and z, and AdamW moments for all three."""
    W_master: torch.Tensor
    W: torch.Tensor
    s: torch.Tensor
    z: torch.Tensor
    moments: dict = field(default_factory=dict)
    ws: torch.Tensor | None = None
    grads: tuple | None = None

    @staticmethod
    def from_weight(W_fp32: torch.Tensor, bits: int, group: int, M: int) -> "QuantLinearState":
        W = W_fp32.to(torch.bfloat16)
        s, z = minmax_init(W, bits, group)
        st = QuantLinearState(W_fp32.clone(), W, s, z)
        for name, t in (("W", st.W_master), ("s", s), ("z", z)):
            st.moments[name] = (torch.zeros_like(t, dtype=torch.float32), torch.zeros_like(t, dtype=torch.float32))
        N, K = W.shape
        st.ws = workspace(M, N, K, bits, group, torch.bfloat16, W.device)
        return st


@dataclass
class BlockAPConfig:
    bits: int = 2
    group: int = 64
    lr_w: float = 2e-5        # weights (2-bit setting of the pages)
    lr_q: float = 1e-4        # step sizes and zero points
    lr_min: float = 0.0       # cosine floor
    total_steps: int = 4096   # schedule length (2 epochs of 4096 samples at batch 2)
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.0


def blockap_step(linears, inputs, targets, cfg: BlockAPConfig, step: int, losses=None, reducer=None):
    """One step (step >= 1).  linears: QuantLinearState per linear; inputs[i] X [M, K_i] bf16,
    targets[i] T [M, N_i] bf16.  Returns the per-linear losses as one fp64 CUDA tensor.
    With data parallelism over tokens, `reducer` (dp.OverlappedGradReducer) averages each
    linear's dW, ds, dz over ranks while the next linear computes."""
    n = len(linears)
    if losses is None:
        losses = torch.empty(n, dtype=torch.float64, device=linears[0].W.device)
    for i, (L, X, T) in enumerate(zip(linears, inputs, targets)):
        dY, _ = fq_linear_fwd_mse(X, L.W, L.s, L.z, T, cfg.bits, cfg.group, ws=L.ws, loss=losses[i:i + 1])
        _, dW, ds, dz = fq_linear_bwd(X, L.W, L.s, L.z, dY, cfg.bits, cfg.group, need_dx=False, ws=L.ws,
                                      out=L.grads, w_hat_in_ws=True)
        L.grads = (None, dW, ds, dz)
        if reducer is not None:
            reducer.submit([dW, ds, dz], tag=i)
    if reducer is not None:
        reducer.wait()
    # the schedules are indexed from 0: step t uses the rate of position t - 1
    lr_w = cosine_lr(cfg.lr_w, cfg.lr_min, step - 1, cfg.total_steps)
    lr_q = cosine_lr(cfg.lr_q, cfg.lr_min, step - 1, cfg.total_steps)
    groups = [dict(lr=lr_w, beta1=cfg.beta1, beta2=cfg.beta2, eps=cfg.eps, weight_decay=cfg.weight_decay),
              dict(lr=lr_q, beta1=cfg.beta1, beta2=cfg.beta2, eps=cfg.eps, weight_decay=cfg.weight_decay)]
    entries = []
    for L in linears:
        _, dW, ds, dz = L.grads
        entries.append((L.W_master, dW, *L.moments["W"], L.W, 0))
        entries.append((L.s, ds, *L.moments["s"], None, 1))
        entries.append((L.z, dz, *L.moments["z"], None, 1))
    for i in range(0, len(entries), 32):
        adamw_step(entries[i:i + 32], groups, step)
    return losses
