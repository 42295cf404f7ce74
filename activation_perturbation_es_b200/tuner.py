"""Choosing sigma and gamma by the cosine criterion, on the library's kernels.

cnblogs Dust explainer, section "真正的工作量：压住干扰" (last paragraph): the
cheap way to set sigma (and gamma) per layer type is to maximise, on a single
batch, the cosine between the Dust estimate and the backprop gradient; a high
single-batch cosine screens candidates, training decides.  Section
"梯度是"长"出来的": the cosine grows with the population as
cos(K) = c_max / sqrt(1 + c/K).

This module only orchestrates calls of the C ABI (head steps over draw
ranges, the head's closed-form backprop gradient, the reward scan, draw
reduction and weight estimate of a hidden layer, the device cosine); the
two-parameter law is fitted on the host from the handful of cosines.  For a
hidden layer the backprop gradient and the perturbed forward belong to the
caller's model, so hidden_sweep takes both from the caller.
With the literal sign of the error equation the estimate approaches
-grad_W, so the cosines are taken against -G_bp.
"""
from __future__ import annotations

import numpy as np
import torch

from . import dust


def _neg_cos(G_W: torch.Tensor, G_bp: torch.Tensor) -> float:
    return float(dust.cosine(G_W, -G_bp)[3].item())


def head_population_sweep(X: torch.Tensor, W: torch.Tensor, targets: torch.Tensor, Vc: int, Ks, sigma: float,
                          seed: int = 0, layer: int = 0, Z: torch.Tensor | None = None):
    """cos(G_W(K), -G_bp) for increasing populations K (one pass over the
    largest K: the draws are added range by range with accumulate = 1; the
    cosine does not depend on the 1/(K sigma) scale).  Returns (Ks, cosines)."""
    Ks = sorted(int(k) for k in Ks)
    if Z is None:
        Z = dust.logits(X, W)
    G_bp = dust.head_bp_grad(Z, targets, X)
    K_max = Ks[-1]
    g = None
    coss, prev = [], 0
    G_W = torch.empty(W.shape[0], X.shape[1], dtype=torch.float32, device=X.device)
    g16 = torch.empty(Z.shape, dtype=torch.bfloat16, device=X.device) if X.dtype == torch.bfloat16 else None
    for K in Ks:
        nz = dust.Noise(seed, layer, prev, K - prev, K_max, sigma)
        out = dust.head_step(targets, Vc, nz, Z=Z, g_hat=g, g_hat_bf16=g16, accumulate=g is not None)
        g = out["g_hat"]
        dust.weight_grad(g16 if g16 is not None else g, X, G_W=G_W)
        coss.append(_neg_cos(G_W, G_bp))
        prev = K
    return np.array(Ks), np.array(coss)


def head_sigma_sweep(X, W, targets, Vc: int, K: int, sigmas, seed: int = 0, layer: int = 0, Z=None):
    """cos(G_W, -G_bp) at population K for each sigma; returns (sigmas, cosines, best sigma)."""
    if Z is None:
        Z = dust.logits(X, W)
    G_bp = dust.head_bp_grad(Z, targets, X)
    coss = []
    for s in sigmas:
        out = dust.head_step(targets, Vc, dust.Noise(seed, layer, 0, K, K, float(s)), Z=Z, X=X, want_G_W=True,
                             want_bf16=X.dtype == torch.bfloat16)
        coss.append(_neg_cos(out["G_W"], G_bp))
    coss = np.array(coss)
    return np.array(sigmas, dtype=float), coss, float(np.asarray(sigmas)[int(np.argmax(coss))])


def cosine_with(G_W: torch.Tensor, G_ref: torch.Tensor) -> float:
    """cos(G_W, G_ref) on the device (fixed-order double reduction)."""
    return float(dust.cosine(G_W.contiguous(), G_ref.contiguous())[3].item())


def hidden_sweep(costs_fn, X: torch.Tensor, seq_offsets: torch.Tensor, d_out: int, G_ref: torch.Tensor, K: int,
                 sigmas, gammas, seed: int = 0, layer: int = 0):
    """sigma and gamma of a hidden layer by the cosine criterion.

    costs_fn(noise) -> c [draw_count][T] fp32 (device) is the caller's scoring of
    its perturbed forward for the draws of `noise` (c = l~ - l per token): the
    library cannot run a model's suffix, so the caller supplies it, as it
    supplies G_ref, its backprop gradient of the summed loss w.r.t. the
    layer's weights ([d_out][d_in] fp32; pass -grad_W, the direction the
    estimate approaches, or grad_W and read the cosines negated).  For each
    sigma the costs are scored once; every gamma then reuses them through the
    reward scan (a4), the draw reduction (a5) and the weight estimate (a6).
    Returns (sigmas, gammas, cosines [len(sigmas)][len(gammas)], (best sigma, best gamma))."""
    sigmas = [float(x) for x in sigmas]
    gammas = [float(x) for x in gammas]
    coss = np.zeros((len(sigmas), len(gammas)))
    G_W = torch.empty(d_out, X.shape[1], dtype=torch.float32, device=X.device)
    for i, s in enumerate(sigmas):
        nz = dust.Noise(seed, layer, 0, K, K, s)
        c = costs_fn(nz)
        for j, gm in enumerate(gammas):
            g, g16 = dust.layer_estimate(c, False, seq_offsets, gm, nz, d_out,
                                         g_hat_bf16=X.dtype == torch.bfloat16)
            dust.weight_grad(g16 if g16 is not None else g, X, G_W=G_W)
            coss[i, j] = cosine_with(G_W, G_ref)
    i, j = np.unravel_index(int(np.argmax(coss)), coss.shape)
    return np.array(sigmas), np.array(gammas), coss, (sigmas[i], gammas[j])


def fit_cosine_law(Ks, coss):
    """Least-squares fit of cos(K) = c_max / sqrt(1 + c/K): with y = 1/cos^2,
    y = (1 + c/K) / c_max^2 is linear in 1/K.  Returns (c_max, c)."""
    Ks = np.asarray(Ks, dtype=float)
    y = 1.0 / np.asarray(coss, dtype=float) ** 2
    A = np.stack([np.ones_like(Ks), 1.0 / Ks], axis=1)
    (a0, a1), *_ = np.linalg.lstsq(A, y, rcond=None)
    c_max = 1.0 / np.sqrt(a0)
    return float(c_max), float(a1 / a0)
