"""Float64 torch autograd through the toy causal suffix: the comparator of the
end-to-end convergence pins (test helper; it shares no code with the oracle
or the library).

The suffix is the hidden-layer workload's model: y = X W^T; one causal softmax
attention head per sequence (q, k, v = y Wq^T, y Wk^T, y Wv^T, scores scaled
by 1/sqrt(dh)) on a residual stream h = y + o Wo^T; logits z = h Wout^T;
per-token cross entropy.  Autograd differentiates it exactly, so it gives

  J[s][t] = dl_s / dy_t                      (one backward per s),
  g_gamma[t] = -sum_{s >= t, same sequence} gamma^(s-t) J[s][t],
  G_gamma = g_gamma^T X,

the first-order expectation of the Dust estimate with discount gamma (cnblogs
Dust explainer, section "信用分配：一次前向，两种奖励": reward, error and
weight equations), and -grad_W sum_t l_t, which G_1 equals because the causal
mask makes dl_s/dy_t vanish for s < t.
"""
from __future__ import annotations

import numpy as np
import torch


def _t(a):
    return torch.tensor(np.asarray(a, np.float64))


def suffix_losses(Y: torch.Tensor, p: dict) -> torch.Tensor:
    """Per-token clean losses of the suffix for the layer output Y [T][d] (float64)."""
    q, k, v = Y @ _t(p["Wq"]).T, Y @ _t(p["Wk"]).T, Y @ _t(p["Wv"]).T
    dh = q.shape[1]
    off = np.asarray(p["off"])
    outs = []
    for s in range(len(off) - 1):
        a, b = int(off[s]), int(off[s + 1])
        sc = q[a:b] @ k[a:b].T / np.sqrt(dh)
        sc = sc.masked_fill(torch.triu(torch.ones(b - a, b - a, dtype=torch.bool), 1), float("-inf"))
        outs.append(torch.softmax(sc, dim=1) @ v[a:b])
    o = torch.cat(outs)
    h = Y + o @ _t(p["Wo"]).T
    z = h @ _t(p["Wout"]).T
    T = Y.shape[0]
    return torch.logsumexp(z, dim=1) - z[torch.arange(T), torch.tensor(np.asarray(p["y"], np.int64))]


def clean_losses(p: dict) -> np.ndarray:
    with torch.no_grad():
        return suffix_losses(_t(p["X"]) @ _t(p["W"]).T, p).numpy()


def backprop_gradient(p: dict) -> np.ndarray:
    """grad_W sum_t l_t, [d][d_in]."""
    W = _t(p["W"]).requires_grad_(True)
    suffix_losses(_t(p["X"]) @ W.T, p).sum().backward()
    return W.grad.numpy()


def loss_jacobian(p: dict) -> np.ndarray:
    """J[s][t][j] = dl_s / dy_t[j] by one backward per s."""
    Y = (_t(p["X"]) @ _t(p["W"]).T).detach().requires_grad_(True)
    L = suffix_losses(Y, p)
    T = Y.shape[0]
    J = np.zeros((T,) + tuple(Y.shape))
    for s in range(T):
        (g,) = torch.autograd.grad(L[s], Y, retain_graph=True)
        J[s] = g.numpy()
    return J


def discounted_gradient(p: dict, J: np.ndarray, gamma: float):
    """(G_gamma [d][d_in], g_gamma [T][d]) by the double sum over s >= t in each sequence."""
    T, d = J.shape[1], J.shape[2]
    g = np.zeros((T, d))
    off = np.asarray(p["off"])
    for q in range(len(off) - 1):
        for t in range(int(off[q]), int(off[q + 1])):
            for s in range(t, int(off[q + 1])):
                g[t] -= gamma ** (s - t) * J[s][t]
    return g.T @ np.asarray(p["X"], np.float64), g


def tiny_problem(seed: int = 30, n_seq: int = 2, seq_len: int = 16, d_in: int = 8, d: int = 16, dh: int = 8,
                 V: int = 12) -> dict:
    """The hidden-layer workload's model at a size the brute force handles: 2 sequences
    of 16 tokens, X ~ N(0, 1), every weight ~ N(0, 1/fan_in), uniform targets."""
    r = np.random.Generator(np.random.PCG64(seed))
    f = lambda s, *shape: (r.standard_normal(shape) * s).astype(np.float32)
    T = n_seq * seq_len
    return dict(X=f(1.0, T, d_in), W=f(1 / np.sqrt(d_in), d, d_in), Wq=f(1 / np.sqrt(d), dh, d),
                Wk=f(1 / np.sqrt(d), dh, d), Wv=f(1 / np.sqrt(d), dh, d), Wo=f(1 / np.sqrt(dh), d, dh),
                Wout=f(1 / np.sqrt(d), V, d), y=r.integers(0, V, T).astype(np.int32),
                off=np.arange(0, T + 1, seq_len).astype(np.int32))
