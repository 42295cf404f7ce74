"""Parity at full configuration sizes, in the launch configuration bench.py
times, on outputs the oracle can compute one by one (sampled tokens of g_hat,
sampled rows of G_W).

The oracle computes a token's error estimate from its own costs row and the
noise specification, so sampling tokens is exact; a row of G_W is a dot
product over all tokens of the GPU's bf16 g_hat with X, which the oracle
recomputes in double."""
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from activation_perturbation_es_b200 import dust  # noqa: E402
from activation_perturbation_es_b200 import inputs as I  # noqa: E402

pytestmark = pytest.mark.gpu
FP32_TOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dust.lib()


def rel_err(gpu, orc):
    return float(np.max(np.abs(np.asarray(gpu, np.float64) - orc)) / np.max(np.abs(orc)))


def host(t):
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


def test_scaled_workload_as_benchmarked(orc):
    """SCALED (64 x 1024 tokens, 1024 -> 4096, 4096 -> 1024, head d = 1024,
    V = 4096, Vc = 1024, K = 4096): one bench step, then sampled checks."""
    import bench
    w = I.SCALED
    step = bench.Step(w, w.K, rank=0, world=1)
    step.run()
    torch.cuda.synchronize()
    rs = np.random.Generator(np.random.PCG64(11))
    off = I.uniform_offsets(w.n_seq, w.seq_len)
    for L in step.hidden:
        hl = L["hl"]
        toks = np.sort(rs.choice(w.T, 3, replace=False))
        c = host(L["c"])
        g_ref = orc.layer_estimate(c, False, hl.d_out, off, w.gamma, L["nz"].seed, hl.layer, 0, w.K, w.sigma, toks)
        assert rel_err(host(L["g"])[toks], g_ref) < FP32_TOL, hl.name
        rows = rs.choice(hl.d_out, 2, replace=False)
        X = host(L["X"])
        G_ref = orc.weight_grad(host(L["g16"]), X, rows=rows)
        assert rel_err(host(L["G"])[rows], G_ref) < 1e-4, hl.name
    H = step.head
    toks = np.sort(rs.choice(w.T, 3, replace=False))
    Z = host(H["Z"])
    Xh, Wh = host(H["X"]), host(H["W"])
    # the logits GEMM (tensor cores) against the oracle on the sampled rows
    assert rel_err(Z[toks], orc.logits(Xh, Wh, toks)) < 1e-5
    y = host(H["y"])
    _, g_ref = orc.head_step(Z[toks], y[toks], toks, w.Vc, H["nz"].seed, w.head_layer, 0, w.K, w.K, w.sigma,
                             want_c=False)
    assert rel_err(host(H["g"])[toks], g_ref) < FP32_TOL
    rows = rs.choice(w.V, 2, replace=False)
    assert rel_err(host(H["G"])[rows], orc.weight_grad(host(H["g16"]), Xh, rows=rows)) < 1e-4


def test_head_pages_K1024_sampled(orc):
    w = I.HEAD_PAGES
    K = 1024
    h = I.head_inputs(w)
    X, W, y = (torch.from_numpy(h["X"]).cuda().to(torch.bfloat16), torch.from_numpy(h["W"]).cuda().to(torch.bfloat16),
               torch.from_numpy(h["y"]).cuda())
    nz = dust.Noise(w.seed, w.head_layer, 0, K, K, w.sigma)
    out = dust.head_step(y, w.Vc, nz, X=X, W=W, want_c=True)
    toks = np.array([0, 8191, 16383])
    Zs = orc.logits(h["X"], h["W"], toks).astype(np.float32)
    c_ref, g_ref = orc.head_step(Zs, h["y"][toks], toks, w.Vc, nz.seed, nz.layer, 0, K, K, w.sigma)
    assert rel_err(host(out["g_hat"])[toks], g_ref) < FP32_TOL
    assert rel_err(host(out["c"])[:, :, toks], c_ref) < FP32_TOL


def test_hidden_sweep_K16384_sampled(orc):
    """The largest population of the sweep (K = 16384) on the 512 -> 2048 layer."""
    w = I.HIDDEN_SWEEP
    K = 16384
    layer = w.hidden[2]
    li = I.layer_inputs(w, layer)
    off = I.uniform_offsets(w.n_seq, w.seq_len)
    nz = dust.Noise(w.seed, layer.layer, 0, K, K, w.sigma)
    c = dust.synth_costs(torch.from_numpy(li["u"]).cuda(), nz, w.eps_scale)
    goff = torch.from_numpy(off).cuda()
    r = dust.reward_scan(c, goff, w.gamma)
    g, g16 = dust.layer_estimate(r, True, goff, w.gamma, nz, layer.d_out, g_hat_bf16=True)
    G = dust.weight_grad(g16, torch.from_numpy(li["X"]).cuda().to(torch.bfloat16))
    toks = np.array([5, 10000])
    r_h = host(r)
    g_ref = orc.layer_estimate(r_h, True, layer.d_out, off, w.gamma, w.seed, layer.layer, 0, K, w.sigma, toks)
    assert rel_err(host(g)[toks], g_ref) < FP32_TOL
    # the scan at this size against the oracle's recurrence on sampled draws
    ks = np.array([0, 9999, 16383])
    ref = orc.reward_scan(host(c)[ks], off, w.gamma)
    assert rel_err(r_h[ks], ref) < 1e-5
    rows = np.array([0, 2047])
    assert rel_err(host(G)[rows], orc.weight_grad(host(g16), li["X"], rows=rows)) < 1e-4
