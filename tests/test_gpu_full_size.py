"""Parity at full configuration sizes, in the launch configuration bench.py
times, on outputs the oracle can compute one by one.

Every oracle input comes from the seeded generators: the benchmarked step's
costs are replaced by seeded costs before it runs, so the oracle can follow
the same chain (scan -> reduction -> weight estimate) from the same bytes.
Sampled draws of r, sampled tokens of g_hat (16 per layer) and sampled rows of
G_W (8 per layer: the oracle's g over every token at those channels, rounded
as the kernels round it) are checked.  For the scaled head a vocabulary column
of g over its 65536 tokens x 4096 draws is beyond the oracle, so its G_W is
checked as the weight GEMM of its g; the pages-shaped head's G_W rows
(16384 tokens, K = 64) are checked against the oracle's chain in
test_gpu_parity."""
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from activation_perturbation_es_b200 import dust  # noqa: E402
from activation_perturbation_es_b200 import inputs as I  # noqa: E402

import oracle_chains  # noqa: E402

pytestmark = pytest.mark.gpu
FP32_TOL = 1e-3
BF16_G_TOL = 1e-3      # G_W rows from bf16 g: rounding decisions may differ at binary32 ties


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dust.lib()


def rel_err(gpu, orc):
    return float(np.max(np.abs(np.asarray(gpu, np.float64) - orc)) / np.max(np.abs(orc)))


def host(t):
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


def _bench_step_on_seeded_costs(w, K, seed0):
    """One bench step of workload w at population K with the hidden layers'
    costs replaced by seeded ones (returned, for the oracle)."""
    import bench
    step = bench.Step(w, K, rank=0, world=1)
    costs = []
    for i, L in enumerate(step.hidden):
        c = I.normal((K, w.T), 0.02, seed=seed0 + i)
        L["c"].copy_(torch.from_numpy(c))
        costs.append(c)
    step.run()
    torch.cuda.synchronize()
    return step, costs


def _check_hidden_layers(orc, w, K, step, costs, rs, n_tok=16, n_rows=8):
    off = I.uniform_offsets(w.n_seq, w.seq_len)
    for L, c in zip(step.hidden, costs):
        hl = L["hl"]
        ks = rs.choice(K, 3, replace=False)
        assert rel_err(host(L["r"])[ks], orc.reward_scan(c[ks], off, w.gamma)) < 1e-5, hl.name
        toks = np.sort(rs.choice(w.T, n_tok, replace=False))
        g_ref = orc.layer_estimate(c, False, hl.d_out, off, w.gamma, L["nz"].seed, hl.layer, 0, K, w.sigma, toks)
        assert rel_err(host(L["g"])[toks], g_ref) < FP32_TOL, hl.name
        rows = np.sort(rs.choice(hl.d_out, n_rows, replace=False))
        G_ref = oracle_chains.weight_rows(orc, c, False, hl.d_out, off, w.gamma, L["nz"].seed, hl.layer, 0, K,
                                          w.sigma, host(L["X"]), rows)
        assert rel_err(host(L["G"])[rows], G_ref) < BF16_G_TOL, hl.name


@pytest.mark.parametrize("gamma", [None, 0.0])
def test_scaled_workload_as_benchmarked(orc, gamma):
    """SCALED (64 x 1024 tokens, 1024 -> 4096, 4096 -> 1024, head d = 1024,
    V = 4096, Vc = 1024, K = 4096): one bench step on seeded costs, with the
    workload's discount gamma = 0.99 and with gamma = 0 (r = c), then sampled
    checks of every layer, the head's costs included."""
    import dataclasses
    w = I.SCALED if gamma is None else dataclasses.replace(I.SCALED, gamma=gamma)
    step, costs = _bench_step_on_seeded_costs(w, w.K, 500)
    rs = np.random.Generator(np.random.PCG64(11))
    _check_hidden_layers(orc, w, w.K, step, costs, rs)
    if gamma is not None:
        return                                   # the head does not depend on the hidden layers' gamma
    H = step.head
    toks = np.sort(rs.choice(w.T, 16, replace=False))
    Xh, Wh = host(H["X"]), host(H["W"])
    Z_orc = orc.logits(Xh, Wh, toks)
    # the logits GEMM (tensor cores) against the oracle on the sampled rows
    assert rel_err(host(H["Z"])[toks], Z_orc) < 1e-5
    y = host(H["y"])
    c_ref, g_ref = orc.head_step(Z_orc.astype(np.float32), y[toks], toks, w.Vc, H["nz"].seed, w.head_layer, 0, w.K,
                                 w.K, w.sigma, want_c=True)
    assert rel_err(host(H["g"])[toks], g_ref) < FP32_TOL
    # the costs of the benchmarked head (the timed step does not write them out):
    # the same call with c requested, on the same cached logits
    out = dust.head_step(H["y"], w.Vc, H["nz"], Z=H["Z"], want_c=True)
    assert torch.equal(out["g_hat"], H["g"])
    assert rel_err(host(out["c"][:, :, torch.from_numpy(toks).cuda()]), c_ref) < FP32_TOL
    G2 = dust.weight_grad(H["g16"], H["X"])
    assert rel_err(host(H["G"]), host(G2).astype(np.float64)) < 1e-6


def test_hidden_sweep_K1024_all_layers(orc):
    """HIDDEN_SWEEP at K = 1024 (16 x 1024 tokens; 512 -> 1536, 512 -> 512,
    512 -> 2048, 2048 -> 512; gamma 0.95), as benchmarked: every layer."""
    w = I.HIDDEN_SWEEP
    step, costs = _bench_step_on_seeded_costs(w, 1024, 700)
    _check_hidden_layers(orc, w, 1024, step, costs, np.random.Generator(np.random.PCG64(12)))


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
    """The largest population of the sweep (K = 16384) on the 512 -> 2048 layer,
    on seeded costs: scan rows, estimate tokens and weight rows."""
    w = I.HIDDEN_SWEEP
    K = 16384
    layer = w.hidden[2]
    li = I.layer_inputs(w, layer)
    off = I.uniform_offsets(w.n_seq, w.seq_len)
    nz = dust.Noise(w.seed, layer.layer, 0, K, K, w.sigma)
    c = I.normal((K, w.T), 0.02, seed=77)
    goff = torch.from_numpy(off).cuda()
    r = dust.reward_scan(torch.from_numpy(c).cuda(), goff, w.gamma)
    g, g16 = dust.layer_estimate(r, True, goff, w.gamma, nz, layer.d_out, g_hat_bf16=True)
    G = dust.weight_grad(g16, torch.from_numpy(li["X"]).cuda().to(torch.bfloat16))
    ks = np.array([0, 9999, 16383])
    assert rel_err(host(r)[ks], orc.reward_scan(c[ks], off, w.gamma)) < 1e-5
    toks = np.array([5, 10000])
    g_ref = orc.layer_estimate(c, False, layer.d_out, off, w.gamma, w.seed, layer.layer, 0, K, w.sigma, toks)
    assert rel_err(host(g)[toks], g_ref) < FP32_TOL
    rows = np.array([0, 2047])
    G_ref = oracle_chains.weight_rows(orc, c, False, layer.d_out, off, w.gamma, w.seed, layer.layer, 0, K, w.sigma,
                                      li["X"], rows)
    assert rel_err(host(G)[rows], G_ref) < BF16_G_TOL
