"""Attention-internal scoring on the GPU against the oracle, and the estimate
built on it (reward scan with gamma = 1, draw reduction over the dh
projection channels, weight estimate against the projection's input)."""
import numpy as np
import pytest
import torch

from activation_perturbation_es_b200 import dust
from activation_perturbation_es_b200 import inputs as I

import oracle_chains  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dust.lib()


def rel_err(gpu, orc):
    return float(np.max(np.abs(np.asarray(gpu, np.float64) - orc)) / np.max(np.abs(orc)))


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _block(T=1024, n_seq=4, d=256, dh=64, seed=50):
    r = np.random.Generator(np.random.PCG64(seed))
    f = lambda *s, sc=1.0: (r.standard_normal(s) * sc).astype(np.float32)
    return dict(Y=f(T, d), Wq=f(dh, d, sc=d ** -0.5), Wk=f(dh, d, sc=d ** -0.5), Wv=f(dh, d, sc=d ** -0.5),
                Wo=f(d, dh, sc=dh ** -0.5), G=f(T, d, sc=0.1), off=I.uniform_offsets(n_seq, T // n_seq))


@pytest.mark.parametrize("which", [0, 1, 2])
def test_attention_costs_parity(orc, which):
    p = _block()
    nz = dust.Noise(3, 20 + which, 7, 5, 5, 0.01)
    c = dust.attention_internal_costs(cu(p["Y"]), cu(p["off"]), cu(p["Wq"]), cu(p["Wk"]), cu(p["Wv"]), cu(p["Wo"]),
                                      which, cu(p["G"]), nz).cpu().numpy()
    ref = orc.attention_internal_costs(p["Y"], p["off"], p["Wq"], p["Wk"], p["Wv"], p["Wo"], which, p["G"], 3,
                                       20 + which, 0.01, np.arange(7, 12))
    # c is a difference of attention outputs (perturbed minus clean) in fp32
    assert rel_err(c, ref) < 1e-3


def test_value_projection_estimate_end_to_end(orc):
    """The value projection's costs for every draw against the oracle's, then
    the estimator and the weight estimate on the oracle's costs."""
    p = _block(seed=51)
    K, dh = 48, 64
    nz = dust.Noise(4, 22, 0, K, K, 0.01)
    goff = cu(p["off"])
    c = dust.attention_internal_costs(cu(p["Y"]), goff, cu(p["Wq"]), cu(p["Wk"]), cu(p["Wv"]), cu(p["Wo"]), 2,
                                      cu(p["G"]), nz)
    c_orc = orc.attention_internal_costs(p["Y"], p["off"], p["Wq"], p["Wk"], p["Wv"], p["Wo"], 2, p["G"], 4, 22,
                                         0.01, np.arange(K)).astype(np.float32)
    assert rel_err(c.cpu().numpy(), c_orc) < 1e-3
    g, _ = dust.layer_estimate(cu(c_orc), False, goff, 1.0, nz, dh)
    G_W = dust.weight_grad(g, cu(p["Y"]))                  # the value projection's input is Y
    toks = np.array([0, 255, 256, 1023])
    g_ref = orc.layer_estimate(c_orc, False, dh, p["off"], 1.0, 4, 22, 0, K, 0.01, toks)
    assert rel_err(g.cpu().numpy()[toks], g_ref) < 1e-3
    rows = np.array([0, 63])
    G_ref = oracle_chains.weight_rows(orc, c_orc, False, dh, p["off"], 1.0, 4, 22, 0, K, 0.01, p["Y"], rows,
                                      bf16=False)
    assert rel_err(G_W.cpu().numpy()[rows], G_ref) < 1e-4


def test_value_estimate_converges_through_uniform_attention():
    """Wq = Wk = 0: E[g_hat_t] = sum_{s >= t} (G_s Wo) / n_s (backprop of <z, G> to v_t)."""
    T, d, dh, K, sigma = 64, 16, 16, 65536, 0.05
    p = _block(T=T, n_seq=2, d=d, dh=dh, seed=52)
    p["Wq"][:] = 0
    p["Wk"][:] = 0
    off = p["off"]
    w = p["G"].astype(np.float64) @ p["Wo"].astype(np.float64)
    target = np.zeros((T, dh))
    for q in range(2):
        for t in range(off[q], off[q + 1]):
            for s in range(t, off[q + 1]):
                target[t] += w[s] / (s - off[q] + 1)
    nz = dust.Noise(5, 23, 0, K, K, sigma)
    goff = cu(off)
    c = dust.attention_internal_costs(cu(p["Y"]), goff, cu(p["Wq"]), cu(p["Wk"]), cu(p["Wv"]), cu(p["Wo"]), 2,
                                      cu(p["G"]), nz)
    g, _ = dust.layer_estimate(c, False, goff, 1.0, nz, dh)
    g = g.cpu().numpy().astype(np.float64)
    cos = np.sum(g * target) / (np.linalg.norm(g) * np.linalg.norm(target))
    assert cos > 0.98, cos


def _gated(p, seed):
    """Add a gate Wg ~ N(0, 1/d) and value embeddings E ~ N(0, 0.5^2) to a block."""
    r = np.random.Generator(np.random.PCG64(seed))
    T, d = p["Y"].shape
    dh = p["Wq"].shape[0]
    return dict(p, Wg=(r.standard_normal((dh, d)) * d ** -0.5).astype(np.float32),
                E=(r.standard_normal((T, dh)) * 0.5).astype(np.float32))


@pytest.mark.parametrize("which", [0, 2, 3, 4])
def test_gate_and_value_embedding_costs_parity(orc, which):
    """Gated value embeddings on the values: the gate's and the embedding's draws
    (and q / v draws of the same head) against the oracle."""
    p = _gated(_block(seed=53), 54)
    nz = dust.Noise(3, 30 + which, 2, 6, 6, 0.01)
    c = dust.attention_internal_costs(cu(p["Y"]), cu(p["off"]), cu(p["Wq"]), cu(p["Wk"]), cu(p["Wv"]), cu(p["Wo"]),
                                      which, cu(p["G"]), nz, Wg=cu(p["Wg"]), E=cu(p["E"])).cpu().numpy()
    ref = orc.attention_internal_costs(p["Y"], p["off"], p["Wq"], p["Wk"], p["Wv"], p["Wo"], which, p["G"], 3,
                                       30 + which, 0.01, np.arange(2, 8), Wg=p["Wg"], E=p["E"])
    assert rel_err(c, ref) < 1e-3


def test_gate_and_value_embedding_rejected_without_their_inputs():
    p = _block(T=64, n_seq=1, d=16, dh=16, seed=55)
    nz = dust.Noise(0, 1, 0, 2, 2, 0.01)
    args = [cu(p[k]) for k in ("Y", "off", "Wq", "Wk", "Wv", "Wo")]
    for which, kw in ((3, {}), (3, {"E": cu(np.zeros((64, 16), np.float32))}), (4, {}), (5, {})):
        with pytest.raises(dust.DustError) as e:
            dust.attention_internal_costs(*args, which, cu(p["G"]), nz, **kw)
        assert e.value.status == 1


@pytest.mark.parametrize("which", [3, 4])
def test_gate_and_value_embedding_estimates_converge(which):
    """Uniform attention (Wq = Wk = 0), gamma = 1: the estimate approaches the
    backprop of <z, G> to the perturbed quantity, sum_{s >= t} (G_s Wo)/n_s
    times s'(g_t) E_t (gate) or s(g_t) (value embedding)."""
    T, d, dh, K, sigma = 64, 16, 16, 65536, 0.02
    p = _gated(_block(T=T, n_seq=2, d=d, dh=dh, seed=56), 57)
    p["Wq"][:] = 0
    p["Wk"][:] = 0
    off = p["off"]
    w = p["G"].astype(np.float64) @ p["Wo"].astype(np.float64)
    target = np.zeros((T, dh))
    for q in range(2):
        for t in range(off[q], off[q + 1]):
            for s in range(t, off[q + 1]):
                target[t] += w[s] / (s - off[q] + 1)
    gp = 1.0 / (1.0 + np.exp(-(p["Y"].astype(np.float64) @ p["Wg"].astype(np.float64).T)))
    target *= gp * (1 - gp) * p["E"] if which == 3 else gp
    nz = dust.Noise(6, 40 + which, 0, K, K, sigma)
    goff = cu(off)
    c = dust.attention_internal_costs(cu(p["Y"]), goff, cu(p["Wq"]), cu(p["Wk"]), cu(p["Wv"]), cu(p["Wo"]), which,
                                      cu(p["G"]), nz, Wg=cu(p["Wg"]), E=cu(p["E"]))
    g, _ = dust.layer_estimate(c, False, goff, 1.0, nz, dh)
    g = g.cpu().numpy().astype(np.float64)
    cos = np.sum(g * target) / (np.linalg.norm(g) * np.linalg.norm(target))
    assert cos > 0.97, cos
