"""End-to-end pin of the hidden-layer chain on the toy causal suffix (CPU oracle).

cnblogs Dust explainer, section "信用分配：一次前向，两种奖励": with the perturbed
losses of the suffix, c = l~ - l, the reward r_t = sum_{s>=t} gamma^(s-t) c_s,
the error g_t = -(1/(K sigma)) sum_i r_t^(i) a_t^(i) and G_W = sum_t g_t x_t^T
converge, to first order in sigma, to
  G_gamma = -sum_t sum_{s >= t} gamma^(s-t) (dl_s/dy_t) x_t^T,
which at gamma = 1 is -grad_W sum_t l_t (backprop).  The comparator is float64
torch autograd through the same model (tests/suffix_autograd.py); the oracle
computes the whole chain.  2 sequences x 16 tokens, K up to 16384.
"""
import numpy as np
import pytest
import scipy.optimize as so

import suffix_autograd as SA

SEED, LAYER, SIGMA = 0, 5, 0.01
KS = np.array([64, 256, 1024, 4096, 16384])


@pytest.fixture(scope="module")
def chain(orc):
    p = SA.tiny_problem()
    args = (p["X"], p["W"], p["off"], p["Wq"], p["Wk"], p["Wv"], p["Wo"], p["Wout"], p["y"], SEED, LAYER)
    clean = orc.toy_suffix_losses(*args, SIGMA, [0], with_noise=False)[0]
    loss = orc.toy_suffix_losses(*args, SIGMA, np.arange(KS[-1]))
    c = (loss - clean[None, :]).astype(np.float32)
    return p, clean, c, SA.loss_jacobian(p)


def test_autograd_comparator_is_the_oracle_model(orc, chain):
    """The torch model is the oracle's suffix (clean losses), and the brute-force
    discounted gradient at gamma = 1 is minus backprop's gradient."""
    p, clean, _, J = chain
    np.testing.assert_allclose(SA.clean_losses(p), clean, rtol=1e-12)
    G1, _ = SA.discounted_gradient(p, J, 1.0)
    Gbp = SA.backprop_gradient(p)
    np.testing.assert_allclose(G1, -Gbp, rtol=0, atol=1e-12 * np.abs(Gbp).max())
    # causality: dl_s/dy_t = 0 for s < t and across sequences
    T = J.shape[0]
    off = p["off"]
    seq = np.searchsorted(off, np.arange(T), side="right") - 1
    for s in range(T):
        for t in range(T):
            if t > s or seq[t] != seq[s]:
                assert not J[s][t].any()


def _estimates(orc, p, c, gamma):
    T, d = p["X"].shape[0], p["W"].shape[0]
    out = []
    for K in KS:
        g = orc.layer_estimate(c[:K], False, d, p["off"], gamma, SEED, LAYER, 0, int(K), SIGMA, np.arange(T))
        out.append(orc.weight_grad(g.astype(np.float32), p["X"]))
    return out


@pytest.mark.parametrize("gamma,final", [(1.0, 0.12), (0.9, 0.09), (0.0, 0.06)])
def test_weight_estimate_converges_to_discounted_gradient(orc, chain, gamma, final):
    """||G_W - G_gamma|| / ||G_gamma|| falls like K^-1/2 (fitted log-log slope
    -0.5 +- 0.08) down to a few percent at K = 16384."""
    p, _, c, J = chain
    Gref, _ = SA.discounted_gradient(p, J, gamma)
    errs = [np.linalg.norm(G - Gref) / np.linalg.norm(Gref) for G in _estimates(orc, p, c, gamma)]
    slope = np.polyfit(np.log(KS), np.log(errs), 1)[0]
    assert -0.58 <= slope <= -0.42, (slope, errs)
    assert errs[-1] < final, errs


def test_backprop_cosine_follows_the_cosine_law(orc, chain):
    """gamma = 1: cos(G_W, -grad_W sum l) rises toward 1 and follows
    cos(K) = c_max / sqrt(1 + c/K) (section "梯度是"长"出来的") with c_max ~ 1."""
    p, _, c, _ = chain
    Gbp = -SA.backprop_gradient(p)
    coss = np.array([np.sum(G * Gbp) / (np.linalg.norm(G) * np.linalg.norm(Gbp)) for G in _estimates(orc, p, c, 1.0)])
    assert np.all(np.diff(coss) > 0), coss
    assert coss[-1] > 0.99, coss
    (cmax, cc), _ = so.curve_fit(lambda k, a, b: a / np.sqrt(1 + b / k), KS, coss, p0=[1.0, 100.0])
    assert abs(cmax - 1.0) < 0.03, (cmax, cc)
    assert cc > 0
