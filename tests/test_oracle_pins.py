"""Pins of the CPU oracle's estimator arithmetic (CPU only).

Each oracle function is checked against something other than itself: a brute
force on tiny inputs, a closed form, a special case that reduces to a library
routine (numpy/scipy/torch autograd in float64), or the first-order behaviour
the pages state (cnblogs Dust explainer, section "信用分配：一次前向，两种奖励":
the reward-weighted noise is the gradient plus an error with no preferred
direction, so across draws the signal grows like K and the error like sqrt(K);
section "梯度是"长"出来的": cos(K) = c_max / sqrt(1 + c/K)).
Sign convention: the formulas are implemented literally, so c = l~ - l gives
g ~ -dl/dy and G_W ~ -grad_W (the descent direction).
"""
import mpmath as mp
import numpy as np
import pytest
import scipy.optimize as so
import scipy.special as sp
import torch

from activation_perturbation_es_b200 import inputs as I


# ------------------------------------------------------------------ a4 reward scan

@pytest.mark.parametrize("gamma", [0.0, 0.5, 0.9, 0.95, 1.0])
def test_scan_recurrence_equals_brute_force(orc, gamma):
    lengths = [5, 0, 1, 17, 3, 0, 33, 2]                 # ragged, with empty sequences
    off = I.offsets_from_lengths(lengths)
    T = int(off[-1])
    c = I.normal((7, T), 1.0, seed=1)
    r = orc.reward_scan(c, off, gamma)
    rb = orc.reward_scan(c, off, gamma, brute=True)
    np.testing.assert_allclose(r, rb, rtol=1e-12, atol=1e-12)


def test_scan_special_cases(orc):
    off = I.offsets_from_lengths([9, 1, 14, 6])
    T = int(off[-1])
    c = I.normal((5, T), 1.0, seed=2)
    # gamma = 0: identity (0^0 = 1)
    np.testing.assert_array_equal(orc.reward_scan(c, off, 0.0), c.astype(np.float64))
    # gamma = 1: reversed cumulative sums inside each sequence (numpy)
    r1 = orc.reward_scan(c, off, 1.0)
    for q in range(len(off) - 1):
        seg = c[:, off[q]:off[q + 1]].astype(np.float64)
        np.testing.assert_allclose(r1[:, off[q]:off[q + 1]], np.cumsum(seg[:, ::-1], axis=1)[:, ::-1], rtol=1e-13)
    # last token of every sequence: r = c; nothing leaks across a boundary
    r9 = orc.reward_scan(c, off, 0.9)
    for q in range(len(off) - 1):
        np.testing.assert_array_equal(r9[:, off[q + 1] - 1], c[:, off[q + 1] - 1].astype(np.float64))
    c2 = c.copy()
    c2[:, off[2]:] += 100.0                              # change later sequences only
    np.testing.assert_array_equal(orc.reward_scan(c2, off, 0.9)[:, :off[2]], r9[:, :off[2]])


def test_scan_rejects_bad_offsets(orc):
    c = np.zeros((1, 10), np.float32)
    with pytest.raises(ValueError):
        orc.reward_scan(c, np.array([0, 5, 9], np.int32), 0.5)
    with pytest.raises(ValueError):
        orc.reward_scan(c, np.array([0, 6, 5, 10], np.int32), 0.5)


# ------------------------------------------------------------------ a5 error estimate

def test_estimate_single_draw_closed_form(orc):
    """K = 1, T = 1: g = -(r / sigma) a, with a the spec's Gaussian."""
    sigma, r = 0.01, 0.37
    g = orc.layer_estimate(np.array([[r]], np.float32), True, 8, [0, 1], 0.0, 5, 3, 11, 1, sigma, [0])
    a = np.array([orc.gauss(5, 3, 11, 0, j) for j in range(8)], np.float64)
    np.testing.assert_allclose(g[0], -(float(np.float32(r)) / sigma) * a, rtol=1e-15)
    # the same token placed at global index 70000 of a sharded batch draws that token's noise
    g = orc.layer_estimate(np.array([[r]], np.float32), True, 8, [0, 1], 0.0, 5, 3, 11, 1, sigma, [0],
                           token_begin=70000)
    a = np.array([orc.gauss(5, 3, 11, 70000, j) for j in range(8)], np.float64)
    np.testing.assert_allclose(g[0], -(float(np.float32(r)) / sigma) * a, rtol=1e-15)


def test_estimate_reward_path_and_draw_split(orc):
    off = I.offsets_from_lengths([40, 24])
    T, K, d = 64, 12, 10
    c = I.normal((K, T), 0.01, seed=3)
    toks = np.array([0, 5, 39, 40, 63])
    g_c = orc.layer_estimate(c, False, d, off, 0.9, 0, 1, 0, K, 0.01, toks)
    r = orc.reward_scan(c, off, 0.9).astype(np.float32)
    g_r = orc.layer_estimate(r, True, d, off, 0.9, 0, 1, 0, K, 0.01, toks)
    np.testing.assert_allclose(g_c, g_r, rtol=1e-5, atol=1e-7 * np.abs(g_c).max())
    # draw ranges add up (same K_total scale): [0, K) = [0, 5) + [5, K)
    g_a = orc.layer_estimate(c[:5], False, d, off, 0.9, 0, 1, 0, K, 0.01, toks)
    g_b = orc.layer_estimate(c[5:], False, d, off, 0.9, 0, 1, 5, K, 0.01, toks)
    np.testing.assert_allclose(g_a + g_b, g_c, rtol=1e-12, atol=1e-15)
    # channel subsets are the same numbers
    g_sub = orc.layer_estimate(c, False, d, off, 0.9, 0, 1, 0, K, 0.01, toks, chans=[7, 2])
    np.testing.assert_array_equal(g_sub, g_c[:, [7, 2]])


def _linear_costs(orc, u, sigma, K, layer):
    """c[i, s] = sigma <u_s, a_s^(i)> exactly (observation noise off)."""
    T = u.shape[0]
    draws = np.repeat(np.arange(K), T)
    toks = np.tile(np.arange(T), K)
    return orc.synth_costs(u, 0, layer, sigma, 0.0, draws, toks).reshape(K, T).astype(np.float32)


def test_estimate_converges_like_inverse_sqrt_K(orc):
    """Synthetic linear costs: E[g_t] = -u_t exactly; the normwise error falls
    like K^-1/2 and the per-token cosine follows cos(K) = c_max/sqrt(1 + c/K)
    with c_max ~ 1 and c ~ d_out + 1."""
    T, d, sigma = 48, 24, 0.01
    u = I.normal((T, d), 1.0, seed=4)
    Kmax = 4096
    c = _linear_costs(orc, u, sigma, Kmax, layer=17)
    off = [0, T]
    Ks = np.array([16, 32, 64, 128, 256, 512, 1024, 2048, 4096])
    errs, coss = [], []
    for K in Ks:
        g = orc.layer_estimate(c[:K], True, d, off, 0.0, 0, 17, 0, K, sigma, np.arange(T))
        errs.append(np.mean(np.linalg.norm(g + u, axis=1) / np.linalg.norm(u, axis=1)))
        coss.append(np.mean(np.sum(g * -u, axis=1) / (np.linalg.norm(g, axis=1) * np.linalg.norm(u, axis=1))))
    slope = np.polyfit(np.log(Ks), np.log(errs), 1)[0]
    assert -0.55 <= slope <= -0.45, slope
    (cmax, cc), _ = so.curve_fit(lambda k, a, b: a / np.sqrt(1 + b / k), Ks, np.array(coss), p0=[1.0, d])
    assert abs(cmax - 1.0) < 0.03, cmax
    assert abs(cc - (d + 1)) < 0.15 * (d + 1), cc
    # the theory's error level itself: ||g + u||/||u|| ~ sqrt((d+1)/K)
    np.testing.assert_allclose(errs, np.sqrt((d + 1) / Ks), rtol=0.15)


def test_estimate_observation_noise_raises_the_cosine_constant(orc):
    """Synthetic linear costs with observation noise, c = sigma <u, a> + eps e
    (gamma = 0, so r = c): g stays unbiased and, per token,
    K E||g + u||^2 / ||u||^2 = d + 1 + d (eps / sigma)^2 / ||u||^2
    (Var g_j = (||u||^2 + u_j^2 + eps^2 / sigma^2) / K), the constant c of the
    cosine law cos(K) = c_max / sqrt(1 + c / K).  At eps / sigma = 5 the noise
    term roughly doubles c, so the pin separates it from the noiseless d + 1."""
    T, d, sigma, eps, K = 64, 24, 0.01, 0.05, 2048
    u = I.normal((T, d), 1.0, seed=6)
    draws = np.repeat(np.arange(K), T)
    toks = np.tile(np.arange(T), K)
    c = orc.synth_costs(u, 0, 19, sigma, eps, draws, toks).reshape(K, T).astype(np.float32)
    g = orc.layer_estimate(c, True, d, [0, T], 0.0, 0, 19, 0, K, sigma, np.arange(T))
    u2 = np.sum(u.astype(np.float64) ** 2, axis=1)
    c_emp = K * np.sum((g + u) ** 2, axis=1) / u2
    c_th = d + 1 + d * (eps / sigma) ** 2 / u2
    assert abs(np.mean(c_emp) / np.mean(c_th) - 1) < 0.10, (np.mean(c_emp), np.mean(c_th))
    assert np.mean(c_th) > 1.6 * (d + 1)                     # the noise term is what is being pinned
    # unbiased: the token-mean of g + u is within a few standard errors of zero
    se = np.sqrt(np.mean(c_th * u2) / K / d)
    assert np.all(np.abs(np.mean(g + u, axis=0)) < 5 * se / np.sqrt(T))


# ------------------------------------------------------------------ a6 weight estimate

def test_weight_grad_input_invariance_autograd(orc):
    """Feeding the exact dl/dy (torch autograd, float64) into the weight
    estimate reproduces autograd's grad_W: the outer product with the same
    input is shared by backprop and Dust (section "信用分配", last paragraph)."""
    T, d_in, d_out, V = 40, 12, 9, 7
    X = I.normal((T, d_in), 1.0, seed=5)
    W = I.normal((d_out, d_in), 0.3, seed=6)
    W2 = I.normal((V, d_out), 0.3, seed=7)
    y_t = I.targets(T, V, seed=8)
    Xt = torch.tensor(X, dtype=torch.float64)
    Wt = torch.tensor(W, dtype=torch.float64, requires_grad=True)
    Y = Xt @ Wt.T
    Y.retain_grad()
    loss = torch.nn.functional.cross_entropy(torch.tanh(Y) @ torch.tensor(W2, dtype=torch.float64).T,
                                             torch.tensor(y_t, dtype=torch.int64), reduction="sum")
    loss.backward()
    dy = Y.grad.numpy().astype(np.float32)
    G = orc.weight_grad(dy, X)
    np.testing.assert_allclose(G, Wt.grad.numpy(), rtol=1e-6, atol=1e-6 * np.abs(Wt.grad.numpy()).max())
    # and a row subset equals float64 matmul rows
    Gs = orc.weight_grad(dy, X, rows=[8, 0, 3])
    np.testing.assert_allclose(Gs, (dy.astype(np.float64).T @ X.astype(np.float64))[[8, 0, 3]], rtol=1e-13)


def test_logits_equal_matmul(orc):
    X = I.normal((9, 13), 1.0, seed=9)
    W = I.normal((21, 13), 1.0, seed=10)
    Z = orc.logits(X, W, toks=[0, 4, 8])
    np.testing.assert_allclose(Z, (X.astype(np.float64) @ W.astype(np.float64).T)[[0, 4, 8]], rtol=1e-13)


# ------------------------------------------------------------------ a2/a3 head

def test_head_costs_brute_force_mpmath(orc):
    """Tiny vocab: c = CE(z + sigma a 1_chunk, y) - CE(z, y) recomputed in mpmath."""
    n, V, Vc, nd, sigma = 3, 12, 4, 3, 0.05
    Z = I.normal((n, V), 2.0, seed=11)
    y = np.array([0, 7, 11], np.int32)
    toks = np.array([5, 6, 100], np.int32)
    c, g = orc.head_step(Z, y, toks, Vc, 9, 4, 2, nd, nd, sigma)
    lse, ell = orc.head_clean(Z, y)
    mp.mp.prec = 120
    for m in range(n):
        z = [mp.mpf(float(v)) for v in Z[m]]
        l0 = mp.log(mp.fsum(mp.exp(v) for v in z)) - z[y[m]]
        assert abs(float(l0) - ell[m]) < 1e-12
        assert abs(float(mp.log(mp.fsum(mp.exp(v) for v in z))) - lse[m]) < 1e-12
        acc = [mp.mpf(0)] * V
        for ch in range(V // Vc):
            for k in range(nd):
                zp = list(z)
                a = {}
                for v in range(ch * Vc, (ch + 1) * Vc):
                    a[v] = mp.mpf(float(orc.gauss(9, 4, 2 + k, int(toks[m]), v)))
                    zp[v] += sigma * a[v]
                cc = mp.log(mp.fsum(mp.exp(v) for v in zp)) - zp[y[m]] - l0
                assert abs(float(cc) - c[ch, k, m]) < 1e-12 * max(1.0, abs(float(cc)))
                for v in a:
                    acc[v] += cc * a[v]
        np.testing.assert_allclose(g[m], [float(-x / (nd * sigma)) for x in acc], rtol=1e-11, atol=1e-14)


def test_head_first_order_closed_form(orc):
    """gamma = 0 head: E[g_t] -> -(softmax(z_t) - e_{y_t}) to first order in sigma;
    the error falls like K^-1/2 and the cosine approaches 1."""
    n, V, Vc, sigma = 6, 16, 8, 1e-3
    Z = I.normal((n, V), 1.0, seed=12)
    y = I.targets(n, V, seed=13)
    target = -(sp.softmax(Z.astype(np.float64), axis=1) - np.eye(V)[y])
    errs = []
    Ks = [256, 1024, 4096, 16384]
    for K in Ks:
        _, g = orc.head_step(Z, y, np.arange(n), Vc, 0, 2, 0, K, K, sigma, want_c=False)
        errs.append(np.mean(np.linalg.norm(g - target, axis=1) / np.linalg.norm(target, axis=1)))
        cos = np.sum(g * target, axis=1) / (np.linalg.norm(g, axis=1) * np.linalg.norm(target, axis=1))
    slope = np.polyfit(np.log(Ks), np.log(errs), 1)[0]
    assert -0.6 <= slope <= -0.4, slope
    assert cos.min() > 0.98, cos
    # chunking does not change what is estimated: Vc = V converges to the same target
    _, g1 = orc.head_step(Z, y, np.arange(n), V, 0, 2, 0, 16384, 16384, sigma, want_c=False)
    assert np.mean(np.linalg.norm(g1 - target, axis=1) / np.linalg.norm(target, axis=1)) < 2.5 * errs[-1]


def test_head_rejects_bad_chunk(orc):
    with pytest.raises(ValueError):
        orc.head_step(np.zeros((1, 10), np.float32), [0], [0], 3, 0, 0, 0, 1, 1, 0.01)


# ------------------------------------------------------------------ synthetic costs

def test_synth_costs_moments(orc):
    T, d, sigma, eps = 32, 64, 0.01, 0.01
    u = I.normal((T, d), 1.0, seed=14)
    K = 512
    draws = np.repeat(np.arange(K), T)
    toks = np.tile(np.arange(T), K)
    c = orc.synth_costs(u, 0, 3, sigma, eps, draws, toks).reshape(K, T)
    var_th = sigma**2 * np.sum(u.astype(np.float64)**2, axis=1) + eps**2
    z = c / np.sqrt(var_th)                                  # standardised: N(0, 1)
    assert abs(z.mean()) < 4 / np.sqrt(z.size)
    assert abs(z.var() - 1) < 4 * np.sqrt(2 / z.size)
    # sigma = 0 leaves the observation noise alone: eps * gauss(stream 1, channel 0)
    c0 = orc.synth_costs(u, 0, 3, 0.0, eps, [4, 9], [2, 31])
    np.testing.assert_array_equal(c0, [eps * float(orc.gauss(0, 3, 4, 2, 0, 1)), eps * float(orc.gauss(0, 3, 9, 31, 0, 1))])


# ------------------------------------------------------------------ toy causal suffix

def _suffix_small(seed=20):
    T, d_in, d, dh, V = 12, 6, 8, 4, 10
    r = np.random.Generator(np.random.PCG64(seed))
    f = lambda *s: r.standard_normal(s).astype(np.float32) * np.float32(0.5)
    return dict(X=f(T, d_in), W=f(d, d_in), Wq=f(dh, d), Wk=f(dh, d), Wv=f(dh, d), Wo=f(d, dh),
                Wout=f(V, d), y=r.integers(0, V, T).astype(np.int32), off=np.array([0, 5, 5, 12], np.int32))


def _ytilde(orc, p, draw, sigma, layer=1):
    T, d = p["X"].shape[0], p["W"].shape[0]
    a = orc.noise_block(0, layer, draw, 1, np.arange(T), 0, d)[0].astype(np.float64)
    return p["X"].astype(np.float64) @ p["W"].astype(np.float64).T + sigma * a


def test_suffix_reduces_to_readout_ce(orc):
    """Wq = Wk = Wv = Wo = 0: the suffix is the readout + cross entropy (scipy)."""
    p = _suffix_small()
    for k in ("Wq", "Wk", "Wv", "Wo"):
        p[k] = np.zeros_like(p[k])
    loss = orc.toy_suffix_losses(p["X"], p["W"], p["off"], p["Wq"], p["Wk"], p["Wv"], p["Wo"], p["Wout"],
                                 p["y"], 0, 1, 0.3, [3])
    z = _ytilde(orc, p, 3, 0.3) @ p["Wout"].astype(np.float64).T
    ref = sp.logsumexp(z, axis=1) - z[np.arange(len(p["y"])), p["y"]]
    np.testing.assert_allclose(loss[0], ref, rtol=1e-12)


def test_suffix_uniform_attention_is_causal_running_mean(orc):
    """Wq = Wk = 0: every causal score is equal, so attention is the running
    mean of v over the token's own sequence prefix (numpy cumsum)."""
    p = _suffix_small()
    p["Wq"] = np.zeros_like(p["Wq"])
    p["Wk"] = np.zeros_like(p["Wk"])
    loss = orc.toy_suffix_losses(p["X"], p["W"], p["off"], p["Wq"], p["Wk"], p["Wv"], p["Wo"], p["Wout"],
                                 p["y"], 0, 1, 0.2, [0])
    yt = _ytilde(orc, p, 0, 0.2)
    v = yt @ p["Wv"].astype(np.float64).T
    o = np.zeros_like(v)
    off = p["off"]
    for q in range(len(off) - 1):
        seg = v[off[q]:off[q + 1]]
        if len(seg):
            o[off[q]:off[q + 1]] = np.cumsum(seg, axis=0) / np.arange(1, len(seg) + 1)[:, None]
    h = yt + o @ p["Wo"].astype(np.float64).T
    z = h @ p["Wout"].astype(np.float64).T
    ref = sp.logsumexp(z, axis=1) - z[np.arange(len(p["y"])), p["y"]]
    np.testing.assert_allclose(loss[0], ref, rtol=1e-12)


def test_suffix_clean_losses_and_small_sigma_linearity(orc):
    p = _suffix_small()
    args = (p["X"], p["W"], p["off"], p["Wq"], p["Wk"], p["Wv"], p["Wo"], p["Wout"], p["y"], 0, 1)
    clean = orc.toy_suffix_losses(*args, 0.01, [0, 1], with_noise=False)
    np.testing.assert_array_equal(clean[0], clean[1])
    same = orc.toy_suffix_losses(*args, 0.0, [5])
    np.testing.assert_array_equal(same[0], clean[0])
    # differentiability: (l~ - l)/sigma converges as sigma -> 0 (first order)
    c1 = (orc.toy_suffix_losses(*args, 1e-4, [2])[0] - clean[0]) / 1e-4
    c2 = (orc.toy_suffix_losses(*args, 5e-5, [2])[0] - clean[0]) / 5e-5
    np.testing.assert_allclose(c1, c2, rtol=2e-3, atol=1e-3 * np.abs(c1).max())
    # causality: the first token of each sequence sees only itself, so perturbing
    # later tokens is invisible to it -- compare with the one-token suffix
    for q in (0, 2):
        t0 = int(p["off"][q])
        one = {k: v for k, v in p.items()}
        X1 = p["X"][t0:t0 + 1]
        l1 = orc.toy_suffix_losses(X1, p["W"], np.array([0, 1], np.int32), p["Wq"], p["Wk"], p["Wv"],
                                   p["Wo"], p["Wout"], p["y"][t0:t0 + 1], 0, 1, 0.0, [0])
        np.testing.assert_allclose(l1[0, 0], clean[0, t0], rtol=1e-13)


# ------------------------------------------------------------------ cosine tuner support

def test_head_bp_grad_equals_autograd(orc):
    """The head's backprop gradient (comparator of the cosine criterion)
    against torch autograd in float64 (a library routine)."""
    T, d, V = 30, 7, 11
    X = I.normal((T, d), 1.0, seed=30)
    W = I.normal((V, d), 0.5, seed=31)
    y = I.targets(T, V, seed=32)
    Wt = torch.tensor(W, dtype=torch.float64, requires_grad=True)
    Z = torch.tensor(X, dtype=torch.float64) @ Wt.T
    torch.nn.functional.cross_entropy(Z, torch.tensor(y, dtype=torch.int64), reduction="sum").backward()
    Zf = (X.astype(np.float64) @ W.astype(np.float64).T).astype(np.float32)
    G = orc.head_bp_grad(Zf, y, X)
    np.testing.assert_allclose(G, Wt.grad.numpy(), rtol=1e-5, atol=1e-5 * np.abs(Wt.grad.numpy()).max())


def test_cosine_equals_numpy(orc):
    a = I.normal(1000, 1.0, seed=33)
    b = I.normal(1000, 1.0, seed=34) + 0.5 * a
    ref = float(np.dot(a.astype(np.float64), b) / (np.linalg.norm(a.astype(np.float64)) * np.linalg.norm(b.astype(np.float64))))
    assert abs(orc.cosine(a, b) - ref) < 1e-12


def test_cosine_law_fit_recovers_parameters():
    from activation_perturbation_es_b200 import tuner
    Ks = np.array([64, 128, 256, 1024, 4096, 16384])
    c_max, c = 0.93, 850.0
    cm, cc = tuner.fit_cosine_law(Ks, c_max / np.sqrt(1 + c / Ks))
    assert abs(cm - c_max) < 1e-9 and abs(cc - c) < 1e-6


# ------------------------------------------------------------------ attention-internal scoring

def _attn_small(seed=40, T=14, d=8, dh=4):
    r = np.random.Generator(np.random.PCG64(seed))
    f = lambda *s: r.standard_normal(s).astype(np.float32) * np.float32(0.5)
    return dict(Y=f(T, d), Wq=f(dh, d), Wk=f(dh, d), Wv=f(dh, d), Wo=f(d, dh), G=f(T, d),
                off=np.array([0, 6, 6, T], np.int32))


def test_attention_costs_zero_when_the_projection_cannot_matter(orc):
    """q has no effect when Wk = 0 (every score is 0), k none when Wq = 0."""
    p = _attn_small()
    args = lambda P, which: (P["Y"], P["off"], P["Wq"], P["Wk"], P["Wv"], P["Wo"], which, P["G"], 0, 5, 0.1, [0, 3])
    pq = dict(p, Wk=np.zeros_like(p["Wk"]))
    assert np.all(orc.attention_internal_costs(*args(pq, 0)) == 0.0)
    pk = dict(p, Wq=np.zeros_like(p["Wq"]))
    assert np.all(orc.attention_internal_costs(*args(pk, 1)) == 0.0)
    # but the value projection matters in both cases
    assert np.any(orc.attention_internal_costs(*args(pq, 2)) != 0.0)


def test_attention_costs_uniform_attention_closed_form(orc):
    """Wq = Wk = 0: attention is the causal running mean, so a value perturbation
    changes the output by (running mean of sigma a) Wo^T (numpy cumsum)."""
    p = _attn_small()
    p["Wq"] = np.zeros_like(p["Wq"])
    p["Wk"] = np.zeros_like(p["Wk"])
    sigma, T, dh = 0.1, p["Y"].shape[0], p["Wq"].shape[0]
    c = orc.attention_internal_costs(p["Y"], p["off"], p["Wq"], p["Wk"], p["Wv"], p["Wo"], 2, p["G"], 0, 5, sigma, [2])
    a = orc.noise_block(0, 5, 2, 1, np.arange(T), 0, dh)[0].astype(np.float64)
    dz = np.zeros((T, p["Y"].shape[1]))
    off = p["off"]
    for q in range(len(off) - 1):
        seg = a[off[q]:off[q + 1]]
        if len(seg):
            m = np.cumsum(seg, axis=0) / np.arange(1, len(seg) + 1)[:, None]
            dz[off[q]:off[q + 1]] = sigma * m @ p["Wo"].astype(np.float64).T
    np.testing.assert_allclose(c[0], -np.sum(dz * p["G"], axis=1), rtol=1e-10, atol=1e-14)


def test_attention_value_estimate_converges_to_backprop_through_uniform_attention(orc):
    """With uniform attention the value-projection costs are linear in the noise,
    and with gamma = 1 the estimate's expectation is exactly the backprop of
    <z, g> to v_t: E[g_hat_t] = sum_{s >= t, same seq} (G_s Wo) / n_s, n_s the
    size of s's causal prefix.  The error falls like K^-1/2."""
    p = _attn_small(seed=41, T=10, d=6, dh=8)
    p["Wq"] = np.zeros_like(p["Wq"])
    p["Wk"] = np.zeros_like(p["Wk"])
    off = np.array([0, 4, 10], np.int32)
    T, dh, sigma = 10, 8, 0.05
    target = np.zeros((T, dh))
    w = p["G"].astype(np.float64) @ p["Wo"].astype(np.float64)       # G_s Wo
    for q in range(2):
        for t in range(off[q], off[q + 1]):
            for s in range(t, off[q + 1]):
                target[t] += w[s] / (s - off[q] + 1)
    Kmax = 8192
    c = orc.attention_internal_costs(p["Y"], off, p["Wq"], p["Wk"], p["Wv"], p["Wo"], 2, p["G"], 1, 7, sigma,
                                     np.arange(Kmax)).astype(np.float32)
    errs = []
    Ks = [128, 512, 2048, 8192]
    for K in Ks:
        g = orc.layer_estimate(c[:K], False, dh, off, 1.0, 1, 7, 0, K, sigma, np.arange(T))
        errs.append(np.linalg.norm(g - target) / np.linalg.norm(target))
    slope = np.polyfit(np.log(Ks), np.log(errs), 1)[0]
    assert -0.6 <= slope <= -0.4, (slope, errs)
    assert errs[-1] < 0.2, errs


def _gated_values(seed=43, T=14, d=8, dh=4):
    p = _attn_small(seed=seed, T=T, d=d, dh=dh)
    r = np.random.Generator(np.random.PCG64(seed + 100))
    p["Wg"] = (r.standard_normal((dh, d)) * 0.5).astype(np.float32)
    p["E"] = (r.standard_normal((T, dh)) * 0.7).astype(np.float32)
    return p


def _costs(orc, p, which, sigma, draws, seed=0, layer=5, off=None):
    return orc.attention_internal_costs(p["Y"], p["off"] if off is None else off, p["Wq"], p["Wk"], p["Wv"], p["Wo"],
                                        which, p["G"], seed, layer, sigma, draws, Wg=p.get("Wg"), E=p.get("E"))


def test_gate_and_value_embedding_special_cases(orc):
    """The gate matters only through the value embedding (E = 0: every gate cost
    is 0); with Wg = 0 the gate is s(0) = 1/2 everywhere, so a value-embedding
    draw moves v by half of what the same draw does to the value projection,
    and since the attention output is linear in v its costs are half the
    value-projection costs (under any q, k)."""
    p = _gated_values()
    p0 = dict(p, E=np.zeros_like(p["E"]))
    assert np.all(_costs(orc, p0, 3, 0.1, [0, 4]) == 0.0)
    ph = dict(p, Wg=np.zeros_like(p["Wg"]))
    np.testing.assert_allclose(_costs(orc, ph, 4, 0.1, [1, 2]), 0.5 * _costs(orc, ph, 2, 0.1, [1, 2]), rtol=1e-10,
                               atol=1e-15)
    # the clean values carry the gated embedding: q draws see it (their costs change with E)
    assert not np.allclose(_costs(orc, p, 0, 0.1, [3]), _costs(orc, p0, 0, 0.1, [3]))


@pytest.mark.parametrize("which", [3, 4])
def test_gate_and_value_embedding_uniform_attention_closed_form(orc, which):
    """Wq = Wk = 0: the output change is the causal running mean of the values'
    change, (s(g + sigma a) - s(g)) e for the gate and s(g) sigma a for the value
    embedding (numpy, scipy's logistic function)."""
    p = _gated_values()
    p["Wq"] = np.zeros_like(p["Wq"])
    p["Wk"] = np.zeros_like(p["Wk"])
    sigma, T, dh = 0.3, p["Y"].shape[0], p["Wq"].shape[0]
    c = _costs(orc, p, which, sigma, [5])
    a = orc.noise_block(0, 5, 5, 1, np.arange(T), 0, dh)[0].astype(np.float64)
    g = p["Y"].astype(np.float64) @ p["Wg"].astype(np.float64).T
    dv = (sp.expit(g + sigma * a) - sp.expit(g)) * p["E"] if which == 3 else sp.expit(g) * sigma * a
    dz = np.zeros((T, p["Y"].shape[1]))
    off = p["off"]
    for q in range(len(off) - 1):
        seg = dv[off[q]:off[q + 1]]
        if len(seg):
            m = np.cumsum(seg, axis=0) / np.arange(1, len(seg) + 1)[:, None]
            dz[off[q]:off[q + 1]] = m @ p["Wo"].astype(np.float64).T
    np.testing.assert_allclose(c[0], -np.sum(dz * p["G"], axis=1), rtol=1e-10, atol=1e-14)


@pytest.mark.parametrize("which", [3, 4])
def test_gate_and_value_embedding_estimates_converge_to_backprop(orc, which):
    """Uniform attention, gamma = 1: the estimate's expectation is the backprop of
    <z, G> to the perturbed quantity, the value path's sum_{s >= t} (G_s Wo)/n_s
    times dv/dx: s'(g) e for the gate, s(g) for the value embedding (first
    order in sigma).  The error falls like K^-1/2."""
    p = _gated_values(seed=44, T=10, d=6, dh=8)
    p["Wq"] = np.zeros_like(p["Wq"])
    p["Wk"] = np.zeros_like(p["Wk"])
    off = np.array([0, 4, 10], np.int32)
    T, dh, sigma = 10, 8, 0.02
    w = p["G"].astype(np.float64) @ p["Wo"].astype(np.float64)
    target = np.zeros((T, dh))
    for q in range(2):
        for t in range(off[q], off[q + 1]):
            for s in range(t, off[q + 1]):
                target[t] += w[s] / (s - off[q] + 1)
    gp = sp.expit(p["Y"].astype(np.float64) @ p["Wg"].astype(np.float64).T)
    target *= gp * (1 - gp) * p["E"] if which == 3 else gp
    Kmax = 8192
    c = _costs(orc, p, which, sigma, np.arange(Kmax), seed=1, layer=7, off=off).astype(np.float32)
    errs = []
    Ks = [128, 512, 2048, 8192]
    for K in Ks:
        g = orc.layer_estimate(c[:K], False, dh, off, 1.0, 1, 7, 0, K, sigma, np.arange(T))
        errs.append(np.linalg.norm(g - target) / np.linalg.norm(target))
    slope = np.polyfit(np.log(Ks), np.log(errs), 1)[0]
    assert -0.6 <= slope <= -0.4, (slope, errs)
    assert errs[-1] < 0.2, errs


def test_suffix_hard_self_attention_limit(orc):
    """Orthonormal layer outputs y_t, Wq = lam A and Wk = lam A^-T for a
    non-orthogonal A: the score of token t on u is q_t . k_u / sqrt(dh) =
    lam^2 <y_t, y_u> / sqrt(dh) = lam^2 delta_tu / sqrt(dh) (while q_t . q_u and
    k_t . k_u are not), so for large lam every token attends only to itself,
    o_t = v_t, and the suffix is the residual + readout of y_t + Wo Wv y_t
    (numpy/scipy closed form).  Together with the uniform case (which pins the
    causal mask and the value path) this pins the score path q_t . k_u."""
    d = dh = 8
    T = 8
    r = np.random.Generator(np.random.PCG64(60))
    Q, _ = np.linalg.qr(r.standard_normal((d, d)))
    X = Q.astype(np.float32)                           # rows orthonormal
    W = np.eye(d, dtype=np.float32)                    # y = X
    lam = np.sqrt(300.0 * np.sqrt(dh))                 # self score 300, others 0
    A = np.linalg.qr(r.standard_normal((d, d)))[0] @ np.diag(np.linspace(0.5, 2.0, d)) @ \
        np.linalg.qr(r.standard_normal((d, d)))[0].T
    Wq = (lam * A).astype(np.float32)
    Wk = (lam * np.linalg.inv(A).T).astype(np.float32)
    Wv = (r.standard_normal((dh, d)) * 0.5).astype(np.float32)
    Wo = (r.standard_normal((d, dh)) * 0.5).astype(np.float32)
    Wout = (r.standard_normal((10, d)) * 0.5).astype(np.float32)
    y = r.integers(0, 10, T).astype(np.int32)
    off = np.array([0, 3, T], np.int32)
    loss = orc.toy_suffix_losses(X, W, off, Wq, Wk, Wv, Wo, Wout, y, 0, 1, 0.0, [0], with_noise=False)[0]
    Y = X.astype(np.float64)
    h = Y + Y @ Wv.astype(np.float64).T @ Wo.astype(np.float64).T
    z = h @ Wout.astype(np.float64).T
    ref = sp.logsumexp(z, axis=1) - z[np.arange(T), y]
    # Wq, Wk are rounded to binary32: the off-diagonal scores are ~lam^2 * 1e-7, far from mattering
    np.testing.assert_allclose(loss, ref, rtol=1e-6)
