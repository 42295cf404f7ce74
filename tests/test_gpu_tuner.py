"""Cosine-criterion support on the GPU: the head's backprop gradient, the
device cosine, and the tuner's population / sigma sweeps against the oracle."""
import numpy as np
import pytest
import torch

from activation_perturbation_es_b200 import dust, tuner
from activation_perturbation_es_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dust.lib()


def rel_err(gpu, orc):
    return float(np.max(np.abs(np.asarray(gpu, np.float64) - orc)) / np.max(np.abs(orc)))


def _head(T=512, d=64, V=512, seed=0):
    X = I.bf16_round(I.normal((T, d), 1.0, seed=seed))
    W = I.bf16_round(I.normal((V, d), 1.0 / np.sqrt(d), seed=seed + 1))
    y = I.targets(T, V, seed=seed + 2)
    return X, W, y


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_head_bp_grad_parity(orc, dt):
    X, W, y = _head(T=700, d=48, V=384)
    Xg = torch.from_numpy(X).cuda().to(dt)
    # both sides get the oracle's logits (binary32); the logits GEMM is pinned on its own
    Z = orc.logits(X, W).astype(np.float32)
    G = dust.head_bp_grad(torch.from_numpy(Z).cuda(), torch.from_numpy(y).cuda(), Xg).cpu().numpy()
    ref = orc.head_bp_grad(Z, y, X)
    # bf16: the softmax difference is rounded to bf16 before the tensor-core GEMM
    assert rel_err(G, ref) < (2e-2 if dt == torch.bfloat16 else 1e-5)


def test_device_cosine(orc):
    a = I.normal(1_000_003, 1.0, seed=1)
    b = I.normal(1_000_003, 1.0, seed=2) + 0.3 * a
    out = dust.cosine(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()).cpu().numpy()
    assert abs(out[3] - orc.cosine(a, b)) < 1e-12
    assert abs(out[0] - float(np.dot(a.astype(np.float64), b))) < 1e-9 * abs(out[0])


def test_population_sweep_follows_the_cosine_law(orc):
    X, W, y = _head()
    Xg, Wg, yg = (torch.from_numpy(X).cuda().to(torch.bfloat16), torch.from_numpy(W).cuda().to(torch.bfloat16),
                  torch.from_numpy(y).cuda())
    Ks, coss = tuner.head_population_sweep(Xg, Wg, yg, 256, [64, 256, 1024, 4096, 16384], sigma=1e-2, seed=0, layer=4)
    assert np.all(np.diff(coss) > 0), coss
    c_max, c = tuner.fit_cosine_law(Ks, coss)
    assert 0.85 < c_max < 1.02 and c > 0, (c_max, c, coss)
    # the first point against the oracle's own estimate and backprop gradient
    Z = (X.astype(np.float64) @ W.astype(np.float64).T).astype(np.float32)
    _, g = orc.head_step(Z, y, np.arange(len(y)), 256, 0, 4, 0, 64, 16384, 1e-2, want_c=False)
    G_orc = g.T @ X.astype(np.float64)
    G_bp = orc.head_bp_grad(Z, y, X)
    cos_orc = orc.cosine(G_orc.astype(np.float32), (-G_bp).astype(np.float32))
    assert abs(coss[0] - cos_orc) < 2e-3, (coss[0], cos_orc)


def test_sigma_sweep(orc):
    X, W, y = _head(seed=7)
    Xg, Wg, yg = (torch.from_numpy(X).cuda().to(torch.bfloat16), torch.from_numpy(W).cuda().to(torch.bfloat16),
                  torch.from_numpy(y).cuda())
    sig, coss, best = tuner.head_sigma_sweep(Xg, Wg, yg, 512, 2048, [1e-3, 1e-2, 1e-1, 3.0], seed=1, layer=2)
    assert best in (1e-3, 1e-2, 1e-1)
    assert coss[-1] < max(coss[:-1])            # far outside the first-order regime the cosine drops
    assert abs(coss[0] - coss[1]) < 0.05        # inside it the cosine barely depends on sigma


def test_hidden_sweep_picks_gamma_one_against_backprop(orc):
    """A hidden layer of the toy causal suffix (2 sequences x 16 tokens): the
    caller scores its perturbed forward (the library's toy suffix) and supplies
    -grad_W sum l from float64 autograd; against the full backprop gradient the
    discount that keeps every later token's loss, gamma = 1, wins, and each
    cosine matches the oracle chain's on the same costs."""
    import suffix_autograd as SA
    p = SA.tiny_problem()
    G_ref = -SA.backprop_gradient(p)
    cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    Y = dust.logits(cu(p["X"]), cu(p["W"]))
    off = cu(p["off"])

    def costs(nz):
        return dust.toy_suffix_losses(Y, off, cu(p["Wq"]), cu(p["Wk"]), cu(p["Wv"]), cu(p["Wo"]), cu(p["Wout"]),
                                      cu(p["y"]), nz)[1]

    K, d = 8192, p["W"].shape[0]
    sigmas, gammas = [1e-3, 1e-2], [0.0, 0.5, 0.9, 1.0]
    _, _, coss, best = tuner.hidden_sweep(costs, cu(p["X"]), off, d, cu(G_ref.astype(np.float32)), K, sigmas,
                                          gammas, seed=0, layer=5)
    assert best[1] == 1.0, coss
    assert np.all(np.diff(coss, axis=1) > 0), coss           # more of the future helps, for either sigma
    assert coss[1, -1] > 0.99, coss
    # the sweep's cosine at (1e-2, 0.9) against the oracle's chain on the same costs
    c = costs(dust.Noise(0, 5, 0, K, K, 1e-2)).cpu().numpy()
    T = p["X"].shape[0]
    g = orc.layer_estimate(c, False, d, p["off"], 0.9, 0, 5, 0, K, 1e-2, np.arange(T))
    G = orc.weight_grad(g.astype(np.float32), p["X"])
    ref = np.sum(G * G_ref) / (np.linalg.norm(G) * np.linalg.norm(G_ref))
    assert abs(coss[1, 2] - ref) < 2e-3, (coss[1, 2], ref)
