"""GPU parity on random small shapes (hypothesis, derandomized so every run
draws the same examples): ragged and empty sequences, odd token counts,
channel counts not divisible by 4, draw ranges split over calls, gamma's
special values, vocabulary chunk counts and chunk ranges, tokens placed at
random global offsets (token_begin), and the fused reduction + weight
estimate.  Every expected value comes from the oracle on the same seeded
inputs."""
import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings, strategies as st

from activation_perturbation_es_b200 import dust
from activation_perturbation_es_b200 import inputs as I

import oracle_chains  # noqa: E402

pytestmark = pytest.mark.gpu
FP32_TOL = 1e-3
SETTINGS = dict(max_examples=50, deadline=None, derandomize=True,
                suppress_health_check=[HealthCheck.function_scoped_fixture, HealthCheck.too_slow])

lengths_st = st.lists(st.integers(min_value=0, max_value=70), min_size=1, max_size=5).filter(lambda l: sum(l) > 0)
gamma_st = st.sampled_from([0.0, 0.5, 0.95, 1.0])


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dust.lib()


def rel_err(gpu, orc):
    scale = np.max(np.abs(orc))
    return float(np.max(np.abs(np.asarray(gpu, np.float64) - orc)) / scale) if scale > 0 else float(
        np.max(np.abs(gpu)))


def cu(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.to(dtype)


@settings(**SETTINGS)
@given(lengths=lengths_st, d_out=st.integers(1, 70), K=st.integers(1, 9), split=st.integers(1, 8),
       gamma=gamma_st, seed=st.integers(0, 10_000), tb=st.integers(0, 2**31 - 1000))
def test_estimate_random_shapes(orc, lengths, d_out, K, split, gamma, seed, tb):
    """Scan + reduction against the oracle, with the draws split over two
    calls (accumulate = 1) at a random point and the tokens at global offset tb."""
    off = I.offsets_from_lengths(lengths)
    T = int(off[-1])
    c = I.normal((K, T), 0.02, seed=seed)
    a = min(split, K)
    nz_all = dust.Noise(seed % 7, 3, 5, K, K, 0.01, tb)
    goff = cu(off)
    g, _ = dust.layer_estimate(cu(c[:a]), False, goff, gamma, dust.Noise(seed % 7, 3, 5, a, K, 0.01, tb), d_out)
    if a < K:
        dust.layer_estimate(cu(c[a:]), False, goff, gamma, dust.Noise(seed % 7, 3, 5 + a, K - a, K, 0.01, tb),
                            d_out, g_hat=g, accumulate=True)
    ref = orc.layer_estimate(c, False, d_out, off, gamma, nz_all.seed, 3, 5, K, 0.01, np.arange(T), token_begin=tb)
    assert rel_err(g.cpu().numpy(), ref) < FP32_TOL


@settings(**dict(SETTINGS, max_examples=40))
@given(T=st.integers(1, 40), n_chunks=st.integers(1, 4), Vc=st.sampled_from([128, 256, 384, 1024]),
       K=st.integers(1, 6), sigma=st.sampled_from([0.005, 0.02, 0.05, 0.3]), seed=st.integers(0, 10_000),
       first=st.integers(0, 3), tb=st.integers(0, 2**31 - 1000))
def test_head_random_shapes(orc, T, n_chunks, Vc, K, sigma, seed, first, tb):
    """Head step (cached logits) over a random range of its chunks, with the
    tokens at global offset tb, against the oracle: c per chunk and g."""
    V = n_chunks * Vc
    cb = first % n_chunks
    cc = n_chunks - cb
    Z = I.normal((T, V), 1.5, seed=seed)
    y = I.targets(T, V, seed=seed + 1)
    nz = dust.Noise(seed % 5, 9, 2, K, K, sigma, tb)
    out = dust.head_step(cu(y), Vc, nz, Z=cu(Z), want_c=True, chunk_begin=cb, chunk_count=cc)
    c_ref, g_ref = orc.head_step(Z, y, tb + np.arange(T), Vc, nz.seed, nz.layer, 2, K, K, sigma)
    assert rel_err(out["g_hat"].cpu().numpy(), g_ref[:, cb * Vc:]) < FP32_TOL
    assert rel_err(out["c"].cpu().numpy(), c_ref[cb:]) < FP32_TOL


@settings(**dict(SETTINGS, max_examples=30))
@given(lengths=lengths_st, d_out=st.integers(1, 300), d_in=st.sampled_from([64, 128, 192, 256, 320, 384, 448, 512]),
       K=st.integers(1, 7), gamma=gamma_st, seed=st.integers(0, 10_000), tb=st.integers(0, 2**31 - 1000))
def test_fused_random_shapes(orc, lengths, d_out, d_in, K, gamma, seed, tb):
    """Fused reduction + weight estimate against the oracle's chain (tokens at global offset tb)."""
    off = I.offsets_from_lengths(lengths)
    T = int(off[-1])
    c = I.normal((K, T), 0.02, seed=seed)
    X = I.bf16_round(I.normal((T, d_in), 1.0, seed=seed + 1))
    nz = dust.Noise(seed % 3, 4, 0, K, K, 0.01, tb)
    G, g = dust.layer_estimate_weight_grad(cu(c), False, cu(off), gamma, nz, cu(X, torch.bfloat16), d_out,
                                           g_hat=True)
    g_ref = orc.layer_estimate(c, False, d_out, off, gamma, nz.seed, 4, 0, K, 0.01, np.arange(T), token_begin=tb)
    assert rel_err(g.cpu().numpy(), g_ref) < FP32_TOL
    G_ref = oracle_chains.weight_rows(orc, c, False, d_out, off, gamma, nz.seed, 4, 0, K, 0.01, X, np.arange(d_out),
                                      token_begin=tb)
    assert rel_err(G.cpu().numpy(), G_ref) < FP32_TOL


@settings(**dict(SETTINGS, max_examples=40))
@given(T=st.integers(1, 70), d=st.integers(1, 300), K=st.integers(1, 40), draw0=st.integers(0, 1 << 20),
       seed=st.integers(0, 2**32 - 1), tb=st.integers(0, 1 << 30))
def test_noise_sum_random_shapes(orc, T, d, K, draw0, seed, tb):
    """The ceiling kernel on random shapes: within the fp32 bound of a
    fixed-order sum, |out - sum a| <= (K + 1) 2^-24 sum |a|, of the oracle's
    noise summed in float64."""
    nz = dust.Noise(seed, 4, draw0, K, K, 1e-2, token_begin=tb)
    got = dust.noise_sum(nz, T, d).cpu().numpy().astype(np.float64)
    a = orc.noise_block(seed, 4, draw0, K, np.arange(T) + tb, 0, d).astype(np.float64)
    assert np.all(np.abs(got - a.sum(axis=0)) <= (K + 1) * 2.0 ** -24 * np.abs(a).sum(axis=0) + 1e-30)
