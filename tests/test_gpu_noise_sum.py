"""dust_noise_sum (the generator's ceiling kernel) against the oracle's noise.

out[t][j] = sum over the draw range of a(seed, layer, draw, token_begin + t, j).
Pins that do not depend on the summation order:
- one draw: each term is fma(rho, cos, 0) = the binary32 noise value itself, so
  the output equals the oracle's noise bit for bit;
- two draws: the two noise values added once in fp32, again bit for bit;
- any draw count: within the fp32 summation bound of a fixed-order sum,
  |out - sum| <= (n + 1) 2^-24 sum |a| per element, against the oracle's noise
  summed in float64.
Shapes cover ragged channel counts (d not a multiple of 4), the draw loop's
remainders (K mod 4), several thread blocks per row and the grid-stride path
over tokens (more tokens than one grid column covers)."""
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from activation_perturbation_es_b200 import dust  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dust.lib()


def oracle_sum(orc, seed, layer, draw0, nd, tokens, d):
    a = orc.noise_block(seed, layer, draw0, nd, tokens, 0, d).astype(np.float64)   # [nd][T][d]
    return a.sum(axis=0), np.abs(a).sum(axis=0), a


@pytest.mark.parametrize("T,d,K,draw0,tok0", [
    (37, 13, 1, 0, 0), (37, 13, 2, 5, 100), (37, 13, 7, 5, 100), (64, 256, 9, 0, 7),
    (33, 1024, 6, 1000, 0), (5, 3, 33, 2, 1 << 20), (1, 1, 1, 0, 0), (300, 516, 67, 11, 3),
])
def test_noise_sum_matches_oracle(orc, T, d, K, draw0, tok0):
    seed, layer = 1234, 9
    nz = dust.Noise(seed, layer, draw0, K, K, 1e-2, token_begin=tok0)
    out = dust.noise_sum(nz, T, d)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    s, sabs, a = oracle_sum(orc, seed, layer, draw0, K, np.arange(T) + tok0, d)
    if K == 1:
        assert np.array_equal(got, a[0].astype(np.float32))
    elif K == 2:
        assert np.array_equal(got, (a[0].astype(np.float32) + a[1].astype(np.float32)))
    bound = (K + 1) * 2.0 ** -24 * sabs + 1e-30
    assert np.all(np.abs(got.astype(np.float64) - s) <= bound)


def test_noise_sum_grid_stride_tokens(orc):
    """More tokens than one grid column covers (65535 blocks of 2 token rows at
    d = 512): sampled tokens, including ones past the first sweep, bit-exact at
    one draw."""
    T, d = 140000, 512
    nz = dust.Noise(7, 3, 42, 1, 1, 1e-2)
    out = dust.noise_sum(nz, T, d)
    toks = np.array([0, 1, 65535 * 2 - 1, 65535 * 2, 131071, 139999])
    ref = orc.noise_block(7, 3, 42, 1, toks, 0, d)[0]
    assert np.array_equal(out[torch.from_numpy(toks).cuda()].cpu().numpy(), ref)


def test_noise_sum_is_the_reduction_at_unit_rewards(orc):
    """With every reward 1 the draw reduction is the scaled noise sum:
    g = -(1/(K sigma)) sum_k a; the two kernels round differently (the
    reduction scales r rho first), so they agree within fp32 rounding."""
    T, d, K, sigma = 96, 64, 40, 0.5
    nz = dust.Noise(5, 2, 0, K, K, sigma)
    ones = torch.ones(K, T, dtype=torch.float32, device="cuda")
    g, _ = dust.layer_estimate(ones, True, None, 0.0, nz, d)
    s = dust.noise_sum(nz, T, d)
    ref = -s / (K * sigma)
    err = float((g - ref).abs().max() / ref.abs().max())
    assert err < 1e-5


def test_noise_sum_as_benchmarked(orc):
    """The launch the benchmark times as the generator's ceiling on the scaled
    workload: 256 draws over 64 x 1024 tokens x 4096 channels (the widest
    layer), the noise of its layer; 16 sampled tokens against the oracle."""
    from activation_perturbation_es_b200 import inputs as I
    w = I.SCALED
    hl = max(w.hidden, key=lambda h: h.d_out)
    T, d, K = w.T, hl.d_out, 256
    nz = dust.Noise(w.seed, hl.layer, 0, K, K, w.sigma)
    out = dust.noise_sum(nz, T, d)
    rs = np.random.Generator(np.random.PCG64(21))
    toks = np.sort(rs.choice(T, 16, replace=False))
    got = out[torch.from_numpy(toks).cuda()].cpu().numpy().astype(np.float64)
    s, sabs, _ = oracle_sum(orc, w.seed, hl.layer, 0, K, toks, d)
    assert np.all(np.abs(got - s) <= (K + 1) * 2.0 ** -24 * sabs + 1e-30)
