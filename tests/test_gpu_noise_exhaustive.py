"""Exhaustive bit-exactness of the GPU Box-Muller step against the oracle.

The transform sees only 2^23 distinct radius uniforms (the top 23 bits of the
first word) and 2^26 distinct angles (octant + 23 fraction bits of the
second).  These tests run every radius value (paired with varied angle words)
and every angle fraction in every octant (paired with varied radius words),
so every ln / sqrt / sin / cos evaluation the generator can ever perform is
checked bit for bit, in both lanes of the packed generator the hot kernels
inline.  The draw reduction itself is checked against the oracle's noise
where its arithmetic is exact (one draw, sigma = 1, r = 1: g = -a)."""
import numpy as np
import pytest
import torch

from activation_perturbation_es_b200 import dust

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dust.lib()


def _check(orc, a, b):
    """The kernel runs element i in the low lane and element i + n/2 in the high
    lane of the packed (two-pair) generator; the inputs are checked in both
    placements, so every value passes through both lanes."""
    rne, rno = orc.box_muller_batch(a, b)
    h = a.size // 2
    for shift in (0, h):
        sa, sb = np.roll(a, shift), np.roll(b, shift)
        ne, no = dust.box_muller_words(torch.from_numpy(sa.view(np.int32)).cuda(),
                                       torch.from_numpy(sb.view(np.int32)).cuda())
        np.testing.assert_array_equal(np.roll(ne.cpu().numpy(), -shift).view(np.uint32), rne.view(np.uint32))
        np.testing.assert_array_equal(np.roll(no.cpu().numpy(), -shift).view(np.uint32), rno.view(np.uint32))


def test_every_radius_uniform(orc):
    k = np.arange(2**23, dtype=np.uint32)
    a = (k << 9) | (k & 0x1FF)                      # every value of a >> 9
    b = (k * np.uint32(2654435761)) & np.uint32(0xFFFFFFFF)
    _check(orc, a, b.astype(np.uint32))


@pytest.mark.parametrize("octant", range(8))
def test_every_angle_fraction(orc, octant):
    k = np.arange(2**23, dtype=np.uint32)
    b = (np.uint32(octant) << 29) | (k << 6) | (k & 0x3F)   # every fraction in this octant
    a = (k * np.uint32(2246822519)) & np.uint32(0xFFFFFFFF)
    _check(orc, a.astype(np.uint32), b.astype(np.uint32))


@pytest.mark.parametrize("d_out,with_bf16", [(4096, True), (1021, False)])
def test_draw_reduction_reproduces_the_noise(orc, d_out, with_bf16):
    """One draw with sigma = 1 and r = 1: every step of the reduction is exact
    (r rho = rho, fma(rho, cos, 0) = rho cos, scale = -1), so g = -a value for
    value (zeros may differ in sign).  This runs the packed generator as the
    hot kernel inlines it, on 4096 tokens x d_out channels."""
    T = 4096
    nz = dust.Noise(7, 3, 11, 1, 1, 1.0)
    r = torch.ones(1, T, dtype=torch.float32, device="cuda")
    g, g16 = dust.layer_estimate(r, True, None, 0.0, nz, d_out, g_hat_bf16=with_bf16)
    a = orc.noise_block(7, 3, 11, 1, np.arange(T), 0, d_out)[0]
    gh = g.cpu().numpy()
    assert np.array_equal(gh, -a)
    if with_bf16:
        assert torch.equal(g16, g.to(torch.bfloat16))


def test_noise_fill_and_synth_costs_use_the_same_noise(orc):
    """noise_fill (the gauss4 path that the head and the synthetic costs
    inline) against the oracle, bit for bit, on a block that spans many quads."""
    nz = dust.Noise(5, 2, 3, 4, 4, 0.01)
    out = dust.noise_fill(nz, 100, 64, 0, 1024)
    ref = orc.noise_block(5, 2, 3, 4, np.arange(100, 164), 0, 1024)
    np.testing.assert_array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
