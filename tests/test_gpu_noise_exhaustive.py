"""Exhaustive bit-exactness of the GPU Box-Muller step against the oracle.

The transform sees only 2^23 distinct radius uniforms (the top 23 bits of the
first word) and 2^26 distinct angles (octant + 23 fraction bits of the
second).  These tests run every radius value (paired with varied angle words)
and every angle fraction in every octant (paired with varied radius words),
so every ln / sqrt / sin / cos evaluation the generator can ever perform is
checked bit for bit."""
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
    ne, no = dust.box_muller_words(torch.from_numpy(a.view(np.int32)).cuda(), torch.from_numpy(b.view(np.int32)).cuda())
    rne, rno = orc.box_muller_batch(a, b)
    np.testing.assert_array_equal(ne.cpu().numpy().view(np.uint32), rne.view(np.uint32))
    np.testing.assert_array_equal(no.cpu().numpy().view(np.uint32), rno.view(np.uint32))


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
