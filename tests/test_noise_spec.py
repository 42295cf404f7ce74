"""Pins of the oracle's noise specification (CPU only).

The pages fix only a_t ~ N(0, I) (cnblogs Dust explainer, section
"信用分配：一次前向，两种奖励").  The oracle's generator is pinned to things
other than itself:
  - Philox4x32-10 against PyTorch's independent open-source host engine
    (ATen/core/PhiloxRNGEngine.h, compiled here into a tiny program);
  - ln and sin/cos against float64 libm (and mpmath spot checks), over EVERY
    input the generator can feed them;
  - the Box-Muller pair against the exact transform of the same uniforms;
  - the distribution (moments, KS test, cross-correlations);
  - a frozen fixture written by tests/golden/make_golden.py from the oracle.
"""
import os
import subprocess
import tempfile

import mpmath as mp
import numpy as np
import pytest
import scipy.stats as st
import torch

HERE = os.path.dirname(os.path.abspath(__file__))

PHILOX_PROG = r"""
#include <ATen/core/PhiloxRNGEngine.h>
#include <cstdio>
int main() {
  unsigned k0, k1, c0, c1, c2, c3;
  while (std::scanf("%u %u %u %u %u %u", &k0, &k1, &c0, &c1, &c2, &c3) == 6) {
    // torch: key = seed (lo, hi); counter = (offset lo, offset hi, subsequence lo, hi)
    at::philox_engine e((uint64_t(k1) << 32) | k0, (uint64_t(c3) << 32) | c2, 0);
    e.set_offset((uint64_t(c1) << 32) | c0);
    unsigned a = e(), b = e(), c = e(), d = e();
    std::printf("%u %u %u %u\n", a, b, c, d);
  }
}
"""


@pytest.fixture(scope="module")
def torch_philox():
    inc = os.path.join(os.path.dirname(torch.__file__), "include")
    d = tempfile.mkdtemp(prefix="philox_pin_")
    src, exe = os.path.join(d, "p.cpp"), os.path.join(d, "p")
    with open(src, "w") as f:
        f.write(PHILOX_PROG)
    subprocess.run(["g++", "-O1", "-std=c++17", "-I" + inc, src, "-o", exe], check=True)

    def run(keys, ctrs):
        lines = "\n".join(" ".join(str(int(v)) for v in (*k, *c)) for k, c in zip(keys, ctrs))
        out = subprocess.run([exe], input=lines, capture_output=True, text=True, check=True).stdout
        return np.array([[int(v) for v in ln.split()] for ln in out.strip().splitlines()], np.uint64).astype(np.uint32)
    return run


def test_philox_matches_torch_engine(orc, torch_philox):
    r = np.random.Generator(np.random.PCG64(11))
    keys = r.integers(0, 2**32, size=(3000, 2), dtype=np.uint64).astype(np.uint32)
    ctrs = r.integers(0, 2**32, size=(3000, 4), dtype=np.uint64).astype(np.uint32)
    # corners: all zeros, all ones, small counters as used by the kernels
    keys[:4] = [[0, 0], [0xFFFFFFFF, 0xFFFFFFFF], [0, 3], [7, 2]]
    ctrs[:4] = [[0, 0, 0, 0], [0xFFFFFFFF] * 4, [511, 16383, 16383, 0], [255, 12345, 1023, 1]]
    ref = torch_philox(keys, ctrs)
    got = orc.philox_batch(ctrs, keys)
    np.testing.assert_array_equal(got, ref)


def _ulp_err(got32, exact64):
    ulp = np.spacing(np.abs(exact64).astype(np.float32)).astype(np.float64)
    return np.abs(got32.astype(np.float64) - exact64) / ulp


def test_ln_exhaustive_within_2ulp(orc):
    k = np.arange(2**23, dtype=np.uint32)
    u = (np.float32(2.0) - (np.uint32(0x3F800000) | k).view(np.float32)).astype(np.float32)
    got = orc.ln_batch(u)
    exact = np.log(u.astype(np.float64))
    assert got[0] == 0.0 and u[0] == 1.0
    nz = exact != 0
    assert _ulp_err(got[nz], exact[nz]).max() <= 2.0
    # spot-check the float64 reference itself against mpmath
    mp.mp.prec = 80
    for idx in np.linspace(1, 2**23 - 1, 33).astype(int):
        assert abs(float(mp.log(mp.mpf(float(u[idx])))) - exact[idx]) <= 1e-15 * abs(exact[idx])


def test_sincos_exhaustive_within_1ulp(orc):
    k = np.arange(2**23, dtype=np.uint32)
    f = ((np.uint32(0x3F800000) | k).view(np.float32) - np.float32(1.0)).astype(np.float32)
    phi = (f * np.float32(np.pi / 4)).astype(np.float32)
    s, c = orc.sincos_batch(phi)
    es, ec = np.sin(phi.astype(np.float64)), np.cos(phi.astype(np.float64))
    nz = es != 0
    assert _ulp_err(s[nz], es[nz]).max() <= 1.0
    assert _ulp_err(c, ec).max() <= 1.0
    assert s[0] == 0.0 and c[0] == 1.0


def test_box_muller_matches_exact_transform(orc):
    r = np.random.Generator(np.random.PCG64(5))
    a = r.integers(0, 2**32, size=400_000, dtype=np.uint64).astype(np.uint32)
    b = r.integers(0, 2**32, size=400_000, dtype=np.uint64).astype(np.uint32)
    # include the extremes of the radius and every octant boundary
    a[:8] = [0, 0xFFFFFFFF, 0x1FF, 0x200, 0x80000000, 1, 0xFFFFFE00, 0x7FFFFFFF]
    b[:8] = np.arange(8, dtype=np.uint32) << 29
    ne, no = orc.box_muller_batch(a, b)
    # exact transform of the same uniforms in float64
    u = 2.0 - (1.0 + (a >> 9).astype(np.float64) * 2.0**-23)
    o = (b >> 29).astype(np.float64)
    f = ((b >> 6) & 0x7FFFFF).astype(np.float64) * 2.0**-23
    theta = (o + f) * (np.pi / 4)
    rho = np.sqrt(-2.0 * np.log(u))
    tol = 8 * 2.0**-24 * np.maximum(rho, 1e-30) + 1e-37
    assert np.all(np.abs(ne - rho * np.cos(theta)) <= tol)
    assert np.all(np.abs(no - rho * np.sin(theta)) <= tol)
    # the radius uniform is never 0 and the largest |a| is sqrt(46 ln 2)
    assert np.abs(np.concatenate([ne, no])).max() <= np.sqrt(46 * np.log(2)) * (1 + 1e-6)


def test_gauss_channel_layout(orc):
    """Channels 4q..4q+3 come from one Philox call: (x0,x1) -> 4q, 4q+1; (x2,x3) -> 4q+2, 4q+3."""
    for (seed, layer, draw, tok, q) in [(0, 0, 0, 0, 0), (3, 5, 17, 900, 77)]:
        x = orc.philox4x32_10([q, tok, draw, 0], [seed, layer])
        e0, o0 = orc.box_muller(int(x[0]), int(x[1]))
        e1, o1 = orc.box_muller(int(x[2]), int(x[3]))
        got = [orc.gauss(seed, layer, draw, tok, 4 * q + j) for j in range(4)]
        assert np.array_equal(np.array(got, np.float32), np.array([e0, o0, e1, o1], np.float32))


def test_gauss_distribution(orc):
    toks = np.arange(256)
    a = orc.noise_block(0, 0, 0, 8, toks, 0, 512)          # 8 draws x 256 tokens x 512 channels
    x = a.ravel().astype(np.float64)
    n = x.size
    assert abs(x.mean()) < 4 / np.sqrt(n)
    assert abs(x.var() - 1.0) < 4 * np.sqrt(2.0 / n)
    assert abs(st.skew(x)) < 4 * np.sqrt(6.0 / n)
    assert abs(st.kurtosis(x)) < 4 * np.sqrt(24.0 / n)
    assert st.kstest(x[: 2**20], "norm").pvalue > 1e-3
    # independence across channels, tokens, draws (adjacent and one Philox call apart)
    lim = 4 / np.sqrt(a[:, :, :-1].size)
    for sl0, sl1 in [((slice(None), slice(None), slice(0, -1)), (slice(None), slice(None), slice(1, None))),
                     ((slice(None), slice(None), slice(0, -4)), (slice(None), slice(None), slice(4, None))),
                     ((slice(None), slice(0, -1), slice(None)), (slice(None), slice(1, None), slice(None))),
                     ((slice(0, -1), slice(None), slice(None)), (slice(1, None), slice(None), slice(None)))]:
        assert abs(np.corrcoef(a[sl0].ravel(), a[sl1].ravel())[0, 1]) < lim
    # even/odd (cosine/sine) branches of one pair are uncorrelated, also in squares
    ev, od = a[..., 0::2].ravel(), a[..., 1::2].ravel()
    assert abs(np.corrcoef(ev, od)[0, 1]) < lim
    assert abs(np.corrcoef(ev**2, od**2)[0, 1]) < 2 * lim
    # streams are independent too
    e1 = np.array([orc.gauss(0, 0, i, t, 0, 1) for i in range(4) for t in range(512)])
    e0 = np.array([orc.gauss(0, 0, i, t, 0, 0) for i in range(4) for t in range(512)])
    assert abs(np.corrcoef(e0, e1)[0, 1]) < 4 / np.sqrt(e0.size)


def test_frozen_fixture(orc):
    path = os.path.join(HERE, "golden", "noise_spec_seed0.txt")
    n = 0
    with open(path) as f:
        for line in f:
            if line.startswith("#"):
                continue
            left, right = line.split("|")
            s, l, d, t, c, stream, bits = left.split()
            v = orc.gauss(int(s), int(l), int(d), int(t), int(c), int(stream))
            assert int(v.view(np.uint32)) == int(bits, 16), line
            words = orc.philox4x32_10([int(c) >> 2, int(t), int(d), int(stream)], [int(s), int(l)])
            assert [f"{int(w):08x}" for w in words] == right.split(), line
            n += 1
    assert n >= 10
