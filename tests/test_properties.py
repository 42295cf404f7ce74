"""Property tests (hypothesis) on random small shapes: the oracle's invariants
and the data-parallel range helpers.  CPU only."""
import numpy as np
from hypothesis import given, settings, strategies as st

from activation_perturbation_es_b200 import dp
from activation_perturbation_es_b200 import inputs as I

lengths_st = st.lists(st.integers(min_value=0, max_value=9), min_size=1, max_size=6).filter(lambda l: sum(l) > 0)


@settings(max_examples=40, deadline=None)
@given(lengths=lengths_st, K=st.integers(1, 4), gamma=st.sampled_from([0.0, 0.3, 0.9, 1.0]),
       seed=st.integers(0, 1000))
def test_scan_recurrence_matches_brute_force(orc, lengths, K, gamma, seed):
    off = I.offsets_from_lengths(lengths)
    c = I.normal((K, int(off[-1])), 1.0, seed=seed)
    np.testing.assert_allclose(orc.reward_scan(c, off, gamma), orc.reward_scan(c, off, gamma, brute=True),
                               rtol=1e-12, atol=1e-12)


@settings(max_examples=25, deadline=None)
@given(lengths=lengths_st, d=st.integers(1, 9), K=st.integers(2, 6), split=st.integers(1, 5),
       gamma=st.sampled_from([0.0, 0.5, 1.0]), seed=st.integers(0, 1000))
def test_estimate_is_additive_over_draw_ranges(orc, lengths, d, K, split, gamma, seed):
    split = min(split, K - 1)
    off = I.offsets_from_lengths(lengths)
    T = int(off[-1])
    c = I.normal((K, T), 0.01, seed=seed)
    toks = np.arange(T)
    full = orc.layer_estimate(c, False, d, off, gamma, seed, 1, 0, K, 0.01, toks)
    a = orc.layer_estimate(c[:split], False, d, off, gamma, seed, 1, 0, K, 0.01, toks)
    b = orc.layer_estimate(c[split:], False, d, off, gamma, seed, 1, split, K, 0.01, toks)
    np.testing.assert_allclose(a + b, full, rtol=1e-11, atol=1e-13)


@settings(max_examples=25, deadline=None)
@given(T=st.integers(1, 6), V=st.sampled_from([4, 8, 12]), nd=st.integers(1, 3), seed=st.integers(0, 1000))
def test_head_costs_vanish_when_sigma_does(orc, T, V, nd, seed):
    """c = l~ - l is 0 when the perturbation is 0; its even part in sigma is
    second order (|c(s) + c(-s)| <= s^2 sum_chunk a^2, the curvature of the
    cross entropy being at most 1/2 per squared logit change), and the
    first-order coefficient (c(s) - c(-s)) / 2s agrees at two step sizes up to
    O(s^2)."""
    Z = I.normal((T, V), 1.0, seed=seed)
    y = I.targets(T, V, seed=seed + 1)
    run = lambda s: orc.head_step(Z, y, np.arange(T), V // 2, seed, 0, 0, nd, nd, s)[0]
    assert np.all(np.abs(run(1e-30)) < 1e-25)
    s = 1e-3
    a2 = np.zeros((2, nd, T))                       # two chunks of V/2
    for ch in range(2):
        blk = orc.noise_block(seed, 0, 0, nd, np.arange(T), ch * (V // 2), V // 2)
        a2[ch] = np.sum(blk.astype(np.float64) ** 2, axis=2)
    cp, cm = run(s), run(-s)
    assert np.all(np.abs(cp + cm) <= s * s * a2 + 1e-12)
    d1 = (cp - cm) / (2 * s)
    d2 = (run(2 * s) - run(-2 * s)) / (4 * s)
    assert np.all(np.abs(d1 - d2) <= 10 * s * s * a2 * np.sqrt(a2) + 1e-9)


@given(K=st.integers(1, 10_000), world=st.integers(1, 16))
def test_draw_ranges_partition(K, world):
    rs = [dp.draw_range(K, world, r) for r in range(world)]
    assert rs[0][0] == 0 and sum(n for _, n in rs) == K
    for (b0, n0), (b1, _) in zip(rs, rs[1:]):
        assert b0 + n0 == b1
    assert max(n for _, n in rs) - min(n for _, n in rs) <= 1


@given(n_seq=st.integers(1, 500), world=st.integers(1, 16))
def test_sequence_ranges_partition(n_seq, world):
    rs = [dp.sequence_range(n_seq, world, r) for r in range(world)]
    assert rs[0][0] == 0 and rs[-1][1] == n_seq
    assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
