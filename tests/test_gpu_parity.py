"""GPU parity: every C-ABI entry point against the CPU oracle.

Bars (from the estimator's statement): noise and indices bit-exact; floating
point within max relative error 1e-3 (fp32 paths) and 2e-2 (bf16-input GEMM
paths), with err = max_k |gpu_k - orc_k| / max_k |orc_k| per output tensor.
Where both sides consume identical inputs the tests also assert the tighter
bound the fp32 arithmetic itself allows (noted per test).
"""
import numpy as np
import pytest
import torch

from activation_perturbation_es_b200 import dust
from activation_perturbation_es_b200 import inputs as I

import oracle_chains  # noqa: E402

pytestmark = pytest.mark.gpu

FP32_TOL = 1e-3
BF16_TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dust.lib()


def rel_err(gpu, orc):
    gpu = np.asarray(gpu, np.float64)
    orc = np.asarray(orc, np.float64)
    return float(np.max(np.abs(gpu - orc)) / max(np.max(np.abs(orc)), 1e-300))


def cu(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.to(dtype)


def host(t):
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


# ------------------------------------------------------------------ a1 noise
@pytest.mark.parametrize("seed,layer,d0,nd,t0,nt,j0,nc,stream", [
    (0, 0, 0, 3, 0, 17, 0, 64, 0),
    (7, 2, 1021, 4, 12340, 9, 1, 13, 0),         # odd channel start / count, crossing quads
    (0, 9, 4095, 2, 65530, 6, 4090, 6, 0),        # large indices
    (123456789, 42, 77, 3, 88, 5, 0, 3, 1),       # observation-noise stream
    (2**32 - 1, 2**32 - 1, 2**32 - 3, 3, 0, 4, 1021, 7, 0),
])
def test_noise_bit_exact(orc, seed, layer, d0, nd, t0, nt, j0, nc, stream):
    nz = dust.Noise(seed, layer, d0, nd, nd, 1.0)
    gpu = host(dust.noise_fill(nz, t0, nt, j0, nc, stream_id=stream))
    ref = orc.noise_block(seed, layer, d0, nd, np.arange(t0, t0 + nt), j0, nc, stream=stream)
    np.testing.assert_array_equal(gpu.view(np.uint32), ref.view(np.uint32))


def test_noise_bit_exact_bulk(orc):
    """A 2 x 512 x 512 block (2^19 values) -- every Box-Muller branch is hit."""
    nz = dust.Noise(3, 4, 100, 2, 2, 1.0)
    gpu = host(dust.noise_fill(nz, 1000, 512, 0, 512))
    ref = orc.noise_block(3, 4, 100, 2, np.arange(1000, 1512), 0, 512)
    np.testing.assert_array_equal(gpu.view(np.uint32), ref.view(np.uint32))


# ------------------------------------------------------------------ a4 scan
SCAN_CASES = [
    ([5, 0, 1, 17, 3, 0, 33, 2], 7),        # ragged with empty sequences, odd T (61)
    ([3000, 1, 1500], 3),                    # multi-chunk sequences (carry across chunks)
    ([1024] * 4, 5),
    ([1], 2),                                # single token
]


@pytest.mark.parametrize("lengths,K", SCAN_CASES)
@pytest.mark.parametrize("gamma", [0.0, 0.5, 0.9, 0.95, 0.99, 1.0])
def test_reward_scan_parity(orc, lengths, K, gamma):
    off = I.offsets_from_lengths(lengths)
    T = int(off[-1])
    c = I.normal((K, T), 0.01, seed=K + T)
    ref = orc.reward_scan(c, off, gamma)
    gc, goff = cu(c), cu(off)
    r = host(dust.reward_scan(gc, goff, gamma))
    assert rel_err(r, ref) < 1e-5          # fp32 scan: ~L eps at worst
    if gamma == 0.0:
        np.testing.assert_array_equal(r.view(np.uint32), c.view(np.uint32))
    inplace = gc.clone()
    dust.reward_scan(inplace, goff, gamma, out=inplace)
    np.testing.assert_array_equal(host(inplace).view(np.uint32), r.view(np.uint32))


SPLIT_CASES = [
    ([70000], 3),                                   # one long sequence (69 chunks)
    ([1500, 1, 0, 2047, 1024, 3000, 5], 4),         # boundaries inside and at chunk edges, empty sequences
    ([5, 0, 1, 17, 3, 0, 33, 2], 7),                # many sequences inside one chunk
    ([1], 2),
]


@pytest.mark.parametrize("lengths,K", SPLIT_CASES)
@pytest.mark.parametrize("gamma", [0.0, 0.5, 0.99, 1.0])
def test_reward_scan_split_parity(orc, lengths, K, gamma):
    """The chunked scan gives the same rewards as the oracle's recurrence (and the
    per-sequence scan), in place too."""
    off = I.offsets_from_lengths(lengths)
    T = int(off[-1])
    c = I.normal((K, T), 0.01, seed=K + T + 1)
    ref = orc.reward_scan(c, off, gamma)
    gc, goff = cu(c), cu(off)
    r = host(dust.reward_scan_split(gc, goff, gamma))
    assert rel_err(r, ref) < 1e-5
    if gamma == 0.0:
        np.testing.assert_array_equal(r.view(np.uint32), c.view(np.uint32))
    inplace = gc.clone()
    dust.reward_scan_split(inplace, goff, gamma, out=inplace)
    np.testing.assert_array_equal(host(inplace).view(np.uint32), r.view(np.uint32))


def test_reward_scan_split_one_very_long_sequence(orc):
    """The case the chunked scan is timed on: one sequence of 262144 tokens
    (256 chunks per draw row), K = 16, gamma = 0.99; every reward against the
    oracle's recurrence, and the per-sequence scan's rewards."""
    T, K, gamma = 262144, 16, 0.99
    off = np.array([0, T], np.int32)
    c = I.normal((K, T), 0.01, seed=2026)
    ref = orc.reward_scan(c, off, gamma)
    gc, goff = cu(c), cu(off)
    r = host(dust.reward_scan_split(gc, goff, gamma))
    assert rel_err(r, ref) < 1e-5
    assert rel_err(host(dust.reward_scan(gc, goff, gamma)), ref) < 1e-5


def test_layer_estimate_long_sequence_uses_chunked_scan(orc):
    """K x n_seq small and one long sequence: the estimate runs the chunked scan internally."""
    T, K, d = 9000, 4, 16
    off = np.array([0, T], np.int32)
    c = I.normal((K, T), 0.01, seed=77)
    g, _ = dust.layer_estimate(cu(c), False, cu(off), 0.97, dust.Noise(2, 3, 0, K, K, 0.01), d)
    toks = np.array([0, 1023, 1024, 4500, 8999])
    ref = orc.layer_estimate(c, False, d, off, 0.97, 2, 3, 0, K, 0.01, toks)
    assert rel_err(host(g)[toks], ref) < 1e-5


# ------------------------------------------------------------------ a5 estimate
@pytest.mark.parametrize("T,d_out,K,gamma,is_r", [
    (37, 10, 9, 0.9, False),
    (64, 64, 16, 0.0, False),
    (130, 130, 5, 0.95, True),
    (256, 13, 33, 1.0, False),
])
def test_layer_estimate_parity(orc, T, d_out, K, gamma, is_r):
    off = I.offsets_from_lengths(I.ragged_lengths(T, 3, seed=T, allow_empty=False))
    c = I.normal((K, T), 0.01, seed=T + K)
    arr = orc.reward_scan(c, off, gamma).astype(np.float32) if is_r else c
    nz = dust.Noise(5, 11, 3, K, K, 0.01)
    g, g16 = dust.layer_estimate(cu(arr), is_r, cu(off), gamma, nz, d_out, g_hat_bf16=True)
    ref = orc.layer_estimate(arr, is_r, d_out, off, gamma, 5, 11, 3, K, 0.01, np.arange(T))
    assert rel_err(host(g), ref) < 1e-5
    # bf16 copy is round-to-nearest-even of the fp32 result
    np.testing.assert_array_equal(host(g16), I.bf16_round(host(g)))


def test_layer_estimate_draw_split_additivity(orc):
    T, d, K = 48, 20, 12
    off = I.uniform_offsets(2, 24)
    c = I.normal((K, T), 0.01, seed=3)
    gc, goff = cu(c), cu(off)
    full, _ = dust.layer_estimate(gc, False, goff, 0.9, dust.Noise(0, 1, 0, K, K, 0.01), d)
    part, _ = dust.layer_estimate(gc[:5].contiguous(), False, goff, 0.9, dust.Noise(0, 1, 0, 5, K, 0.01), d)
    dust.layer_estimate(gc[5:].contiguous(), False, goff, 0.9, dust.Noise(0, 1, 5, K - 5, K, 0.01), d,
                        g_hat=part, accumulate=True)
    assert rel_err(host(part), host(full)) < 1e-6


def test_synth_costs_parity(orc):
    T, d, K = 200, 36, 40
    u = I.normal((T, d), 1.0, seed=9)
    c = host(dust.synth_costs(cu(u), dust.Noise(0, 3, 10, K, K, 0.01), 0.01))
    rs = np.random.Generator(np.random.PCG64(1))
    ks, ts = rs.integers(0, K, 300), rs.integers(0, T, 300)
    ref = orc.synth_costs(u, 0, 3, 0.01, 0.01, ks + 10, ts)
    assert rel_err(c[ks, ts], ref) < 1e-5


# ------------------------------------------------------------------ a6 / a2 GEMMs
@pytest.mark.parametrize("T,d_in,d_out", [(100, 24, 40), (333, 7, 65), (4096, 64, 96)])
def test_weight_grad_f32(orc, T, d_in, d_out):
    g = I.normal((T, d_out), 1.0, seed=T)
    X = I.normal((T, d_in), 1.0, seed=T + 1)
    G = host(dust.weight_grad(cu(g), cu(X)))
    assert rel_err(G, orc.weight_grad(g, X)) < 1e-5


@pytest.mark.parametrize("T,d_in,d_out", [(256, 64, 128), (1000, 48, 32), (16384, 512, 512), (2048, 2048, 512),
                                          (16384, 512, 4096), (16384, 520, 136)])
def test_weight_grad_bf16(orc, T, d_in, d_out):
    """(16384, 520, 136) splits k, and its tiles are ragged in both output
    dimensions: the split slabs' TMA stores are clipped by the 3-D map."""
    g = I.bf16_round(I.normal((T, d_out), 1.0, seed=T))
    X = I.bf16_round(I.normal((T, d_in), 1.0, seed=T + 1))
    G = host(dust.weight_grad(cu(g, torch.bfloat16), cu(X, torch.bfloat16)))
    rows = np.arange(d_out) if d_out * T <= 2**22 else np.random.Generator(np.random.PCG64(0)).integers(0, d_out, 24)
    assert rel_err(G[rows], orc.weight_grad(g, X, rows=rows)) < 1e-4   # same bf16 inputs, fp32 accumulation


@pytest.mark.parametrize("T,d_in,d_out", [(200, 24, 40), (777, 520, 136), (64, 64, 64)])
def test_weight_grad_bf16_ragged_and_accumulate(orc, T, d_in, d_out):
    """Tensor-core path with tails in every dimension (M, N not multiples of the
    tile, T not a multiple of the 64-deep k block) and accumulate = 1."""
    g = I.bf16_round(I.normal((T, d_out), 1.0, seed=T + 5))
    X = I.bf16_round(I.normal((T, d_in), 1.0, seed=T + 6))
    G0 = I.normal((d_out, d_in), 1.0, seed=T + 7)
    G = cu(G0)
    dust.weight_grad(cu(g, torch.bfloat16), cu(X, torch.bfloat16), G_W=G, accumulate=True)
    ref = orc.weight_grad(g, X) + G0.astype(np.float64)
    assert rel_err(host(G), ref) < 1e-5


@pytest.mark.parametrize("g_bf16", [False, True])
@pytest.mark.parametrize("T,d_in,d_out", [(1000, 72, 40), (4096, 256, 130)])
def test_weight_grad_mixed_dtypes(orc, g_bf16, T, d_in, d_out):
    """fp32 g with bf16 X and bf16 g with fp32 X (the reduction's fp32 g against
    a bf16 layer input, or its bf16 copy against an fp32 input): the bf16
    operand is widened exactly, so the bar is fp32 accumulation's."""
    g = I.normal((T, d_out), 1.0, seed=T + 11)
    X = I.normal((T, d_in), 1.0, seed=T + 12)
    if g_bf16:
        g = I.bf16_round(g)
    else:
        X = I.bf16_round(X)
    G0 = I.normal((d_out, d_in), 1.0, seed=T + 13)
    G = cu(G0)
    dust.weight_grad(cu(g, torch.bfloat16 if g_bf16 else torch.float32),
                     cu(X, torch.float32 if g_bf16 else torch.bfloat16), G_W=G, accumulate=True)
    assert rel_err(host(G), orc.weight_grad(g, X) + G0.astype(np.float64)) < 1e-5


@pytest.mark.parametrize("T,d_in,V", [(1000, 64, 520), (256, 1024, 4096), (1000, 64, 522)])
def test_logits_bf16_tensor_cores(orc, T, d_in, V):
    """V = 522: a row pitch that is not a multiple of 16 bytes, which the
    epilogue writes with row stores instead of TMA stores."""
    X = I.bf16_round(I.normal((T, d_in), 1.0, seed=T))
    W = I.bf16_round(I.normal((V, d_in), 1.0 / np.sqrt(d_in), seed=V))
    Z = dust.logits(cu(X, torch.bfloat16), cu(W, torch.bfloat16))
    toks = np.arange(0, T, 7)
    assert rel_err(host(Z)[toks], orc.logits(X, W, toks)) < 1e-5


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_logits_and_row_stats(orc, dt):
    T, d_in, V = 300, 64, 512
    X = I.bf16_round(I.normal((T, d_in), 1.0, seed=1))
    W = I.bf16_round(I.normal((V, d_in), 0.125, seed=2))
    y = I.targets(T, V, seed=3)
    Z = dust.logits(cu(X, dt), cu(W, dt))
    toks = np.arange(T)
    assert rel_err(host(Z), orc.logits(X, W, toks)) < 1e-5
    # row statistics on a seeded logits matrix (an input of their own)
    Zh = I.normal((T, V), 1.5, seed=4)
    lse, ell = dust.head_row_stats(cu(Zh), cu(y))
    ref_lse, ref_ell = orc.head_clean(Zh, y)
    assert rel_err(host(lse), ref_lse) < 1e-6
    assert np.max(np.abs(host(ell) - ref_ell)) < 1e-5 * np.max(np.abs(ref_lse))


# ------------------------------------------------------------------ head
def _head_check(orc, Z, y, toks, Vc, nz, out, tol):
    c_ref, g_ref = orc.head_step(Z[toks], y[toks], toks, Vc, nz.seed, nz.layer, nz.draw_begin, nz.draw_count,
                                 nz.K_total, nz.sigma)
    g = host(out["g_hat"])[toks]
    assert rel_err(g, g_ref) < tol
    if out["c"] is not None:
        assert rel_err(host(out["c"])[:, :, toks], c_ref) < tol


def test_head_step_small_fp32(orc):
    """HEAD_SMALL: T = 256, d = 64, V = Vc = 512, K = 16, fp32; cached and recomputed logits."""
    w = I.HEAD_SMALL
    h = I.head_inputs(w)
    X, W, y = cu(h["X"]), cu(h["W"]), cu(h["y"])
    nz = dust.Noise(w.seed, w.head_layer, 0, w.K, w.K, w.sigma)
    Zr = orc.logits(h["X"], h["W"]).astype(np.float32)
    toks = np.arange(w.T)
    cached = dust.head_step(y, w.Vc, nz, Z=cu(Zr), X=X, want_c=True, want_G_W=True)
    _head_check(orc, Zr, h["y"], toks, w.Vc, nz, cached, FP32_TOL)
    rec = dust.head_step(y, w.Vc, nz, X=X, W=W, want_c=True, want_G_W=True)
    _head_check(orc, Zr, h["y"], toks, w.Vc, nz, rec, FP32_TOL)
    # G_W = g^T X from the oracle's g
    _, g_ref = orc.head_step(Zr, h["y"], toks, w.Vc, nz.seed, nz.layer, 0, w.K, w.K, w.sigma, want_c=False)
    G_ref = g_ref.T @ h["X"].astype(np.float64)
    assert rel_err(host(rec["G_W"]), G_ref) < FP32_TOL
    assert rel_err(host(cached["G_W"]), G_ref) < FP32_TOL


@pytest.mark.parametrize("sigma", [0.005, 0.02, 0.05, 0.1, 0.3])   # the four expm1 tiers of the head kernel
                                                                   # (0.05 and 0.1: the x^8 series)
def test_head_step_chunks_and_split(orc, sigma):
    """Several chunks, draw split with accumulate, target ids on chunk edges."""
    T, V, Vc, K = 40, 768, 256, 10
    Z = I.normal((T, V), 1.5, seed=5)
    y = I.targets(T, V, seed=6)
    y[:6] = [0, 255, 256, 511, 512, 767]
    gz, gy = cu(Z), cu(y)
    full = dust.head_step(gy, Vc, dust.Noise(1, 2, 0, K, K, sigma), Z=gz, want_c=True)
    _head_check(orc, Z, y, np.arange(T), Vc, dust.Noise(1, 2, 0, K, K, sigma), full, 1e-4)
    part = dust.head_step(gy, Vc, dust.Noise(1, 2, 0, 4, K, sigma), Z=gz)
    dust.head_step(gy, Vc, dust.Noise(1, 2, 4, K - 4, K, sigma), Z=gz, g_hat=part["g_hat"], accumulate=True)
    assert rel_err(host(part["g_hat"]), host(full["g_hat"])) < 1e-6


@pytest.mark.parametrize("V,Vc,sigma", [(2560, 1280, 0.01), (4096, 2048, 0.05), (5120, 2560, 0.01),
                                         (4096, 4096, 0.02)])
def test_head_wide_chunks(orc, V, Vc, sigma):
    """Chunks wider than 1024 ids (2 or 4 warps per token, partial sums met in
    shared memory), including the whole-vocabulary reading Vc = V."""
    T, K = 24, 6
    Z = I.normal((T, V), 1.5, seed=V + Vc)
    y = I.targets(T, V, seed=V)
    sub = Vc // (2 if Vc <= 2048 else 4)        # ids per warp
    y[:6] = [0, sub - 1, sub, Vc - 1, Vc % V, V - 1]   # targets on warp and chunk edges
    nz = dust.Noise(2, 8, 3, K, K, sigma)
    out = dust.head_step(cu(y), Vc, nz, Z=cu(Z), want_c=True)
    _head_check(orc, Z, y, np.arange(T), Vc, nz, out, 1e-4)


@pytest.mark.parametrize("K", [64])
def test_head_pages_sampled(orc, K):
    """HEAD_PAGES at full size (16 x 1024 tokens, V = 4096, Vc = 1024, bf16 X/W),
    logits recomputed on the tensor cores: sampled tokens against the oracle
    (given the oracle's own logits rows), and G_W as the weight GEMM of g."""
    w = I.HEAD_PAGES
    h = I.head_inputs(w)
    X, W, y = cu(h["X"], torch.bfloat16), cu(h["W"], torch.bfloat16), cu(h["y"])
    nz = dust.Noise(w.seed, w.head_layer, 0, K, K, w.sigma)
    out = dust.head_step(y, w.Vc, nz, X=X, W=W, want_c=True, want_bf16=True, want_G_W=True)
    toks = np.random.Generator(np.random.PCG64(7)).choice(w.T, 12, replace=False)
    Zs = orc.logits(h["X"], h["W"], toks).astype(np.float32)
    # the oracle gets the same tokens' logits rows (double -> fp32) and the global token ids
    c_ref, g_ref = orc.head_step(Zs, h["y"][toks], toks, w.Vc, nz.seed, nz.layer, 0, K, K, w.sigma)
    assert rel_err(host(out["g_hat"])[toks], g_ref) < FP32_TOL
    assert rel_err(host(out["c"])[:, :, toks], c_ref) < FP32_TOL
    # G_W rows against the oracle's chain: its g over all 16384 tokens (the
    # logits are the float64 product X W^T, rounded to binary32 as the oracle's
    # logits are), held in binary32 and rounded to bf16 as the kernels hold it
    X64, W64 = h["X"].astype(np.float64), h["W"].astype(np.float64)
    Z_all = (X64 @ W64.T).astype(np.float32)
    _, g_all = orc.head_step(Z_all, h["y"], np.arange(w.T), w.Vc, nz.seed, nz.layer, 0, K, K, w.sigma,
                             want_c=False)
    rows = np.sort(np.random.Generator(np.random.PCG64(8)).choice(w.V, 8, replace=False))
    g_rows = torch.from_numpy(np.ascontiguousarray(g_all[:, rows]).astype(np.float32)).to(torch.bfloat16)
    G_ref = orc.weight_grad(g_rows.float().numpy(), h["X"], rows=np.arange(len(rows)))
    assert rel_err(host(out["G_W"])[rows], G_ref) < 1e-3


# ------------------------------------------------------------------ hidden layer, config-sized
def test_hidden_sweep_sampled(orc):
    """HIDDEN_SWEEP (T = 16 x 1024, gamma = 0.95) for every layer shape at K = 64,
    in the launch configuration the benchmark times.  The synthetic costs are
    checked on sampled (draw, token) pairs; scan, reduction and weight estimate
    then run on seeded costs, and sampled tokens / rows of g and G_W are
    checked against the oracle's chain on the same costs."""
    w = I.HIDDEN_SWEEP
    K = 64
    off = I.uniform_offsets(w.n_seq, w.seq_len)
    for layer in w.hidden:
        li = I.layer_inputs(w, layer)
        nz = dust.Noise(w.seed, layer.layer, 0, K, K, w.sigma)
        rs = np.random.Generator(np.random.PCG64(layer.layer))
        toks = np.sort(rs.choice(w.T, 6, replace=False))
        c_gpu = host(dust.synth_costs(cu(li["u"]), nz, w.eps_scale))
        ks = rs.integers(0, K, 64)
        assert rel_err(c_gpu[ks, toks[ks % 6]],
                       orc.synth_costs(li["u"], w.seed, layer.layer, w.sigma, w.eps_scale, ks, toks[ks % 6])) < 1e-5
        c = I.normal((K, w.T), 0.02, seed=100 + layer.layer)
        g, g16 = dust.layer_estimate(cu(c), False, cu(off), w.gamma, nz, layer.d_out, g_hat_bf16=True)
        G = dust.weight_grad(g16, cu(li["X"], torch.bfloat16))
        g_ref = orc.layer_estimate(c, False, layer.d_out, off, w.gamma, w.seed, layer.layer, 0, K, w.sigma, toks)
        assert rel_err(host(g)[toks], g_ref) < FP32_TOL
        rows = rs.choice(layer.d_out, 4, replace=False)
        G_ref = oracle_chains.weight_rows(orc, c, False, layer.d_out, off, w.gamma, w.seed, layer.layer, 0, K,
                                          w.sigma, li["X"], rows)
        assert rel_err(host(G)[rows], G_ref) < 1e-3


# ------------------------------------------------------------------ toy suffix (hidden layer, fp32)
def test_hidden_suffix_end_to_end(orc):
    """HIDDEN_SUFFIX: losses of the toy suffix against the oracle, then the
    estimator on the oracle's costs for gamma in {0, 0.9, 1}."""
    w = I.HIDDEN_SUFFIX
    s = I.suffix_inputs(w)
    off = I.uniform_offsets(w.n_seq, w.seq_len)
    layer = w.hidden[0]
    Y = dust.logits(cu(s["X"]), cu(s["W"]))       # the layer's clean output y = X W^T
    nz = dust.Noise(w.seed, layer.layer, 0, w.K, w.K, w.sigma)
    loss, c = dust.toy_suffix_losses(Y, cu(off), cu(s["Wq"]), cu(s["Wk"]), cu(s["Wv"]), cu(s["Wo"]),
                                     cu(s["Wout"]), cu(s["y"]), nz)
    draws = np.array([0, 17, 63])
    ref = orc.toy_suffix_losses(s["X"], s["W"], off, s["Wq"], s["Wk"], s["Wv"], s["Wo"], s["Wout"], s["y"],
                                w.seed, layer.layer, w.sigma, draws)
    clean = orc.toy_suffix_losses(s["X"], s["W"], off, s["Wq"], s["Wk"], s["Wv"], s["Wo"], s["Wout"], s["y"],
                                  w.seed, layer.layer, w.sigma, [0], with_noise=False)[0]
    loss_h = host(loss)
    assert rel_err(loss_h[0], clean) < 1e-5
    assert rel_err(loss_h[1 + draws], ref) < 1e-5
    # c = l~ - l: a difference of two O(log V) numbers in fp32; its bar is
    # relative to max|c| with the fp32 loss rounding (|loss| eps ~ 1e-6) on top.
    c_ref = ref - clean[None, :]
    assert rel_err(host(c)[draws], c_ref) < 5e-3
    # every draw's costs from the oracle; the GPU estimator runs on them
    all_ref = orc.toy_suffix_losses(s["X"], s["W"], off, s["Wq"], s["Wk"], s["Wv"], s["Wo"], s["Wout"], s["y"],
                                    w.seed, layer.layer, w.sigma, np.arange(w.K))
    c_orc = (all_ref - clean[None, :]).astype(np.float32)
    assert rel_err(host(c), c_orc) < 5e-3
    X32 = cu(s["X"])
    rows = np.arange(0, 256, 37)
    for gamma in w.notes["gammas"]:
        g, _ = dust.layer_estimate(cu(c_orc), False, cu(off), gamma, nz, layer.d_out)
        toks = np.array([0, 1, 255, 256, 700, 1023])
        g_ref = orc.layer_estimate(c_orc, False, layer.d_out, off, gamma, w.seed, layer.layer, 0, w.K, w.sigma, toks)
        assert rel_err(host(g)[toks], g_ref) < FP32_TOL
        G = dust.weight_grad(g, X32)
        G_ref = oracle_chains.weight_rows(orc, c_orc, False, layer.d_out, off, gamma, w.seed, layer.layer, 0, w.K,
                                          w.sigma, s["X"], rows, bf16=False)
        assert rel_err(host(G)[rows], G_ref) < 1e-4
