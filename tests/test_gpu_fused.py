"""Parity of the fused draw reduction + weight estimate
(dust_layer_estimate_weight_grad): g produced in shared memory as the tensor
cores' operand, G_W's row block in TMEM.  Against the oracle's chain on the
same seeded costs, against the unfused calls, with ragged tokens, ragged
channel blocks, every supported width class and accumulate."""
import numpy as np
import pytest
import torch

from activation_perturbation_es_b200 import dust
from activation_perturbation_es_b200 import inputs as I

import oracle_chains  # noqa: E402

pytestmark = pytest.mark.gpu
FP32_TOL = 1e-3
BF16_G_TOL = 1e-3      # G_W from bf16 g: rounding decisions may differ at binary32 ties


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dust.lib()


def rel_err(gpu, orc):
    return float(np.max(np.abs(np.asarray(gpu, np.float64) - orc)) / np.max(np.abs(orc)))


def cu(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.to(dtype)


def host(t):
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


CASES = [
    # T, d_out, d_in, K, gamma, n_seq
    (300, 200, 128, 8, 0.9, 5),     # ragged 48-token stages, ragged 128-channel block, scan inside
    (1000, 128, 512, 5, 0.0, 3),    # the whole TMEM (two 256-wide MMAs), odd K, gamma = 0 (r = c)
    (97, 40, 64, 16, 1.0, 2),       # fewer tokens than a stage, narrowest width
    (512, 384, 384, 12, 0.5, 4),    # 256 + 128 wide MMAs, three channel blocks
]


@pytest.mark.parametrize("T,d_out,d_in,K,gamma,n_seq", CASES)
def test_fused_against_oracle(orc, T, d_out, d_in, K, gamma, n_seq):
    off = I.offsets_from_lengths(I.ragged_lengths(T, n_seq, seed=T + n_seq))
    c = I.normal((K, T), 0.02, seed=T + 1)
    X = I.bf16_round(I.normal((T, d_in), 1.0, seed=T + 2))
    nz = dust.Noise(3, 9, 2, K, K, 0.01)
    G, g = dust.layer_estimate_weight_grad(cu(c), False, cu(off), gamma, nz, cu(X, torch.bfloat16), d_out,
                                           g_hat=True)
    g_ref = orc.layer_estimate(c, False, d_out, off, gamma, 3, 9, 2, K, 0.01, np.arange(T))
    assert rel_err(host(g), g_ref) < FP32_TOL
    G_ref = oracle_chains.weight_rows(orc, c, False, d_out, off, gamma, 3, 9, 2, K, 0.01, X, np.arange(d_out))
    assert rel_err(host(G), G_ref) < BF16_G_TOL


@pytest.mark.parametrize("T,d_out,d_in,K,gamma,n_seq", CASES)
def test_fused_equals_unfused(T, d_out, d_in, K, gamma, n_seq):
    """The fused kernel's g is the standalone reduction's bit for bit; G_W
    matches the tensor-core weight GEMM of its bf16 copy up to fp32
    accumulation order; accumulate = 1 adds."""
    off = cu(I.offsets_from_lengths(I.ragged_lengths(T, n_seq, seed=T + n_seq)))
    c = cu(I.normal((K, T), 0.02, seed=T + 1))
    X = cu(I.bf16_round(I.normal((T, d_in), 1.0, seed=T + 2)), torch.bfloat16)
    nz = dust.Noise(3, 9, 2, K, K, 0.01)
    G, g = dust.layer_estimate_weight_grad(c, False, off, gamma, nz, X, d_out, g_hat=True)
    g1, g16 = dust.layer_estimate(c, False, off, gamma, nz, d_out, g_hat_bf16=True)
    assert torch.equal(g, g1)
    G1 = dust.weight_grad(g16, X)
    assert rel_err(host(G), host(G1).astype(np.float64)) < 1e-5
    G0 = cu(I.normal((d_out, d_in), 1.0, seed=5))
    base = host(G0).astype(np.float64)
    dust.layer_estimate_weight_grad(c, False, off, gamma, nz, X, d_out, G_W=G0, accumulate=True)
    assert rel_err(host(G0), base + host(G)) < 1e-6


def test_fused_hidden_sweep_layer_full_size(orc):
    """HIDDEN_SWEEP's 512 -> 2048 layer at full size (T = 16 x 1024, K = 64,
    gamma = 0.95) on seeded costs: sampled tokens of g and rows of G_W
    against the oracle's chain, g against the standalone reduction."""
    w = I.HIDDEN_SWEEP
    K = 64
    layer = w.hidden[2]
    li = I.layer_inputs(w, layer)
    off = I.uniform_offsets(w.n_seq, w.seq_len)
    nz = dust.Noise(w.seed, layer.layer, 0, K, K, w.sigma)
    c = I.normal((K, w.T), 0.02, seed=91)
    X = cu(li["X"], torch.bfloat16)
    G, g = dust.layer_estimate_weight_grad(cu(c), False, cu(off), w.gamma, nz, X, layer.d_out, g_hat=True)
    g1, _ = dust.layer_estimate(cu(c), False, cu(off), w.gamma, nz, layer.d_out)
    assert torch.equal(g, g1)
    toks = np.array([3, 4096, 16383])
    g_ref = orc.layer_estimate(c, False, layer.d_out, off, w.gamma, w.seed, layer.layer, 0, K, w.sigma, toks)
    assert rel_err(host(g)[toks], g_ref) < FP32_TOL
    rows = np.array([0, 777, 2047])
    G_ref = oracle_chains.weight_rows(orc, c, False, layer.d_out, off, w.gamma, w.seed, layer.layer, 0, K, w.sigma,
                                      li["X"], rows)
    assert rel_err(host(G)[rows], G_ref) < BF16_G_TOL


def test_fused_rejects_unsupported_width():
    T, K = 64, 4
    c = torch.zeros(K, T, device="cuda")
    nz = dust.Noise(0, 0, 0, K, K, 0.01)
    for d_in in (1024, 96):
        X = torch.zeros(T, d_in, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(dust.DustError) as e:
            dust.layer_estimate_weight_grad(c, True, None, 0.0, nz, X, 32)
        assert e.value.status == 2


@pytest.mark.parametrize("split", [1, 3, 5])
def test_fused_draw_ranges_add_up(orc, split):
    """Draw sharding (each call a range of the draws, all scaled by K_total):
    the fused calls added with accumulate = 1 give the one-call G_W up to the
    fp32 order of the sums."""
    T, d_out, d_in, K, gamma = 400, 160, 256, 8, 0.9
    off_h = I.offsets_from_lengths(I.ragged_lengths(T, 3, seed=4))
    off = cu(off_h)
    c = I.normal((K, T), 0.02, seed=6)
    X_h = I.bf16_round(I.normal((T, d_in), 1.0, seed=7))
    X = cu(X_h, torch.bfloat16)
    G_all, _ = dust.layer_estimate_weight_grad(cu(c), False, off, gamma, dust.Noise(1, 2, 0, K, K, 0.01), X, d_out)
    G = torch.zeros(d_out, d_in, device="cuda")
    dust.layer_estimate_weight_grad(cu(c[:split]), False, off, gamma, dust.Noise(1, 2, 0, split, K, 0.01), X, d_out,
                                    G_W=G, accumulate=True)
    dust.layer_estimate_weight_grad(cu(c[split:]), False, off, gamma, dust.Noise(1, 2, split, K - split, K, 0.01), X,
                                    d_out, G_W=G, accumulate=True)
    # each call rounds its own partial g to bf16: the oracle chain does the same per range
    rows = np.arange(d_out)
    G_ref = (oracle_chains.weight_rows(orc, c[:split], False, d_out, off_h, gamma, 1, 2, 0, K, 0.01, X_h, rows) +
             oracle_chains.weight_rows(orc, c[split:], False, d_out, off_h, gamma, 1, 2, split, K, 0.01, X_h, rows))
    assert rel_err(host(G), G_ref) < BF16_G_TOL
    # and against the one-call estimate at bf16 resolution (the roundings differ)
    assert rel_err(host(G), host(G_all).astype(np.float64)) < 2e-2
