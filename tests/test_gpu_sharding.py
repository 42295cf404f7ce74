"""The library's two sharding arguments on one GPU: token_begin (a call on
whole sequences of a batch draws, token for token, the noise of one call over
the whole batch) and the head's chunk range (the vocabulary-chunk passes split
over calls give the full step's g columns and costs bit for bit).  These are
the per-rank calls of the multi-GPU shardings; the host composition is tested
with gloo ranks on CPU."""
import numpy as np
import pytest
import torch

from activation_perturbation_es_b200 import dust
from activation_perturbation_es_b200 import inputs as I

pytestmark = pytest.mark.gpu

FP32_TOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dust.lib()


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def rel_err(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / np.max(np.abs(b)))


def bits(t):
    return t.contiguous().view(torch.int32).cpu().numpy()


def test_sequence_shard_draws_the_whole_batch_noise(orc):
    """Sequences [2, 5) of a ragged batch with token_begin = their first token:
    g equals the whole-batch call's rows bit for bit (rewards given), and the
    oracle's whole-batch rows when the scan runs (costs given)."""
    lengths = [37, 0, 64, 33, 128, 9]
    off = I.offsets_from_lengths(lengths)
    T, K, d_out, gamma = int(off[-1]), 40, 70, 0.9
    c = I.normal((K, T), 0.02, seed=21)
    r = I.normal((K, T), 0.02, seed=22)
    nz = dust.Noise(3, 9, 5, K, 2 * K, 0.01)
    t0, t1 = int(off[2]), int(off[5])
    off_r = (off[2:6] - t0).astype(np.int32)
    nz_r = dust.Noise(3, 9, 5, K, 2 * K, 0.01, token_begin=t0)
    g_full, _ = dust.layer_estimate(cu(r), True, cu(off), gamma, nz, d_out)
    g_r, _ = dust.layer_estimate(cu(r[:, t0:t1]), True, cu(off_r), gamma, nz_r, d_out)
    np.testing.assert_array_equal(bits(g_r), bits(g_full)[t0:t1])
    g_c, _ = dust.layer_estimate(cu(c[:, t0:t1]), False, cu(off_r), gamma, nz_r, d_out)
    toks = np.array([t0, t0 + 1, t0 + 63, t0 + 64, t1 - 1])
    ref = orc.layer_estimate(c, False, d_out, off, gamma, 3, 9, 5, 2 * K, 0.01, toks)
    assert rel_err(g_c.cpu().numpy()[toks - t0], ref) < FP32_TOL
    # without token_begin the shard would draw other noise
    g_wrong, _ = dust.layer_estimate(cu(r[:, t0:t1]), True, cu(off_r), gamma, nz, d_out)
    assert not np.array_equal(bits(g_wrong), bits(g_full)[t0:t1])


def test_token_begin_in_harness_kernels():
    """Synthetic costs and the noise fill of a token range with token_begin
    equal the whole batch's (bit for bit)."""
    T, d, K, t0, t1 = 300, 24, 33, 120, 250
    u = I.normal((T, d), 1.0, seed=23)
    nz = dust.Noise(1, 4, 0, K, K, 0.01)
    nz_r = dust.Noise(1, 4, 0, K, K, 0.01, token_begin=t0)
    c_full = dust.synth_costs(cu(u), nz, 0.01)
    c_r = dust.synth_costs(cu(u[t0:t1]), nz_r, 0.01)
    np.testing.assert_array_equal(bits(c_r), bits(c_full)[:, t0:t1])
    a_full = dust.noise_fill(nz, 0, T, 0, d)
    a_r = dust.noise_fill(nz_r, 0, t1 - t0, 0, d)
    np.testing.assert_array_equal(bits(a_r), bits(a_full)[:, t0:t1])


@pytest.mark.parametrize("Vc,ranges", [(256, [(0, 2), (2, 2)]), (128, [(0, 3), (3, 1), (4, 4)])])
def test_head_chunk_ranges_compose(orc, Vc, ranges):
    """The head's chunk passes split over calls: g columns and costs equal the
    full step's bit for bit, G_W rows within fp32 GEMM rounding; the pieces
    also match the oracle."""
    T, d, V, K = 256, 64, 1024, 12
    X = I.bf16_round(I.normal((T, d), 1.0, seed=31))
    W = I.bf16_round(I.normal((V, d), 1.0 / np.sqrt(d), seed=32))
    y = I.targets(T, V, seed=33)
    Xg, Wg, yg = cu(X).to(torch.bfloat16), cu(W).to(torch.bfloat16), cu(y)
    nz = dust.Noise(0, 2, 0, K, K, 0.01)
    Z = dust.logits(Xg, Wg)
    full = dust.head_step(yg, Vc, nz, Z=Z, X=Xg, want_c=True, want_bf16=True, want_G_W=True)
    g_cols, c_rows, G_rows = [], [], []
    for cb, cc in ranges:
        part = dust.head_step(yg, Vc, nz, Z=Z, X=Xg, want_c=True, want_bf16=True, want_G_W=True,
                              chunk_begin=cb, chunk_count=cc)
        assert part["g_hat"].shape == (T, cc * Vc) and part["G_W"].shape == (cc * Vc, d)
        g_cols.append(bits(part["g_hat"]))
        c_rows.append(bits(part["c"]))
        G_rows.append(part["G_W"].cpu().numpy())
    np.testing.assert_array_equal(np.concatenate(g_cols, axis=1), bits(full["g_hat"]))
    np.testing.assert_array_equal(np.concatenate(c_rows, axis=0), bits(full["c"]))
    G_full = full["G_W"].cpu().numpy()
    assert rel_err(np.concatenate(G_rows, axis=0), G_full) < 1e-5
    toks = np.array([0, 1, 100, 255])
    _, g_ref = orc.head_step(Z.cpu().numpy()[toks], y[toks], toks, Vc, 0, 2, 0, K, K, 0.01, want_c=False)
    assert rel_err(full["g_hat"].cpu().numpy()[toks], g_ref) < FP32_TOL


def test_head_token_shard():
    """Tokens [t0, t1) of the head with token_begin = t0: the full step's rows."""
    T, V, Vc, K, t0, t1 = 192, 512, 128, 8, 64, 160
    Z = cu(I.normal((T, V), 1.0, seed=41))
    y = cu(I.targets(T, V, seed=42))
    full = dust.head_step(y, Vc, dust.Noise(0, 6, 0, K, K, 0.01), Z=Z, want_c=True)
    part = dust.head_step(y[t0:t1].contiguous(), Vc, dust.Noise(0, 6, 0, K, K, 0.01, token_begin=t0),
                          Z=Z[t0:t1].contiguous(), want_c=True)
    np.testing.assert_array_equal(bits(part["g_hat"]), bits(full["g_hat"])[t0:t1])
    np.testing.assert_array_equal(bits(part["c"]), bits(full["c"])[:, :, t0:t1])
