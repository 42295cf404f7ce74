"""dust_layer_estimate_noalloc against dust_layer_estimate (GPU).

The allocation-free entry point serves callers that cannot call cudaMalloc
(a plugin whose host framework owns all device memory and hands it only its
input and output pointers).  It must give what the workspace entry point
gives, call after call, although every call reuses the same static scratch.
This file is collected last so that a failure here cannot hide the others.
"""
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


def rel_err(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.max(np.abs(a - b)) / np.max(np.abs(b)))


def test_noalloc_matches_workspace_entry_point_twice(orc):
    """Two calls in a row with different shapes, costs and discounts: the same
    bits as dust_layer_estimate (the same kernels on the same rewards; the
    third case takes the chunked scan in both), and the oracle's values."""
    cases = [
        (I.offsets_from_lengths([700, 0, 301, 23]), 48, 0.95, 1000, 3),
        (I.uniform_offsets(4, 256), 130, 0.5, 32, 7),
        (I.uniform_offsets(1, 5000), 20, 0.9, 16, 9),        # few long sequences: chunked scan
    ]
    for off, d_out, gamma, K, seed in cases:
        T = int(off[-1])
        c_np = I.normal((K, T), 0.01, seed=seed)
        c = torch.from_numpy(c_np).cuda()
        goff = torch.from_numpy(off).cuda()
        nz = dust.Noise(seed, 5, 0, K, K, 0.01)
        ref, ref16 = dust.layer_estimate(c, False, goff, gamma, nz, d_out, g_hat_bf16=True)
        g16 = torch.empty(T, d_out, dtype=torch.bfloat16, device="cuda")
        got, got16 = dust.layer_estimate_noalloc(c, goff, gamma, nz, d_out, g_hat_bf16=g16)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
        assert torch.equal(got16, ref16)
        toks = np.array([0, T // 2, T - 1])
        g_orc = orc.layer_estimate(c_np, False, d_out, off, gamma, seed, 5, 0, K, 0.01, toks)
        assert rel_err(got[toks], torch.from_numpy(g_orc)) < FP32_TOL


def test_noalloc_rejects_sizes_beyond_the_scratch():
    T, K = 4096, 1025                     # 4198400 > 4194304 floats
    c = torch.zeros(K, T, device="cuda")
    off = torch.tensor([0, T], dtype=torch.int32, device="cuda")
    with pytest.raises(dust.DustError) as e:
        dust.layer_estimate_noalloc(c, off, 0.9, dust.Noise(0, 0, 0, K, K, 0.01), 8)
    assert e.value.status == 4 and "static scratch" in str(e.value)
    # gamma = 0 needs no scratch, so the same size is accepted
    g, _ = dust.layer_estimate_noalloc(c, off, 0.0, dust.Noise(0, 0, 0, K, K, 0.01), 8)
    torch.cuda.synchronize()
    assert float(g.abs().max()) == 0.0
