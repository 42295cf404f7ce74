"""Failure detection without a GPU fault: a bounded wait on a barrier that
nothing completes gives up, records the status word, and the host reads
DUST_ERR_TIMEOUT; the context stays usable afterwards."""
import pytest
import torch

from activation_perturbation_es_b200 import dust

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dust.lib()


def test_bounded_wait_times_out_and_reports():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    dust.poll_status(ws)                                  # clean workspace: OK
    dust.selftest_bounded_wait(ws, polls=2000)
    with pytest.raises(dust.DustError) as e:
        dust.poll_status(ws)
    assert e.value.status == 6
    dust.poll_status(ws)                                  # read-and-clear: OK again
    # the context is still usable: a tensor-core GEMM runs and is right
    g = torch.randn(128, 64, device="cuda").to(torch.bfloat16)
    X = torch.randn(128, 32, device="cuda").to(torch.bfloat16)
    G = dust.weight_grad(g, X)
    ref = g.float().T @ X.float()
    assert float((G - ref).abs().max()) <= 1e-3 * float(ref.abs().max())


def test_selftest_rejects_bad_poll_counts():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(dust.DustError):
        dust.selftest_bounded_wait(ws, polls=0)
    with pytest.raises(dust.DustError):
        dust.selftest_bounded_wait(ws, polls=(1 << 20) + 1)
