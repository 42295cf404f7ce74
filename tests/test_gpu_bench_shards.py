"""The benchmark's per-rank partition of a step, on one GPU: the ranks of a
draw split (hidden layers) and of a vocabulary split (LM head) are built one
after the other as bench.Step(rank, world = 2) without a process group (their
exchange is skipped), and their weight estimates are combined here as the NCCL
collectives would combine them: summed for draws, rows concatenated for
vocabulary chunks.  The result must be the single-rank step's."""
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from activation_perturbation_es_b200 import dust  # noqa: E402
from activation_perturbation_es_b200 import inputs as I  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dust.lib()


def rel_err(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / np.max(np.abs(b)))


def _run(w, K, rank, world, shard):
    import bench
    step = bench.Step(w, K, rank=rank, world=world, shard=shard)
    step.run()
    torch.cuda.synchronize()
    return step


def test_draw_split_of_the_hidden_sweep():
    w = I.HIDDEN_SWEEP
    K = 64
    whole = _run(w, K, 0, 1, "sequences")
    parts = [_run(w, K, r, 2, "draws") for r in range(2)]
    assert [p.draws for p in parts] == [32, 32]
    for i, L in enumerate(whole.hidden):
        # the fp32 error estimate is linear in the draws: the ranks' parts add up to the whole
        g = sum(p.hidden[i]["g"].double() for p in parts).cpu().numpy()
        assert rel_err(g, L["g"].cpu().numpy()) < 1e-5, L["hl"].name
        # each rank rounds its own part of g to bf16 for the tensor-core GEMM, so the summed weight
        # estimates differ from the whole's by bf16 rounding (2^-8 relative), the bf16 GEMM path's bar
        G = sum(p.hidden[i]["G"].double() for p in parts).cpu().numpy()
        assert rel_err(G, L["G"].cpu().numpy()) < 2e-2, L["hl"].name


def test_vocabulary_split_of_the_head():
    w = I.HEAD_PAGES
    K = 64
    whole = _run(w, K, 0, 1, "vocab")
    parts = [_run(w, K, r, 2, "vocab") for r in range(2)]
    assert [p.head["chunks"] for p in parts] == [(0, 2), (2, 2)]
    # the vocabulary chunks' g columns are the whole step's bit for bit
    g = torch.cat([p.head["g"] for p in parts], dim=1)
    assert torch.equal(g, whole.head["g"])
    G = torch.cat([p.head["G"] for p in parts]).cpu().numpy()
    assert rel_err(G, whole.head["G"].cpu().numpy()) < 1e-5
    # and a third rank of three gets a share too (4 chunks over 3 ranks: 1, 1, 2)
    assert [_run(w, 8, r, 3, "vocab").head["chunks"] for r in range(3)] == [(0, 1), (1, 1), (2, 2)]
