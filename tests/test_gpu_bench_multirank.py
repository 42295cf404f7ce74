"""bench.py's multi-rank flow end to end on the real kernels: two ranks
launched by torch.distributed.run, as the multi-GPU benchmark is, sharing the
one GPU over a gloo process group (DUST_BENCH_DIST_BACKEND=gloo; no kernel of
this library waits on another rank, so ranks may share a device; the
collectives go through host copies).  Each sharding runs its exchange (the sum
all-reduce, and the row gather of the head's vocabulary chunks), the
max-over-ranks timing and the end-to-end leg; rank 0 alone prints the line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("shard,workload", [("sequences", "hidden_sweep_bf16"), ("draws", "hidden_sweep_bf16"),
                                            ("vocab", "head_pages_bf16")])
def test_two_ranks_share_one_gpu_over_gloo(shard, workload):
    env = dict(os.environ, DUST_BENCH_DIST_BACKEND="gloo")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           "bench.py", "--gpus", "2", "--workload", workload, "--draws", "64", "--steps", "2", "--warmup", "3",
           "--no-cpu-baseline", "--shard", shard]
    out = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, (out.stdout[-2000:], out.stderr[-3000:])
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]          # rank 0 only
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["status"] == "ok"
    assert line["config"]["shard"] == shard and line["config"]["dist_backend"] == "gloo"
    assert line["scaling"] == ("weak" if shard == "sequences" else "strong")
    assert line["config"]["parallelism"] == {"sequences": "dp2", "draws": "draws2",
                                             "vocab": "draws2+head_vocab2"}[shard]
    assert line["value"] > 0 and line["e2e"]["value"] > 0 and line["gpu_launches"] > 0
    # the throughput counts every rank's units: the whole batch's once (draws, vocab) or each rank's own batch
    w_T = line["config"]["tokens_per_rank"]
    n_layers = len(line["config"]["hidden"]) + (1 if line["config"]["head"] else 0)
    units = 64 * w_T * n_layers * (2 if shard == "sequences" else 1)
    assert line["value"] == pytest.approx(units / (line["ms_per_step"] / 1e3), rel=1e-9)
