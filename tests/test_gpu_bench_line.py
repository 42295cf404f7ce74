"""bench.py's one JSON line, run as a user runs it, on small workloads: the
keys the measurement contract names are present and consistent, the device
status word reads ok, and every ALU-bound kernel carries its fraction of the
generator's measured ceiling."""
import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


def run_bench(*args):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "2", "--warmup", "3", "--no-cpu-baseline",
           *args]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("workload,draws", [("head_small_fp32", 16), ("hidden_sweep_bf16", 64)])
def test_bench_line_contract(workload, draws):
    line = run_bench("--workload", workload, "--draws", str(draws))
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks",
                "status", "noise_ceiling", "kernels", "layers"):
        assert key in line, key
    assert line["status"] == "ok"
    assert line["n_gpus"] == 1 and line["steps"] == 2 and line["warmup"] == 3
    assert line["config"]["workload"] == workload and line["config"]["draws"] == draws
    assert line["value"] > 0 and line["gpu_launches"] > 0
    e2e = line["e2e"]
    assert e2e["value"] > 0 and e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    roof = line["roofline"]
    assert roof["bound"] in ("alu", "hbm", "tensor") and 0 < roof["frac"] == pytest.approx(
        roof["achieved"] / roof["peak"])
    # the metric per layer step: each layer's draws x tokens over its own stages, which add up to the step
    names = {L["layer"] for L in line["layers"]}
    assert names == {k["name"].split(":")[0] for k in line["kernels"]}
    stage_ms = sum(L["ms"] for L in line["layers"])
    assert stage_ms <= line["ms_per_step"] * 1.001 + 1e-3
    if workload == "hidden_sweep_bf16":          # not launch-bound: the stages fill the step
        assert stage_ms == pytest.approx(line["ms_per_step"], rel=0.02)
    for L in line["layers"]:
        assert L["draws_x_tokens_per_s"] == pytest.approx(draws * line["config"]["tokens_per_rank"] / (L["ms"] / 1e3))
    ceil = line["noise_ceiling"]
    assert ceil["kernel"] == "noise_sum_kernel" and ceil["gaussians_per_s"] > 0
    alu = [k for k in line["kernels"] if k.get("bound") == "alu"]
    assert alu
    for k in alu:
        assert k["noise_ceiling_frac"] == pytest.approx(k["gaussians_per_s"] / ceil["gaussians_per_s"])
        assert 0 < k["noise_ceiling_frac"]
    if workload == "hidden_sweep_bf16":
        # the draw reduction is the generator plus one load-free multiply per pair: near the ceiling
        for k in alu:
            assert 0.5 < k["noise_ceiling_frac"] < 1.1, k


def test_end_to_end_leg_computes_the_same_step():
    """The end-to-end leg (double-buffered device inputs, copied from pinned
    host memory while the previous step computes) leaves every weight estimate
    equal, bit for bit, to the device-resident step's."""
    import sys as _sys
    _sys.path.insert(0, ROOT)
    import argparse
    import bench
    from activation_perturbation_es_b200 import inputs as I
    w = I.HIDDEN_SWEEP
    step = bench.Step(w, 64, rank=0, world=1)
    step.run()
    torch.cuda.synchronize()
    ref = [L["G"].clone() for L in step.hidden]
    out = bench.e2e_run(step, argparse.Namespace(steps=3), 1)
    torch.cuda.synchronize()
    assert out["value"] > 0 and out["h2d_bytes_per_step"] > 0
    for L, G in zip(step.hidden, ref):
        assert torch.equal(L["G"], G), L["hl"].name
    # the step is bound to its own input tensors again
    step.run()
    torch.cuda.synchronize()
    for L, G in zip(step.hidden, ref):
        assert torch.equal(L["G"], G), L["hl"].name
