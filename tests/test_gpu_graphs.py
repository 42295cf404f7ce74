"""The library's calls enqueue only (no allocation, no synchronisation), so a
whole estimator step can be captured in a CUDA graph and replayed; the replay
gives the eager results bit for bit."""
import numpy as np
import pytest
import torch

from activation_perturbation_es_b200 import dust
from activation_perturbation_es_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dust.lib()


def test_step_replays_from_a_cuda_graph():
    T, d_in, d_out, V, Vc, K = 2048, 64, 96, 512, 256, 32
    off = torch.from_numpy(I.uniform_offsets(4, T // 4)).cuda()
    X = torch.from_numpy(I.bf16_round(I.normal((T, d_in), 1.0, seed=1))).cuda().to(torch.bfloat16)
    W = torch.from_numpy(I.bf16_round(I.normal((V, d_in), 0.125, seed=2))).cuda().to(torch.bfloat16)
    y = torch.from_numpy(I.targets(T, V, seed=3)).cuda()
    u = torch.from_numpy(I.normal((T, d_out), 1.0, seed=4)).cuda()
    nz_h, nz_l = dust.Noise(0, 1, 0, K, K, 0.01), dust.Noise(0, 2, 0, K, K, 0.01)
    c = dust.synth_costs(u, nz_l, 0.01)
    r = torch.empty_like(c)
    g = torch.empty(T, d_out, device="cuda")
    g16 = torch.empty(T, d_out, device="cuda", dtype=torch.bfloat16)
    G = torch.empty(d_out, d_in, device="cuda")
    Z = torch.empty(T, V, device="cuda")
    gh = torch.empty(T, V, device="cuda")
    gh16 = torch.empty(T, V, device="cuda", dtype=torch.bfloat16)
    GH = torch.empty(V, d_in, device="cuda")
    GF = torch.empty(d_out, d_in, device="cuda")
    stream = torch.cuda.Stream()

    def step():
        dust.reward_scan(c, off, 0.9, out=r)
        dust.layer_estimate(r, True, off, 0.9, nz_l, d_out, g_hat=g, g_hat_bf16=g16)
        dust.weight_grad(g16, X, G_W=G)
        dust.logits(X, W, Z=Z)
        dust.head_step(y, Vc, nz_h, Z=Z, g_hat=gh, g_hat_bf16=gh16)
        dust.weight_grad(gh16, X, G_W=GH)
        dust.layer_estimate_weight_grad(r, True, off, 0.9, nz_l, X, d_out, G_W=GF)   # fused a5 + a6

    with torch.cuda.stream(stream):
        step()                                   # warm-up: workspaces, kernel attributes
    torch.cuda.synchronize()
    eager = [t.clone() for t in (g, G, gh, GH, GF)]
    for t in (g, G, gh, GH, GF):
        t.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    graph.replay()
    torch.cuda.synchronize()
    for a, b in zip(eager, (g, G, gh, GH, GF)):
        assert torch.equal(a, b)
