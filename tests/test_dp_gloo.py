"""World-size-2 data-parallel composition on CPU (gloo), checked with the oracle.

Each rank computes its part with the CPU oracle -- its sequences, or its range
of draws with the whole-population scale -- and the parts are summed with the
same all-reduce helper the benchmark uses on GPUs.  The sum must equal the
single-process estimate over the whole batch / population."""
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, mode, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import oracle
    from activation_perturbation_es_b200 import dp
    from activation_perturbation_es_b200 import inputs as I
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        n_seq, L, K, d_in, d_out, gamma, sigma = 4, 12, 24, 6, 10, 0.9, 0.01
        T = n_seq * L
        c = I.normal((K, T), 0.01, seed=1)
        X = I.normal((T, d_in), 1.0, seed=2)
        off = I.uniform_offsets(n_seq, L)
        if mode == "draws":
            b, n = dp.draw_range(K, world, rank)
            g = oracle.layer_estimate(c[b:b + n], False, d_out, off, gamma, 0, 3, b, K, sigma, np.arange(T))
            G = oracle.weight_grad(g.astype(np.float32), X)
        else:
            G = _shard_estimate(oracle, dp, I, rank, world)
        Gt = torch.from_numpy(G.astype(np.float32))
        dp.allreduce_sum_([Gt])
        if rank == 0:
            q.put(Gt.numpy())
    finally:
        dist.destroy_process_group()


def _shard_estimate(oracle, dp, I, rank, world):
    """Sequence shard of `rank`: local token ids and offsets, the rank folded
    into the noise seed so that ranks draw independent noise."""
    n_seq, L, K, d_in, d_out, gamma, sigma = 4, 12, 24, 6, 10, 0.9, 0.01
    T = n_seq * L
    c = I.normal((K, T), 0.01, seed=1)
    X = I.normal((T, d_in), 1.0, seed=2)
    off = I.uniform_offsets(n_seq, L)
    q0, q1 = dp.sequence_range(n_seq, world, rank)
    t0, t1 = int(off[q0]), int(off[q1])
    off_r = (off[q0:q1 + 1] - t0).astype(np.int32)
    g_r = oracle.layer_estimate(np.ascontiguousarray(c[:, t0:t1]), False, d_out, off_r, gamma, rank, 3, 0, K,
                                sigma, np.arange(t1 - t0))
    return oracle.weight_grad(g_r.astype(np.float32), X[t0:t1])


def _run(mode, port):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, mode, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return out


def _reference(mode):
    sys.path.insert(0, ROOT)
    import oracle
    from activation_perturbation_es_b200 import dp
    from activation_perturbation_es_b200 import inputs as I
    if mode == "sequences":
        return sum(_shard_estimate(oracle, dp, I, r, 2) for r in range(2))
    n_seq, L, K, d_in, d_out, gamma, sigma = 4, 12, 24, 6, 10, 0.9, 0.01
    T = n_seq * L
    c = I.normal((K, T), 0.01, seed=1)
    X = I.normal((T, d_in), 1.0, seed=2)
    off = I.uniform_offsets(n_seq, L)
    g = oracle.layer_estimate(c, False, d_out, off, gamma, 0, 3, 0, K, sigma, np.arange(T))
    return oracle.weight_grad(g.astype(np.float32), X)


@pytest.mark.parametrize("mode,port", [("draws", 29611), ("sequences", 29612)])
def test_two_rank_composition(mode, port):
    got = _run(mode, port)
    ref = _reference(mode)
    assert np.max(np.abs(got - ref)) / np.max(np.abs(ref)) < 1e-5


def test_ranges_partition():
    from activation_perturbation_es_b200 import dp
    for K in (1, 7, 64, 4096):
        for world in (1, 2, 3, 8):
            got = [dp.draw_range(K, world, r) for r in range(world)]
            assert got[0][0] == 0 and sum(n for _, n in got) == K
            assert all(got[i][0] + got[i][1] == got[i + 1][0] for i in range(world - 1))
    assert [dp.sequence_range(5, 2, r) for r in range(2)] == [(0, 2), (2, 5)]
    with pytest.raises(ValueError):
        dp.draw_range(4, 2, 2)
