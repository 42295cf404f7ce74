"""World-size-2 composition of the three shardings on CPU (gloo), checked with
the oracle.

Each rank computes its part with the CPU oracle and the parts are combined
with the same helpers the benchmark uses on GPUs (dp.allreduce_sum_,
dp.allgather_rows):
  * draws: rank r takes its range of the global draw indices, scaled by the
    whole population; the sum is the K-draw estimate;
  * sequences: rank r takes whole sequences, rebased offsets and the global
    index of its first token as token_begin; the sum equals ONE single-process
    estimate over the whole batch (same noise, token for token);
  * vocab: rank r runs a range of the head's vocabulary-chunk passes; the
    gathered G_W rows equal the single-process head estimate.
"""
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

N_SEQ, L, K, D_IN, D_OUT, GAMMA, SIGMA = 4, 12, 24, 6, 10, 0.9, 0.01
HT, HD, HV, HVC, HK = 24, 8, 640, 128, 16          # head: tokens, d_in, vocabulary (5 chunks), chunk, draws


def _hidden_inputs(I):
    T = N_SEQ * L
    c = I.normal((K, T), 0.01, seed=1)
    X = I.normal((T, D_IN), 1.0, seed=2)
    off = I.uniform_offsets(N_SEQ, L)
    return T, c, X, off


def _head_inputs(I):
    Z = I.normal((HT, HV), 1.0, seed=11)
    y = I.targets(HT, HV, seed=12)
    X = I.normal((HT, HD), 1.0, seed=13)
    return Z, y, X


def _part(mode, rank, world):
    """This rank's contribution, computed with the oracle."""
    sys.path.insert(0, ROOT)
    import oracle
    from activation_perturbation_es_b200 import dp
    from activation_perturbation_es_b200 import inputs as I
    if mode == "vocab":
        Z, y, X = _head_inputs(I)
        cb, cc = dp.chunk_range(HV // HVC, world, rank)
        _, g = oracle.head_step(Z, y, np.arange(HT), HVC, 0, 7, 0, HK, HK, SIGMA, want_c=False)
        g_mine = np.ascontiguousarray(g[:, cb * HVC:(cb + cc) * HVC]).astype(np.float32)
        return oracle.weight_grad(g_mine, X), [dp.chunk_range(HV // HVC, world, r)[1] * HVC for r in range(world)]
    T, c, X, off = _hidden_inputs(I)
    if mode == "draws":
        b, n = dp.draw_range(K, world, rank)
        g = oracle.layer_estimate(c[b:b + n], False, D_OUT, off, GAMMA, 0, 3, b, K, SIGMA, np.arange(T))
        return oracle.weight_grad(g.astype(np.float32), X), None
    q0, q1 = dp.sequence_range(N_SEQ, world, rank)
    t0, t1 = int(off[q0]), int(off[q1])
    off_r = (off[q0:q1 + 1] - t0).astype(np.int32)
    g_r = oracle.layer_estimate(np.ascontiguousarray(c[:, t0:t1]), False, D_OUT, off_r, GAMMA, 0, 3, 0, K, SIGMA,
                                np.arange(t1 - t0), token_begin=t0)
    return oracle.weight_grad(g_r.astype(np.float32), X[t0:t1]), None


def _worker(rank, world, port, mode, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from activation_perturbation_es_b200 import dp
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        G, counts = _part(mode, rank, world)
        Gt = torch.from_numpy(G.astype(np.float32))
        if mode == "vocab":
            Gt = dp.allgather_rows(Gt, counts)
        else:
            dp.allreduce_sum_([Gt])
        if rank == 0:
            q.put(Gt.numpy())
    finally:
        dist.destroy_process_group()


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


def _single_process(mode):
    """One estimate over the whole batch / population / vocabulary."""
    sys.path.insert(0, ROOT)
    import oracle
    from activation_perturbation_es_b200 import inputs as I
    if mode == "vocab":
        Z, y, X = _head_inputs(I)
        _, g = oracle.head_step(Z, y, np.arange(HT), HVC, 0, 7, 0, HK, HK, SIGMA, want_c=False)
        return oracle.weight_grad(g.astype(np.float32), X)
    T, c, X, off = _hidden_inputs(I)
    g = oracle.layer_estimate(c, False, D_OUT, off, GAMMA, 0, 3, 0, K, SIGMA, np.arange(T))
    return oracle.weight_grad(g.astype(np.float32), X)


@pytest.mark.parametrize("mode,port", [("draws", 29611), ("sequences", 29612), ("vocab", 29613)])
def test_two_rank_composition(mode, port):
    got = _run(mode, port)
    ref = _single_process(mode)
    assert got.shape == ref.shape
    assert np.max(np.abs(got - ref)) / np.max(np.abs(ref)) < 1e-5


def test_sequence_shard_noise_is_the_whole_batch_noise(orc):
    """A sequence shard's estimate with token_begin = its first token equals the
    rows of the whole-batch estimate (the oracle computes both from c)."""
    from activation_perturbation_es_b200 import inputs as I
    T, c, X, off = _hidden_inputs(I)
    t0, t1 = int(off[1]), int(off[3])
    g_full = orc.layer_estimate(c, False, D_OUT, off, GAMMA, 0, 3, 0, K, SIGMA, np.arange(T))
    off_r = (off[1:4] - t0).astype(np.int32)
    g_r = orc.layer_estimate(np.ascontiguousarray(c[:, t0:t1]), False, D_OUT, off_r, GAMMA, 0, 3, 0, K, SIGMA,
                             np.arange(t1 - t0), token_begin=t0)
    np.testing.assert_array_equal(g_r, g_full[t0:t1])
    g_wrong = orc.layer_estimate(np.ascontiguousarray(c[:, t0:t1]), False, D_OUT, off_r, GAMMA, 0, 3, 0, K, SIGMA,
                                 np.arange(t1 - t0))
    assert np.max(np.abs(g_wrong - g_full[t0:t1])) > 0.1 * np.max(np.abs(g_full))


def test_ranges_partition():
    from activation_perturbation_es_b200 import dp
    for K_ in (1, 7, 64, 4096):
        for world in (1, 2, 3, 8):
            for fn in (dp.draw_range, dp.chunk_range):
                got = [fn(K_, world, r) for r in range(world)]
                assert got[0][0] == 0 and sum(n for _, n in got) == K_
                assert all(got[i][0] + got[i][1] == got[i + 1][0] for i in range(world - 1))
    assert [dp.sequence_range(5, 2, r) for r in range(2)] == [(0, 2), (2, 5)]
    assert [dp.chunk_range(4, 8, r)[1] for r in range(8)] == [0, 1, 0, 1, 0, 1, 0, 1]
    with pytest.raises(ValueError):
        dp.draw_range(4, 2, 2)
    with pytest.raises(ValueError):
        dp.chunk_range(4, 2, -1)
