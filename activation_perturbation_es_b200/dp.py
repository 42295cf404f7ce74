"""Data-parallel plumbing for the estimator (host side, torch.distributed).

The estimator shards three ways without changing what it computes:
  * by sequences (data parallel): each rank owns whole sequences -- the reward
    scan never crosses a sequence -- and passes the global index of its first
    token as the noise's token_begin, so every token draws the noise it would
    draw in one run over the whole batch; the weight estimates of all ranks
    are summed, G_W = sum_t g_t x_t^T over the global batch (cnblogs Dust
    explainer, credit-assignment section, weight equation);
  * by draws: each rank takes a contiguous range of the global draw indices
    and scales by the whole population K_total, so the sum over ranks of the
    partial estimates is the K-draw estimate (error equation, linear in the
    draws);
  * the LM head by vocabulary chunk (the interference-suppression section's
    third measure perturbs one chunk per pass): each rank runs a contiguous
    range of the chunk passes; their g columns and G_W rows are disjoint, so
    the rows are gathered, not summed.
The exchange is one sum all-reduce per step (and one gather of the head's
rows when the head is split by chunk).
"""
from __future__ import annotations

import torch


def draw_range(K: int, world: int, rank: int) -> tuple[int, int]:
    """(draw_begin, draw_count) of `rank` when K draws are split over `world` ranks."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    b = K * rank // world
    e = K * (rank + 1) // world
    return b, e - b


def sequence_range(n_seq: int, world: int, rank: int) -> tuple[int, int]:
    """[first, last) sequence index of `rank` when n_seq whole sequences are split."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return n_seq * rank // world, n_seq * (rank + 1) // world


def chunk_range(n_chunks: int, world: int, rank: int) -> tuple[int, int]:
    """(chunk_begin, chunk_count) of `rank` when n_chunks vocabulary chunks are
    split over `world` ranks (chunk_count is 0 for ranks beyond n_chunks)."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    b = n_chunks * rank // world
    e = n_chunks * (rank + 1) // world
    return b, e - b


def _host_staged(group, t: torch.Tensor) -> bool:
    """A gloo process group exchanges device tensors through host copies (the
    plumbing of a multi-process run on CPU ranks or on one shared GPU)."""
    import torch.distributed as dist
    return t.is_cuda and dist.get_backend(group) == "gloo"


def allgather_rows(local: torch.Tensor, counts, group=None) -> torch.Tensor:
    """Concatenate every rank's row block (rank order): local is [counts[rank]][...];
    blocks are padded to the largest count for the collective and trimmed after."""
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return local
    world = dist.get_world_size(group)
    if len(counts) != world:
        raise ValueError("one row count per rank")
    most = max(counts)
    rest = tuple(local.shape[1:])
    pad = torch.zeros((most,) + rest, dtype=local.dtype, device=local.device)
    pad[:local.shape[0]].copy_(local)
    if _host_staged(group, pad):
        host = pad.cpu()
        parts = [torch.empty_like(host) for _ in range(world)]
        dist.all_gather(parts, host, group=group)
        parts = [p.to(local.device) for p in parts]
    else:
        parts = [torch.empty_like(pad) for _ in range(world)]
        dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:n] for p, n in zip(parts, counts)])


def allreduce_sum_(tensors, group=None) -> None:
    """Sum each tensor over the ranks, in place, with one collective per dtype:
    the tensors are packed into one flat buffer (fewer launches than one
    all-reduce per layer)."""
    import torch.distributed as dist
    if not tensors or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return
    by_dtype = {}
    for t in tensors:
        by_dtype.setdefault(t.dtype, []).append(t)
    for ts in by_dtype.values():
        flat = torch.cat([t.reshape(-1) for t in ts])
        if _host_staged(group, flat):
            host = flat.cpu()
            dist.all_reduce(host, op=dist.ReduceOp.SUM, group=group)
            flat.copy_(host)
        else:
            dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
        off = 0
        for t in ts:
            n = t.numel()
            t.copy_(flat[off:off + n].view_as(t))
            off += n
