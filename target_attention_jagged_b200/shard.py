"""Data-parallel sharding of a jagged STCA batch over ranks (host logic only).

Requests never interact: each request's output depends only on its own
history and targets ("Make It Long, Keep It Fast" digest §2.2), so a batch
shards over GPUs by whole requests with no exchange on the data path.  This
module balances requests by their work and cuts the jagged arrays; the
per-rank forward is the ordinary single-GPU call.
"""
from __future__ import annotations

import heapq
from typing import List, Sequence

import numpy as np


def request_work(lengths, target_counts, d: int, h: int, M: int, r: int) -> np.ndarray:
    """Work estimate per request: M layers of the encoder (6 d rd per history
    token) plus the attention (4 h d per history token and target)."""
    L = np.asarray(lengths, dtype=np.float64)
    T = np.asarray(target_counts, dtype=np.float64)
    return M * (6.0 * d * r * d * L + 4.0 * h * d * T * L)


def partition_requests(work: Sequence[float], world: int) -> List[np.ndarray]:
    """Greedy longest-processing-time: each request, heaviest first, goes to the
    rank with the least work so far.  Returns each rank's request indices in
    increasing order (the order of the original batch)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    w = np.asarray(work, dtype=np.float64)
    heap = [(0.0, k) for k in range(world)]
    owned: List[list] = [[] for _ in range(world)]
    for i in np.argsort(-w, kind="stable"):
        load, k = heapq.heappop(heap)
        owned[k].append(int(i))
        heapq.heappush(heap, (load + float(w[i]), k))
    return [np.asarray(sorted(o), dtype=np.int64) for o in owned]


def shard_offsets(offsets, target_offsets, requests):
    """Rows of X, rows of the targets and the new offset arrays of a shard."""
    off = np.asarray(offsets, dtype=np.int64)
    toff = np.asarray(target_offsets, dtype=np.int64)
    reqs = np.asarray(requests, dtype=np.int64)
    x_rows = np.concatenate([np.arange(off[q], off[q + 1]) for q in reqs]) if len(reqs) else \
        np.zeros(0, dtype=np.int64)
    t_rows = np.concatenate([np.arange(toff[q], toff[q + 1]) for q in reqs]) if len(reqs) else \
        np.zeros(0, dtype=np.int64)
    new_off = np.concatenate([[0], np.cumsum(off[reqs + 1] - off[reqs])]).astype(np.int64)
    new_toff = np.concatenate([[0], np.cumsum(toff[reqs + 1] - toff[reqs])]).astype(np.int64)
    return x_rows, t_rows, new_off, new_toff


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of `value` over the default process group (identity
    without one): a timed region ends when its slowest rank does."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gather_outputs(Z_local, t_rows, T_total: int):
    """The whole batch's output, (T_total, ...) in the batch's target order, on
    every rank, from each rank's rows Z_local of its targets t_rows.

    Not part of the data path: Z normally stays with the rank that owns the
    request.  For a caller that wants it everywhere, this is an all-gather of
    unequal parts -- one all-gather of the row counts, then one of the rows
    padded to the largest count and one of their target indices -- so every
    rank takes the same three collectives in the same order.  Without a
    process group (or with one rank) it only scatters Z_local into place."""
    import torch
    import torch.distributed as dist
    dev = Z_local.device
    inner = tuple(Z_local.shape[1:])
    rows = torch.as_tensor(np.asarray(t_rows, dtype=np.int64).reshape(-1), device=dev)
    # checked before any collective, so a mismatch fails on its own rank
    # instead of scattering rows to the wrong targets
    if rows.shape[0] != Z_local.shape[0]:
        raise ValueError(f"gather_outputs: {rows.shape[0]} target indices for "
                         f"{Z_local.shape[0]} rows of Z_local")
    if rows.numel() and (int(rows.min()) < 0 or int(rows.max()) >= int(T_total)):
        raise ValueError("gather_outputs: a target index lies outside [0, T_total)")
    out = torch.zeros((int(T_total),) + inner, dtype=Z_local.dtype, device=dev)
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        out[rows] = Z_local
        return out
    world = dist.get_world_size()
    n = torch.tensor([Z_local.shape[0]], dtype=torch.int64, device=dev)
    counts = [torch.zeros_like(n) for _ in range(world)]
    dist.all_gather(counts, n)
    counts = [int(c.item()) for c in counts]
    width = max(1, max(counts))
    part = torch.zeros((width,) + inner, dtype=Z_local.dtype, device=dev)
    part[:Z_local.shape[0]] = Z_local
    idx = torch.full((width,), -1, dtype=torch.int64, device=dev)
    idx[:rows.shape[0]] = rows
    parts = [torch.empty_like(part) for _ in range(world)]
    idxs = [torch.empty_like(idx) for _ in range(world)]
    dist.all_gather(parts, part)
    dist.all_gather(idxs, idx)
    for p, i, c in zip(parts, idxs, counts):
        out[i[:c]] = p[:c]
    return out


def broadcast_weights(weights, src: int = 0):
    """Rank `src`'s weight dict (numpy arrays, lists of them, None) on every
    rank: the weights are replicated, sent once before the first stca_init.
    Other ranks may pass None.  Identity without a process group."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return weights
    box = [weights if dist.get_rank() == src else None]
    dist.broadcast_object_list(box, src=src)
    return box[0]
