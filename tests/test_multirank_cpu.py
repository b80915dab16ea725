"""The multi-rank host logic on the CPU: world-size-2 gloo process groups.

Requests are independent, so sharding a batch over ranks by whole requests
and running each shard alone must reproduce the unsharded result exactly
(here with the fp64 oracle standing in for each rank's GPU forward), and the
timing reduction must return the slowest rank's time.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from gen import make_workload
from target_attention_jagged_b200.shard import (broadcast_weights, gather_outputs, max_over_ranks,
                                                partition_requests, request_work, shard_offsets)

WORLD = 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    from oracle import stca_oracle as O
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = make_workload(lengths=[40, 7, 63, 1, 25, 90, 3], targets=[2, 1, 0, 3, 1, 2, 1],
                           d=16, h=2, M=2, r=1, dtype="f32", seed=31)
        # rank 0's weights, replicated once; the others start from nothing
        W = broadcast_weights(wl.weights if rank == 0 else None)
        assert all(np.array_equal(W[k][i], wl.weights[k][i]) for k in ("Wu", "Wq") for i in range(wl.M))
        work = request_work(wl.lengths, wl.target_counts, wl.d, wl.h, wl.M, wl.r)
        mine = partition_requests(work, world)[rank]
        x_rows, t_rows, off, toff = shard_offsets(wl.offsets, wl.target_offsets, mine)
        Z = O.forward(wl.X[x_rows], off, wl.targets[t_rows], toff, W, wl.h)
        gathered = [None] * world
        dist.all_gather_object(gathered, (mine.tolist(), t_rows.tolist(), Z))
        # the helper a caller uses to see every target's Z on every rank
        Z_all = gather_outputs(torch.from_numpy(Z), t_rows, wl.T).numpy()
        np.save(os.path.join(out_dir, f"gathered{rank}.npy"), Z_all)
        slowest = max_over_ranks(10.0 * (rank + 1))
        if rank == 0:
            full = O.forward_workload(wl)
            got = np.zeros_like(full)
            covered = []
            for reqs, rows, z in gathered:
                covered += reqs
                got[np.asarray(rows, dtype=np.int64)] = z
            np.save(os.path.join(out_dir, "got.npy"), got)
            np.save(os.path.join(out_dir, "want.npy"), full)
            with open(os.path.join(out_dir, "meta.txt"), "w") as f:
                f.write(f"{sorted(covered)} {slowest}\n")
    finally:
        dist.destroy_process_group()


def test_sharded_batch_matches_unsharded(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(WORLD, port, str(tmp_path)), nprocs=WORLD,
                       start_method="spawn", join=True)
    got = np.load(tmp_path / "got.npy")
    want = np.load(tmp_path / "want.npy")
    assert np.array_equal(got, want)          # request independence: bit-identical
    covered, slowest = open(tmp_path / "meta.txt").read().rsplit(" ", 1)
    assert covered == str(list(range(7)))      # every request exactly once
    assert float(slowest) == 20.0              # max over the two ranks
    for rank in range(WORLD):                  # gather_outputs: the whole Z on every rank
        assert np.array_equal(np.load(tmp_path / f"gathered{rank}.npy"), want)


def test_gather_outputs_without_a_group():
    import torch
    Z = torch.arange(12, dtype=torch.float64).reshape(3, 4)
    out = gather_outputs(Z, [4, 0, 2], 5)
    assert out.shape == (5, 4)
    assert torch.equal(out[[4, 0, 2]], Z) and torch.count_nonzero(out[[1, 3]]) == 0


def test_gather_outputs_rejects_mismatched_rows():
    import torch
    Z = torch.zeros((3, 4), dtype=torch.float64)
    with pytest.raises(ValueError):
        gather_outputs(Z, [4, 0], 5)               # two indices for three rows
    with pytest.raises(ValueError):
        gather_outputs(Z, [4, 0, 5], 5)            # index past T_total


def test_partition_is_balanced_and_complete():
    rng = np.random.default_rng(0)
    L = rng.integers(100, 10000, size=256)
    T = 1 + rng.poisson(8, size=256)
    work = request_work(L, T, 256, 8, 4, 2)
    for world in (1, 2, 4, 8):
        parts = partition_requests(work, world)
        allr = np.sort(np.concatenate(parts))
        assert np.array_equal(allr, np.arange(256))
        loads = [work[p].sum() for p in parts]
        # LPT bound: max load <= mean + largest single item
        assert max(loads) <= np.mean(loads) + work.max() + 1e-6


def test_shard_offsets_roundtrip():
    off = np.array([0, 3, 3 + 5, 3 + 5 + 2])
    toff = np.array([0, 1, 1, 4])
    x_rows, t_rows, noff, ntoff = shard_offsets(off, toff, [0, 2])
    assert x_rows.tolist() == [0, 1, 2, 8, 9]
    assert t_rows.tolist() == [0, 1, 2, 3]
    assert noff.tolist() == [0, 3, 5] and ntoff.tolist() == [0, 1, 4]
    with pytest.raises(ValueError):
        partition_requests([1.0], 0)
