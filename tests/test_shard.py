"""Sharding users across ranks: a partition, balanced, and numerically a no-op.

The distributed check runs two `gloo` ranks on the CPU: each rank evaluates
the float64 oracle on its own users, the results are gathered and must equal
the unsharded evaluation bit for bit (users are independent)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gen import make_case
from hstu_sequential_transduction_jagged_b200.shard import gather_rows, shard_users, user_cost


def test_shard_is_a_balanced_partition():
    rng = np.random.default_rng(0)
    lengths = rng.integers(1, 4096, 64)
    for world in (1, 2, 3, 8):
        parts = shard_users(lengths, world)
        flat = sorted(u for p in parts for u in p)
        assert flat == list(range(64))
        loads = [sum(user_cost(int(lengths[u])) for u in p) for p in parts]
        biggest = max(user_cost(int(n)) for n in lengths)
        assert max(loads) - min(loads) <= biggest + 1e-6


def test_gather_rows():
    offs = np.array([0, 3, 3, 7, 9])
    rows, sub = gather_rows(offs, [2, 0])
    assert list(rows) == [3, 4, 5, 6, 0, 1, 2]
    assert list(sub) == [0, 4, 7]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from oracle import hstu as O
    case = make_case("small-bf16", seed=5, lengths=[40, 7, 120, 64, 3], num_layers=1)
    parts = shard_users(case.lengths, world)
    mine = parts[rank]
    rows, sub = gather_rows(case.offsets, mine)
    y, _ = O.forward(case.x[rows], sub, case.timestamps[rows], case.layers, case.cfg)
    gathered = [None] * world
    dist.all_gather_object(gathered, (mine, rows.tolist(), y))
    if rank == 0:
        full = np.full((case.total_tokens, case.cfg.d_model), np.nan)
        for users, r, yy in gathered:
            full[np.array(r, dtype=np.int64)] = yy
        ref, _ = O.forward(case.x, case.offsets, case.timestamps, case.layers, case.cfg)
        np.save(out_path, np.array([np.array_equal(full, ref)]))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_gloo_sharded_forward_matches(tmp_path):
    out = str(tmp_path / "ok.npy")
    mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, join=True,
                       start_method="spawn")
    assert bool(np.load(out)[0])
