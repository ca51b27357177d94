"""Assigning users of a jagged batch to ranks (one process per GPU).

Users are independent in the HSTU layer (each user's rows attend only to that
user's rows, normalised by that user's length), so a batch shards by users
with no collective in the forward pass.  Work per user grows as
a*n + b*n^2 (the linear layers and the causal attention); users are placed
longest-first on the least loaded rank (greedy LPT).
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np

# per-token linear work (f1 + f2 at d = 512, H = 8) and per causal pair attention work (flop)
LINEAR_FLOP_PER_TOKEN = 2.6e6
ATTN_FLOP_PER_PAIR = 2048.0


def user_cost(n: int, a: float = LINEAR_FLOP_PER_TOKEN, b: float = ATTN_FLOP_PER_PAIR) -> float:
    return a * n + b * n * (n + 1) / 2


def shard_users(lengths: Sequence[int], world_size: int) -> List[List[int]]:
    """Greedy longest-processing-time assignment; returns user indices per rank."""
    if world_size < 1:
        raise ValueError("world_size must be >= 1")
    order = sorted(range(len(lengths)), key=lambda u: (-user_cost(int(lengths[u])), u))
    load = [0.0] * world_size
    parts: List[List[int]] = [[] for _ in range(world_size)]
    for u in order:
        r = min(range(world_size), key=lambda k: (load[k], k))
        parts[r].append(u)
        load[r] += user_cost(int(lengths[u]))
    return [sorted(p) for p in parts]


def gather_rows(offsets: np.ndarray, users: Sequence[int]) -> Tuple[np.ndarray, np.ndarray]:
    """Row indices of `users` (in order) and the offsets of the sub-batch they form."""
    offsets = np.asarray(offsets, dtype=np.int64)
    idx = [np.arange(offsets[u], offsets[u + 1]) for u in users]
    rows = np.concatenate(idx) if idx else np.zeros(0, dtype=np.int64)
    lens = [int(offsets[u + 1] - offsets[u]) for u in users]
    sub = np.zeros(len(users) + 1, dtype=np.int64)
    sub[1:] = np.cumsum(lens)
    return rows, sub
