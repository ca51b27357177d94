"""Stochastic Length (SL) subsampling of jagged user sequences, float64 / exact integer oracle.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call this
module; only the tests, the entry-point smoke check and the benchmark's CPU
baseline leg do.  It shares no code with the CUDA library.

Source: the review of "Actions Speak Louder than Words" (xllm-io paper review
of arXiv 2402.17152), section 三 技术架构 / Stochastic Length: a user's
sequence of n events is shortened to L = min(n, ceil(n * u^(1/alpha))) with
u ~ Uniform(0, 1) and alpha controlling the sparsity.

Readings taken where the pages leave a step open:
  * which L events are kept: a uniformly random subset of size L, kept in
    time order (the same reading as the input generator's sl-bf16 workload);
  * randomness: one counter-based generator, Philox4x64-10 (Salmon, Moraes,
    Dror and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011),
    keyed by (seed, 0); the CUDA sampler implements the same published
    definition, so both sides draw the same numbers:
      - user u's length draw: counter (0, u, step, 0), first output word x,
        u = ((x >> 11) + 1) * 2^-53, in (0, 1];
      - the rank key of position p of user u: counter (p, u, step, 1), first
        output word;
    the kept subset is the L positions with the smallest rank keys (ties,
    which need equal 64-bit draws, go to the lower position), in time order;
  * the length decision n * u^(1/alpha) is taken in float64 (the CUDA side
    too); two correctly working pow implementations can differ in the last
    bit, which moves L only when n * u^(1/alpha) lies within about 1e-16
    relative of an integer.
"""
from __future__ import annotations

import math
from typing import Tuple

import numpy as np

MASK64 = (1 << 64) - 1
# Philox4x64 round multipliers and key increments (the published constants)
PHILOX_M0, PHILOX_M1 = 0xD2E7470EE14C6C93, 0xCA5A826395121157
PHILOX_W0, PHILOX_W1 = 0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B


def philox4x64_10(counter, key):
    """Philox4x64 with 10 rounds: 4 x 64-bit counter words, 2 x 64-bit key words
    -> 4 x 64-bit output words (Python integers)."""
    c = [int(v) & MASK64 for v in counter]
    k = [int(v) & MASK64 for v in key]
    for _ in range(10):
        p0 = PHILOX_M0 * c[0]
        p1 = PHILOX_M1 * c[2]
        hi0, lo0 = p0 >> 64, p0 & MASK64
        hi1, lo1 = p1 >> 64, p1 & MASK64
        c = [(hi1 ^ c[1] ^ k[0]) & MASK64, lo1, (hi0 ^ c[3] ^ k[1]) & MASK64, lo0]
        k = [(k[0] + PHILOX_W0) & MASK64, (k[1] + PHILOX_W1) & MASK64]
    return c


def length_uniform(seed: int, step: int, user: int) -> float:
    """The uniform u in (0, 1] of the user's length draw."""
    x = philox4x64_10((0, user, step, 0), (seed, 0))[0]
    return float(((x >> 11) + 1) * 2.0 ** -53)


def sl_length(n: int, alpha: float, seed: int, step: int, user: int) -> int:
    """L = min(n, ceil(n * u^(1/alpha))), 0 for an empty user."""
    if n <= 0:
        return 0
    u = length_uniform(seed, step, user)
    return int(min(n, math.ceil(n * math.pow(u, 1.0 / alpha))))


def rank_key(seed: int, step: int, user: int, pos: int) -> int:
    return philox4x64_10((pos, user, step, 1), (seed, 0))[0]


def sl_kept_positions(n: int, length: int, seed: int, step: int, user: int) -> np.ndarray:
    """The `length` positions with the smallest rank keys, in time order."""
    keys = [(rank_key(seed, step, user, p), p) for p in range(n)]
    keys.sort()
    return np.sort(np.array([p for _, p in keys[:length]], dtype=np.int64))


def stochastic_length(offsets, timestamps, x, alpha: float, seed: int,
                      step: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray, np.ndarray]:
    """Subsample every user of a jagged batch.

    Returns (offsets_out [B+1], timestamps_out [T_out], x_out [T_out, d],
    kept_index [T_out]) where kept_index holds each kept row's row in the input.
    """
    B = len(offsets) - 1
    lens = [sl_length(int(offsets[u + 1] - offsets[u]), alpha, seed, step, u) for u in range(B)]
    offs = np.zeros(B + 1, dtype=np.int64)
    offs[1:] = np.cumsum(lens)
    kept = []
    for u in range(B):
        n = int(offsets[u + 1] - offsets[u])
        kept.append(int(offsets[u]) + sl_kept_positions(n, lens[u], seed, step, u))
    kept_index = np.concatenate(kept) if kept else np.zeros(0, dtype=np.int64)
    kept_index = kept_index.astype(np.int64)
    return offs, np.asarray(timestamps)[kept_index], np.asarray(x)[kept_index], kept_index
