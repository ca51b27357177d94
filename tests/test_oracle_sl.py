"""Pins for the Stochastic Length oracle (CPU only).

The method: the review of "Actions Speak Louder than Words" (xllm-io paper
review), section 三, Stochastic Length: L = min(n, ceil(n * u^(1/alpha))),
u ~ Uniform(0, 1).  The generator is Philox4x64-10, pinned here against
numpy's implementation of the same published generator."""
import math

import numpy as np
import pytest

from oracle import sl as S


def test_philox_matches_numpy():
    """numpy.random.Philox draws the block of counter c + 1 first."""
    for key in ([0x123456789ABCDEF0, 0x0FEDCBA987654321], [7, 0], [2 ** 64 - 1, 2 ** 63]):
        for ctr in ([0, 0, 0, 0], [5, 7, 9, 11], [2 ** 64 - 2, 3, 0, 1]):
            bg = np.random.Philox(key=np.array(key, dtype=np.uint64),
                                  counter=np.array(ctr, dtype=np.uint64))
            raw = [int(v) for v in bg.random_raw(4)]
            c1 = list(ctr)
            c1[0] = (c1[0] + 1) % 2 ** 64
            carry = c1[0] == 0
            for w in range(1, 4):  # numpy's counter is one 256-bit integer
                if not carry:
                    break
                c1[w] = (c1[w] + 1) % 2 ** 64
                carry = c1[w] == 0
            assert S.philox4x64_10(c1, key) == raw


def test_length_draw_distribution():
    """E[L] for L = min(n, ceil(n u^(1/alpha))): n alpha/(alpha+1) + 1/2 to within a
    small correction; 20000 draws, compared within 4 standard errors."""
    n, alpha = 4096, 1.6
    L = np.array([S.sl_length(n, alpha, 11, 3, u) for u in range(20000)], dtype=np.float64)
    assert L.min() >= 1 and L.max() <= n
    # exact mean of ceil(n V) with V = u^(1/alpha): sum_k P(n V > k) for k = 0..n-1
    k = np.arange(n)
    exact = float(np.sum(1.0 - (k / n) ** alpha))
    se = L.std() / math.sqrt(len(L))
    assert abs(L.mean() - exact) < 4 * se
    assert abs(exact - (n * alpha / (alpha + 1) + 0.5)) < 1.0


def test_length_is_the_printed_formula():
    for u_idx in range(50):
        for n in (1, 2, 17, 4096):
            u = S.length_uniform(5, 0, u_idx)
            assert 0.0 < u <= 1.0
            assert S.sl_length(n, 1.6, 5, 0, u_idx) == min(n, math.ceil(n * u ** (1 / 1.6)))
    assert S.sl_length(0, 1.6, 5, 0, 0) == 0


def test_kept_positions_sorted_unique_and_uniform():
    """Each position of an n-event user is kept with probability L/n: over 4000
    draws of L = 8 of n = 32 the per-position counts match 1000 within 5 sigma."""
    n, L, draws = 32, 8, 4000
    counts = np.zeros(n)
    for u in range(draws):
        kept = S.sl_kept_positions(n, L, 9, 1, u)
        assert len(kept) == L and np.all(np.diff(kept) > 0)
        assert kept.min() >= 0 and kept.max() < n
        counts[kept] += 1
    p = L / n
    sigma = math.sqrt(draws * p * (1 - p))
    assert np.all(np.abs(counts - draws * p) < 5 * sigma)


def test_batch_subsample_layout():
    rng = np.random.default_rng(0)
    lens = [0, 1, 40, 7]
    offsets = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T = int(offsets[-1])
    ts = np.arange(T, dtype=np.int64) * 10
    x = rng.standard_normal((T, 4))
    offs, ts_out, x_out, kept = S.stochastic_length(offsets, ts, x, 1.6, 3, 2)
    assert offs[0] == 0 and np.all(np.diff(offs) <= np.diff(offsets))
    assert np.all(np.diff(offs)[np.array(lens) > 0] >= 1)
    for u in range(len(lens)):
        rows = kept[offs[u]:offs[u + 1]]
        assert np.all((rows >= offsets[u]) & (rows < offsets[u + 1]))
        assert np.all(np.diff(rows) > 0)
    assert np.array_equal(ts_out, ts[kept]) and np.array_equal(x_out, x[kept])
