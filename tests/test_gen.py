"""Input generator checks: Stochastic Length draws, shapes, dtypes, determinism."""
import math

import numpy as np
import pytest

from gen import CONFIGS, make_case, round_bf16, stochastic_length


def test_stochastic_length_distribution():
    """L = min(n, ceil(n u^(1/alpha))) (review of "Actions Speak Louder than Words",
    section 三 核心公式, Stochastic Length): 1 <= L <= n and, since u^(1/alpha) has
    mean alpha/(alpha+1), E[L] = n alpha/(alpha+1) + (ceil rounding, about 1/2)."""
    rng = np.random.default_rng(123)
    n, alpha, draws = 4096, 1.6, 100_000
    L = np.array([stochastic_length(rng, n, alpha) for _ in range(draws)])
    assert L.min() >= 1 and L.max() <= n
    mean_exact = n * alpha / (alpha + 1) + 0.5
    # Var[n u^(1/a)] = n^2 (a/(a+2) - (a/(a+1))^2)
    sd = n * math.sqrt(alpha / (alpha + 2) - (alpha / (alpha + 1)) ** 2)
    assert abs(L.mean() - mean_exact) < 3 * sd / math.sqrt(draws) + 0.5


def test_sl_case_positions_sorted_and_timestamps_monotone():
    case = make_case("sl-bf16", seed=2, batch=5, num_layers=1)
    for u in range(5):
        s, e = case.offsets[u], case.offsets[u + 1]
        assert 1 <= e - s <= 4096
        assert np.all(np.diff(case.timestamps[s:e]) >= 0)


def test_round_bf16():
    x = np.array([1.0, 1.00390625, 1.005859375, -3.14159, 0.0], dtype=np.float32)
    r = round_bf16(x)
    # values exactly representable stay; halfway rounds to even; others to nearest
    assert r[0] == 1.0 and r[1] == 1.0 and r[2] == np.float32(1.0078125)
    assert (r.view(np.uint32) & 0xFFFF == 0).all()
    assert abs(r[3] - x[3]) <= 2 ** -7 * 4


@pytest.mark.parametrize("name", ["tiny-fp32", "small-bf16"])
def test_case_shapes_and_determinism(name):
    a = make_case(name)
    b = make_case(name)
    cfg = CONFIGS[name]
    assert a.x.shape == (a.total_tokens, cfg.d_model)
    assert np.array_equal(a.x, b.x) and np.array_equal(a.timestamps, b.timestamps)
    lw = a.layers[0]
    assert lw.w1.shape == (cfg.n1, cfg.d_model)
    assert lw.w2.shape == (cfg.d_model, cfg.num_heads * cfg.dv)
    assert lw.rab_pos.shape == (cfg.num_heads, cfg.num_pos_buckets)
    assert lw.rab_time.shape == (cfg.num_heads, cfg.num_time_buckets)
    lens = a.lengths
    assert lens.min() >= cfg.len_lo and lens.max() <= cfg.len_hi
    if cfg.dtype == "bf16":
        assert (a.x.view(np.uint32) & 0xFFFF == 0).all()


def test_mfalcon_case():
    case = make_case("mfalcon", batch=2, lengths=[10, 3], num_layers=1, num_cand=4)
    assert case.cand_emb.shape == (8, case.cfg.d_model)
    assert list(case.cand_offsets) == [0, 4, 8]
    for u in range(2):
        assert case.request_ts[u] >= case.timestamps[case.offsets[u + 1] - 1]
