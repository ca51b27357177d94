"""Parity at the full workload sizes, in the launch configuration bench.py times.

The float64 oracle cannot evaluate whole 65k-token batches in seconds, so these
tests check sampled rows the oracle can compute one user-prefix at a time
(rows 0..m-1 of a user depend only on its first m tokens), plus properties
that hold at any size and are checked bit-exactly on the GPU: a user's rows do
not depend on the other users of the batch."""
import numpy as np
import pytest
import torch

from gen import make_case
from gen.device import tensor
from oracle import hstu as O
from hstu_testutil import assert_close, binding, config_of, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    return binding()


def _prefix_check(case, y, user, m, what):
    cfg = case.cfg
    want, _ = O.forward(case.x, case.offsets, case.timestamps, case.layers, cfg,
                        users=[user], prefix=[m])
    s = int(case.offsets[user])
    L = cfg.num_layers
    assert_close(y[s:s + m], want[s:s + m], f"{what} user {user} rows 0..{m - 1}",
                 max_abs=2e-2 * np.sqrt(L))


def _single_user_rows(H, case, t, cfg, weights, user):
    """GPU forward of one user alone (same kernels, a one-user batch)."""
    s, e = int(case.offsets[user]), int(case.offsets[user + 1])
    offs = torch.tensor([0, e - s], dtype=torch.int64, device="cuda")
    jag = H.Jagged(offs, t["timestamps"][s:e].contiguous(), e - s, e - s)
    return H.forward(cfg, weights, jag, t["x"][s:e].contiguous()).cpu()


def test_long_sequence_full_batch(H):
    """8 users x 8192 tokens, 2 layers: the benchmark workload itself."""
    case = make_case("long-bf16")
    t, jag, weights = upload(H, case)
    cfg = config_of(H, case.cfg)
    y = H.forward(cfg, weights, jag, t["x"]).cpu()
    assert H.device_status() == 0
    yn = y.numpy()
    _prefix_check(case, yn, 3, 700, "long-bf16")
    _prefix_check(case, yn, 7, 300, "long-bf16")
    # user 5 alone gives bit-identical rows
    s, e = int(case.offsets[5]), int(case.offsets[6])
    assert torch.equal(_single_user_rows(H, case, t, cfg, weights, 5), y[s:e])


def test_stochastic_length_full_batch(H):
    """64 users, Stochastic Length (alpha 1.6) over 4096, 4 layers."""
    case = make_case("sl-bf16")
    t, jag, weights = upload(H, case)
    cfg = config_of(H, case.cfg)
    y = H.forward(cfg, weights, jag, t["x"]).cpu()
    assert H.device_status() == 0
    yn = y.numpy()
    lens = case.lengths
    shortest = [int(u) for u in np.argsort(lens)[:3]]
    for u in shortest:
        _prefix_check(case, yn, u, int(lens[u]), "sl-bf16")
    longest = int(np.argmax(lens))
    _prefix_check(case, yn, longest, 300, "sl-bf16")
    s, e = int(case.offsets[longest]), int(case.offsets[longest + 1])
    assert torch.equal(_single_user_rows(H, case, t, cfg, weights, longest), y[s:e])


def test_longest_supported_sequence(H):
    """One user at the longest supported length (16384): the position table no
    longer fits twice in shared memory and the single-copy path runs."""
    cfg0 = make_case("long-bf16").cfg.replace(full_len=16384, num_pos_buckets=16384)
    case = make_case(cfg0, seed=41, batch=1, num_layers=1)
    t, jag, weights = upload(H, case)
    cfg = config_of(H, case.cfg)
    y = H.forward(cfg, weights, jag, t["x"]).cpu().numpy()
    assert H.device_status() == 0
    _prefix_check(case, y, 0, 400, "max length")


def test_mfalcon_full_size_sampled(H):
    """16 users x 4096 history, 2048 candidates each, b_m 256, 4 layers."""
    case = make_case("mfalcon")
    t, jag, weights = upload(H, case)
    cfg = config_of(H, case.cfg)
    L, T, hv = case.cfg.num_layers, case.total_tokens, case.cfg.num_heads * 64
    kv = torch.empty((L, T, 2 * hv), dtype=torch.bfloat16, device="cuda")
    H.forward(cfg, weights, jag, t["x"], kv_cache_out=kv)
    sc = H.mfalcon_score(cfg, weights, jag, kv, t["cand_offsets"], t["cand_emb"],
                         t["request_ts"], case.cfg.microbatch, case.cfg.num_cand).cpu().numpy()
    assert H.device_status() == 0
    assert np.all(np.isfinite(sc))
    # oracle on one user's history and a few of its candidates
    u = 2
    hs, he = int(case.offsets[u]), int(case.offsets[u + 1])
    offs = np.array([0, he - hs], dtype=np.int64)
    m = case.cfg.num_cand
    pick = [0, 1, 255, 256, 1023, m - 1]
    rows = np.array([u * m + c for c in pick])
    want = O.mfalcon_scores(case.x[hs:he], offs, case.timestamps[hs:he], case.layers, case.cfg,
                            np.array([0, len(pick)], dtype=np.int64), case.cand_emb[rows],
                            case.request_ts[u:u + 1], 2)
    got = sc[rows]
    scale = max(1.0, float(np.sqrt(np.mean(want ** 2))))
    assert_close(got / scale, want / scale, "mfalcon full-size sampled",
                 max_abs=2e-2 * np.sqrt(L))
