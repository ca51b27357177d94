"""Parity at the full workload sizes, in the launch configuration bench.py times.

The float64 oracle cannot evaluate whole 65k-token batches in seconds, so these
tests check sampled rows the oracle can compute one user-prefix at a time
(rows 0..m-1 of a user depend only on its first m tokens), plus properties
that hold at any size and are checked bit-exactly on the GPU: a user's rows do
not depend on the other users of the batch."""
import numpy as np
import pytest
import torch

from gen import make_case, to_dtype
from gen.device import tensor
from oracle import hstu as O
from hstu_testutil import assert_close, binding, check_scores, config_of, errors, record, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    return binding()


def _prefix_check(case, y, user, m, what):
    cfg = case.cfg
    want, _ = O.forward(case.x, case.offsets, case.timestamps, case.layers, cfg,
                        users=[user], prefix=[m])
    s = int(case.offsets[user])
    assert_close(y[s:s + m], want[s:s + m], f"{what} user {user} rows 0..{m - 1}")


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


def _per_layer_prefix_check(H, case, users, prefix, what):
    """Each layer at the stated tolerance (max abs 2e-2, rel-L2 5e-3) on the
    full batch, in the launch configuration of the forward: layer l runs over
    every user with the oracle's layer l-1 output in the checked prefix rows
    and the GPU's own layer l-1 output elsewhere, as the fp32 residual input
    that f1 reads rounded to fp16 (x_in = None, as inside a stack).  Rows before m of a user depend on its first m inputs only
    (the mask is causal and N = n_u is fixed), so the prefix rows of layer l
    are compared with the oracle's layer l on the same inputs."""
    t, jag, weights = upload(H, case)
    cfg = config_of(H, case.cfg)
    rows = np.concatenate([np.arange(int(case.offsets[u]), int(case.offsets[u]) + m)
                           for u, m in zip(users, prefix)])
    rows_t = torch.from_numpy(rows).cuda()
    cur_o = case.x.astype(np.float64)          # oracle input of this layer (prefix rows valid)
    x_lp, x_res = t["x"], None                  # GPU input of this layer
    for l, lw in enumerate(case.layers):
        want = O.layer_fwd(cur_o, case.offsets, case.timestamps, lw, case.cfg,
                           keep_stages=False, users=users, prefix=prefix)["y"]
        if l > 0:
            x_res = y_gpu.clone()
            x_res[rows_t] = tensor(cur_o[rows].astype(np.float32), torch.float32, "cuda")
            x_lp = None
        y_gpu = H.layer_fwd(cfg, weights[l], jag, x_lp, x_res=x_res)
        assert H.device_status() == 0
        got = y_gpu[rows_t].cpu().numpy()
        assert_close(got, want[rows], f"{what} layer {l} rows of users {users}")
        base = cur_o[rows]
        dma, drl = errors(got - base, want[rows] - base)
        record(f"{what} layer {l} delta", dma, drl, None, 2e-2)
        assert drl <= 2e-2, f"{what} layer {l} delta rel_l2={drl:.3e}"
        cur_o = want


def test_long_sequence_per_layer(H):
    """The bench workload, layer by layer at the stated bound, on a 2500-row
    prefix of user 3 and a 700-row prefix of user 7."""
    _per_layer_prefix_check(H, make_case("long-bf16"), [3, 7], [2500, 700], "long-bf16")


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
    longer fits twice in shared memory and the single-copy path runs.  One
    layer, so the stated bound applies directly."""
    cfg0 = make_case("long-bf16").cfg.replace(full_len=16384, num_pos_buckets=16384)
    case = make_case(cfg0, seed=41, batch=1, num_layers=1)
    t, jag, weights = upload(H, case)
    cfg = config_of(H, case.cfg)
    y = H.forward(cfg, weights, jag, t["x"]).cpu().numpy()
    assert H.device_status() == 0
    _prefix_check(case, y, 0, 1200, "max length")


def test_stochastic_length_per_layer(H):
    """sl-bf16 (64 users, 4 layers) layer by layer on the full batch: the
    shortest user whole and 400 rows of the longest."""
    case = make_case("sl-bf16")
    lens = case.lengths
    shortest, longest = int(np.argmin(lens)), int(np.argmax(lens))
    _per_layer_prefix_check(H, case, [shortest, longest], [int(lens[shortest]), 400], "sl-bf16")


def test_mfalcon_full_size_sampled(H):
    """16 users x 4096 history, 2048 candidates each, b_m 256, 4 layers: the
    final rows y_c and the scores of sampled candidates of one user."""
    case = make_case("mfalcon")
    t, jag, weights = upload(H, case)
    cfg = config_of(H, case.cfg)
    L, T, hv = case.cfg.num_layers, case.total_tokens, case.cfg.num_heads * 64
    kv = torch.empty((L, T, 2 * hv), dtype=cfg.cache_dtype, device="cuda")
    H.forward(cfg, weights, jag, t["x"], kv_cache_out=kv)
    M = case.cand_emb.shape[0]
    y = torch.empty((M, case.cfg.d_model), dtype=torch.float32, device="cuda")
    sc = H.mfalcon_score(cfg, weights, jag, kv, t["cand_offsets"], t["cand_emb"],
                         t["request_ts"], case.cfg.microbatch, case.cfg.num_cand,
                         cand_y_out=y).cpu().numpy()
    assert H.device_status() == 0
    assert np.all(np.isfinite(sc))
    # oracle on two users' histories and 48 candidates of each (every microbatch
    # boundary of b_m = 256 among them)
    m = case.cfg.num_cand
    rng = np.random.default_rng(5)
    pick = sorted(set([0, 1, 255, 256, 511, 512, 1023, 1024, m - 1]
                      + [int(c) for c in rng.choice(m, 39, replace=False)]))[:48]
    yn = y.cpu().numpy()
    got_y, want_y, got_s, want_s, emb = [], [], [], [], []
    for u in (2, 11):
        hs, he = int(case.offsets[u]), int(case.offsets[u + 1])
        offs = np.array([0, he - hs], dtype=np.int64)
        rows = np.array([u * m + c for c in pick])
        ws, wy = O.mfalcon_scores(case.x[hs:he], offs, case.timestamps[hs:he], case.layers,
                                  case.cfg, np.array([0, len(pick)], dtype=np.int64),
                                  case.cand_emb[rows], case.request_ts[u:u + 1], 16,
                                  return_rows=True)
        got_y.append(yn[rows]); want_y.append(wy)
        got_s.append(sc[rows]); want_s.append(ws); emb.append(case.cand_emb[rows])
    assert_close(np.concatenate(got_y), np.concatenate(want_y), "mfalcon full-size final rows")
    check_scores(np.concatenate(got_s), np.concatenate(want_s), np.concatenate(emb),
                 "mfalcon full-size scores")
