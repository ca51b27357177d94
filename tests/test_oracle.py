"""Pins for the float64 oracle: checks against hand-worked values, closed forms,
brute force and structural invariants fixed by the method (CPU only).

The method: the review of "Actions Speak Louder than Words" (xllm-io paper
review of arXiv 2402.17152), section 三 核心公式 Eq. 1-3 and the M-FALCON
paragraph.
"""
import os

import numpy as np
import pytest

from gen import make_case, CONFIGS
from oracle import brute, hstu as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _tiny_cfg(**kw):
    base = CONFIGS["small-bf16"].replace(d_model=8, num_heads=2, dqk=4, dv=4,
                                         num_pos_buckets=3, num_time_buckets=6,
                                         dtype="fp32", num_layers=1)
    return base.replace(**kw)


def _brute_args(case, layer):
    return dict(offsets=[int(v) for v in case.offsets], ts=[int(v) for v in case.timestamps],
                w1=layer.w1.astype(float).tolist(), b1=layer.b1.astype(float).tolist(),
                w2=layer.w2.astype(float).tolist(), b2=layer.b2.astype(float).tolist(),
                rab_pos=layer.rab_pos.astype(float).tolist(),
                rab_time=layer.rab_time.astype(float).tolist(),
                gamma=None if layer.ln_gamma is None else layer.ln_gamma.astype(float).tolist(),
                beta=None if layer.ln_beta is None else layer.ln_beta.astype(float).tolist())


# --------------------------------------------------------------------------- buckets

def test_time_bucket_golden():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "time_buckets.txt"))
            if l.strip() and not l.startswith("#")]
    dts = np.array([int(r[0]) for r in rows], dtype=np.int64)
    want = np.array([int(r[1]) for r in rows])
    assert np.array_equal(O.time_bucket(dts, 128), want)


def test_time_bucket_monotone_and_thresholds():
    thr = O.time_bucket_thresholds(128)
    assert thr[0] == 0 and np.all(np.diff(thr) >= 0)
    for k in range(1, 128):
        assert O.time_bucket(thr[k], 128) >= k
        if thr[k] > 0:
            assert O.time_bucket(thr[k] - 1, 128) < k
    dt = np.arange(0, 200000, dtype=np.int64)
    b = O.time_bucket(dt, 128)
    assert np.all(np.diff(b) >= 0)
    # bucket k covers [e^{0.301 k} - 1, e^{0.301 (k+1)} - 1): check against the
    # exponential form of the boundary rather than the logarithm
    for k in (2, 5, 10, 27, 40):
        lo = np.exp(0.301 * k) - 1
        hi = np.exp(0.301 * (k + 1)) - 1
        inside = dt[(dt >= np.ceil(lo)) & (dt < np.floor(hi))]
        assert np.all(b[inside] == k)


def test_pos_bucket():
    assert list(O.pos_bucket([0, 1, 5, 63, 64, 1000], 64)) == [0, 1, 5, 63, 63, 63]


# --------------------------------------------------------------------------- phi

def test_phi_closed_forms():
    x = np.linspace(-30, 30, 2001)
    s = O.phi(x, "silu")
    # SiLU via the tanh identity x/2 (1 + tanh(x/2)) and odd-part identity
    assert np.allclose(s, 0.5 * x * (1 + np.tanh(0.5 * x)), rtol=1e-13, atol=1e-13)
    assert np.allclose(s - O.phi(-x, "silu"), x, atol=1e-12)
    assert O.phi(np.array([0.0]), "silu")[0] == 0.0
    assert np.array_equal(O.phi(x, "relu"), np.where(x > 0, x, 0.0))
    assert np.array_equal(O.phi(x, "identity"), x)


# --------------------------------------------------------------------------- attention

def test_tiny_attention_golden():
    q = np.array([[1.0, 0.0], [0.5, 2.0]])
    k = np.array([[2.0, 1.0], [1.0, -1.0]])
    v = np.array([[1.0, 2.0], [3.0, -1.0]])
    ts = np.array([100, 103], dtype=np.int64)
    rp = np.array([[0.1, 0.2, 0.3, 0.4]])
    rt = np.array([[0.01, 0.02, 0.03, 0.04, 0.05, 0.06, 0.07, 0.08]])
    rows = [l.split() for l in open(os.path.join(GOLDEN, "tiny_attention.txt"))
            if l.strip() and not l.startswith("#")]
    for kind in ("identity", "relu"):
        av = O.user_attention(q, k, v, ts, rp, rt, 2, 1, 2, 2, kind)
        for r in rows:
            if r[0] == kind:
                i = int(r[1])
                assert np.allclose(av[i], [float(r[2]), float(r[3])], atol=1e-12)


def test_single_token_case():
    rng = np.random.default_rng(5)
    q, k, v = rng.standard_normal((1, 8)), rng.standard_normal((1, 8)), rng.standard_normal((1, 8))
    rp, rt = rng.standard_normal((1, 4)), rng.standard_normal((1, 4))
    av = O.user_attention(q, k, v, np.array([7]), rp, rt, 1, 1, 8, 8, "silu")
    s = float(q[0] @ k[0]) + rp[0, 0] + rt[0, 0]
    want = s / (1 + np.exp(-s)) * v[0]
    assert np.allclose(av[0], want, rtol=1e-14)


@pytest.mark.parametrize("n", [1, 2, 17, 64])
def test_closed_form_linear_recurrence(n):
    """rab = 0, phi2 = identity: (QK^T (.) M) V / N equals q_i (sum_{j<=i} k_j v_j^T) / N."""
    rng = np.random.default_rng(n)
    H, dh = 2, 5
    q, k, v = (rng.standard_normal((n, H * dh)) for _ in range(3))
    ts = np.sort(rng.integers(0, 10**6, n))
    zeros_p, zeros_t = np.zeros((H, 8)), np.zeros((H, 8))
    N = n + 3  # any normaliser; the oracle must divide by exactly this
    av = O.user_attention(q, k, v, ts, zeros_p, zeros_t, N, H, dh, dh, "identity")
    for h in range(H):
        sl = slice(h * dh, (h + 1) * dh)
        state = np.zeros((dh, dh))
        for i in range(n):
            state += np.outer(k[i, sl], v[i, sl])
            assert np.allclose(av[i, sl], q[i, sl] @ state / N, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("phi2", ["silu", "softmax"])
def test_jagged_equals_padded_and_masked(phi2):
    """Jagged users equal a padded batch with a key-padding mask.  The padding
    sits BEFORE each user's rows (left padding), where the causal mask alone
    would let every real row see it: only the key-padding mask removes the
    garbage keys, positions count from the user's first real row and N = n_u.
    A jagged implementation that leaked across users, miscounted positions or
    used the padded length as N would differ."""
    case = make_case(_tiny_cfg(phi2=phi2), seed=3, lengths=[5, 1, 9, 3])
    cfg, lw = case.cfg, case.layers[0]
    x = case.x.astype(np.float64)
    ref = O.layer_fwd(x, case.offsets, case.timestamps, lw, cfg)["av"]
    Lp = case.max_len + 4
    rng = np.random.default_rng(0)
    H, dqk, dv = cfg.num_heads, cfg.dqk, cfg.dv
    rp, rt = lw.rab_pos.astype(float), lw.rab_time.astype(float)
    for uu in range(len(case.offsets) - 1):
        s, e = case.offsets[uu], case.offsets[uu + 1]
        n = e - s
        padn = Lp - n
        seq = np.concatenate([rng.standard_normal((padn, cfg.d_model)) * 100.0, x[s:e]])
        ts = np.concatenate([rng.integers(0, 10**9, padn), case.timestamps[s:e]])
        pos = np.arange(Lp) - padn                      # real rows at positions 0..n-1
        real = pos >= 0
        mask = (pos[None, :] <= pos[:, None]) & real[None, :]
        u, v, q, k = O.projection(seq, lw.w1.astype(float), lw.b1.astype(float), H, dqk, dv)
        av = np.zeros((Lp, H * dv))
        for h in range(H):
            sh = (q[:, h * dqk:(h + 1) * dqk] @ k[:, h * dqk:(h + 1) * dqk].T
                  + O.rab_matrix(ts, ts, pos, pos, rp[h], rt[h]))
            a = O.attention_weights(sh, mask, phi2, n)
            av[:, h * dv:(h + 1) * dv] = a @ v[:, h * dv:(h + 1) * dv]
        assert np.allclose(av[padn:], ref[s:e], rtol=1e-12, atol=1e-12)


def test_softmax_rows_sum_to_one():
    """Softmax ablation: the weights of each row sum to 1 over its visible keys,
    so with V = 1 every output entry is exactly 1 (up to rounding), whatever Q, K, rab."""
    rng = np.random.default_rng(21)
    n, H, dh = 13, 2, 4
    q, k = rng.standard_normal((n, H * dh)) * 3, rng.standard_normal((n, H * dh)) * 3
    v = np.ones((n, H * dh))
    ts = np.sort(rng.integers(0, 10**7, n))
    rp, rt = rng.standard_normal((H, 20)), rng.standard_normal((H, 40))
    av = O.user_attention(q, k, v, ts, rp, rt, n, H, dh, dh, "softmax")
    assert np.allclose(av, 1.0, rtol=0, atol=1e-13)


def test_softmax_equals_torch_attention():
    """Softmax ablation against torch's scaled_dot_product_attention (float64,
    scale 1, additive bias = rab plus -inf above the diagonal)."""
    import torch
    rng = np.random.default_rng(22)
    n, H, dh = 11, 3, 4
    q, k, v = (rng.standard_normal((n, H * dh)) for _ in range(3))
    ts = np.sort(rng.integers(0, 10**6, n))
    rp, rt = rng.standard_normal((H, 6)), rng.standard_normal((H, 32))
    av = O.user_attention(q, k, v, ts, rp, rt, n, H, dh, dh, "softmax")
    pos = np.arange(n)
    for h in range(H):
        bias = O.rab_matrix(ts, ts, pos, pos, rp[h], rt[h])
        bias = np.where(pos[None, :] <= pos[:, None], bias, -np.inf)
        sl = slice(h * dh, (h + 1) * dh)
        want = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[None, None, :, sl]), torch.from_numpy(k[None, None, :, sl]),
            torch.from_numpy(v[None, None, :, sl]), attn_mask=torch.from_numpy(bias[None, None]),
            scale=1.0)[0, 0].numpy()
        assert np.allclose(av[:, sl], want, rtol=1e-12, atol=1e-12)


def test_softmax_invariant_to_constant_bias():
    """Adding one constant to every rab entry leaves the softmax weights unchanged
    (and changes the pointwise result, which has no such invariance)."""
    rng = np.random.default_rng(23)
    n, H, dh = 9, 1, 4
    q, k, v = (rng.standard_normal((n, H * dh)) for _ in range(3))
    ts = np.sort(rng.integers(0, 10**6, n))
    rp, rt = rng.standard_normal((H, 5)), rng.standard_normal((H, 30))
    a = O.user_attention(q, k, v, ts, rp, rt, n, H, dh, dh, "softmax")
    b = O.user_attention(q, k, v, ts, rp + 0.7, rt, n, H, dh, dh, "softmax")
    assert np.allclose(a, b, rtol=1e-12, atol=1e-12)
    c = O.user_attention(q, k, v, ts, rp, rt, n, H, dh, dh, "silu")
    d = O.user_attention(q, k, v, ts, rp + 0.7, rt, n, H, dh, dh, "silu")
    assert not np.allclose(c, d)


# --------------------------------------------------------------------------- whole layer

@pytest.mark.parametrize("phi2", ["silu", "relu", "identity", "softmax"])
@pytest.mark.parametrize("affine", [False, True])
def test_brute_force_equals_vectorised(phi2, affine):
    cfg = _tiny_cfg(phi2=phi2)
    case = make_case(cfg, seed=11, lengths=[5, 0, 1, 4], ln_affine=affine)
    lw = case.layers[0]
    # stretch the timestamps so several time buckets and the Tb-1 clamp are hit
    ts = case.timestamps.copy()
    ts[case.offsets[0]:case.offsets[1]] = [0, 1, 3, 30, 10**6]
    y_vec = O.layer_fwd(case.x, case.offsets, ts, lw, cfg)["y"]
    y_bru = brute.layer(case.x.astype(float).tolist(), H=cfg.num_heads, dqk=cfg.dqk,
                        dv=cfg.dv, phi1=cfg.phi1, phi2=phi2, eps=cfg.ln_eps,
                        **{**_brute_args(case, lw), "ts": [int(t) for t in ts]})
    assert np.allclose(y_vec, np.array(y_bru), rtol=1e-12, atol=1e-12)


def test_split_order_u_v_q_k():
    """Eq. 1 splits phi1(f1(X)) into U, V, Q, K in that order."""
    H, dh, d = 2, 3, 4
    n1 = 4 * H * dh
    w1 = np.zeros((n1, d))
    for blk in range(4):
        w1[blk * H * dh:(blk + 1) * H * dh, 0] = blk + 1  # block b scales x[0] by b+1
    x = np.array([[1.0, 0, 0, 0]])
    u, v, q, k = O.projection(x, w1, np.zeros(n1), H, dh, dh)
    assert (u == 1).all() and (v == 2).all() and (q == 3).all() and (k == 4).all()


def test_causality():
    case = make_case("small-bf16", seed=1, batch=3, num_layers=2)
    cfg = case.cfg
    y0, _ = O.forward(case.x, case.offsets, case.timestamps, case.layers, cfg)
    s, e = case.offsets[1], case.offsets[2]
    cut = s + (e - s) // 2
    x2 = case.x.astype(np.float64).copy()
    x2[cut + 1:e] += 5.0
    ts2 = case.timestamps.copy()
    ts2[cut + 1:e] += 12345
    y1, _ = O.forward(x2, case.offsets, ts2, case.layers, cfg)
    assert np.array_equal(y0[s:cut + 1], y1[s:cut + 1])
    assert not np.allclose(y0[cut + 1:e], y1[cut + 1:e])


def test_per_user_independence_and_permutation():
    case = make_case("small-bf16", seed=2, batch=4, num_layers=1)
    cfg = case.cfg
    y0, _ = O.forward(case.x, case.offsets, case.timestamps, case.layers, cfg)
    perm = [2, 0, 3, 1]
    segs = [(case.offsets[u], case.offsets[u + 1]) for u in range(4)]
    xs = np.concatenate([case.x[s:e] for s, e in (segs[p] for p in perm)])
    ts = np.concatenate([case.timestamps[s:e] for s, e in (segs[p] for p in perm)])
    lens = [segs[p][1] - segs[p][0] for p in perm]
    offs = np.concatenate([[0], np.cumsum(lens)])
    y1, _ = O.forward(xs, offs, ts, case.layers, cfg)
    for new, old in enumerate(perm):
        s, e = segs[old]
        assert np.array_equal(y1[offs[new]:offs[new + 1]], y0[s:e])
    # changing another user's inputs leaves user 0 unchanged
    x3 = case.x.astype(np.float64).copy()
    x3[segs[3][0]:segs[3][1]] *= -1
    y3, _ = O.forward(x3, case.offsets, case.timestamps, case.layers, cfg)
    assert np.array_equal(y3[segs[0][0]:segs[0][1]], y0[segs[0][0]:segs[0][1]])


def test_prefix_rows_equal_full_rows():
    case = make_case("small-bf16", seed=4, batch=2, num_layers=2)
    cfg = case.cfg
    full, _ = O.forward(case.x, case.offsets, case.timestamps, case.layers, cfg)
    part, _ = O.forward(case.x, case.offsets, case.timestamps, case.layers, cfg,
                        users=[1], prefix=[37])
    s = case.offsets[1]
    assert np.array_equal(part[s:s + 37], full[s:s + 37])


def test_layer_norm_textbook():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(9)
    o = rng.standard_normal((7, 32)) * 3 + 1
    g, b = rng.standard_normal(32), rng.standard_normal(32)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(o), (32,), torch.from_numpy(g),
                                         torch.from_numpy(b), eps=1e-5).numpy()
    assert np.allclose(O.layer_norm(o, 1e-5, g, b), ref, rtol=1e-12, atol=1e-12)
    y = O.layer_norm(o, 1e-5)
    var = o.var(axis=1)
    assert np.allclose(y.mean(axis=1), 0, atol=1e-12)
    assert np.allclose(y.var(axis=1), var / (var + 1e-5), rtol=1e-12)


# --------------------------------------------------------------------------- M-FALCON

def _mf_case(seed=7, lengths=(6, 1, 0, 11), m=5):
    cfg = _tiny_cfg(num_layers=2, num_cand=m, microbatch=2)
    return make_case(cfg, seed=seed, lengths=list(lengths))


@pytest.mark.parametrize("phi2", ["silu", "softmax"])
def test_mfalcon_equals_scoring_alone(phi2):
    case = _mf_case()
    case.cfg = case.cfg.replace(phi2=phi2)
    cfg = case.cfg
    sc = O.mfalcon_scores(case.x, case.offsets, case.timestamps, case.layers, cfg,
                          case.cand_offsets, case.cand_emb, case.request_ts, 2)
    alone = O.score_alone(case.x, case.offsets, case.timestamps, case.layers, cfg,
                          case.cand_offsets, case.cand_emb, case.request_ts,
                          list(range(len(sc))))
    assert np.allclose(sc, alone, rtol=1e-11, atol=1e-11)


def test_mfalcon_microbatch_invariance_and_permutation():
    case = _mf_case(seed=8)
    cfg = case.cfg
    args = (case.x, case.offsets, case.timestamps, case.layers, cfg)
    ref = O.mfalcon_scores(*args, case.cand_offsets, case.cand_emb, case.request_ts, 1)
    for bm in (2, 3, 5, 100):
        sc = O.mfalcon_scores(*args, case.cand_offsets, case.cand_emb, case.request_ts, bm)
        assert np.allclose(sc, ref, rtol=1e-12, atol=1e-12)
    # permuting the candidates of one user permutes their scores
    m = cfg.num_cand
    perm = np.arange(len(ref))
    perm[m:2 * m] = perm[m:2 * m][::-1]
    sc = O.mfalcon_scores(*args, case.cand_offsets, case.cand_emb[perm], case.request_ts, 2)
    assert np.allclose(sc, ref[perm], rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------- planted mistakes

def test_planted_mistakes_are_caught(monkeypatch):
    """A wrong oracle must fail at least one pin; plants live in the oracle, on the CPU."""
    q = np.array([[1.0, 0.0], [0.5, 2.0]])
    k = np.array([[2.0, 1.0], [1.0, -1.0]])
    v = np.array([[1.0, 2.0], [3.0, -1.0]])
    ts = np.array([100, 103], dtype=np.int64)
    rp = np.array([[0.1, 0.2, 0.3, 0.4]])
    rt = np.array([[0.01, 0.02, 0.03, 0.04, 0.05, 0.06, 0.07, 0.08]])
    good = O.user_attention(q, k, v, ts, rp, rt, 2, 1, 2, 2, "identity")
    assert np.allclose(good[1], [-0.46, 3.945])
    # (1) time bucket off by one
    real_tb = O.time_bucket
    monkeypatch.setattr(O, "time_bucket", lambda dt, Tb: np.minimum(real_tb(dt, Tb) + 1, Tb - 1))
    bad = O.user_attention(q, k, v, ts, rp, rt, 2, 1, 2, 2, "identity")
    assert not np.allclose(bad[1], [-0.46, 3.945])
    monkeypatch.setattr(O, "time_bucket", real_tb)
    # (2) position index transposed (j - i instead of i - j)
    real_rm = O.rab_matrix
    monkeypatch.setattr(O, "rab_matrix", lambda tq, tk, pq, pk, a, b: real_rm(tk, tq, pk, pq, a, b).T)
    bad = O.user_attention(q, k, v, ts, rp, rt, 2, 1, 2, 2, "identity")
    assert not np.allclose(bad[1], [-0.46, 3.945])
    monkeypatch.setattr(O, "rab_matrix", real_rm)
    # (3) split order U/V swapped: brute force disagrees
    cfg = _tiny_cfg()
    case = make_case(cfg, seed=12, lengths=[4, 3])
    lw = case.layers[0]
    real_proj = O.projection

    def swapped(*a, **kw):
        u, v_, q_, k_ = real_proj(*a, **kw)
        return v_, u, q_, k_
    monkeypatch.setattr(O, "projection", swapped)
    y_bad = O.layer_fwd(case.x, case.offsets, case.timestamps, lw, cfg)["y"]
    monkeypatch.setattr(O, "projection", real_proj)
    y_bru = brute.layer(case.x.astype(float).tolist(), H=cfg.num_heads, dqk=cfg.dqk, dv=cfg.dv,
                        phi2=cfg.phi2, **_brute_args(case, lw))
    assert not np.allclose(y_bad, np.array(y_bru), rtol=1e-9)


# --------------------------------------------------------------------------- generalised masks

def _seg_case(phi2="silu", lens=(9, 1, 12, 6), seed=41):
    case = make_case(_tiny_cfg(phi2=phi2, num_pos_buckets=5), seed=seed, lengths=list(lens))
    return case


@pytest.mark.parametrize("phi2", ["silu", "identity", "softmax"])
def test_segments_all_history_is_causal(phi2):
    """n_us = 0 and n_r = n (no profile, no candidates) is the causal layer."""
    case = _seg_case(phi2)
    segs = [[0, int(n)] for n in case.lengths]
    a = O.layer_fwd(case.x, case.offsets, case.timestamps, case.layers[0], case.cfg)["y"]
    b = O.layer_fwd(case.x, case.offsets, case.timestamps, case.layers[0], case.cfg,
                    segments=segs)["y"]
    assert np.array_equal(a, b)


@pytest.mark.parametrize("phi2", ["silu", "softmax"])
def test_segments_brute_force_equals_vectorised(phi2):
    case = _seg_case(phi2)
    segs = [[3, 4], [1, 0], [4, 5], [0, 2]]  # n_c = 2, 0, 3, 4
    lw = case.layers[0]
    ts = case.timestamps.copy()
    s0, e0 = case.offsets[2], case.offsets[3]
    ts[s0:e0] = np.sort(ts[s0:e0])
    ts[e0 - 3:e0] = ts[s0 + 6]  # candidates timed inside R: they see only part of it
    y_vec = O.layer_fwd(case.x, case.offsets, ts, lw, case.cfg, segments=segs)["y"]
    y_bru = brute.layer(case.x.astype(float).tolist(), H=case.cfg.num_heads, dqk=case.cfg.dqk,
                        dv=case.cfg.dv, phi1=case.cfg.phi1, phi2=phi2, eps=case.cfg.ln_eps,
                        segments=segs, **{**_brute_args(case, lw), "ts": [int(t) for t in ts]})
    assert np.allclose(y_vec, np.array(y_bru), rtol=1e-12, atol=1e-12)


def _av(case, ts, segs, x=None):
    x = case.x if x is None else x
    return O.layer_fwd(x, case.offsets, ts, case.layers[0], case.cfg, segments=segs)["av"]


def test_segments_visibility_invariants():
    """U+S rows ignore R and C; R rows ignore later R and C; a candidate ignores
    the other candidates and the R events after its time."""
    case = _seg_case("silu", lens=(14,))
    n_us, n_r = 4, 6  # rows 0-3 U+S, 4-9 R, 10-13 C
    segs = [[n_us, n_r]]
    ts = np.sort(case.timestamps.copy())
    ts[10:] = ts[7]  # candidates at the time of R row 7: they see R rows 4..7
    base = _av(case, ts, segs)
    rng = np.random.default_rng(1)

    def perturbed(rows):
        x = case.x.copy()
        x[rows] += rng.standard_normal((len(rows), x.shape[1]))
        return _av(case, ts, segs, x)
    a = perturbed(list(range(4, 14)))            # every R and C token
    assert np.array_equal(a[:4], base[:4])
    b = perturbed([8, 9, 10, 11, 12, 13])         # R rows 8, 9 and the candidates
    assert np.array_equal(b[:8], base[:8])
    c = perturbed([8, 9, 11, 12, 13])             # later R and the other candidates
    assert np.array_equal(c[10], base[10])
    assert not np.array_equal(perturbed([7])[10], base[10])   # R row 7 is visible to it
    assert not np.array_equal(perturbed([10])[10], base[10])  # and so is itself


def test_segment_mask_rules():
    ts = np.array([0, 0, 5, 10, 20, 30, 15, 30, 1], dtype=np.int64)
    m = O.segment_mask(ts, 2, 4)  # U+S 0-1, R 2-5, C 6-8
    assert m[0].tolist() == [1, 1, 0, 0, 0, 0, 0, 0, 0]
    assert m[3].tolist() == [1, 1, 1, 1, 0, 0, 0, 0, 0]
    assert m[6].tolist() == [1, 1, 1, 1, 0, 0, 1, 0, 0]   # t = 15: R events at 5 and 10
    assert m[7].tolist() == [1, 1, 1, 1, 1, 1, 0, 1, 0]   # t = 30: all of R
    assert m[8].tolist() == [1, 1, 0, 0, 0, 0, 0, 0, 1]   # t = 1: no R event yet
