"""Float64 CPU oracle for the HSTU layer forward and M-FALCON candidate scoring.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call this
module; only the tests, the entry-point smoke check and the benchmark's CPU
baseline leg do.  It shares no code with the CUDA library.

Source of every step: the review of "Actions Speak Louder than Words"
(xllm-io paper-review of arXiv 2402.17152), section 三 技术架构 / 核心公式:
  Eq. 1  U, V, Q, K = Split(phi1(f1(X))),  f_i(X) = W_i X + b_i, phi1 = ReLU
  Eq. 2  A(X)V(X) = phi2(Q K^T + rab^{p,t}) V(X)   (pointwise, replaces softmax)
  Eq. 3  Y(X) = f2(Norm(A(X)V(X)) (.) U(X))
  tree   "Residual Connections between layers"
and its M-FALCON paragraph (section 三, M-FALCON 推理算法): candidates are
scored in microbatches whose attention ops are identical, reusing the cached
history keys/values.

Readings taken where the pages leave a step open (each is a parameter or a
documented constant here, never hidden):
  * phi2 is selectable: "silu" (default), "relu" or "identity".  The pages only
    say "pointwise aggregated normalisation".  Parity for the choice itself is
    unpinned.
  * the normaliser is 1/N with N = n_u, the user's own sequence length, applied
    to every row of that user (also to M-FALCON candidates).
  * no 1/sqrt(d) on Q K^T; rab is added before phi2; the causal mask zeroes
    a_ij for j > i after phi2.
  * rab^{p,t}_ij = rab_pos[h, min(i-j, P-1)] + rab_time[h, b_t(t_i - t_j)] with
    b_t(dt) = clamp(floor(ln(dt + 1) / 0.301), 0, Tb-1), dt in integer seconds
    (dt < 0 maps to bucket 0).
  * Norm is LayerNorm over the H*dv concatenated heads of one token, biased
    variance, eps = 1e-5, optional affine (gamma, beta).
  * Residual: Y = X + f2(...).  No pre-norm, no final norm.
  * phi2 = "softmax" is the ablation "HSTU (-rab, Softmax)" of the review's
    section 六 (消融实验, HSTU 组件消融) and section 五 (industrial streaming
    table): the pointwise phi2 and its 1/N are replaced by a row-wise softmax
    over the visible keys of the same pre-activation Q K^T + rab (no extra
    scale; "-rab" is the same with zero bias tables).
  * Generalised (MTGR-style) masks, from the RecSysChannel digest of "MTGR:
    Industrial-Scale Generative Recommendation Framework in Meituan" (Dynamic
    Masking): a user's tokens are ordered U+S (profile and long history),
    then R (short history), then C (candidates), with n_us and n_r given per
    user.  U+S keys are visible to every row, U+S rows see only U+S
    (both directions); R rows are causal; a candidate sees U+S, the R events
    at or before its own timestamp ("the preceding part of R") and itself,
    not the other candidates.  Positions are the token indices; the position
    bucket of a key after the row (inside U+S) is min(|i - j|, P - 1); the
    time bucket of a negative difference is 0.  N = n_u, all the user's tokens.
  * M-FALCON: a candidate sits at position n_u with timestamp t_req, attends to
    the user's cached history rows (keys/values of every layer) and to itself
    (position bucket 0, time bucket 0); its score is <y_c^(L), e_c>.  Its
    normaliser is max(n_u, 1), so a user with an empty history still scores.

Layouts (row-major): X [T, d]; W1 [2H(dqk+dv), d] rows ordered U, V, Q, K with
head h occupying rows h*dh:(h+1)*dh of each block; W2 [d, H*dv]; jagged users
given by offsets [B+1].
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence

import numpy as np

TIME_BUCKET_DIVISOR = 0.301


def phi(x: np.ndarray, kind: str) -> np.ndarray:
    """Pointwise nonlinearity: phi1 = ReLU (核心公式, 其中), phi2 per reading."""
    if kind == "relu":
        return np.maximum(x, 0.0)
    if kind == "silu":
        return x / (1.0 + np.exp(-x))
    if kind == "identity":
        return x
    raise ValueError(kind)


def time_bucket(dt, num_time_buckets: int) -> np.ndarray:
    """Log-time bucket of a timestamp difference (rab^{p,t}, time part).

    b_t = clamp(floor(ln(dt + 1) / 0.301), 0, Tb - 1); negative dt -> 0.
    """
    dt = np.asarray(dt, dtype=np.int64)
    pos = np.maximum(dt, 0).astype(np.float64)
    b = np.floor(np.log(pos + 1.0) / TIME_BUCKET_DIVISOR).astype(np.int64)
    b = np.where(dt < 0, 0, b)
    return np.clip(b, 0, num_time_buckets - 1)


def pos_bucket(delta, num_pos_buckets: int) -> np.ndarray:
    """Position bucket of i - j (rab^{p,t}, position part): min(i - j, P - 1)."""
    return np.minimum(np.asarray(delta, dtype=np.int64), num_pos_buckets - 1)


def projection(x: np.ndarray, w1: np.ndarray, b1: np.ndarray, H: int, dqk: int, dv: int,
               phi1: str = "relu"):
    """Eq. 1: U, V, Q, K = Split(phi1(W1 x + b1)), split in the order U, V, Q, K."""
    z = phi(x @ w1.T + b1, phi1)
    hv, hq = H * dv, H * dqk
    u = z[:, 0:hv]
    v = z[:, hv:2 * hv]
    q = z[:, 2 * hv:2 * hv + hq]
    k = z[:, 2 * hv + hq:2 * hv + 2 * hq]
    return u, v, q, k


def rab_matrix(ts_q: np.ndarray, ts_k: np.ndarray, pos_q: np.ndarray, pos_k: np.ndarray,
               rab_pos_h: np.ndarray, rab_time_h: np.ndarray) -> np.ndarray:
    """rab^{p,t} for one head between query rows and key rows (dense matrix)."""
    P, Tb = rab_pos_h.shape[0], rab_time_h.shape[0]
    dpos = pos_q[:, None] - pos_k[None, :]
    dts = ts_q[:, None].astype(np.int64) - ts_k[None, :].astype(np.int64)
    # |i - j|: keys after the row only occur inside the bidirectional U+S block
    bp = pos_bucket(np.abs(dpos), P)
    bt = time_bucket(dts, Tb)
    return rab_pos_h[bp] + rab_time_h[bt]


def attention_weights(s: np.ndarray, mask: np.ndarray, phi2: str, n_norm: int) -> np.ndarray:
    """Attention weights from the pre-activations s = Q K^T + rab of one head.

    Pointwise phi2 (Eq. 2): a_ij = phi2(s_ij) / N for visible keys, 0 otherwise.
    Softmax ablation: a_ij = exp(s_ij) / sum over visible j' of exp(s_ij') for
    visible keys (a row with no visible key gets all zeros); N is not used.
    """
    if phi2 == "softmax":
        z = np.where(mask, s, -np.inf)
        m = z.max(axis=1, keepdims=True)
        m = np.where(np.isfinite(m), m, 0.0)
        e = np.where(mask, np.exp(np.where(mask, s, 0.0) - m), 0.0)
        den = e.sum(axis=1, keepdims=True)
        return e / np.where(den > 0.0, den, 1.0)
    return np.where(mask, phi(s, phi2), 0.0) / float(n_norm)


def segment_mask(ts, n_us: int, n_r: int) -> np.ndarray:
    """Visibility of the generalised (MTGR-style) mask for one user: rows i,
    keys j over the user's n tokens ordered U+S, R, C."""
    ts = np.asarray(ts, dtype=np.int64)
    n = len(ts)
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    r_end = n_us + n_r
    key_us = j < n_us
    key_r = (j >= n_us) & (j < r_end)
    row_us = i < n_us
    row_r = (i >= n_us) & (i < r_end)
    row_c = i >= r_end
    vis = key_us & (row_us | row_r | row_c)              # U+S: visible to all
    vis |= row_r & key_r & (j <= i)                       # R: causal
    vis |= row_c & key_r & (ts[None, :] <= ts[:, None])   # C: R events up to its time
    vis |= row_c & (j == i)                               # C: itself only
    return vis


def user_attention(q, k, v, ts, rab_pos, rab_time, n_norm: int, H: int, dqk: int, dv: int,
                   phi2: str = "silu", mask=None) -> np.ndarray:
    """Eq. 2 for one user: causal pointwise attention, per head, divided by N
    (or the softmax ablation, see attention_weights); `mask` (bool [n, n])
    replaces the causal mask (the generalised masks of segment_mask).

    q, k: [n, H*dqk]; v: [n, H*dv]; ts: [n] int64; returns AV [n, H*dv].
    """
    n = q.shape[0]
    out = np.zeros((n, H * dv))
    if n == 0:
        return out
    pos = np.arange(n)
    if mask is None:
        mask = np.tril(np.ones((n, n), dtype=bool))
    for h in range(H):
        qh = q[:, h * dqk:(h + 1) * dqk]
        kh = k[:, h * dqk:(h + 1) * dqk]
        vh = v[:, h * dv:(h + 1) * dv]
        s = qh @ kh.T + rab_matrix(ts, ts, pos, pos, rab_pos[h], rab_time[h])
        a = attention_weights(s, mask, phi2, n_norm)
        out[:, h * dv:(h + 1) * dv] = a @ vh
    return out


def layer_norm(o: np.ndarray, eps: float, gamma=None, beta=None) -> np.ndarray:
    """Norm of Eq. 3 read as LayerNorm over the whole H*dv row, biased variance."""
    mu = o.mean(axis=1, keepdims=True)
    var = ((o - mu) ** 2).mean(axis=1, keepdims=True)
    y = (o - mu) / np.sqrt(var + eps)
    if gamma is not None:
        y = y * gamma
    if beta is not None:
        y = y + beta
    return y


def output(x, av, u, w2, b2, eps, gamma=None, beta=None):
    """Eq. 3 plus the residual: Y = X + W2 (Norm(AV) (.) U) + b2."""
    g = layer_norm(av, eps, gamma, beta) * u
    return x + g @ w2.T + b2, g


def _f64(a):
    return None if a is None else np.asarray(a, dtype=np.float64)


def layer_fwd(x, offsets, timestamps, layer, cfg, *, keep_stages: bool = True,
              users: Optional[Sequence[int]] = None, prefix: Optional[Sequence[int]] = None,
              segments=None):
    """One HSTU layer over a jagged batch.

    Returns a dict with Y [T, d] and (if keep_stages) U, V, Q, K, AV, G = Norm(AV) (.) U.
    `users` restricts work to some users (other rows are left NaN); `prefix[i]`
    computes only the first prefix[i] rows of users[i] (valid because the layer
    is causal and N = n_u does not depend on the prefix).  `segments` ([B, 2]:
    n_us, n_r per user) selects the generalised masks (no prefix then).
    """
    x = _f64(x)
    H, dqk, dv = cfg.num_heads, cfg.dqk, cfg.dv
    T = x.shape[0]
    res = {"y": np.full((T, cfg.d_model), np.nan)}
    if keep_stages:
        for name, width in (("u", H * dv), ("v", H * dv), ("q", H * dqk), ("k", H * dqk),
                            ("av", H * dv), ("g", H * dv)):
            res[name] = np.full((T, width), np.nan)
    B = len(offsets) - 1
    users = range(B) if users is None else users
    w1, b1, w2, b2 = _f64(layer.w1), _f64(layer.b1), _f64(layer.w2), _f64(layer.b2)
    rp, rt = _f64(layer.rab_pos), _f64(layer.rab_time)
    gamma, beta = _f64(layer.ln_gamma), _f64(layer.ln_beta)
    for idx, uu in enumerate(users):
        s, e = int(offsets[uu]), int(offsets[uu + 1])
        n_u = e - s
        if prefix is not None:
            e = s + min(n_u, int(prefix[idx]))
        if e == s:
            continue
        xu = x[s:e]
        u, v, q, k = projection(xu, w1, b1, H, dqk, dv, cfg.phi1)
        mask = None
        if segments is not None:
            assert prefix is None
            mask = segment_mask(timestamps[s:e], int(segments[uu][0]), int(segments[uu][1]))
        av = user_attention(q, k, v, timestamps[s:e], rp, rt, n_u, H, dqk, dv, cfg.phi2, mask)
        y, g = output(xu, av, u, w2, b2, cfg.ln_eps, gamma, beta)
        res["y"][s:e] = y
        if keep_stages:
            for name, val in (("u", u), ("v", v), ("q", q), ("k", k), ("av", av), ("g", g)):
                res[name][s:e] = val
    return res


def forward(x, offsets, timestamps, layers, cfg, *, keep_stages: bool = False,
            users=None, prefix=None, segments=None):
    """Stack of HSTU layers (the residual stream is carried in float64)."""
    cur = _f64(x)
    stages = []
    for layer in layers:
        r = layer_fwd(cur, offsets, timestamps, layer, cfg, keep_stages=keep_stages,
                      users=users, prefix=prefix, segments=segments)
        stages.append(r)
        cur = r["y"]
    return cur, stages


def history_kv(x, offsets, timestamps, layers, cfg):
    """Encode the history and keep every layer's K and V rows (the cacheable ops)."""
    cur = _f64(x)
    ks, vs = [], []
    for layer in layers:
        r = layer_fwd(cur, offsets, timestamps, layer, cfg, keep_stages=True)
        ks.append(r["k"])
        vs.append(r["v"])
        cur = r["y"]
    return cur, ks, vs


def mfalcon_scores(hist_x, offsets, timestamps, layers, cfg, cand_offsets, cand_emb,
                   request_ts, microbatch: int, kv=None, return_rows: bool = False):
    """M-FALCON: score every candidate against its user's cached history.

    Candidates of a user are taken b_m at a time; inside a microbatch each
    candidate's row only sees the history keys/values and its own key/value,
    so the microbatch size changes the schedule, not the result.
    `kv` = (per-layer K list, per-layer V list) replaces the history encode.
    With return_rows the final residual-stream rows y_c^(L) are returned too.
    """
    H, dqk, dv = cfg.num_heads, cfg.dqk, cfg.dv
    if kv is None:
        _, ks, vs = history_kv(hist_x, offsets, timestamps, layers, cfg)
    else:
        ks, vs = kv
    e_all = _f64(cand_emb)
    scores = np.zeros(e_all.shape[0])
    rows = np.zeros_like(e_all)
    B = len(offsets) - 1
    for uu in range(B):
        hs, he = int(offsets[uu]), int(offsets[uu + 1])
        n_u = he - hs
        cs, ce = int(cand_offsets[uu]), int(cand_offsets[uu + 1])
        t_req = int(request_ts[uu])
        for mb in range(cs, ce, max(1, microbatch)):
            mend = min(ce, mb + max(1, microbatch))
            e = e_all[mb:mend]
            xc = e.copy()
            m = xc.shape[0]
            for li, layer in enumerate(layers):
                w1, b1, w2, b2 = _f64(layer.w1), _f64(layer.b1), _f64(layer.w2), _f64(layer.b2)
                rp, rt = _f64(layer.rab_pos), _f64(layer.rab_time)
                u, v, q, k = projection(xc, w1, b1, H, dqk, dv, cfg.phi1)
                kh_all = ks[li][hs:he]
                vh_all = vs[li][hs:he]
                av = np.zeros((m, H * dv))
                pos_k = np.arange(n_u)
                pos_q = np.full(m, n_u)
                ts_q = np.full(m, t_req, dtype=np.int64)
                for h in range(H):
                    qh = q[:, h * dqk:(h + 1) * dqk]
                    kh = kh_all[:, h * dqk:(h + 1) * dqk]
                    vh = vh_all[:, h * dv:(h + 1) * dv]
                    s_hist = qh @ kh.T + rab_matrix(ts_q, timestamps[hs:he], pos_q, pos_k,
                                                    rp[h], rt[h])
                    own_k = k[:, h * dqk:(h + 1) * dqk]
                    own_v = v[:, h * dv:(h + 1) * dv]
                    s_self = np.einsum("cd,cd->c", qh, own_k) + rp[h, 0] + rt[h, 0]
                    # keys of a candidate row: the n_u history rows, then itself
                    s_all = np.concatenate([s_hist, s_self[:, None]], axis=1)
                    a = attention_weights(s_all, np.ones(s_all.shape, dtype=bool), cfg.phi2,
                                          max(n_u, 1))
                    o = a[:, :n_u] @ vh + a[:, n_u:n_u + 1] * own_v
                    av[:, h * dv:(h + 1) * dv] = o
                xc, _ = output(xc, av, u, w2, b2, cfg.ln_eps, _f64(layer.ln_gamma),
                               _f64(layer.ln_beta))
            scores[mb:mend] = np.einsum("cd,cd->c", xc, e)
            rows[mb:mend] = xc
    return (scores, rows) if return_rows else scores


def score_alone(hist_x, offsets, timestamps, layers, cfg, cand_offsets, cand_emb,
                request_ts, cand_index: List[int]) -> np.ndarray:
    """Score candidates one at a time by running the encoder on [history ; c].

    The candidate row gets timestamp t_req and the normaliser stays N = n_u.
    This is the full-recompute definition the cached path must reproduce.
    """
    x = _f64(hist_x)
    e_all = _f64(cand_emb)
    out = []
    B = len(offsets) - 1
    for c in cand_index:
        uu = int(np.searchsorted(cand_offsets, c, side="right") - 1)
        assert 0 <= uu < B
        hs, he = int(offsets[uu]), int(offsets[uu + 1])
        n_u = he - hs
        seq = np.concatenate([x[hs:he], e_all[c:c + 1]], axis=0)
        ts = np.concatenate([timestamps[hs:he], [int(request_ts[uu])]]).astype(np.int64)
        cur = seq
        for layer in layers:
            u, v, q, k = projection(cur, _f64(layer.w1), _f64(layer.b1), cfg.num_heads,
                                    cfg.dqk, cfg.dv, cfg.phi1)
            av = user_attention(q, k, v, ts, _f64(layer.rab_pos), _f64(layer.rab_time),
                                max(n_u, 1), cfg.num_heads, cfg.dqk, cfg.dv, cfg.phi2)
            cur, _ = output(cur, av, u, _f64(layer.w2), _f64(layer.b2), cfg.ln_eps,
                            _f64(layer.ln_gamma), _f64(layer.ln_beta))
        out.append(float(cur[n_u] @ e_all[c]))
    return np.array(out)


def time_bucket_thresholds(num_time_buckets: int) -> np.ndarray:
    """Smallest integer dt reaching each bucket k (k = 0..Tb-1), by the formula above.

    Buckets that no dt below 2^62 reaches get INT64_MAX.  Used only by tests to
    probe bucket edges (dt = thr[k] - 1 and thr[k]).
    """
    cap = 1 << 62
    thr = np.zeros(num_time_buckets, dtype=np.int64)
    for k in range(1, num_time_buckets):
        if int(time_bucket(cap, 1 << 30)) < k:
            thr[k] = np.iinfo(np.int64).max
            continue
        lo, hi = 0, 1
        while int(time_bucket(hi, 1 << 30)) < k:
            hi = min(hi * 2, cap)
        while lo < hi:
            mid = (lo + hi) // 2
            if int(time_bucket(mid, 1 << 30)) >= k:
                hi = mid
            else:
                lo = mid + 1
        thr[k] = lo
    return thr
