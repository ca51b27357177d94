"""Pure-Python loop version of the HSTU layer (tiny inputs only).

TEST INFRASTRUCTURE ONLY: used to pin the vectorised oracle in `oracle.hstu`.
It is written independently of that module (scalar loops and the `math`
module, no numpy arithmetic) so that an indexing, ordering or sign mistake in
either one shows up as a disagreement.

Follows the review of "Actions Speak Louder than Words" (xllm-io paper-review
of arXiv 2402.17152), section 三 核心公式 Eq. 1-3, with the same readings as
`oracle.hstu` (SiLU/ReLU/identity phi2 with 1/n_u, or the softmax ablation
over the visible keys; LayerNorm over H*dv,
ln(dt+1)/0.301 time buckets, min(i-j, P-1) position buckets, residual).
"""
from __future__ import annotations

import math


def _act(x, kind):
    if kind == "relu":
        return x if x > 0.0 else 0.0
    if kind == "silu":
        # x * sigmoid(x), written in the numerically safe form for both signs
        if x >= 0:
            return x / (1.0 + math.exp(-x))
        ex = math.exp(x)
        return x * ex / (1.0 + ex)
    if kind == "identity":
        return x
    raise ValueError(kind)


def _tbucket(dt, Tb):
    if dt < 0:
        return 0
    b = int(math.floor(math.log(float(dt) + 1.0) / 0.301))
    return max(0, min(Tb - 1, b))


def _visible(i, j, n_us, n_r, t):
    """Generalised (MTGR-style) mask, row by row: U+S seen by all and seeing only
    U+S, R causal, a candidate seeing U+S, the R events up to its time, itself."""
    r_end = n_us + n_r
    if j < n_us:
        return True
    if i < n_us:
        return False
    if i < r_end:
        return j <= i
    if j < r_end:
        return t[j] <= t[i]
    return j == i


def layer(x, offsets, ts, w1, b1, w2, b2, rab_pos, rab_time, H, dqk, dv,
          phi1="relu", phi2="silu", eps=1e-5, gamma=None, beta=None, segments=None):
    """One layer with explicit loops.  All arguments are nested lists / scalars;
    `segments` [[n_us, n_r], ...] selects the generalised masks (else causal)."""
    T = len(x)
    d = len(x[0]) if T else 0
    n1 = len(w1)
    P, Tb = len(rab_pos[0]), len(rab_time[0])
    hv = H * dv
    y = [[0.0] * d for _ in range(T)]
    for uu in range(len(offsets) - 1):
        s, e = offsets[uu], offsets[uu + 1]
        n = e - s
        # Eq. 1, row by row
        z = []
        for i in range(s, e):
            row = []
            for c in range(n1):
                acc = b1[c]
                for t in range(d):
                    acc += w1[c][t] * x[i][t]
                row.append(_act(acc, phi1))
            z.append(row)
        U = [r[0:hv] for r in z]
        V = [r[hv:2 * hv] for r in z]
        Q = [r[2 * hv:2 * hv + H * dqk] for r in z]
        K = [r[2 * hv + H * dqk:2 * hv + 2 * H * dqk] for r in z]
        tu = ts[s:e]
        for i in range(n):
            # Eq. 2 for row i, every head
            if segments is None:
                keys = list(range(i + 1))
            else:
                keys = [j for j in range(n) if _visible(i, j, segments[uu][0], segments[uu][1], tu)]
            o = [0.0] * hv
            for h in range(H):
                pre = []
                for j in keys:
                    dot = 0.0
                    for t in range(dqk):
                        dot += Q[i][h * dqk + t] * K[j][h * dqk + t]
                    bp = min(abs(i - j), P - 1)
                    bt = _tbucket(ts[s + i] - ts[s + j], Tb)
                    pre.append(dot + rab_pos[h][bp] + rab_time[h][bt])
                if phi2 == "softmax":
                    # ablation: softmax over the visible keys, no 1/n
                    top = max(pre)
                    ex = [math.exp(val - top) for val in pre]
                    tot = sum(ex)
                    weights = [val / tot for val in ex]
                else:
                    weights = [_act(val, phi2) / n for val in pre]
                for idx, j in enumerate(keys):
                    for t in range(dv):
                        o[h * dv + t] += weights[idx] * V[j][h * dv + t]
            # Eq. 3: LayerNorm over all heads, gate with U, project, residual
            mean = sum(o) / hv
            var = sum((val - mean) * (val - mean) for val in o) / hv
            inv = 1.0 / math.sqrt(var + eps)
            g = []
            for c in range(hv):
                nv = (o[c] - mean) * inv
                if gamma is not None:
                    nv *= gamma[c]
                if beta is not None:
                    nv += beta[c]
                g.append(nv * U[i][c])
            for c in range(d):
                acc = b2[c]
                for t in range(hv):
                    acc += w2[c][t] * g[t]
                y[s + i][c] = x[s + i][c] + acc
    return y
