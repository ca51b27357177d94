"""Float64 CPU oracle for the backward pass of one HSTU layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call this
module; only the tests and the benchmark's CPU baseline leg do.  It shares no
code with the CUDA library.

The pages state the forward (review of "Actions Speak Louder than Words",
xllm-io paper review, section 三 技术架构 / 核心公式, Eq. 1-3, with the residual
between layers) and train it (section 五 编码器效率: training throughput); they
print no backward.  The backward is therefore the derivative of the forward of
oracle/hstu.py, taken step by step with the chain rule, in the forward's
notation.  Given dY = dL/dY for a loss L of the layer output Y:

  Y = X + G W2^T + b2           dX  = dY (+ the path through f1 below)
                                db2 = sum_rows dY,  dW2 = dY^T G,  dG = dY W2
  G = Ln (.) U, Ln = n*gamma+beta,  n = (AV - mu) * rstd  (LayerNorm over H*dv)
                                dU = dG (.) Ln,  dLn = dG (.) U
                                dgamma = sum_rows dLn (.) n,  dbeta = sum_rows dLn
                                dn = dLn (.) gamma
                                dAV = rstd * (dn - mean(dn) - n * mean(dn (.) n))
  per head, O = A V, A = phi2(S)/N on visible pairs, S = Q K^T + rab:
                                dV = A^T dO,  dA = dO V^T
                                dS = dA (.) phi2'(S) / N        (pointwise phi2)
                                dS = A (.) (dA - rowsum(dA (.) A))  (softmax ablation)
                                dQ = dS K,  dK = dS^T Q
                                drab_pos[h, b] = sum of dS over visible pairs in position bucket b
                                drab_time[h, b] = the same over time bucket b
  Z = phi1(X W1^T + b1) = [U | V | Q | K]:
                                dZpre = [dU | dV | dQ | dK] (.) phi1'(X W1^T + b1)
                                db1 = sum_rows dZpre,  dW1 = dZpre^T X,  dX += dZpre W1

Readings (the pages are silent on all of them):
  * derivatives at the kinks: ReLU'(0) = 0;
  * SiLU'(x) = sigmoid(x) (1 + x (1 - sigmoid(x)));
  * the bucket indices are integers and carry no gradient; the tables receive
    the sum of dS over the pairs that read each entry;
  * masked pairs (invisible keys) carry no gradient.
"""
from __future__ import annotations

from typing import Optional

import numpy as np

from . import hstu as F


def phi_grad(x: np.ndarray, kind: str) -> np.ndarray:
    """Derivative of the pointwise nonlinearity (ReLU'(0) = 0)."""
    if kind == "relu":
        return (x > 0.0).astype(np.float64)
    if kind == "silu":
        sg = 1.0 / (1.0 + np.exp(-x))
        return sg * (1.0 + x * (1.0 - sg))
    if kind == "identity":
        return np.ones_like(x)
    raise ValueError(kind)


def layer_norm_bwd(dn: np.ndarray, nrm: np.ndarray, rstd: np.ndarray) -> np.ndarray:
    """Gradient through n = (o - mean(o)) * rstd over a row of m entries (biased
    variance): do = rstd * (dn - mean(dn) - n * mean(dn (.) n))."""
    return rstd * (dn - dn.mean(axis=1, keepdims=True) -
                   nrm * (dn * nrm).mean(axis=1, keepdims=True))


def _buckets(ts, n, P, Tb):
    """Position and time bucket index matrices of one user (rows i, keys j)."""
    pos = np.arange(n)
    bp = F.pos_bucket(np.abs(pos[:, None] - pos[None, :]), P)
    dts = np.asarray(ts, dtype=np.int64)[:, None] - np.asarray(ts, dtype=np.int64)[None, :]
    bt = F.time_bucket(dts, Tb)
    return bp, bt


def attention_bwd_user(q, k, v, ts, rab_pos, rab_time, n_norm, H, dqk, dv, phi2, dav,
                       mask=None):
    """Backward of the attention of one user (user_attention in oracle/hstu.py).

    Returns dq, dk, dv (same shapes as q, k, v) and the per-head table
    gradients drab_pos [H, P], drab_time [H, Tb].
    """
    n = q.shape[0]
    P, Tb = rab_pos.shape[1], rab_time.shape[1]
    dq, dk, dvv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    drp, drt = np.zeros((H, P)), np.zeros((H, Tb))
    if n == 0:
        return dq, dk, dvv, drp, drt
    if mask is None:
        mask = np.tril(np.ones((n, n), dtype=bool))
    bp, bt = _buckets(ts, n, P, Tb)
    for h in range(H):
        qh = q[:, h * dqk:(h + 1) * dqk]
        kh = k[:, h * dqk:(h + 1) * dqk]
        vh = v[:, h * dv:(h + 1) * dv]
        s = qh @ kh.T + rab_pos[h][bp] + rab_time[h][bt]
        a = F.attention_weights(s, mask, phi2, n_norm)
        do = dav[:, h * dv:(h + 1) * dv]
        dvv[:, h * dv:(h + 1) * dv] = a.T @ do
        da = do @ vh.T
        if phi2 == "softmax":
            ds = a * (da - (da * a).sum(axis=1, keepdims=True))
        else:
            ds = np.where(mask, da * phi_grad(s, phi2), 0.0) / float(n_norm)
        dq[:, h * dqk:(h + 1) * dqk] = ds @ kh
        dk[:, h * dqk:(h + 1) * dqk] = ds.T @ qh
        np.add.at(drp[h], bp[mask], ds[mask])
        np.add.at(drt[h], bt[mask], ds[mask])
    return dq, dk, dvv, drp, drt


def layer_bwd(x, offsets, timestamps, layer, cfg, dy, segments=None, x_f1=None) -> dict:
    """Gradients of sum(dY (.) Y) for one HSTU layer Y = layer_fwd(X).

    `x_f1` is the input f1 reads when it differs from the residual input x (a
    layer handed its input in two precisions, e.g. an fp32 residual stream of
    which f1 reads a 16-bit copy); the rounding between them passes the
    gradient unchanged, so dX = dY + dZpre W1 either way and dW1 = dZpre^T x_f1.

    Returns dx [T, d], dw1 [n1, d], db1 [n1], dw2 [d, H*dv], db2 [d],
    drab_pos [H, P], drab_time [H, Tb], dgamma / dbeta ([H*dv], or None when
    the layer has no affine LayerNorm) and the intermediate gradients dq, dk,
    dv, du [T, H*64] and dav [T, H*dv].
    """
    x = np.asarray(x, dtype=np.float64)
    xf = x if x_f1 is None else np.asarray(x_f1, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    H, dqk, dvw = cfg.num_heads, cfg.dqk, cfg.dv
    hv, hq = H * dvw, H * dqk
    T, d = x.shape
    w1, b1 = np.asarray(layer.w1, np.float64), np.asarray(layer.b1, np.float64)
    w2 = np.asarray(layer.w2, np.float64)
    rp, rt = np.asarray(layer.rab_pos, np.float64), np.asarray(layer.rab_time, np.float64)
    gamma = None if layer.ln_gamma is None else np.asarray(layer.ln_gamma, np.float64)
    beta = None if layer.ln_beta is None else np.asarray(layer.ln_beta, np.float64)
    out = {"dx": dy.copy(), "dw1": np.zeros_like(w1), "db1": np.zeros_like(b1),
           "dw2": np.zeros_like(w2), "db2": np.zeros(d), "drab_pos": np.zeros_like(rp),
           "drab_time": np.zeros_like(rt),
           "dgamma": None if gamma is None else np.zeros(hv),
           "dbeta": None if beta is None else np.zeros(hv)}
    for name, width in (("dq", hq), ("dk", hq), ("dv", hv), ("du", hv), ("dav", hv)):
        out[name] = np.zeros((T, width))
    for u in range(len(offsets) - 1):
        s0, e0 = int(offsets[u]), int(offsets[u + 1])
        n = e0 - s0
        if n == 0:
            continue
        xu, dyu = xf[s0:e0], dy[s0:e0]
        pre = xu @ w1.T + b1
        z = F.phi(pre, cfg.phi1)
        uu, vv = z[:, 0:hv], z[:, hv:2 * hv]
        qq, kk = z[:, 2 * hv:2 * hv + hq], z[:, 2 * hv + hq:2 * hv + 2 * hq]
        mask = None
        if segments is not None:
            mask = F.segment_mask(timestamps[s0:e0], int(segments[u][0]), int(segments[u][1]))
        av = F.user_attention(qq, kk, vv, timestamps[s0:e0], rp, rt, n, H, dqk, dvw, cfg.phi2,
                              mask)
        mu = av.mean(axis=1, keepdims=True)
        var = ((av - mu) ** 2).mean(axis=1, keepdims=True)
        rstd = 1.0 / np.sqrt(var + cfg.ln_eps)
        nrm = (av - mu) * rstd
        ln = nrm * (gamma if gamma is not None else 1.0) + (beta if beta is not None else 0.0)
        g = ln * uu
        # Y = X + G W2^T + b2
        out["db2"] += dyu.sum(axis=0)
        out["dw2"] += dyu.T @ g
        dg = dyu @ w2
        du = dg * ln
        dln = dg * uu
        if gamma is not None:
            out["dgamma"] += (dln * nrm).sum(axis=0)
            dn = dln * gamma
        else:
            dn = dln
        if beta is not None:
            out["dbeta"] += dln.sum(axis=0)
        dav = layer_norm_bwd(dn, nrm, rstd)
        dq, dk, dv, drp, drt = attention_bwd_user(qq, kk, vv, timestamps[s0:e0], rp, rt, n, H,
                                                  dqk, dvw, cfg.phi2, dav, mask)
        out["drab_pos"] += drp
        out["drab_time"] += drt
        dzpre = np.concatenate([du, dv, dq, dk], axis=1) * phi_grad(pre, cfg.phi1)
        out["db1"] += dzpre.sum(axis=0)
        out["dw1"] += dzpre.T @ xu
        out["dx"][s0:e0] += dzpre @ w1
        for name, val in (("dq", dq), ("dk", dk), ("dv", dv), ("du", du), ("dav", dav)):
            out[name][s0:e0] = val
    return out
