"""Pins of the backward oracle (oracle/hstu_bwd.py) against central finite
differences of the forward oracle (oracle/hstu.py) in float64.

The forward is the review's section 三 核心公式 Eq. 1-3 with the residual; the
backward is its derivative.  Finite differences of L = sum(dY (.) Y(theta))
check every gradient the oracle returns (X, W1, b1, W2, b2, both rab tables,
the LayerNorm affine) without sharing any of its formulas.  A mistake planted
in the oracle (a wrong SiLU derivative, a dropped LayerNorm term, a transposed
dS) must fail the comparison."""
import types

import numpy as np
import pytest

from oracle import hstu as F
from oracle import hstu_bwd as B

EPS = 1e-6


def _case(phi2, seed, lengths=(3, 5, 1), affine=True, d=8, H=2, dh=4, P=4, Tb=6):
    rng = np.random.default_rng(seed)
    cfg = types.SimpleNamespace(num_heads=H, dqk=dh, dv=dh, d_model=d, phi1="relu", phi2=phi2,
                                ln_eps=1e-5)
    n1 = 2 * H * (dh + dh)
    layer = types.SimpleNamespace(
        w1=rng.standard_normal((n1, d)) * 0.5, b1=rng.standard_normal(n1) * 0.3,
        w2=rng.standard_normal((d, H * dh)) * 0.5, b2=rng.standard_normal(d) * 0.3,
        rab_pos=rng.standard_normal((H, P)) * 0.3, rab_time=rng.standard_normal((H, Tb)) * 0.3,
        ln_gamma=(1.0 + 0.2 * rng.standard_normal(H * dh)) if affine else None,
        ln_beta=(0.2 * rng.standard_normal(H * dh)) if affine else None)
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(offsets[-1])
    # gaps from 0 s to a few hundred s: several time buckets, some equal times
    ts = np.zeros(T, dtype=np.int64)
    for u in range(len(lengths)):
        s, e = offsets[u], offsets[u + 1]
        ts[s:e] = 1000 + np.cumsum(rng.integers(0, 300, e - s))
    x = rng.standard_normal((T, d))
    dy = rng.standard_normal((T, d))
    return cfg, layer, offsets, ts, x, dy


def _loss(x, offsets, ts, layer, cfg, dy, segments=None):
    y = F.layer_fwd(x, offsets, ts, layer, cfg, keep_stages=False, segments=segments)["y"]
    return float(np.sum(dy * y))


def _fd_check(cfg, layer, offsets, ts, x, dy, got, segments=None, tol=2e-6):
    """Every entry of every gradient against a central difference."""
    def fd(arr, set_back):
        g = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + EPS
            lp = _loss(x, offsets, ts, layer, cfg, dy, segments)
            arr[idx] = old - EPS
            lm = _loss(x, offsets, ts, layer, cfg, dy, segments)
            arr[idx] = old
            g[idx] = (lp - lm) / (2 * EPS)
        set_back()
        return g

    checks = [("dx", x), ("dw1", layer.w1), ("db1", layer.b1), ("dw2", layer.w2),
              ("db2", layer.b2), ("drab_pos", layer.rab_pos), ("drab_time", layer.rab_time)]
    if layer.ln_gamma is not None:
        checks += [("dgamma", layer.ln_gamma), ("dbeta", layer.ln_beta)]
    for name, arr in checks:
        want = fd(arr, lambda: None)
        err = np.abs(got[name] - want).max()
        scale = max(1.0, np.abs(want).max())
        assert err <= tol * scale, f"{name}: max |analytic - fd| = {err:.3e} (scale {scale:.2e})"


@pytest.mark.parametrize("phi2", ["silu", "relu", "identity", "softmax"])
def test_layer_gradients_match_finite_differences(phi2):
    cfg, layer, offsets, ts, x, dy = _case(phi2, seed=3)
    got = B.layer_bwd(x, offsets, ts, layer, cfg, dy)
    _fd_check(cfg, layer, offsets, ts, x, dy, got)


def test_gradients_without_affine_layernorm():
    cfg, layer, offsets, ts, x, dy = _case("silu", seed=4, affine=False)
    got = B.layer_bwd(x, offsets, ts, layer, cfg, dy)
    assert got["dgamma"] is None and got["dbeta"] is None
    _fd_check(cfg, layer, offsets, ts, x, dy, got)


@pytest.mark.parametrize("phi2", ["silu", "softmax"])
def test_gradients_under_generalised_masks(phi2):
    """U+S / R / candidate masks: keys after the row inside U+S (|i - j| buckets),
    candidates that see part of R and themselves."""
    cfg, layer, offsets, ts, x, dy = _case(phi2, seed=5, lengths=(6, 4))
    segments = [[2, 2], [0, 3]]
    got = B.layer_bwd(x, offsets, ts, layer, cfg, dy, segments=segments)
    _fd_check(cfg, layer, offsets, ts, x, dy, got, segments=segments)


def test_position_and_time_clamps_receive_gradient():
    """P = 2 and Tb = 3 clamp most pairs into the last bucket; the clamped
    entries collect the sum of dS over all of them."""
    cfg, layer, offsets, ts, x, dy = _case("silu", seed=6, lengths=(5,), P=2, Tb=3)
    got = B.layer_bwd(x, offsets, ts, layer, cfg, dy)
    assert np.all(got["drab_pos"][:, -1] != 0.0) and np.all(got["drab_time"][:, -1] != 0.0)
    _fd_check(cfg, layer, offsets, ts, x, dy, got)


def test_attention_gradient_is_linear_in_do_for_identity_phi2():
    """phi2 = identity, rab = 0: O = (Q K^T (.) M) V / N, so dV = A^T dO with
    A = (Q K^T (.) M) / N and dQ = (dO V^T (.) M) K / N: closed forms."""
    rng = np.random.default_rng(7)
    n, H, dh = 6, 1, 3
    q, k, v = (rng.standard_normal((n, dh)) for _ in range(3))
    do = rng.standard_normal((n, dh))
    ts = np.arange(n, dtype=np.int64) * 10
    rp, rt = np.zeros((H, 4)), np.zeros((H, 5))
    dq, dk, dv, _, _ = B.attention_bwd_user(q, k, v, ts, rp, rt, n, H, dh, dh, "identity", do)
    M = np.tril(np.ones((n, n)))
    A = (q @ k.T) * M / n
    dS = (do @ v.T) * M / n
    assert np.allclose(dv, A.T @ do, atol=1e-12)
    assert np.allclose(dq, dS @ k, atol=1e-12)
    assert np.allclose(dk, dS.T @ q, atol=1e-12)


@pytest.mark.parametrize("plant", ["silu_grad", "ln_term", "ds_transpose"])
def test_planted_mistakes_fail_the_pins(monkeypatch, plant):
    cfg, layer, offsets, ts, x, dy = _case("silu", seed=8, lengths=(4, 3))
    if plant == "silu_grad":
        # drop the x (1 - sigmoid) term of SiLU'
        monkeypatch.setattr(B, "phi_grad", lambda s, kind: (1.0 / (1.0 + np.exp(-s)))
                            if kind == "silu" else (s > 0.0).astype(np.float64))
    elif plant == "ln_term":
        # drop the n * mean(dn (.) n) term of the LayerNorm backward
        monkeypatch.setattr(B, "layer_norm_bwd",
                            lambda dn, nrm, rstd: rstd * (dn - dn.mean(axis=1, keepdims=True)))
    elif plant == "ds_transpose":
        real_att = B.attention_bwd_user

        def swapped(q, k, v, *a, **kw):
            dq, dk, dv, drp, drt = real_att(q, k, v, *a, **kw)
            return dk, dq, dv, drp, drt  # dQ and dK exchanged
        monkeypatch.setattr(B, "attention_bwd_user", swapped)
    got = B.layer_bwd(x, offsets, ts, layer, cfg, dy)
    with pytest.raises(AssertionError):
        _fd_check(cfg, layer, offsets, ts, x, dy, got)


def test_separate_f1_input_reduces_to_the_pinned_gradient():
    """x_f1 (the input f1 reads) differing from the residual input: every
    gradient equals that of the layer fed x_f1 alone, because the residual
    term sum(dY (.) X) has gradient dY whichever X it is."""
    cfg, layer, offsets, ts, x, dy = _case("silu", seed=9, lengths=(4, 3))
    xr = np.round(x * 64.0) / 64.0  # a coarser copy, as a 16-bit f1 input would be
    split = B.layer_bwd(x, offsets, ts, layer, cfg, dy, x_f1=xr)
    alone = B.layer_bwd(xr, offsets, ts, layer, cfg, dy)
    for name in ("dx", "dw1", "db1", "dw2", "db2", "drab_pos", "drab_time", "dgamma", "dbeta"):
        assert np.allclose(split[name], alone[name], rtol=0, atol=1e-12), name
