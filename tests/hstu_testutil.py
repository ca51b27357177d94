"""Shared helpers for the GPU parity tests (marshalling and error metrics)."""
import numpy as np
import torch

from gen.device import case_tensors, tensor

# Tolerance for bf16 storage against the float64 oracle (stated for this path):
# max abs error <= 2e-2 and relative L2 error <= 5e-3.
MAX_ABS = 2e-2
REL_L2 = 5e-3


def errors(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    diff = got - want
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    denom = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(diff) / denom) if denom > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_close(got, want, what="", max_abs=MAX_ABS, rel_l2=REL_L2, scaled=False):
    """max |got - want| <= max_abs and ||got - want|| / ||want|| <= rel_l2.

    scaled=True is for bf16-stored intermediates (AV, cached K/V): one bf16 ulp
    is 2^-7 relative, so the max-abs bound is applied to |got - want| / max(1, |want|).
    """
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    ma, rl = errors(got, want)
    if scaled:
        ma = float(np.max(np.abs(got - want) / np.maximum(1.0, np.abs(want)))) if got.size else 0.0
    assert ma <= max_abs and rl <= rel_l2, f"{what}: max_abs={ma:.3e} rel_l2={rl:.3e}"
    return ma, rl


def binding():
    from hstu_sequential_transduction_jagged_b200 import build, hstu
    build.build()
    return hstu


def config_of(H, cfg):
    return H.LayerConfig(d_model=cfg.d_model, num_heads=cfg.num_heads,
                         num_pos_buckets=cfg.num_pos_buckets,
                         num_time_buckets=cfg.num_time_buckets, dqk=cfg.dqk, dv=cfg.dv,
                         phi1=cfg.phi1, phi2=cfg.phi2, ln_eps=cfg.ln_eps, dtype=cfg.dtype)


def upload(H, case, device="cuda"):
    t = case_tensors(case, device)
    jag = H.Jagged(t["offsets"], t["timestamps"], case.max_len, case.total_tokens)
    weights = [H.LayerWeights(**lw) for lw in t["layers"]]
    return t, jag, weights


def upload_attn(H, ac, device="cuda"):
    dt = torch.bfloat16 if ac.dtype == "bf16" else torch.float32
    offs = tensor(ac.offsets, torch.int64, device)
    ts = tensor(ac.timestamps, torch.int64, device)
    lens = np.diff(ac.offsets)
    jag = H.Jagged(offs, ts, int(lens.max()) if len(lens) else 0, int(ac.offsets[-1]))
    q, k, v = (tensor(a, dt, device) for a in (ac.q, ac.k, ac.v))
    rp = tensor(ac.rab_pos, torch.float32, device)
    rt = tensor(ac.rab_time, torch.float32, device)
    return jag, q, k, v, rp, rt
