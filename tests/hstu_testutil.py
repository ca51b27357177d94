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


# Every comparison made through assert_close / record is kept here with its raw
# errors and bounds; conftest writes the list to $HSTU_PARITY_REPORT (JSON) at
# the end of the session when that variable is set.
PARITY_LOG = []


def record(what, max_abs, rel_l2, bound_abs=None, bound_rel=None, note=""):
    PARITY_LOG.append({"what": what, "max_abs": float(max_abs), "rel_l2": float(rel_l2),
                       "bound_max_abs": bound_abs, "bound_rel_l2": bound_rel, "note": note})


def assert_close(got, want, what="", max_abs=MAX_ABS, rel_l2=REL_L2, scaled=False):
    """max |got - want| <= max_abs and ||got - want|| / ||want|| <= rel_l2.

    scaled=True is for bf16-stored intermediates (AV, cached K/V): one bf16 ulp
    is 2^-7 relative, so the max-abs bound is applied to |got - want| / max(1, |want|).
    The raw errors are recorded in PARITY_LOG.
    """
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    ma, rl = errors(got, want)
    raw_ma = ma
    if scaled:
        ma = float(np.max(np.abs(got - want) / np.maximum(1.0, np.abs(want)))) if got.size else 0.0
    record(what, raw_ma, rl, max_abs, rel_l2, "max_abs bound on |err|/max(1,|want|)" if scaled else "")
    assert ma <= max_abs and rl <= rel_l2, f"{what}: max_abs={ma:.3e} rel_l2={rl:.3e}"
    return ma, rl


def check_scores(got, want, emb, what):
    """M-FALCON scores s_c = <y_c, e_c>.  The raw scores meet rel-L2 <= 5e-3 with
    a wide margin, because about ||e_c||^2 (~d) of each score is the input
    itself; so the comparison that can fail is made on the part the layers
    add, s_c - <e_c, e_c> (computed in float64 from the inputs, the same on
    both sides): rel-L2 <= 5e-3.  The max-abs bound is translated to the score
    through e_c: the score error divided by ||e_c|| is the error of y_c along
    the unit vector e_c / ||e_c||, one coordinate of y_c in an orthonormal
    basis, and it is held to the per-coordinate bound of y_c itself (2e-2)."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    e = np.asarray(emb, dtype=np.float64)
    ee = np.einsum("cd,cd->c", e, e)
    _, rl = errors(got - ee, want - ee)
    proj = np.abs(got - want) / np.maximum(np.linalg.norm(e, axis=1), 1e-30)
    pm = float(proj.max()) if proj.size else 0.0
    bound, bound_rel = MAX_ABS, REL_L2
    record(what, pm, rl, bound, bound_rel, "score: max |ds|/||e_c||; rel-L2 of s - <e,e>")
    _, raw_rel = errors(got, want)
    record(what + " (raw scores)", float(np.abs(got - want).max()) if got.size else 0.0, raw_rel,
           None, REL_L2)
    assert np.all(np.isfinite(got)), f"{what}: non-finite scores"
    assert raw_rel <= REL_L2, f"{what}: raw rel_l2={raw_rel:.3e}"
    assert rl <= bound_rel and pm <= bound, \
        f"{what}: rel_l2(s-<e,e>)={rl:.3e} max|ds|/|e|={pm:.3e}"
    return pm, rl


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
    dt = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}[ac.dtype]
    offs = tensor(ac.offsets, torch.int64, device)
    ts = tensor(ac.timestamps, torch.int64, device)
    lens = np.diff(ac.offsets)
    jag = H.Jagged(offs, ts, int(lens.max()) if len(lens) else 0, int(ac.offsets[-1]))
    q, k, v = (tensor(a, dt, device) for a in (ac.q, ac.k, ac.v))
    rp = tensor(ac.rab_pos, torch.float32, device)
    rt = tensor(ac.rab_time, torch.float32, device)
    return jag, q, k, v, rp, rt
