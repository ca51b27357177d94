"""Backward of the causal attention step on the GPU (hstu_attn_bwd) against the
float64 backward oracle (oracle/hstu_bwd.py, pinned by finite differences).

Tolerance (gradients have no stated bound of their own): per output tensor,
rel-L2 <= 5e-3 and max |err| <= 2e-2 * max |ref|, the forward's bound applied
to the gradient's own scale.  The GPU takes P and dS in the operand type
(fp16 or bf16) between its MMAs, with fp32 accumulation."""
import numpy as np
import pytest
import torch

from gen.device import tensor
from gen.inputs import make_attn_case, to_dtype
from oracle import hstu_bwd as OB
from hstu_testutil import binding, record

pytestmark = pytest.mark.gpu

REL, ABS = 5e-3, 2e-2


@pytest.fixture(scope="module")
def H():
    return binding()


def _check(got, want, what):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    diff = got - want
    scale = max(float(np.abs(want).max()), 1e-30)
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(want), 1e-30))
    ma = float(np.abs(diff).max()) / scale
    record(what, ma, rel, ABS, REL, "max-abs relative to max |ref|")
    assert rel <= REL and ma <= ABS, f"{what}: rel_l2={rel:.3e} max_abs/scale={ma:.3e}"


def _run(H, lengths, phi2, dtype, P=512, Tb=128, heads=2, seed=81, gap_kind="exp"):
    ac = make_attn_case(lengths, heads, P, Tb, seed=seed, dtype=dtype, gap_kind=gap_kind)
    rng = np.random.default_rng(seed + 1)
    T = int(ac.offsets[-1])
    do = to_dtype(rng.standard_normal((T, heads * 64), dtype=np.float32) * 0.5, dtype)
    tdt = H.TORCH_DTYPE[dtype]
    jag = H.Jagged(tensor(ac.offsets, torch.int64, "cuda"), tensor(ac.timestamps, torch.int64, "cuda"),
                   max(lengths), T)
    cfg = H.LayerConfig(d_model=heads * 64, num_heads=heads, num_pos_buckets=P,
                        num_time_buckets=Tb, phi2=phi2, dtype=dtype)
    q, k, v, d_o = (tensor(a, tdt, "cuda") for a in (ac.q, ac.k, ac.v, do))
    dq, dk, dv, drp, drt = H.attn_bwd(cfg, jag, q, k, v, d_o, tensor(ac.rab_pos, torch.float32, "cuda"),
                                      tensor(ac.rab_time, torch.float32, "cuda"))
    torch.cuda.synchronize()
    assert H.device_status() == 0
    want = {"dq": np.zeros((T, heads * 64)), "dk": np.zeros((T, heads * 64)),
            "dv": np.zeros((T, heads * 64)), "drp": np.zeros((heads, P)),
            "drt": np.zeros((heads, Tb))}
    for u, n in enumerate(lengths):
        s, e = int(ac.offsets[u]), int(ac.offsets[u + 1])
        if n == 0:
            continue
        a = OB.attention_bwd_user(ac.q[s:e].astype(np.float64), ac.k[s:e].astype(np.float64),
                                  ac.v[s:e].astype(np.float64), ac.timestamps[s:e],
                                  ac.rab_pos.astype(np.float64), ac.rab_time.astype(np.float64),
                                  n, heads, 64, 64, phi2, do[s:e].astype(np.float64))
        want["dq"][s:e], want["dk"][s:e], want["dv"][s:e] = a[0], a[1], a[2]
        want["drp"] += a[3]
        want["drt"] += a[4]
    tag = f"attn bwd {phi2} {dtype} {lengths[:4]}"
    _check(dq.cpu().numpy(), want["dq"], tag + " dq")
    _check(dk.cpu().numpy(), want["dk"], tag + " dk")
    _check(dv.cpu().numpy(), want["dv"], tag + " dv")
    _check(drp.cpu().numpy(), want["drp"], tag + " drab_pos")
    _check(drt.cpu().numpy(), want["drt"], tag + " drab_time")


# one row, partial first tile, exactly one and two tiles, partial second
# tile, an empty user, several tiles
LENGTHS = [1, 100, 128, 129, 256, 0, 300, 700]


@pytest.mark.parametrize("phi2", ["silu", "relu", "identity"])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_attention_backward(H, phi2, dtype):
    _run(H, LENGTHS, phi2, dtype)


def test_attention_backward_clamped_tables(H):
    """P = 64 and Tb = 16: most pairs fall in the last position bucket, many in
    the last time bucket."""
    _run(H, [300, 129, 50], "silu", "fp16", P=64, Tb=16, seed=83)


def test_attention_backward_long_user(H):
    """A 2000-row user with 8 heads (16 key tiles, the longest-first order)."""
    _run(H, [2000, 77], "silu", "fp16", P=4096, heads=8, seed=85)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_attention_backward_lognormal_timeline(H, dtype):
    """The long-sequence workload's timeline (log-normal gaps, mu 7, sigma 2):
    dense bucket changes near the diagonal, slow ones far from it, so the
    steady, two-bucket and general element paths all occur (a host simulation
    of the kernel's path choice over these two users: 12% steady, 53%
    two-bucket, 35% general 32 x 32 blocks)."""
    _run(H, [1500, 900], "silu", dtype, P=4096, heads=4, seed=87, gap_kind="lognormal")


def test_attention_backward_rejects_softmax_and_masks(H):
    ac = make_attn_case([10], 1, 64, 32, seed=1, dtype="fp16")
    jag = H.Jagged(tensor(ac.offsets, torch.int64, "cuda"), tensor(ac.timestamps, torch.int64, "cuda"),
                   10, 10)
    q = tensor(ac.q, torch.float16, "cuda")
    rp = tensor(ac.rab_pos, torch.float32, "cuda")
    rt = tensor(ac.rab_time, torch.float32, "cuda")
    cfg = H.LayerConfig(d_model=64, num_heads=1, num_pos_buckets=64, num_time_buckets=32,
                        phi2="softmax", dtype="fp16")
    with pytest.raises(H.HSTUError):
        H.attn_bwd(cfg, jag, q, q, q, q, rp, rt)
