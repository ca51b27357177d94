"""Generalised (MTGR-style) masks on the GPU against the float64 oracle.

Dynamic Masking of MTGR (RecSysChannel digest of "MTGR: Industrial-Scale
Generative Recommendation Framework in Meituan"): a user's tokens are U+S
(profile and long history), R (short history) and candidates; U+S keys are
visible to every row and U+S rows see U+S in both directions, R rows are
causal, a candidate sees U+S, the R events at or before its own timestamp and
itself.  The kernels take (n_us, n_r) per user."""
import numpy as np
import pytest
import torch

from gen import make_case
from gen.device import case_tensors, tensor
from gen.inputs import make_attn_case
from oracle import hstu as O
from hstu_testutil import assert_close, binding, config_of

pytestmark = pytest.mark.gpu

# (n, n_us, n_r): U+S across a 256-row tile pair, all U+S, all candidates,
# no R, plain causal, one token
SEGMENTS = [(300, 40, 200), (700, 300, 250), (129, 0, 129), (64, 64, 0), (500, 0, 0),
            (257, 10, 0), (1, 0, 0), (900, 120, 600)]


@pytest.fixture(scope="module")
def H():
    return binding()


def _candidate_times(ts, offsets, segs, rng):
    """Candidates get timestamps inside (or around) their user's R span, so each
    sees only part of R; U+S and R stay time-ordered."""
    ts = ts.copy()
    for u, (n, n_us, n_r) in enumerate(segs):
        s = int(offsets[u])
        c0 = s + n_us + n_r
        if n - n_us - n_r == 0:
            continue
        lo = ts[s + n_us] if n_r else ts[s] if n else 0
        hi = ts[c0 - 1] if n_us + n_r else lo
        ts[c0:s + n] = rng.integers(lo - 5000, hi + 5000, s + n - c0)
    return ts


def _segments_tensor(segs):
    return tensor(np.array([[a, b] for _, a, b in segs], dtype=np.int32), torch.int32, "cuda")


@pytest.mark.parametrize("phi2,dtype", [("silu", "fp16"), ("softmax", "fp16"), ("relu", "fp16"),
                                        ("silu", "bf16"), ("softmax", "bf16")])
def test_masked_attention(H, phi2, dtype):
    heads, P, Tb = 2, 512, 128
    lens = [n for n, _, _ in SEGMENTS]
    ac = make_attn_case(lens, heads, P, Tb, seed=61, dtype=dtype)
    rng = np.random.default_rng(62)
    ts = _candidate_times(ac.timestamps, ac.offsets, SEGMENTS, rng)
    jag = H.Jagged(tensor(ac.offsets, torch.int64, "cuda"), tensor(ts, torch.int64, "cuda"),
                   max(lens), int(ac.offsets[-1]), _segments_tensor(SEGMENTS),
                   max(a for _, a, _ in SEGMENTS))
    tdt = H.TORCH_DTYPE[dtype]
    q, k, v = (tensor(a, tdt, "cuda") for a in (ac.q, ac.k, ac.v))
    cfg = H.LayerConfig(d_model=128, num_heads=heads, num_pos_buckets=P, num_time_buckets=Tb,
                        phi2=phi2, dtype=dtype)
    av = H.attn_fwd_f32(cfg, jag, q, k, v, tensor(ac.rab_pos, torch.float32, "cuda"),
                        tensor(ac.rab_time, torch.float32, "cuda")).cpu().numpy()
    assert H.device_status() == 0
    for u, (n, n_us, n_r) in enumerate(SEGMENTS):
        s, e = int(ac.offsets[u]), int(ac.offsets[u + 1])
        mask = O.segment_mask(ts[s:e], n_us, n_r)
        want = O.user_attention(ac.q[s:e].astype(np.float64), ac.k[s:e].astype(np.float64),
                                ac.v[s:e].astype(np.float64), ts[s:e],
                                ac.rab_pos.astype(np.float64), ac.rab_time.astype(np.float64),
                                n, heads, 64, 64, phi2, mask)
        assert_close(av[s:e], want, f"masked user {u} {(n, n_us, n_r)} {phi2} {dtype}",
                     scaled=True)


def _masked_forward(H, case, segs):
    rng = np.random.default_rng(63)
    ts = _candidate_times(case.timestamps, case.offsets,
                          [(int(n), a, b) for n, (a, b) in zip(case.lengths, segs)], rng)
    case.timestamps = ts
    t = case_tensors(case, "cuda")
    seg_t = tensor(np.array(segs, dtype=np.int32), torch.int32, "cuda")
    jag = H.Jagged(t["offsets"], t["timestamps"], case.max_len, case.total_tokens, seg_t,
                   max(a for a, _ in segs))
    weights = [H.LayerWeights(**lw) for lw in t["layers"]]
    y = H.forward(config_of(H, case.cfg), weights, jag, t["x"]).cpu().numpy()
    assert H.device_status() == 0
    want, _ = O.forward(case.x, case.offsets, ts, case.layers, case.cfg, segments=segs)
    return y, want


@pytest.mark.parametrize("phi2", ["silu", "softmax"])
def test_masked_forward_small(H, phi2):
    cfg = make_case("small-bf16").cfg.replace(phi2=phi2)
    case = make_case(cfg, seed=64, lengths=[300, 700, 129, 64, 500])
    segs = [[40, 200], [300, 250], [0, 129], [64, 0], [0, 0]]
    y, want = _masked_forward(H, case, segs)
    assert_close(y, want, f"masked forward small-bf16 {phi2}")


def test_masked_forward_sl_shapes(H):
    """d 512, 8 heads, 4 layers."""
    case = make_case("sl-bf16", seed=65, lengths=[1500, 300, 2600])
    segs = [[200, 1000], [0, 250], [900, 1500]]
    y, want = _masked_forward(H, case, segs)
    assert_close(y, want, "masked forward sl-bf16")


def test_masked_forward_fp32(H):
    case = make_case("tiny-fp32", seed=66, lengths=[40, 64, 9, 30])
    segs = [[5, 20], [0, 0], [9, 0], [3, 27]]
    y, want = _masked_forward(H, case, segs)
    assert_close(y, want, "masked forward tiny-fp32")


def test_inconsistent_segments_are_reported(H):
    """n_us + n_r beyond the user's length is a device-side check failure."""
    lens = [100, 50]
    offs = tensor(np.array([0, 100, 150], dtype=np.int64), torch.int64, "cuda")
    ts = tensor(1_700_000_000 + np.arange(150, dtype=np.int64) * 60, torch.int64, "cuda")
    seg = tensor(np.array([[30, 80], [0, 50]], dtype=np.int32), torch.int32, "cuda")
    jag = H.Jagged(offs, ts, 100, 150, seg, 30)
    x = torch.zeros((150, 64), dtype=torch.float16, device="cuda")
    cfg = H.LayerConfig(d_model=64, num_heads=1, num_pos_buckets=128, num_time_buckets=64,
                        dtype="fp16")
    rp = torch.zeros((1, 128), dtype=torch.float32, device="cuda")
    rt = torch.zeros((1, 64), dtype=torch.float32, device="cuda")
    assert H.device_status() == 0
    H.attn_fwd_f32(cfg, jag, x, x, x, rp, rt)
    assert H.device_status() == 6
