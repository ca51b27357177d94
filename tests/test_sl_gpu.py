"""GPU Stochastic Length sampler against the oracle (review section 三,
Stochastic Length): lengths, kept rows, timestamps and gathered rows are
integer / copy work and must match bit for bit.  The sampler's output then
feeds the layer forward, which is checked against the oracle on the
subsampled batch."""
import numpy as np
import pytest
import torch

from gen import make_case
from gen.device import case_tensors, tensor
from oracle import hstu as O
from oracle import sl as S
from hstu_testutil import assert_close, binding, config_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    return binding()


def _jagged(H, lens, seed=0, d=16):
    rng = np.random.default_rng(seed)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T = int(offs[-1])
    ts = 1_700_000_000 + np.cumsum(rng.integers(0, 5000, T)).astype(np.int64)
    x = rng.standard_normal((T, d)).astype(np.float32)
    jag = H.Jagged(tensor(offs, torch.int64, "cuda"), tensor(ts, torch.int64, "cuda"),
                   max(lens) if lens else 0, T)
    return offs, ts, x, jag


def _check(H, lens, alpha, seed, step):
    offs, ts, x, jag = _jagged(H, lens, seed=seed)
    xd = tensor(x, torch.float32, "cuda")
    out = H.stochastic_length(jag, alpha, seed, step, x=xd)
    assert H.device_status() == 0
    want_offs, want_ts, want_x, want_kept = S.stochastic_length(offs, ts, x, alpha, seed, step)
    got_offs = out["offsets"].cpu().numpy()
    assert np.array_equal(got_offs, want_offs)
    T_out = int(got_offs[-1])
    assert np.array_equal(out["lengths"].cpu().numpy()[:len(lens)], np.diff(want_offs))
    assert int(out["max_len"].item()) == (int(np.diff(want_offs).max()) if len(lens) else 0)
    assert np.array_equal(out["kept_index"].cpu().numpy()[:T_out], want_kept)
    assert np.array_equal(out["timestamps"].cpu().numpy()[:T_out], want_ts)
    assert np.array_equal(out["x"].cpu().numpy()[:T_out], want_x)


@pytest.mark.parametrize("alpha,seed,step", [(1.6, 7, 0), (1.6, 7, 1), (1.9, 123, 5), (1.0, 2, 9)])
def test_sampler_bit_exact(H, alpha, seed, step):
    _check(H, [0, 1, 2, 17, 600, 4096, 513, 0, 3000], alpha, seed, step)


def test_sampler_longest_users(H):
    _check(H, [16384, 16383, 1], 1.6, 99, 3)


def test_sampler_many_users(H):
    """The sl-bf16 shape: 64 users with full timelines of 4096 events."""
    _check(H, [4096] * 64, 1.6, 2024, 11)


def test_sampler_then_forward(H):
    """Subsample a full-timeline batch on the GPU, then run the 4-layer forward
    on it: parity with the oracle's forward of the oracle's subsample."""
    cfg0 = make_case("sl-bf16").cfg
    full = make_case(cfg0.replace(len_kind="fixed", full_len=1500), seed=51, batch=6,
                     num_layers=2)
    t = case_tensors(full, "cuda")
    jag = H.Jagged(t["offsets"], t["timestamps"], full.max_len, full.total_tokens)
    out = H.stochastic_length(jag, 1.6, 5, 0, x=t["x"])
    offs = out["offsets"]
    T_out, max_len = int(offs[-1].item()), int(out["max_len"].item())
    jag2 = H.Jagged(offs, out["timestamps"][:T_out].contiguous(), max_len, T_out)
    weights = [H.LayerWeights(**lw) for lw in t["layers"]]
    cfg = config_of(H, full.cfg)
    y = H.forward(cfg, weights, jag2, out["x"][:T_out].contiguous()).cpu().numpy()
    assert H.device_status() == 0
    w_offs, w_ts, w_x, _ = S.stochastic_length(full.offsets, full.timestamps, full.x, 1.6, 5, 0)
    want, _ = O.forward(w_x, w_offs, w_ts, full.layers, full.cfg)
    assert_close(y, want, "forward after the GPU sampler")
