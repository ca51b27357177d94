"""Backward of one HSTU layer on the GPU (hstu_layer_bwd) against the float64
backward oracle (oracle/hstu_bwd.py, pinned by finite differences of the
forward oracle).

Tolerance (gradients have no stated bound of their own): per gradient tensor,
rel-L2 <= 5e-3 and max |err| <= 2e-2 * max |ref|: the forward's bound on the
gradient's own scale.  The GPU recomputes the forward with its bf16/fp16
kernels and runs the weight-gradient GEMMs in TF32."""
import dataclasses

import numpy as np
import pytest
import torch

from gen import make_case, round_fp16
from gen.device import tensor
from oracle import hstu as O
from oracle import hstu_bwd as OB
from hstu_testutil import binding, config_of, record, upload

pytestmark = pytest.mark.gpu

REL, ABS = 5e-3, 2e-2
NAMES = ("dx", "dw1", "db1", "dw2", "db2", "drab_pos", "drab_time", "dgamma", "dbeta")


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


def _compare(H, case, what, layer=0, x_res_input=False, seed=91):
    t, jag, weights = upload(H, case)
    cfg = config_of(H, case.cfg)
    lw = case.layers[layer]
    rng = np.random.default_rng(seed)
    dy = rng.standard_normal((case.total_tokens, case.cfg.d_model)).astype(np.float32)
    if x_res_input:
        # a layer deeper in the stack: fp32 input (the oracle's previous output)
        x = O.layer_fwd(case.x, case.offsets, case.timestamps, case.layers[0], case.cfg,
                        keep_stages=False)["y"].astype(np.float32)
        x_in, x_res = None, tensor(x, torch.float32, "cuda")
    else:
        x = case.x
        x_in, x_res = t["x"], None
    got = H.layer_bwd(cfg, weights[layer], jag, x_in, tensor(dy, torch.float32, "cuda"), x_res=x_res)
    torch.cuda.synchronize()
    assert H.device_status() == 0
    # with an fp32 input the GPU's f1 reads it rounded to fp16 (x_in = NULL):
    # the oracle takes the same f1 input, since ReLU' turns the rounding of
    # near-zero pre-activations into whole gradient entries
    want = OB.layer_bwd(np.asarray(x, np.float64), case.offsets, case.timestamps, lw, case.cfg,
                        dy.astype(np.float64),
                        x_f1=round_fp16(x).astype(np.float64) if x_res_input else None)
    for name in NAMES:
        if want[name] is None:
            assert got[name] is None
            continue
        _check(got[name].cpu().numpy(), want[name], f"{what} {name}")


def test_layer_backward_small(H):
    case = make_case("small-bf16", seed=92, lengths=[1, 100, 129, 300, 0, 257], num_layers=1)
    _compare(H, case, "layer bwd small-bf16")


def test_layer_backward_d512_affine(H):
    case = make_case("sl-bf16", seed=93, lengths=[700, 130, 1], num_layers=1, ln_affine=True)
    _compare(H, case, "layer bwd d512 affine LN")


def test_layer_backward_fp32_input(H):
    case = make_case("small-bf16", seed=94, lengths=[200, 333], num_layers=2)
    _compare(H, case, "layer bwd fp32 input", layer=1, x_res_input=True)


@pytest.mark.parametrize("phi1,phi2", [("identity", "silu"), ("relu", "relu"), ("relu", "identity")])
def test_layer_backward_other_activations(H, phi1, phi2):
    cfg = make_case("small-bf16").cfg.replace(phi1=phi1, phi2=phi2, num_layers=1)
    case = make_case(cfg, seed=95, lengths=[150, 64, 400])
    _compare(H, case, f"layer bwd phi1={phi1} phi2={phi2}")


def test_layer_backward_rejects_unsupported(H):
    cfg = make_case("small-bf16").cfg.replace(phi2="softmax", num_layers=1)
    case = make_case(cfg, seed=96, lengths=[10])
    t, jag, weights = upload(H, case)
    dy = torch.zeros((case.total_tokens, case.cfg.d_model), dtype=torch.float32, device="cuda")
    with pytest.raises(H.HSTUError):
        H.layer_bwd(config_of(H, case.cfg), weights[0], jag, t["x"], dy)


def test_two_layer_chain(H):
    """The training step's chain: backward through layer 1, then through layer 0
    with the dX of one as the dY of the other; every gradient of both layers
    and the input gradient against the oracle chained the same way.  Layer 1
    takes the oracle's layer-0 output (fp32) on both sides: f1 reads it rounded
    to fp16, and an input that differed by the forward's own rounding would
    flip ReLU' on near-zero pre-activations (whole gradient entries), which a
    chained forward on each side would compare rather than the backward."""
    case = make_case("sl-bf16", seed=97, lengths=[600, 129, 1], num_layers=2)
    t, jag, weights = upload(H, case)
    cfg = config_of(H, case.cfg)
    rng = np.random.default_rng(98)
    dy = rng.standard_normal((case.total_tokens, case.cfg.d_model)).astype(np.float32)
    y0_ref = O.layer_fwd(case.x, case.offsets, case.timestamps, case.layers[0], case.cfg,
                         keep_stages=False)["y"].astype(np.float32)
    g1 = H.layer_bwd(cfg, weights[1], jag, None, tensor(dy, torch.float32, "cuda"),
                     x_res=tensor(y0_ref, torch.float32, "cuda"))
    g0 = H.layer_bwd(cfg, weights[0], jag, t["x"], g1["dx"])
    torch.cuda.synchronize()
    assert H.device_status() == 0
    w1 = OB.layer_bwd(y0_ref.astype(np.float64), case.offsets, case.timestamps, case.layers[1],
                      case.cfg, dy.astype(np.float64),
                      x_f1=round_fp16(y0_ref).astype(np.float64))
    w0 = OB.layer_bwd(case.x, case.offsets, case.timestamps, case.layers[0], case.cfg, w1["dx"])
    for tag, got, want in (("layer 1", g1, w1), ("layer 0", g0, w0)):
        for name in NAMES:
            if want[name] is None:
                continue
            _check(got[name].cpu().numpy(), want[name], f"two-layer chain {tag} {name}")
