"""The layer-fused attention -> Norm(AV) (.) U -> f2 -> residual path against the
float64 oracle and against f2 run as its own kernel.

Review of "Actions Speak Louder than Words" (xllm-io paper review), section 三
核心公式 Eq. 3: Y = f2(Norm(A(X)V(X)) (.) U(X)) with the residual between
layers.  With HSTU_FLAG_FUSED_F2 the causal bf16 layer runs f2 inside the
attention kernel: the last of a query tile pair's head CTAs computes the pair's
256 rows of Y.  Both forms take the same fp16 operands and the same MMA order,
so they are compared bit for bit, and each against the oracle at the stated
bound."""
import dataclasses

import numpy as np
import pytest
import torch

from gen import make_case
from gen.device import tensor
from oracle import hstu as O
from hstu_testutil import assert_close, binding, config_of, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    return binding()


def _layer(H, case, l, cur, fused, with_lp=False):
    t, jag, weights = upload(H, case)
    cfg = dataclasses.replace(config_of(H, case.cfg), fused_f2=fused)
    if l == 0:
        x_in, x_res = t["x"], None
    else:
        x_res = tensor(cur.astype(np.float32), torch.float32, "cuda")
        x_in = None
    lp = None
    if with_lp:
        lp = torch.empty((case.total_tokens, case.cfg.d_model), dtype=torch.bfloat16, device="cuda")
    y = H.layer_fwd(cfg, weights[l], jag, x_in, x_res=x_res, y_out_lp=lp)
    torch.cuda.synchronize()
    assert H.device_status() == 0
    return y.cpu().numpy(), (lp.float().cpu().numpy() if lp is not None else None)


def _both_forms(H, case, what):
    cur = case.x.astype(np.float64)
    for l, lw in enumerate(case.layers):
        want = O.layer_fwd(cur, case.offsets, case.timestamps, lw, case.cfg, keep_stages=False)["y"]
        yf, lpf = _layer(H, case, l, cur, True, with_lp=True)
        yu, lpu = _layer(H, case, l, cur, False, with_lp=True)
        assert_close(yf, want, f"{what} fused layer {l}")
        assert_close(yu, want, f"{what} unfused layer {l}")
        assert np.array_equal(yf, yu), \
            f"{what} layer {l}: fused and unfused differ by {np.abs(yf - yu).max():.3e}"
        assert np.array_equal(lpf, lpu), f"{what} layer {l}: 16-bit copies differ"
        cur = want


# ragged lengths: one row, a partial first tile, exactly one and two tiles,
# a partial second tile of a pair, several pairs
LENGTHS = [1, 100, 128, 129, 255, 256, 257, 700, 0, 1000]


@pytest.mark.parametrize("phi2", ["silu", "softmax"])
def test_fused_matches_oracle_and_unfused_d512(H, phi2):
    cfg = make_case("sl-bf16").cfg.replace(phi2=phi2, num_layers=2)
    case = make_case(cfg, seed=71, lengths=LENGTHS)
    _both_forms(H, case, f"d512 {phi2}")


def test_fused_small_width(H):
    """d 256, 4 heads: one 256-column half, four K blocks."""
    case = make_case("small-bf16", seed=72, lengths=LENGTHS)
    _both_forms(H, case, "small-bf16")


@pytest.mark.parametrize("d,heads", [(64, 1), (320, 5), (512, 2)])
def test_fused_odd_widths(H, d, heads):
    """N below one box (64), N over one half (320: 256 + 64), K below N (512 x 128)."""
    cfg = make_case("small-bf16").cfg.replace(d_model=d, num_heads=heads, num_layers=1)
    case = make_case(cfg, seed=73, lengths=[300, 57, 513])
    _both_forms(H, case, f"d{d} h{heads}")


def test_fused_with_affine_layernorm(H):
    case = make_case("small-bf16", seed=74, lengths=[400, 90], ln_affine=True)
    _both_forms(H, case, "affine LN")


def test_fused_forward_stack(H):
    """hstu_forward (fp16 copies between layers) with the fused layers, at the bound."""
    case = make_case("sl-bf16", seed=76, lengths=[1500, 3, 640, 2049])
    t, jag, weights = upload(H, case)
    cfg = dataclasses.replace(config_of(H, case.cfg), fused_f2=True)
    y = H.forward(cfg, weights, jag, t["x"]).cpu().numpy()
    assert H.device_status() == 0
    want, _ = O.forward(case.x, case.offsets, case.timestamps, case.layers, case.cfg)
    assert_close(y, want, "fused forward sl-bf16 stack")
