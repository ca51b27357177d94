"""GPU parity: the CUDA path through the C ABI against the float64 oracle on the
same seeded inputs (bf16 tolerance: max abs <= 2e-2, relative L2 <= 5e-3;
bucket indices bit-exact)."""
import numpy as np
import pytest
import torch

from gen import make_case, round_bf16, round_fp16, to_dtype
from gen.device import tensor
from gen.inputs import make_attn_case
from oracle import hstu as O
from hstu_testutil import (assert_close, binding, check_scores, config_of, errors, record, upload,
                           upload_attn)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    return binding()


def _status_ok(H):
    assert H.device_status() == 0


# ------------------------------------------------------------------ bucket indices

def test_rab_index_bit_exact(H):
    Tb, P = 128, 64
    thr = O.time_bucket_thresholds(Tb)
    # user 0 walks every bucket edge: differences thr[k]-1 and thr[k] from its first event
    rel = sorted(set([0] + [int(t) for k in range(1, 60) for t in (thr[k] - 1, thr[k])]))
    u0 = 1_700_000_000 + np.array(rel, dtype=np.int64)
    rng = np.random.default_rng(3)
    u1 = 1_700_000_000 + np.floor(np.cumsum(rng.exponential(3600, 300))).astype(np.int64)
    u2 = np.full(5, 1_700_000_000, dtype=np.int64)  # equal timestamps
    u3 = 1_700_000_000 + np.floor(np.cumsum(rng.lognormal(7, 2, 200))).astype(np.int64)
    users = [u0, u1, u2, np.zeros(0, np.int64), u3]
    ts = np.concatenate(users)
    offs = np.concatenate([[0], np.cumsum([len(u) for u in users])]).astype(np.int64)
    jag = H.Jagged(torch.from_numpy(offs).cuda(), torch.from_numpy(ts).cuda(),
                   max(len(u) for u in users), int(offs[-1]))
    blk, pos, tim = H.debug_rab_index(jag, P, Tb)
    pos, tim, blk = pos.cpu().numpy(), tim.cpu().numpy(), blk.cpu().numpy()
    for u, t in enumerate(users):
        n = len(t)
        if n == 0:
            continue
        i, j = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
        low = j <= i
        want_p = np.where(low, O.pos_bucket(i - j, P), -1)
        want_t = np.where(low, O.time_bucket(t[i] - t[j], Tb), -1)
        got_p = pos[blk[u]:blk[u + 1]].reshape(n, n)
        got_t = tim[blk[u]:blk[u + 1]].reshape(n, n)
        assert np.array_equal(got_p, want_p), f"user {u} position buckets"
        assert np.array_equal(got_t, want_t), f"user {u} time buckets"
    _status_ok(H)


# ------------------------------------------------------------------ attention alone

ATTN_LENGTHS = [1, 127, 128, 129, 255, 256, 257, 700, 0, 64]


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("phi2", ["silu", "relu", "identity", "softmax"])
def test_attention_parity(H, phi2, dtype):
    """Attention alone for both operand types: fp16 is what the bf16 layers run
    (f1 writes fp16 Q, K, V), bf16 serves bf16 inputs given directly."""
    P, Tb, heads = 512, 128, 2
    ac = make_attn_case(ATTN_LENGTHS, heads, P, Tb, seed=5, dtype=dtype)
    cfg = H.LayerConfig(d_model=128, num_heads=heads, num_pos_buckets=P, num_time_buckets=Tb,
                        phi2=phi2, dtype=dtype)
    jag, q, k, v, rp, rt = upload_attn(H, ac)
    av = H.attn_fwd(cfg, jag, q, k, v, rp, rt).float().cpu().numpy()
    _status_ok(H)
    for u in range(len(ATTN_LENGTHS)):
        s, e = ac.offsets[u], ac.offsets[u + 1]
        if e == s:
            continue
        want = O.user_attention(ac.q[s:e].astype(np.float64), ac.k[s:e].astype(np.float64),
                                ac.v[s:e].astype(np.float64), ac.timestamps[s:e],
                                ac.rab_pos.astype(np.float64), ac.rab_time.astype(np.float64),
                                e - s, heads, 64, 64, phi2)
        assert_close(av[s:e], want, f"user {u} (n={e - s}) phi2={phi2} {dtype}", scaled=True)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_attention_position_clamp_and_large_bias(H, dtype):
    """P smaller than the sequence (clamped position buckets) and a bias large
    enough that a wrong gather is visible."""
    P, Tb, heads = 48, 16, 1
    ac = make_attn_case([300, 5, 190], heads, P, Tb, seed=8, rab_std=0.5, dtype=dtype)
    cfg = H.LayerConfig(d_model=64, num_heads=heads, num_pos_buckets=P, num_time_buckets=Tb,
                        dtype=dtype)
    jag, q, k, v, rp, rt = upload_attn(H, ac)
    av = H.attn_fwd(cfg, jag, q, k, v, rp, rt).float().cpu().numpy()
    for u in range(3):
        s, e = ac.offsets[u], ac.offsets[u + 1]
        want = O.user_attention(ac.q[s:e].astype(np.float64), ac.k[s:e].astype(np.float64),
                                ac.v[s:e].astype(np.float64), ac.timestamps[s:e],
                                ac.rab_pos.astype(np.float64), ac.rab_time.astype(np.float64),
                                e - s, heads, 64, 64, "silu")
        assert_close(av[s:e], want, f"user {u}", scaled=True)


# ------------------------------------------------------------------ whole layers

def _forward_check(H, case, what, check_delta=True):
    """Whole stack at the stated bound: max abs <= 2e-2 and rel-L2 <= 5e-3
    against the float64 oracle, plus the layer delta Y - X on its own."""
    t, jag, weights = upload(H, case)
    cfg = config_of(H, case.cfg)
    y = H.forward(cfg, weights, jag, t["x"]).cpu().numpy()
    _status_ok(H)
    want, _ = O.forward(case.x, case.offsets, case.timestamps, case.layers, case.cfg)
    ma, rl = assert_close(y, want, what)
    if check_delta:
        # the change Y - X on its own, so the residual cannot hide errors
        x = case.x.astype(np.float64)
        dma, drl = errors(y - x, want - x)
        record(f"{what} delta", dma, drl, None, 2e-2)
        assert drl <= 2e-2, f"{what} delta: max_abs={dma:.3e} rel_l2={drl:.3e}"
    return ma, rl


def _per_layer_check(H, case, what):
    """Every layer on its own at the stated tolerance (max-abs 2e-2, rel-L2 5e-3):
    layer l gets the oracle's layer l-1 output as its fp32 residual input, and
    f1 reads it rounded to fp16 (x_in = None), the way the GPU's own previous
    layer hands it over inside a stack."""
    t, jag, weights = upload(H, case)
    cfg = config_of(H, case.cfg)
    cur = case.x.astype(np.float64)
    for l, lw in enumerate(case.layers):
        want = O.layer_fwd(cur, case.offsets, case.timestamps, lw, case.cfg, keep_stages=False)["y"]
        if l == 0:
            x_in, x_res = t["x"], None
        else:
            x_res = tensor(cur.astype(np.float32), torch.float32, "cuda")
            x_in = None if case.cfg.dtype == "bf16" else x_res
        y = H.layer_fwd(cfg, weights[l], jag, x_in, x_res=x_res).cpu().numpy()
        _status_ok(H)
        assert_close(y, want, f"{what} layer {l}")
        cur = want


def test_tiny_fp32_full_workload(H):
    case = make_case("tiny-fp32")
    _forward_check(H, case, "tiny-fp32")


def test_small_bf16_ragged(H):
    case = make_case("small-bf16", seed=21, lengths=[1, 64, 129, 300, 512, 257, 0, 128])
    _forward_check(H, case, "small-bf16 ragged")


def test_small_bf16_full_workload(H):
    case = make_case("small-bf16")
    _forward_check(H, case, "small-bf16 full")


@pytest.mark.parametrize("phi2", ["relu", "identity", "softmax"])
def test_small_bf16_other_phi2(H, phi2):
    cfg = make_case("small-bf16").cfg.replace(phi2=phi2)
    case = make_case(cfg, seed=22, lengths=[200, 33, 400])
    _forward_check(H, case, f"small-bf16 phi2={phi2}")


def test_softmax_ablation_without_rab(H):
    """The "HSTU (-rab, Softmax)" ablation: softmax phi2 with zero bias tables,
    whole 2-layer stack and each layer at the stated bound."""
    cfg = make_case("small-bf16").cfg.replace(phi2="softmax")
    case = make_case(cfg, seed=28, lengths=[300, 1, 129, 512, 64])
    for lw in case.layers:
        lw.rab_pos[:] = 0.0
        lw.rab_time[:] = 0.0
    _forward_check(H, case, "softmax -rab")
    _per_layer_check(H, case, "softmax -rab")


def test_softmax_sl_bf16_per_layer(H):
    """Softmax ablation on the Stochastic Length shapes (d 512, 8 heads, 4 layers)."""
    cfg = make_case("sl-bf16").cfg.replace(phi2="softmax")
    case = make_case(cfg, seed=29, lengths=[1, 300, 1100, 2500])
    _forward_check(H, case, "softmax sl-bf16")
    _per_layer_check(H, case, "softmax sl-bf16")


def test_softmax_tiny_fp32(H):
    case = make_case(make_case("tiny-fp32").cfg.replace(phi2="softmax"), seed=30)
    _forward_check(H, case, "softmax tiny-fp32")


def test_layernorm_affine(H):
    case = make_case("small-bf16", seed=23, lengths=[150, 270], num_layers=1, ln_affine=True)
    _forward_check(H, case, "affine LayerNorm")


def test_sl_bf16_reduced(H):
    case = make_case("sl-bf16", seed=24, lengths=[1, 300, 1100, 4096])
    _forward_check(H, case, "sl-bf16 reduced")


def test_sl_bf16_reduced_per_layer(H):
    case = make_case("sl-bf16", seed=24, lengths=[1, 300, 1100, 4096])
    _per_layer_check(H, case, "sl-bf16 reduced")


def test_small_bf16_full_per_layer(H):
    _per_layer_check(H, make_case("small-bf16"), "small-bf16 full")


@pytest.mark.parametrize("d_model", [64, 320, 768])
def test_model_widths(H, d_model):
    """f2's tiles cover up to 512 output columns in two 256-column halves: widths
    that use one half (64), a partly filled second half (320), or a second
    column group (768); two layers, so the bf16 copy of Y feeds the next f1."""
    cfg = make_case("small-bf16").cfg.replace(d_model=d_model, num_heads=2)
    case = make_case(cfg, seed=26, lengths=[70, 300, 5], num_layers=2)
    _forward_check(H, case, f"d_model={d_model}")


def test_single_layer_kv_cache_and_lp_copy(H):
    case = make_case("small-bf16", seed=25, lengths=[100, 260], num_layers=1)
    t, jag, weights = upload(H, case)
    cfg = config_of(H, case.cfg)
    T, d, hv = case.total_tokens, case.cfg.d_model, case.cfg.num_heads * 64
    kv = torch.zeros((T, 2 * hv), dtype=cfg.cache_dtype, device="cuda")
    ylp = torch.zeros((T, d), dtype=torch.bfloat16, device="cuda")
    y = H.layer_fwd(cfg, weights[0], jag, t["x"], y_out_lp=ylp, kv_cache_out=kv)
    want = O.layer_fwd(case.x, case.offsets, case.timestamps, case.layers[0], case.cfg)
    assert_close(y.cpu().numpy(), want["y"], "y")
    assert_close(kv[:, :hv].float().cpu().numpy(), want["k"], "cached K", scaled=True)
    assert_close(kv[:, hv:].float().cpu().numpy(), want["v"], "cached V", scaled=True)
    assert torch.equal(ylp, y.to(torch.bfloat16))


# ------------------------------------------------------------------ structural invariants on GPU

def test_per_user_independence_bit_exact(H):
    case = make_case("small-bf16", seed=26, lengths=[300, 77, 512, 129])
    t, jag, weights = upload(H, case)
    cfg = config_of(H, case.cfg)
    y0 = H.forward(cfg, weights, jag, t["x"]).cpu()
    perm = [2, 0, 3, 1]
    segs = [(int(case.offsets[u]), int(case.offsets[u + 1])) for u in range(4)]
    idx = np.concatenate([np.arange(*segs[p]) for p in perm])
    lens = [segs[p][1] - segs[p][0] for p in perm]
    offs = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int64, device="cuda")
    jag2 = H.Jagged(offs, t["timestamps"][torch.from_numpy(idx).cuda()], jag.max_len,
                    jag.total_tokens)
    y1 = H.forward(cfg, weights, jag2, t["x"][torch.from_numpy(idx).cuda()]).cpu()
    assert torch.equal(y1, y0[torch.from_numpy(idx)])


def test_causality_bit_exact(H):
    case = make_case("small-bf16", seed=27, lengths=[400, 200])
    t, jag, weights = upload(H, case)
    cfg = config_of(H, case.cfg)
    y0 = H.forward(cfg, weights, jag, t["x"]).cpu()
    x2 = t["x"].clone()
    x2[251:400] += 3.0
    ts2 = t["timestamps"].clone()
    ts2[251:400] += 99999
    jag2 = H.Jagged(jag.offsets, ts2, jag.max_len, jag.total_tokens)
    y1 = H.forward(cfg, weights, jag2, x2).cpu()
    assert torch.equal(y1[:251], y0[:251])
    assert torch.equal(y1[400:], y0[400:])
    assert not torch.equal(y1[251:400], y0[251:400])


# ------------------------------------------------------------------ M-FALCON

def _mfalcon_case(seed, lengths, m, layers=2):
    cfg = make_case("mfalcon").cfg.replace(num_cand=m)
    return make_case(cfg, seed=seed, lengths=lengths, num_layers=layers)


def _mfalcon_run(H, case, microbatch, rows=False):
    t, jag, weights = upload(H, case)
    cfg = config_of(H, case.cfg)
    L, T, hv = case.cfg.num_layers, case.total_tokens, case.cfg.num_heads * 64
    kv = torch.empty((L, max(T, 1), 2 * hv), dtype=cfg.cache_dtype, device="cuda")
    H.forward(cfg, weights, jag, t["x"], kv_cache_out=kv)
    y = None
    if rows:
        y = torch.empty((case.cand_emb.shape[0], case.cfg.d_model), dtype=torch.float32,
                        device="cuda")
    sc = H.mfalcon_score(cfg, weights, jag, kv, t["cand_offsets"], t["cand_emb"],
                         t["request_ts"], microbatch, case.cfg.num_cand, cand_y_out=y)
    if rows:
        return sc.cpu().numpy(), y.cpu().numpy()
    return sc.cpu().numpy(), t, jag, weights, kv


def test_mfalcon_parity(H):
    """Whole 2-layer M-FALCON pass: each candidate's final row y_c element by
    element, and the scores on the part the layers add (s_c - <e_c, e_c>)."""
    case = _mfalcon_case(31, [300, 0, 129, 1000], m=150)
    sc, y = _mfalcon_run(H, case, 64, rows=True)
    _status_ok(H)
    want, want_y = O.mfalcon_scores(case.x, case.offsets, case.timestamps, case.layers, case.cfg,
                                    case.cand_offsets, case.cand_emb, case.request_ts, 64,
                                    return_rows=True)
    L = case.cfg.num_layers
    assert_close(y, want_y, "mfalcon final rows")
    e = case.cand_emb.astype(np.float64)
    dma, drl = errors(y - e, want_y - e)
    record("mfalcon final rows delta y-e", dma, drl, None, 2e-2)
    assert drl <= 2e-2, f"delta rel_l2={drl:.3e}"
    check_scores(sc, want, case.cand_emb, "mfalcon scores")


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_mfalcon_softmax(H, dtype):
    """M-FALCON with the softmax ablation: a candidate's softmax runs over its
    user's history keys and its own key."""
    cfg = make_case("mfalcon").cfg.replace(num_cand=70, phi2="softmax")
    if dtype == "fp32":
        cfg = cfg.replace(dtype="fp32", d_model=64, num_heads=1)
    case = make_case(cfg, seed=34, lengths=[300, 0, 129, 700], num_layers=2)
    sc, y = _mfalcon_run(H, case, 32, rows=True)
    _status_ok(H)
    want, want_y = O.mfalcon_scores(case.x, case.offsets, case.timestamps, case.layers, case.cfg,
                                    case.cand_offsets, case.cand_emb, case.request_ts, 32,
                                    return_rows=True)
    assert_close(y, want_y, f"mfalcon softmax {dtype} final rows")
    check_scores(sc, want, case.cand_emb, f"mfalcon softmax {dtype} scores")


def test_mfalcon_per_layer(H):
    """Every M-FALCON layer on its own at the stated bound (max abs 2e-2,
    rel-L2 5e-3): layer l gets the oracle's layer l-1 candidate rows and the
    oracle's layer-l history keys/values, rounded to bf16 (rows) and fp16 (the
    cache's type) and given to both sides, so differences come from the GPU
    arithmetic of that layer."""
    case = _mfalcon_case(33, [300, 0, 129, 1000], m=150, layers=4)
    t, jag, weights = upload(H, case)
    cfg = config_of(H, case.cfg)
    T, hv, d = case.total_tokens, case.cfg.num_heads * 64, case.cfg.d_model
    _, ks, vs = O.history_kv(case.x, case.offsets, case.timestamps, case.layers, case.cfg)
    cur = case.cand_emb.astype(np.float64)
    M = cur.shape[0]
    for l, lw in enumerate(case.layers):
        xt = round_bf16(cur)
        kt, vt = round_fp16(ks[l]), round_fp16(vs[l])  # the cache holds fp16
        want_s, want_y = O.mfalcon_scores(None, case.offsets, case.timestamps, [lw], case.cfg,
                                          case.cand_offsets, xt, case.request_ts, 64,
                                          kv=([kt], [vt]), return_rows=True)
        kv = tensor(np.concatenate([kt, vt], axis=1)[None], cfg.cache_dtype, "cuda")
        y = torch.empty((M, d), dtype=torch.float32, device="cuda")
        sc = H.mfalcon_score(cfg, [weights[l]], jag, kv, t["cand_offsets"],
                             tensor(xt, torch.bfloat16, "cuda"), t["request_ts"], 64,
                             case.cfg.num_cand, cand_y_out=y)
        _status_ok(H)
        yn = y.cpu().numpy()
        assert_close(yn, want_y, f"mfalcon layer {l} rows")
        assert_close(yn - xt, want_y - xt, f"mfalcon layer {l} delta", max_abs=2e-2, rel_l2=2e-2)
        check_scores(sc.cpu().numpy(), want_s, xt, f"mfalcon layer {l} scores")
        cur = want_y


def test_mfalcon_microbatch_and_permutation_invariance(H):
    case = _mfalcon_case(32, [200, 333], m=130)
    a, *_ = _mfalcon_run(H, case, 1)
    b, *_ = _mfalcon_run(H, case, 256)
    assert np.array_equal(a, b)
    m = case.cfg.num_cand
    perm = np.arange(2 * m)
    perm[:m] = perm[:m][::-1]
    case2 = _mfalcon_case(32, [200, 333], m=130)
    case2.cand_emb = case.cand_emb[perm]
    c, *_ = _mfalcon_run(H, case2, 7)
    assert np.array_equal(c, a[perm])


# ------------------------------------------------------------------ failure reporting

def test_bounded_wait_reports_timeout(H):
    assert H.device_status() == 0
    H.debug_wait_timeout(2_000_000)  # 2 ms
    assert H.device_status() == 5
    assert H.device_status() == 0  # reading clears it


def test_unsupported_shape_is_rejected(H):
    cfg = H.LayerConfig(d_model=256, num_heads=4, num_pos_buckets=512, num_time_buckets=128,
                        dqk=32, dv=32)
    x = torch.zeros(4, 128, dtype=torch.bfloat16, device="cuda")
    jag = H.Jagged(torch.tensor([0, 4], device="cuda"), torch.zeros(4, dtype=torch.int64,
                                                                    device="cuda"), 4, 4)
    with pytest.raises(H.HSTUError) as e:
        H.attn_fwd(cfg, jag, x, x, x, x, x)
    assert e.value.status == 2
