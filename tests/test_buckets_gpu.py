"""Bit-exact check of the position and time buckets the attention kernels use.

The relative attention bias rab^{p,t} of Eq. 2 (review of "Actions Speak
Louder than Words", section 三 核心公式) is gathered inside the attention
kernel from integer bucket indices: position min(i - j, P - 1) and time
floor(ln(t_i - t_j + 1) / 0.301) clamped to [0, Tb - 1].  These tests make the
attention result an exact integer function of those indices, so the indices
the production kernel picks (its one-bucket fast path, its two-bucket edge
compare and its per-key octave table) are compared index for index with the
float64 oracle:

  * Q = 0, so S = Q K^T = 0 exactly, and phi2 is the identity or ReLU (with
    non-negative biases both give P = rab exactly; the values are small
    integers, exact in fp16 and bf16).  The operands are fp16 -- the kernel
    the bf16 layers run -- unless a test names bf16;
  * V is one-hot by key residue: V[j, c] = 1 iff j mod 64 == c, so
    AV[i, c] * n_u = sum over keys j <= i with j = c (mod 64) of rab_ij, an
    integer below 2^24, which fp32 accumulation and the 1/n_u scale keep to
    well under 0.5;
  * head 0 carries the bucket index itself (rab_time[0, b] = b, or
    rab_pos[0, x] = x mod 97) and every other head a threshold indicator
    (rab[h, b] = 1 iff b >= k_h).  Bucket indices never increase along a row
    (keys are time-ordered), so for each threshold k the set of keys with
    bucket >= k is a prefix of the row; its 64 residue counts fix where that
    prefix ends, and with thresholds across the range every bucket edge of
    every row is pinned.

The expected integers come from the oracle's own bucket functions
(oracle.hstu.time_bucket / pos_bucket) evaluated on every visible pair."""
import numpy as np
import pytest
import torch

from gen import make_case
from gen.device import tensor
from oracle import hstu as O
from hstu_testutil import binding

pytestmark = pytest.mark.gpu

TS0 = 1_700_000_000


@pytest.fixture(scope="module")
def H():
    return binding()


# ------------------------------------------------------------------ expected sums (oracle)

def _time_sums(ts, Tb, ks, blk=512):
    """[n, 1 + len(ks), 64] integer sums per row and key residue: head 0 the
    time bucket index, head 1+t the indicator bucket >= ks[t]; keys j <= i."""
    n = len(ts)
    out = np.zeros((n, 1 + len(ks), 64), dtype=np.int64)
    for r0 in range(0, n, blk):
        r1 = min(n, r0 + blk)
        kmax = (r1 + 63) // 64 * 64
        tsk = np.concatenate([ts, np.zeros(max(0, kmax - n), np.int64)])[:kmax]
        i = np.arange(r0, r1)
        vis = np.arange(kmax)[None, :] <= i[:, None]
        b = np.where(vis, O.time_bucket(ts[i][:, None] - tsk[None, :], Tb), 0)
        out[r0:r1, 0] = b.reshape(r1 - r0, kmax // 64, 64).sum(1)
        for t, k in enumerate(ks):
            out[r0:r1, 1 + t] = ((b >= k) & vis).reshape(r1 - r0, kmax // 64, 64).sum(1)
    return out


def _pos_fn(P, ks):
    """Per head, the position-bias value of bucket x: x mod 97, then indicators x >= k."""
    x = np.arange(P)
    return np.stack([x % 97] + [(x >= k).astype(np.int64) for k in ks])


def _pos_sums(n, P, ks):
    """[n, 1 + len(ks), 64]: sums over keys j <= i (residue c = j mod 64) of
    f_h(pos_bucket(i - j)).  The bias depends on d = i - j only, so the sum
    runs over d = r, r + 64, ... <= i with r = (i - c) mod 64: prefix sums of
    f_h(pos_bucket(d)) along each residue class of d."""
    f = _pos_fn(P, ks)
    m = (n + 63) // 64
    d = np.arange(m * 64)
    g = f[:, O.pos_bucket(d, P)]                         # [heads, m*64]
    G = np.cumsum(g.reshape(f.shape[0], m, 64), axis=1)  # G[h, t, r] = sum_{t'<=t} g(r + 64 t')
    i = np.arange(n)[:, None]
    c = np.arange(64)[None, :]
    r = (i - c) % 64
    t = (i - r) // 64                                    # number of terms - 1 (when i >= r)
    ok = i >= r
    out = np.zeros((n, f.shape[0], 64), dtype=np.int64)
    for h in range(f.shape[0]):
        out[:, h] = np.where(ok, G[h, np.maximum(t, 0), r], 0)
    return out


# ------------------------------------------------------------------ device inputs

def _onehot_v(offsets, heads):
    T = int(offsets[-1])
    rel = np.zeros(T, dtype=np.int64)
    for u in range(len(offsets) - 1):
        rel[offsets[u]:offsets[u + 1]] = np.arange(offsets[u + 1] - offsets[u])
    v = np.zeros((T, 64), dtype=np.float32)
    v[np.arange(T), rel % 64] = 1.0
    return np.tile(v, (1, heads))


def _run_causal(H, ts_users, P, Tb, rab_pos, rab_time, phi2, dtype="fp16"):
    heads = rab_pos.shape[0]
    lens = [len(t) for t in ts_users]
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T = int(offs[-1])
    ts = np.concatenate(ts_users).astype(np.int64)
    jag = H.Jagged(tensor(offs, torch.int64, "cuda"), tensor(ts, torch.int64, "cuda"),
                   max(lens), T)
    tdt = H.TORCH_DTYPE[dtype]
    q = torch.zeros((T, heads * 64), dtype=tdt, device="cuda")
    k = torch.zeros_like(q)
    v = tensor(_onehot_v(offs, heads), tdt, "cuda")
    cfg = H.LayerConfig(d_model=64, num_heads=heads, num_pos_buckets=P, num_time_buckets=Tb,
                        phi2=phi2, dtype=dtype)
    av = H.attn_fwd_f32(cfg, jag, q, k, v, tensor(rab_pos, torch.float32, "cuda"),
                        tensor(rab_time, torch.float32, "cuda"))
    assert H.device_status() == 0
    return offs, av.cpu().numpy().reshape(T, heads, 64).astype(np.float64)


def _as_integers(av_rows, n, what):
    x = av_rows * n
    r = np.rint(x)
    assert np.max(np.abs(x - r)) < 0.25, f"{what}: not integer sums"
    return r.astype(np.int64)


def _time_tables(heads, Tb, ks):
    rt = np.zeros((heads, Tb), dtype=np.float32)
    rt[0] = np.arange(Tb)
    for h, k in enumerate(ks, start=1):
        rt[h] = (np.arange(Tb) >= k).astype(np.float32)
    return rt


def _check_time(H, ts_users, Tb, ks, phi2, P=8192, dtype="fp16"):
    heads = 1 + len(ks)
    rt = _time_tables(heads, Tb, ks)
    rp = np.zeros((heads, P), dtype=np.float32)
    offs, av = _run_causal(H, ts_users, P, Tb, rp, rt, phi2, dtype)
    for u, ts in enumerate(ts_users):
        n = len(ts)
        if n == 0:
            continue
        got = _as_integers(av[offs[u]:offs[u + 1]], n, f"user {u}")
        want = _time_sums(ts, Tb, ks)
        bad = np.argwhere(got != want)
        assert bad.size == 0, f"user {u} (n={n}, Tb={Tb}, phi2={phi2}, {dtype}): first mismatch " \
                              f"(row, head, residue) {tuple(bad[0])}"


def _check_pos(H, lens, P, ks, phi2, Tb=128, dtype="fp16"):
    heads = 1 + len(ks)
    rp = _pos_fn(P, ks).astype(np.float32)
    rt = np.zeros((heads, Tb), dtype=np.float32)
    rng = np.random.default_rng(11)
    ts_users = [TS0 + np.floor(np.cumsum(rng.exponential(3600, n))).astype(np.int64)
                for n in lens]
    offs, av = _run_causal(H, ts_users, P, Tb, rp, rt, phi2, dtype)
    for u, n in enumerate(lens):
        if n == 0:
            continue
        got = _as_integers(av[offs[u]:offs[u + 1]], n, f"user {u}")
        want = _pos_sums(n, P, ks)
        bad = np.argwhere(got != want)
        assert bad.size == 0, f"user {u} (n={n}, P={P}): first mismatch {tuple(bad[0])}"


# ------------------------------------------------------------------ causal kernel

@pytest.mark.parametrize("phi2,dtype", [("identity", "fp16"), ("relu", "fp16"),
                                        ("identity", "bf16")])
def test_time_buckets_long_lognormal_timeline(H, phi2, dtype):
    """The long-sequence workload's timelines (8 users x 8192, log-normal gaps,
    Tb 128): every (row, key) time bucket of the kernel equals the oracle's."""
    case = make_case("long-bf16", num_layers=1)
    ts_users = [case.timestamps[case.offsets[u]:case.offsets[u + 1]] for u in range(case.cfg.batch)]
    _check_time(H, ts_users, 128, [2, 10, 25, 40, 50, 56, 60], phi2, dtype=dtype)


@pytest.mark.parametrize("Tb", [32, 128])
def test_time_buckets_exponential_gaps_and_clamp(H, Tb):
    """Exp(3600 s) gaps (the other workloads' timelines); Tb = 32 clamps every
    gap beyond about 3 hours into the last bucket."""
    rng = np.random.default_rng(12)
    lens = [3000, 1, 700, 129, 0, 64]
    ts_users = [TS0 + np.floor(np.cumsum(rng.exponential(3600, n))).astype(np.int64)
                for n in lens]
    ks = [1, 5, 12, 20, 27, 30, 31] if Tb == 32 else [1, 8, 16, 24, 30, 36, 45]
    _check_time(H, ts_users, Tb, ks, "relu")


def test_time_buckets_equal_timestamp_runs(H):
    """Runs of equal timestamps (dt = 0, bucket 0) mixed with bursts of short
    gaps and long jumps, so warps see many bucket changes per 32-key chunk."""
    rng = np.random.default_rng(13)
    ts_users = []
    for n in (2500, 640, 333):
        gaps = np.where(rng.random(n) < 0.6, 0, np.floor(rng.lognormal(2.0, 3.0, n)))
        ts_users.append(TS0 + np.cumsum(gaps).astype(np.int64))
    _check_time(H, ts_users, 128, [1, 3, 6, 12, 24, 40, 60], "identity")


def test_time_buckets_bucket_edges(H):
    """A timeline whose differences from the first event hit every bucket edge
    thr[k] - 1 and thr[k] (the smallest gaps of each bucket)."""
    thr = O.time_bucket_thresholds(128)
    rel = sorted(set([0] + [int(t) for k in range(1, 62) for t in (thr[k] - 1, thr[k])]))
    ts_users = [TS0 + np.array(rel, dtype=np.int64)]
    _check_time(H, ts_users, 128, [1, 2, 3, 10, 30, 50, 61], "identity")


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_position_buckets_paired_table(H, dtype):
    """Position buckets on the paired (two staggered copies) table path."""
    _check_pos(H, [8192, 1, 700, 2049], 8192, [1, 2, 63, 64, 1000, 4095, 8191], "identity",
               dtype=dtype)


def test_position_buckets_clamped(H):
    """P smaller than the sequence: min(i - j, P - 1) clamps."""
    _check_pos(H, [3000, 450], 300, [1, 2, 64, 150, 298, 299, 300], "relu")


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_position_buckets_longest_sequence(H, dtype):
    """One user at the longest supported length (16384).  With bf16 operands
    the fp32 position table no longer fits twice in shared memory and the
    single-copy path runs; the fp16 table (fp16 operands) still fits twice."""
    _check_pos(H, [16384], 16384, [1, 2, 63, 4096, 9000, 16000, 16383], "identity", dtype=dtype)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_time_buckets_longest_sequence(H, dtype):
    rng = np.random.default_rng(14)
    ts_users = [TS0 + np.floor(np.cumsum(rng.lognormal(7.0, 2.0, 16384))).astype(np.int64)]
    _check_time(H, ts_users, 128, [2, 10, 25, 40, 50, 56, 60], "identity", P=16384, dtype=dtype)


# ------------------------------------------------------------------ candidate mode (M-FALCON)

def _cand_case(rng, hist_lens, cand_lens):
    ts_users = [TS0 + np.floor(np.cumsum(rng.lognormal(7.0, 2.0, n))).astype(np.int64)
                for n in hist_lens]
    req = np.array([(t[-1] if len(t) else TS0) + int(rng.exponential(3600)) for t in ts_users],
                   dtype=np.int64)
    return ts_users, req


def _run_cand(H, ts_users, req, cand_lens, P, Tb, rab_pos, rab_time, dtype="fp16"):
    heads = rab_pos.shape[0]
    hl = [len(t) for t in ts_users]
    hoffs = np.concatenate([[0], np.cumsum(hl)]).astype(np.int64)
    coffs = np.concatenate([[0], np.cumsum(cand_lens)]).astype(np.int64)
    T, M = int(hoffs[-1]), int(coffs[-1])
    ts = np.concatenate(ts_users).astype(np.int64)
    jag = H.Jagged(tensor(hoffs, torch.int64, "cuda"), tensor(ts, torch.int64, "cuda"),
                   max(hl), T)
    tdt = H.TORCH_DTYPE[dtype]
    kh = torch.zeros((max(T, 1), heads * 64), dtype=tdt, device="cuda")
    vh = tensor(_onehot_v(hoffs, heads), tdt, "cuda")
    q = torch.zeros((M, heads * 64), dtype=tdt, device="cuda")
    k = torch.zeros_like(q)
    v = torch.zeros_like(q)  # the self term adds nothing
    cfg = H.LayerConfig(d_model=64, num_heads=heads, num_pos_buckets=P, num_time_buckets=Tb,
                        phi2="identity", dtype=dtype)
    av = H.mfalcon_attn_fwd(cfg, jag, kh, vh, tensor(coffs, torch.int64, "cuda"),
                            max(cand_lens), q, k, v, tensor(req, torch.int64, "cuda"),
                            tensor(rab_pos, torch.float32, "cuda"),
                            tensor(rab_time, torch.float32, "cuda"))
    assert H.device_status() == 0
    return coffs, av.cpu().numpy().reshape(M, heads, 64).astype(np.float64)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_candidate_mode_buckets(H, dtype):
    """Candidate rows sit at position n_u with time t_req: their bucket against
    history key j is min(n_u - j, P - 1) and bt(t_req - t_j)."""
    rng = np.random.default_rng(15)
    hist, cands = [4096, 0, 1000, 77], [256, 3, 100, 513]
    ts_users, req = _cand_case(rng, hist, cands)
    Tb, P = 128, 4096
    ks_t = [2, 10, 25, 40, 50, 56, 60]
    ks_p = [1, 2, 63, 64, 999, 2048, 4095]
    heads = 8
    rt = _time_tables(heads, Tb, ks_t)
    coffs, av_t = _run_cand(H, ts_users, req, cands, P, Tb,
                            np.zeros((heads, P), np.float32), rt, dtype)
    rp = _pos_fn(P, ks_p).astype(np.float32)
    _, av_p = _run_cand(H, ts_users, req, cands, P, Tb, rp, np.zeros((heads, Tb), np.float32),
                        dtype)
    fp = _pos_fn(P, ks_p)
    for u, n in enumerate(hist):
        rows = slice(coffs[u], coffs[u + 1])
        m = cands[u]
        j = np.arange(n)
        pad = (n + 63) // 64 * 64
        b = np.zeros(pad, dtype=np.int64)
        b[:n] = O.time_bucket(req[u] - ts_users[u], Tb)
        vis = np.zeros(pad, dtype=bool)
        vis[:n] = True
        want_t = np.stack([b.reshape(-1, 64).sum(0)]
                          + [((b >= k) & vis).reshape(-1, 64).sum(0) for k in ks_t])
        bp = np.zeros(pad, dtype=np.int64)
        bp[:n] = O.pos_bucket(n - j, P)
        want_p = np.stack([np.where(vis, fp[h][bp], 0).reshape(-1, 64).sum(0)
                           for h in range(heads)])
        nn = max(n, 1)
        got_t = _as_integers(av_t[rows], nn, f"user {u} time")
        got_p = _as_integers(av_p[rows], nn, f"user {u} position")
        assert np.array_equal(got_t, np.broadcast_to(want_t, (m,) + want_t.shape)), f"user {u} time"
        assert np.array_equal(got_p, np.broadcast_to(want_p, (m,) + want_p.shape)), f"user {u} pos"


# ------------------------------------------------------------------ declared lengths

def test_understated_max_len_is_reported(H):
    """A user longer than the declared max_len is reported as a device-side
    check failure (the launch is sized from max_len) instead of being read or
    written out of range.  Understated by only 3 tokens."""
    lens = [300, 130]
    offs = np.array([0, 300, 430], dtype=np.int64)
    ts = TS0 + np.arange(430, dtype=np.int64) * 60
    jag = H.Jagged(tensor(offs, torch.int64, "cuda"), tensor(ts, torch.int64, "cuda"), 297, 430)
    x = torch.zeros((430, 64), dtype=torch.bfloat16, device="cuda")
    cfg = H.LayerConfig(d_model=64, num_heads=1, num_pos_buckets=512, num_time_buckets=128)
    rp = torch.zeros((1, 512), dtype=torch.float32, device="cuda")
    rt = torch.zeros((1, 128), dtype=torch.float32, device="cuda")
    assert H.device_status() == 0
    H.attn_fwd_f32(cfg, jag, x, x, x, rp, rt)
    assert H.device_status() == 6  # HSTU_ERR_DEVICE_CHECK
    # candidate mode: history and candidate counts understated by 2
    coffs = tensor(np.array([0, 40, 90], dtype=np.int64), torch.int64, "cuda")
    qc = torch.zeros((90, 64), dtype=torch.bfloat16, device="cuda")
    req = tensor(np.array([ts[299] + 5, ts[429] + 5], dtype=np.int64), torch.int64, "cuda")
    jag_h = H.Jagged(jag.offsets, jag.timestamps, 298, 430)
    H.mfalcon_attn_fwd(cfg, jag_h, x, x, coffs, 50, qc, qc, qc, req, rp, rt)
    assert H.device_status() == 6
    jag_ok = H.Jagged(jag.offsets, jag.timestamps, 300, 430)
    H.mfalcon_attn_fwd(cfg, jag_ok, x, x, coffs, 48, qc, qc, qc, req, rp, rt)
    assert H.device_status() == 6
    H.mfalcon_attn_fwd(cfg, jag_ok, x, x, coffs, 50, qc, qc, qc, req, rp, rt)
    assert H.device_status() == 0
