"""Seeded synthetic inputs for the HSTU layer forward and M-FALCON scoring.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no projection, attention, bucketing or normalisation).
Both the float64 oracle and the CUDA path consume exactly the arrays built
here, so any difference between them comes from the arithmetic alone.

Workloads (shapes follow the HSTU paper review, "Actions Speak Louder than
Words", section 三 核心公式 Eq. 1-3 and the M-FALCON paragraph):

  tiny-fp32   1 layer, fp32, d=64, 1 head x 64, 4 users, n_u ~ U{8..64},
              64 position / 32 time buckets
  small-bf16  2 layers, bf16, d=256, 4 heads x 64, 32 users, n_u ~ U{64..512},
              512 / 128 buckets
  sl-bf16     4 layers, bf16, d=512, 8 heads x 64, 64 users; full timeline 4096
              subsampled by Stochastic Length (alpha=1.6), 4096 / 128 buckets
  long-bf16   2 layers, bf16, d=512, 8 heads x 64, 8 users x 8192,
              log-normal gaps (mu=7, sigma=2), 8192 / 128 buckets
  mfalcon     4 layers, bf16, d=512, 8 heads x 64, 16 users x history 4096,
              2048 candidates per user scored in microbatches of 256

Recipe (fixed draw order from one numpy Generator seeded with `seed`):
lengths -> timestamps -> X -> per layer (W1, b1, W2, b2, rab_pos, rab_time)
-> candidates.
  * X, candidate embeddings: standard normal (float32 draws), rounded to the
    workload dtype (bf16 round-to-nearest-even, or kept fp32).
  * W1 [2H(dqk+dv), d] and W2 [d, H*dv] (nn.Linear layout, out x in):
    Xavier-uniform, gain 1, rounded to the workload dtype.
  * b1, b2: U(-1/sqrt(fan_in), 1/sqrt(fan_in)), fp32.
  * rab_pos [H, P], rab_time [H, Tb]: N(0, 0.02^2), fp32.
  * timestamps: int64 seconds, 1.7e9 + floor(cumsum(gaps)); gaps Exp(3600 s)
    except the long workload (LogNormal(7, 2)).
  * Stochastic Length: L = min(n, ceil(n * u^(1/alpha))), u ~ U(0,1); the L
    kept positions are drawn uniformly without replacement and sorted; their
    timestamps are those of the full timeline.
  * M-FALCON request time per user: last history timestamp + floor(Exp(3600)).
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

TS_BASE = 1_700_000_000


@dataclass(frozen=True)
class HSTUConfig:
    name: str
    num_layers: int
    dtype: str  # "bf16" or "fp32": storage type of X and the weight matrices
    d_model: int
    num_heads: int
    dqk: int
    dv: int
    num_pos_buckets: int
    num_time_buckets: int
    batch: int
    len_kind: str  # "uniform" | "fixed" | "sl"
    len_lo: int = 0
    len_hi: int = 0
    full_len: int = 0
    sl_alpha: float = 1.6
    gap_kind: str = "exp"  # "exp" (mean 3600 s) | "lognormal" (mu=7, sigma=2)
    num_cand: int = 0      # candidates per user (M-FALCON only)
    microbatch: int = 0    # b_m (M-FALCON only)
    phi1: str = "relu"
    phi2: str = "silu"
    ln_eps: float = 1e-5

    def replace(self, **kw) -> "HSTUConfig":
        return dataclasses.replace(self, **kw)

    @property
    def n1(self) -> int:
        """Width of the f1 output: U, V (H*dv each), Q, K (H*dqk each)."""
        return 2 * self.num_heads * (self.dqk + self.dv)


CONFIGS = {
    "tiny-fp32": HSTUConfig("tiny-fp32", 1, "fp32", 64, 1, 64, 64, 64, 32, 4,
                            "uniform", 8, 64),
    "small-bf16": HSTUConfig("small-bf16", 2, "bf16", 256, 4, 64, 64, 512, 128, 32,
                             "uniform", 64, 512),
    "sl-bf16": HSTUConfig("sl-bf16", 4, "bf16", 512, 8, 64, 64, 4096, 128, 64,
                          "sl", full_len=4096, sl_alpha=1.6),
    "long-bf16": HSTUConfig("long-bf16", 2, "bf16", 512, 8, 64, 64, 8192, 128, 8,
                            "fixed", full_len=8192, gap_kind="lognormal"),
    "mfalcon": HSTUConfig("mfalcon", 4, "bf16", 512, 8, 64, 64, 4096, 128, 16,
                          "fixed", full_len=4096, num_cand=2048, microbatch=256),
}
CONFIG_ORDER = ["tiny-fp32", "small-bf16", "sl-bf16", "long-bf16", "mfalcon"]
DEFAULT_SEED = {name: i for i, name in enumerate(CONFIG_ORDER)}


@dataclass
class LayerWeights:
    w1: np.ndarray        # [n1, d]   (values representable in the workload dtype)
    b1: np.ndarray        # [n1]      fp32
    w2: np.ndarray        # [d, H*dv]
    b2: np.ndarray        # [d]       fp32
    rab_pos: np.ndarray   # [H, P]    fp32
    rab_time: np.ndarray  # [H, Tb]   fp32
    ln_gamma: Optional[np.ndarray] = None  # [H*dv] fp32 or None (identity)
    ln_beta: Optional[np.ndarray] = None


@dataclass
class Case:
    cfg: HSTUConfig
    seed: int
    offsets: np.ndarray     # [B+1] int64
    timestamps: np.ndarray  # [T] int64
    x: np.ndarray           # [T, d] float32 holding dtype-representable values
    layers: List[LayerWeights]
    # M-FALCON only
    cand_offsets: Optional[np.ndarray] = None  # [B+1] int64
    cand_emb: Optional[np.ndarray] = None      # [M, d] float32
    request_ts: Optional[np.ndarray] = None    # [B] int64
    extra: dict = field(default_factory=dict)

    @property
    def lengths(self) -> np.ndarray:
        return np.diff(self.offsets)

    @property
    def total_tokens(self) -> int:
        return int(self.offsets[-1])

    @property
    def max_len(self) -> int:
        return int(self.lengths.max()) if len(self.lengths) else 0


def round_bf16(a) -> np.ndarray:
    """Round to the nearest bfloat16 (ties to even); returns float32 values."""
    a32 = np.ascontiguousarray(a, dtype=np.float32)
    u = a32.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).reshape(a32.shape)


def round_fp16(a) -> np.ndarray:
    """Round to the nearest IEEE half (ties to even); returns float32 values."""
    return np.asarray(a, dtype=np.float32).astype(np.float16).astype(np.float32)


def to_dtype(a, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return round_bf16(a)
    if dtype == "fp16":
        return round_fp16(a)
    if dtype == "fp32":
        return np.ascontiguousarray(a, dtype=np.float32)
    raise ValueError(dtype)


def stochastic_length(rng: np.random.Generator, n: int, alpha: float) -> int:
    """Stochastic Length draw L = min(n, ceil(n * u^(1/alpha))), u ~ U(0,1)."""
    u = rng.random()
    return int(min(n, max(1, math.ceil(n * u ** (1.0 / alpha)))))


def _gaps(rng, kind: str, size: int) -> np.ndarray:
    if kind == "exp":
        return rng.exponential(3600.0, size)
    if kind == "lognormal":
        return rng.lognormal(7.0, 2.0, size)
    raise ValueError(kind)


def _timeline(rng, kind: str, n: int) -> np.ndarray:
    return TS_BASE + np.floor(np.cumsum(_gaps(rng, kind, n))).astype(np.int64)


def _xavier(rng, fan_out: int, fan_in: int) -> np.ndarray:
    a = math.sqrt(6.0 / (fan_in + fan_out))
    return rng.uniform(-a, a, size=(fan_out, fan_in))


def make_layer(rng, cfg: HSTUConfig) -> LayerWeights:
    d, H = cfg.d_model, cfg.num_heads
    n1, hv = cfg.n1, H * cfg.dv
    w1 = to_dtype(_xavier(rng, n1, d), cfg.dtype)
    b1 = rng.uniform(-1 / math.sqrt(d), 1 / math.sqrt(d), n1).astype(np.float32)
    w2 = to_dtype(_xavier(rng, d, hv), cfg.dtype)
    b2 = rng.uniform(-1 / math.sqrt(hv), 1 / math.sqrt(hv), d).astype(np.float32)
    rab_pos = (rng.standard_normal((H, cfg.num_pos_buckets)) * 0.02).astype(np.float32)
    rab_time = (rng.standard_normal((H, cfg.num_time_buckets)) * 0.02).astype(np.float32)
    return LayerWeights(w1, b1, w2, b2, rab_pos, rab_time)


def make_case(cfg, seed: Optional[int] = None, *, batch: Optional[int] = None,
              lengths: Optional[List[int]] = None, num_layers: Optional[int] = None,
              num_cand: Optional[int] = None, ln_affine: bool = False) -> Case:
    """Build one seeded workload.

    `cfg` is an HSTUConfig or a name from CONFIGS.  `batch`, `lengths`,
    `num_layers` and `num_cand` shrink a workload for tests while keeping its
    shapes and value distributions.  `lengths` fixes the per-user kept lengths
    (for the Stochastic Length workload they are the kept counts of a full
    timeline of `full_len` events).
    """
    if isinstance(cfg, str):
        if seed is None:
            seed = DEFAULT_SEED[cfg]
        cfg = CONFIGS[cfg]
    if seed is None:
        seed = 0
    if num_layers is not None:
        cfg = cfg.replace(num_layers=num_layers)
    if num_cand is not None:
        cfg = cfg.replace(num_cand=num_cand)
    if lengths is not None:
        batch = len(lengths)
    B = cfg.batch if batch is None else batch
    rng = np.random.default_rng(seed)

    # lengths (and, for SL, kept positions)
    kept = None
    if lengths is not None:
        lens = [int(v) for v in lengths]
        if cfg.len_kind == "sl":
            kept = [np.sort(rng.choice(cfg.full_len, L, replace=False)) for L in lens]
    elif cfg.len_kind == "uniform":
        lens = [int(v) for v in rng.integers(cfg.len_lo, cfg.len_hi + 1, B)]
    elif cfg.len_kind == "fixed":
        lens = [cfg.full_len] * B
    elif cfg.len_kind == "sl":
        lens, kept = [], []
        for _ in range(B):
            L = stochastic_length(rng, cfg.full_len, cfg.sl_alpha)
            lens.append(L)
            kept.append(np.sort(rng.choice(cfg.full_len, L, replace=False)))
    else:
        raise ValueError(cfg.len_kind)
    offsets = np.zeros(B + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(lens)
    T = int(offsets[-1])

    # timestamps
    ts = np.empty(T, dtype=np.int64)
    for u in range(B):
        if kept is not None:
            full = _timeline(rng, cfg.gap_kind, cfg.full_len)
            ts[offsets[u]:offsets[u + 1]] = full[kept[u]]
        else:
            ts[offsets[u]:offsets[u + 1]] = _timeline(rng, cfg.gap_kind, lens[u])

    # X
    x = to_dtype(rng.standard_normal((T, cfg.d_model), dtype=np.float32), cfg.dtype)

    layers = [make_layer(rng, cfg) for _ in range(cfg.num_layers)]
    if ln_affine:
        hv = cfg.num_heads * cfg.dv
        for lw in layers:
            lw.ln_gamma = (1.0 + 0.1 * rng.standard_normal(hv)).astype(np.float32)
            lw.ln_beta = (0.1 * rng.standard_normal(hv)).astype(np.float32)

    case = Case(cfg, seed, offsets, ts, x, layers)
    if cfg.num_cand:
        m = cfg.num_cand
        case.cand_offsets = np.arange(B + 1, dtype=np.int64) * m
        case.cand_emb = to_dtype(rng.standard_normal((B * m, cfg.d_model), dtype=np.float32),
                                 cfg.dtype)
        req = np.empty(B, dtype=np.int64)
        for u in range(B):
            last = ts[offsets[u + 1] - 1] if lens[u] > 0 else TS_BASE
            req[u] = last + int(math.floor(rng.exponential(3600.0)))
        case.request_ts = req
    return case


def algorithmic_counts(case: Case) -> dict:
    """Work and byte counts per forward, used to express rates."""
    cfg = case.cfg
    n = case.lengths.astype(np.int64)
    pairs = int((n * (n + 1) // 2).sum())
    H, dqk, dv, d = cfg.num_heads, cfg.dqk, cfg.dv, cfg.d_model
    T = case.total_tokens
    attn_flop = pairs * H * (2 * dqk + 2 * dv)
    f1_flop = 2 * T * d * cfg.n1
    f2_flop = 2 * T * (H * dv) * d
    return {"tokens": T, "causal_pairs": pairs, "attn_flop_per_layer": attn_flop,
            "f1_flop_per_layer": f1_flop, "f2_flop_per_layer": f2_flop,
            "layers": cfg.num_layers}


@dataclass
class AttnCase:
    """Inputs of the attention step alone (Eq. 2): Q, K, V per token and head."""
    offsets: np.ndarray
    timestamps: np.ndarray
    q: np.ndarray         # [T, H*64] float32 holding bf16-representable values
    k: np.ndarray
    v: np.ndarray
    rab_pos: np.ndarray   # [H, P] fp32
    rab_time: np.ndarray  # [H, Tb] fp32
    num_heads: int
    dtype: str


def make_attn_case(lengths: List[int], num_heads: int, P: int, Tb: int, seed: int = 0,
                   dtype: str = "bf16", gap_kind: str = "exp", scale: float = 0.6,
                   rab_std: float = 0.02) -> AttnCase:
    """Q, K, V drawn like the projection's outputs: ReLU-shaped half-normals of std `scale`
    (draw order: timestamps, q, k, v, rab_pos, rab_time)."""
    rng = np.random.default_rng(seed)
    offsets = np.zeros(len(lengths) + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(lengths)
    T = int(offsets[-1])
    ts = np.empty(T, dtype=np.int64)
    for u, n in enumerate(lengths):
        ts[offsets[u]:offsets[u + 1]] = _timeline(rng, gap_kind, n)
    w = num_heads * 64
    q, k, v = (to_dtype(np.maximum(rng.standard_normal((T, w), dtype=np.float32) * scale, 0.0)
                        + 0.05 * rng.standard_normal((T, w), dtype=np.float32), dtype)
               for _ in range(3))
    rp = (rng.standard_normal((num_heads, P)) * rab_std).astype(np.float32)
    rt = (rng.standard_normal((num_heads, Tb)) * rab_std).astype(np.float32)
    return AttnCase(offsets, ts, q, k, v, rp, rt, num_heads, dtype)
