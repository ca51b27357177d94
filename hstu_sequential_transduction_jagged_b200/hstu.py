"""ctypes binding of libhstu (include/hstu.h): argument marshalling only.

Every step of the HSTU layer runs in the CUDA library; this module turns torch
tensors into pointers, sizes and structs, allocates outputs/workspaces with
torch (device memory plumbing only) and raises HSTUError on a non-zero status.
There is no CPU fallback: if libhstu.so is missing, loading raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import List, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhstu.so")

ACT = {"identity": 0, "relu": 1, "silu": 2, "softmax": 3}
DTYPE = {"bf16": 0, "fp32": 1, "fp16": 2}
TORCH_DTYPE = {"bf16": torch.bfloat16, "fp32": torch.float32, "fp16": torch.float16}
# dtype of the per-layer key/value cache of a layer configured with `dtype`
CACHE_DTYPE = {"bf16": torch.float16, "fp32": torch.float32}
STATUS = {0: "HSTU_OK", 1: "HSTU_ERR_INVALID_ARGUMENT", 2: "HSTU_ERR_UNSUPPORTED",
          3: "HSTU_ERR_CUDA", 4: "HSTU_ERR_WORKSPACE_TOO_SMALL", 5: "HSTU_ERR_DEVICE_TIMEOUT",
          6: "HSTU_ERR_DEVICE_CHECK"}


class HSTUError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}")
        self.status = status


class JaggedT(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("total_tokens", ctypes.c_int64),
                ("max_len", ctypes.c_int32), ("offsets", ctypes.c_void_p),
                ("timestamps", ctypes.c_void_p), ("segments", ctypes.c_void_p),
                ("max_static", ctypes.c_int32)]


FLAG_FUSED_F2 = 1


class LayerCfgT(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("num_heads", ctypes.c_int32),
                ("dqk", ctypes.c_int32), ("dv", ctypes.c_int32),
                ("num_pos_buckets", ctypes.c_int32), ("num_time_buckets", ctypes.c_int32),
                ("phi1", ctypes.c_int32), ("phi2", ctypes.c_int32), ("ln_eps", ctypes.c_float),
                ("dtype", ctypes.c_int32), ("flags", ctypes.c_int32)]


class KernelTimeT(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_int32),
                ("total_ms", ctypes.c_double)]


class LayerWeightsT(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("w1", "b1", "w2", "b2", "rab_pos", "rab_time", "ln_gamma", "ln_beta")]


EXPORTS = {
    "hstu_version": (ctypes.c_char_p, []),
    "hstu_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "hstu_layer_workspace_bytes": (ctypes.c_size_t, [ctypes.c_void_p, ctypes.c_int64]),
    "hstu_forward_workspace_bytes": (ctypes.c_size_t,
                                     [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64]),
    "hstu_mfalcon_workspace_bytes": (ctypes.c_size_t, [ctypes.c_void_p, ctypes.c_int64]),
    "hstu_attn_fwd": (ctypes.c_int, [ctypes.c_void_p] * 9 + [ctypes.c_size_t, ctypes.c_void_p]),
    "hstu_attn_fwd_f32": (ctypes.c_int, [ctypes.c_void_p] * 9),
    "hstu_attn_bwd": (ctypes.c_int, [ctypes.c_void_p] * 14),
    "hstu_layer_bwd_workspace_bytes": (ctypes.c_size_t, [ctypes.c_void_p, ctypes.c_int64]),
    "hstu_layer_bwd": (ctypes.c_int, [ctypes.c_void_p] * 8 + [ctypes.c_void_p, ctypes.c_size_t,
                                                              ctypes.c_void_p]),
    "mfalcon_attn_fwd": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int64, ctypes.c_int32]
                         + [ctypes.c_void_p] * 8),
    "hstu_layer_fwd": (ctypes.c_int, [ctypes.c_void_p] * 9 + [ctypes.c_size_t, ctypes.c_void_p]),
    "hstu_layer_fwd_static": (ctypes.c_int, [ctypes.c_void_p] * 9),
    "hstu_forward": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32] + [ctypes.c_void_p] * 6
                     + [ctypes.c_size_t, ctypes.c_void_p]),
    "mfalcon_score": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                     ctypes.c_void_p]),
    "hstu_stochastic_length": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                              ctypes.c_float, ctypes.c_uint64, ctypes.c_uint64]
                               + [ctypes.c_void_p] * 7),
    "hstu_get_device_status": (ctypes.c_int, [ctypes.c_void_p]),
    "hstu_profiler_start": (ctypes.c_int, []),
    "hstu_profiler_stop": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p]),
    "hstu_time_bucket_thresholds": (ctypes.c_int, [ctypes.c_int32, ctypes.c_void_p]),
    "hstu_debug_rab_index": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                            ctypes.c_void_p]),
    "hstu_debug_wait_timeout": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_void_p]),
}

_lib = None


def lib():
    """Load libhstu.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m hstu_sequential_transduction_jagged_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in EXPORTS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise HSTUError(status, where)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


@dataclass
class LayerConfig:
    d_model: int
    num_heads: int
    num_pos_buckets: int
    num_time_buckets: int
    dqk: int = 64
    dv: int = 64
    phi1: str = "relu"
    phi2: str = "silu"
    ln_eps: float = 1e-5
    dtype: str = "bf16"
    fused_f2: bool = False  # True sets HSTU_FLAG_FUSED_F2

    def c(self) -> LayerCfgT:
        return LayerCfgT(self.d_model, self.num_heads, self.dqk, self.dv, self.num_pos_buckets,
                         self.num_time_buckets, ACT[self.phi1], ACT[self.phi2], self.ln_eps,
                         DTYPE[self.dtype], FLAG_FUSED_F2 if self.fused_f2 else 0)

    @property
    def torch_dtype(self):
        return TORCH_DTYPE[self.dtype]

    @property
    def cache_dtype(self):
        """dtype of the K/V cache hstu_layer_fwd / hstu_forward write."""
        return CACHE_DTYPE[self.dtype]

    @property
    def n1(self) -> int:
        return 2 * self.num_heads * (self.dqk + self.dv)


@dataclass
class Jagged:
    offsets: torch.Tensor      # int64 [B+1] on the device
    timestamps: torch.Tensor   # int64 [T] on the device
    max_len: int
    total_tokens: int
    segments: Optional[torch.Tensor] = None  # int32 [B, 2] (n_us, n_r): generalised masks
    max_static: int = 0                      # >= every n_us

    @property
    def batch(self) -> int:
        return self.offsets.numel() - 1

    def c(self) -> JaggedT:
        return JaggedT(self.batch, self.total_tokens, self.max_len, self.offsets.data_ptr(),
                       self.timestamps.data_ptr() if self.timestamps.numel() else None,
                       None if self.segments is None else self.segments.data_ptr(),
                       self.max_static)


@dataclass
class LayerWeights:
    w1: torch.Tensor
    b1: torch.Tensor
    w2: torch.Tensor
    b2: torch.Tensor
    rab_pos: torch.Tensor
    rab_time: torch.Tensor
    ln_gamma: Optional[torch.Tensor] = None
    ln_beta: Optional[torch.Tensor] = None

    def c(self) -> LayerWeightsT:
        def ptr(t):
            return None if t is None else t.data_ptr()
        return LayerWeightsT(ptr(self.w1), ptr(self.b1), ptr(self.w2), ptr(self.b2),
                             ptr(self.rab_pos), ptr(self.rab_time), ptr(self.ln_gamma),
                             ptr(self.ln_beta))


def version() -> str:
    return lib().hstu_version().decode()


def layer_workspace_bytes(cfg: LayerConfig, total_tokens: int) -> int:
    c = cfg.c()
    return lib().hstu_layer_workspace_bytes(ctypes.byref(c), total_tokens)


def forward_workspace_bytes(cfg: LayerConfig, num_layers: int, total_tokens: int) -> int:
    c = cfg.c()
    return lib().hstu_forward_workspace_bytes(ctypes.byref(c), num_layers, total_tokens)


def mfalcon_workspace_bytes(cfg: LayerConfig, num_cand: int) -> int:
    c = cfg.c()
    return lib().hstu_mfalcon_workspace_bytes(ctypes.byref(c), num_cand)


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]):
    if workspace is not None:
        return workspace
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)


def attn_fwd(cfg: LayerConfig, jag: Jagged, q, k, v, rab_pos, rab_time, av_out=None,
             stream=None) -> torch.Tensor:
    """Eq. 2 over a jagged batch: AV[T, H*dv] in cfg dtype."""
    if av_out is None:
        av_out = torch.empty((jag.total_tokens, cfg.num_heads * cfg.dv), dtype=cfg.torch_dtype,
                             device=q.device)
    c, j = cfg.c(), jag.c()
    _check(lib().hstu_attn_fwd(ctypes.byref(c), ctypes.byref(j), _p(q), _p(k), _p(v),
                               _p(rab_pos), _p(rab_time), _p(av_out), None, 0,
                               _stream(stream)), "hstu_attn_fwd")
    return av_out


def attn_fwd_f32(cfg: LayerConfig, jag: Jagged, q, k, v, rab_pos, rab_time, av_out=None,
                 stream=None) -> torch.Tensor:
    """Eq. 2 over a jagged batch with the result in fp32: AV[T, H*dv] float32."""
    if av_out is None:
        av_out = torch.empty((jag.total_tokens, cfg.num_heads * cfg.dv), dtype=torch.float32,
                             device=q.device)
    c, j = cfg.c(), jag.c()
    _check(lib().hstu_attn_fwd_f32(ctypes.byref(c), ctypes.byref(j), _p(q), _p(k), _p(v),
                                   _p(rab_pos), _p(rab_time), _p(av_out), _stream(stream)),
           "hstu_attn_fwd_f32")
    return av_out


def attn_bwd(cfg: LayerConfig, jag: Jagged, q, k, v, d_o, rab_pos, rab_time, stream=None):
    """Backward of the causal attention: returns dq, dk, dv ([T, H*64] fp32) and
    drab_pos [H, P], drab_time [H, Tb] (fp32) for dO = d_o.  dq and the table
    gradients are sums of reductions in no fixed order: their last bits vary
    from run to run."""
    dev = rab_pos.device
    T, hv = jag.total_tokens, cfg.num_heads * cfg.dv
    dq, dk, dv = (torch.empty((max(T, 1), hv), dtype=torch.float32, device=dev) for _ in range(3))
    drp = torch.empty((cfg.num_heads, cfg.num_pos_buckets), dtype=torch.float32, device=dev)
    drt = torch.empty((cfg.num_heads, cfg.num_time_buckets), dtype=torch.float32, device=dev)
    c, j = cfg.c(), jag.c()
    _check(lib().hstu_attn_bwd(ctypes.byref(c), ctypes.byref(j), _p(q), _p(k), _p(v), _p(d_o),
                               _p(rab_pos), _p(rab_time), _p(dq), _p(dk), _p(dv), _p(drp),
                               _p(drt), _stream(stream)), "hstu_attn_bwd")
    return dq[:T], dk[:T], dv[:T], drp, drt


class LayerGradsT(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("dw1", "db1", "dw2", "db2", "drab_pos", "drab_time", "dgamma", "dbeta")]


def layer_bwd_workspace_bytes(cfg: LayerConfig, total_tokens: int) -> int:
    c = cfg.c()
    return int(lib().hstu_layer_bwd_workspace_bytes(ctypes.byref(c), total_tokens))


def layer_bwd(cfg: LayerConfig, w: "LayerWeights", jag: Jagged, x_in, dy, x_res=None,
              workspace=None, stream=None) -> dict:
    """Backward of one bf16 layer for dY = dy ([T, d] fp32): returns a dict with
    dx [T, d] and the parameter gradients (fp32): dw1, db1, dw2, db2, drab_pos,
    drab_time and, when the layer has them, dgamma / dbeta."""
    dev = dy.device
    T, d, hv, n1 = jag.total_tokens, cfg.d_model, cfg.num_heads * cfg.dv, cfg.n1
    f32 = dict(dtype=torch.float32, device=dev)
    out = {"dx": torch.empty((max(T, 1), d), **f32), "dw1": torch.empty((n1, d), **f32),
           "db1": torch.empty(n1, **f32), "dw2": torch.empty((d, hv), **f32),
           "db2": torch.empty(d, **f32),
           "drab_pos": torch.empty((cfg.num_heads, cfg.num_pos_buckets), **f32),
           "drab_time": torch.empty((cfg.num_heads, cfg.num_time_buckets), **f32),
           "dgamma": torch.empty(hv, **f32) if w.ln_gamma is not None else None,
           "dbeta": torch.empty(hv, **f32) if w.ln_beta is not None else None}
    g = LayerGradsT(*[None if out[n] is None else out[n].data_ptr() for n in
                      ("dw1", "db1", "dw2", "db2", "drab_pos", "drab_time", "dgamma", "dbeta")])
    ws = _workspace(layer_bwd_workspace_bytes(cfg, T), dev, workspace)
    c, j, wc = cfg.c(), jag.c(), w.c()
    _check(lib().hstu_layer_bwd(ctypes.byref(c), ctypes.byref(wc), ctypes.byref(j), _p(x_in),
                                _p(x_res), _p(dy), _p(out["dx"]), ctypes.byref(g), _p(ws),
                                ws.numel(), _stream(stream)), "hstu_layer_bwd")
    out["dx"] = out["dx"][:T]
    return out


def mfalcon_attn_fwd(cfg: LayerConfig, history: Jagged, k_hist, v_hist, cand_offsets,
                     max_cand: int, q, k, v, request_ts, rab_pos, rab_time, av_out=None,
                     stream=None) -> torch.Tensor:
    """Candidate-mode attention alone (history keys/values plus self): AV [M, H*dv] fp32."""
    M = q.shape[0]
    if av_out is None:
        av_out = torch.empty((M, cfg.num_heads * cfg.dv), dtype=torch.float32, device=q.device)
    c, j = cfg.c(), history.c()
    _check(lib().mfalcon_attn_fwd(ctypes.byref(c), ctypes.byref(j), _p(k_hist), _p(v_hist),
                                  _p(cand_offsets), M, max_cand, _p(q), _p(k), _p(v),
                                  _p(request_ts), _p(rab_pos), _p(rab_time), _p(av_out),
                                  _stream(stream)), "mfalcon_attn_fwd")
    return av_out


def layer_fwd(cfg: LayerConfig, w: LayerWeights, jag: Jagged, x_in, x_res=None, y_out=None,
              y_out_lp=None, kv_cache_out=None, workspace=None, stream=None) -> torch.Tensor:
    """One HSTU layer; returns the fp32 residual-stream output Y [T, d].  For bf16
    layers x_in may be None when x_res (fp32) is given: f1 then reads x_res
    rounded to fp16."""
    dev = (x_in if x_in is not None else x_res).device
    if y_out is None:
        y_out = torch.empty((jag.total_tokens, cfg.d_model), dtype=torch.float32, device=dev)
    nbytes = layer_workspace_bytes(cfg, jag.total_tokens)
    ws = _workspace(nbytes, dev, workspace)
    c, j, wc = cfg.c(), jag.c(), w.c()
    _check(lib().hstu_layer_fwd(ctypes.byref(c), ctypes.byref(wc), ctypes.byref(j), _p(x_in),
                                _p(x_res), _p(y_out), _p(y_out_lp), _p(kv_cache_out), _p(ws),
                                ws.numel(), _stream(stream)), "hstu_layer_fwd")
    return y_out


STATIC_SCRATCH_BYTES = 64 << 20


def layer_fwd_static(cfg: LayerConfig, w: LayerWeights, jag: Jagged, x_in, x_res=None,
                     y_out=None, y_out_lp=None, kv_cache_out=None, stream=None) -> torch.Tensor:
    """hstu_layer_fwd without a caller workspace: the library's fixed scratch array
    (STATIC_SCRATCH_BYTES per GPU) is used, so the C call itself allocates nothing."""
    if y_out is None:
        y_out = torch.empty((jag.total_tokens, cfg.d_model), dtype=torch.float32,
                            device=(x_in if x_in is not None else x_res).device)
    c, j, wc = cfg.c(), jag.c(), w.c()
    _check(lib().hstu_layer_fwd_static(ctypes.byref(c), ctypes.byref(wc), ctypes.byref(j),
                                       _p(x_in), _p(x_res), _p(y_out), _p(y_out_lp),
                                       _p(kv_cache_out), _stream(stream)),
           "hstu_layer_fwd_static")
    return y_out


def forward(cfg: LayerConfig, weights: Sequence[LayerWeights], jag: Jagged, x_in, y_out=None,
            kv_cache_out=None, workspace=None, stream=None) -> torch.Tensor:
    """A stack of HSTU layers; returns Y [T, d] fp32."""
    dev = x_in.device
    L = len(weights)
    if y_out is None:
        y_out = torch.empty((jag.total_tokens, cfg.d_model), dtype=torch.float32, device=dev)
    ws = _workspace(forward_workspace_bytes(cfg, L, jag.total_tokens), dev, workspace)
    arr = (LayerWeightsT * L)(*[w.c() for w in weights])
    c, j = cfg.c(), jag.c()
    _check(lib().hstu_forward(ctypes.byref(c), L, arr, ctypes.byref(j), _p(x_in), _p(y_out),
                              _p(kv_cache_out), _p(ws), ws.numel(), _stream(stream)),
           "hstu_forward")
    return y_out


def mfalcon_score(cfg: LayerConfig, weights: Sequence[LayerWeights], history: Jagged, kv_cache,
                  cand_offsets, cand_emb, request_ts, microbatch: int, max_cand: int,
                  scores=None, cand_y_out=None, workspace=None, stream=None) -> torch.Tensor:
    """M-FALCON candidate scores [num_cand] fp32.  With `cand_y_out` ([num_cand, d]
    float32) each candidate's final residual-stream row is written there too."""
    dev = cand_emb.device
    M = cand_emb.shape[0]
    L = len(weights)
    if scores is None:
        scores = torch.empty(M, dtype=torch.float32, device=dev)
    ws = _workspace(mfalcon_workspace_bytes(cfg, M), dev, workspace)
    arr = (LayerWeightsT * L)(*[w.c() for w in weights])
    c, j = cfg.c(), history.c()
    _check(lib().mfalcon_score(ctypes.byref(c), L, arr, ctypes.byref(j), _p(kv_cache),
                               _p(cand_offsets), M, max_cand, _p(cand_emb), _p(request_ts),
                               microbatch, _p(scores), _p(cand_y_out), _p(ws), ws.numel(),
                               _stream(stream)),
           "mfalcon_score")
    return scores


def stochastic_length(jag: Jagged, alpha: float, seed: int, step: int, x=None, stream=None):
    """Stochastic Length subsampling on the GPU.  Returns a dict with the output
    offsets [B+1], lengths [B], max_len [1], kept_index [T_full] (first T_out
    valid), timestamps [T_full] and, when x is given, the gathered rows
    [T_full, ...] (first T_out valid).  T_out = offsets[B] stays on the device."""
    dev = jag.offsets.device
    B, T = jag.batch, jag.total_tokens
    out = {"offsets": torch.empty(B + 1, dtype=torch.int64, device=dev),
           "lengths": torch.empty(max(B, 1), dtype=torch.int32, device=dev),
           "max_len": torch.zeros(1, dtype=torch.int32, device=dev),
           "kept_index": torch.empty(max(T, 1), dtype=torch.int64, device=dev),
           "timestamps": torch.empty(max(T, 1), dtype=torch.int64, device=dev)}
    row_bytes = 0
    if x is not None:
        out["x"] = torch.empty((max(T, 1),) + tuple(x.shape[1:]), dtype=x.dtype, device=dev)
        row_bytes = x[0].numel() * x.element_size() if T else 16
    j = jag.c()
    _check(lib().hstu_stochastic_length(ctypes.byref(j), _p(x), row_bytes, alpha, seed, step,
                                        _p(out["offsets"]), _p(out["lengths"]),
                                        _p(out["max_len"]), _p(out["kept_index"]),
                                        _p(out["timestamps"]), _p(out.get("x")),
                                        _stream(stream)), "hstu_stochastic_length")
    return out


def device_status(stream=None) -> int:
    """Synchronise, read and clear the library's device status word."""
    return lib().hstu_get_device_status(_stream(stream))


def time_bucket_thresholds(num_time_buckets: int):
    import numpy as np
    out = np.zeros(num_time_buckets, dtype=np.int64)
    _check(lib().hstu_time_bucket_thresholds(num_time_buckets,
                                             out.ctypes.data_as(ctypes.c_void_p)),
           "hstu_time_bucket_thresholds")
    return out


def debug_rab_index(jag: Jagged, num_pos_buckets: int, num_time_buckets: int, stream=None):
    """Per-user n x n blocks of (position bucket, time bucket), -1 above the diagonal."""
    lens = (jag.offsets[1:] - jag.offsets[:-1]).to(torch.int64)
    blk = torch.zeros(jag.batch + 1, dtype=torch.int64, device=jag.offsets.device)
    blk[1:] = torch.cumsum(lens * lens, 0)
    total = int(blk[-1].item())
    pos = torch.full((max(total, 1),), -7, dtype=torch.int32, device=jag.offsets.device)
    tim = torch.full((max(total, 1),), -7, dtype=torch.int32, device=jag.offsets.device)
    j = jag.c()
    _check(lib().hstu_debug_rab_index(ctypes.byref(j), num_pos_buckets, num_time_buckets,
                                      _p(blk), _p(pos), _p(tim), _stream(stream)),
           "hstu_debug_rab_index")
    return blk, pos[:total], tim[:total]


def debug_wait_timeout(timeout_ns: int, stream=None):
    _check(lib().hstu_debug_wait_timeout(timeout_ns, _stream(stream)), "hstu_debug_wait_timeout")


def profiler_start():
    """Start bracketing every library kernel launch with CUDA events."""
    _check(lib().hstu_profiler_start(), "hstu_profiler_start")


def profiler_stop() -> dict:
    """Stop the profiler; returns {kernel name: (launches, total milliseconds)}."""
    arr = (KernelTimeT * 16)()
    n = ctypes.c_int32(0)
    _check(lib().hstu_profiler_stop(arr, 16, ctypes.byref(n)), "hstu_profiler_stop")
    return {arr[i].name.decode(): (arr[i].launches, arr[i].total_ms) for i in range(n.value)}
