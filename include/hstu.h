/*
 * hstu.h -- C ABI of libhstu, a B200 (sm_100a) implementation of the forward
 * pass of the HSTU layer (Hierarchical Sequential Transduction Unit) and of
 * M-FALCON candidate scoring.
 *
 * Source of the method: the review of "Actions Speak Louder than Words:
 * Trillion-Parameter Sequential Transducers for Generative Recommendations"
 * (xllm-io paper-review of arXiv 2402.17152), section 三 技术架构 / 核心公式:
 *   Eq. 1  U, V, Q, K = Split(phi1(f1(X)))            f_i(X) = W_i X + b_i, phi1 = ReLU
 *   Eq. 2  A(X)V(X)   = phi2(Q K^T + rab^{p,t}) V(X)  pointwise attention, no softmax
 *   Eq. 3  Y(X)       = f2(Norm(A(X)V(X)) (.) U(X))   plus the residual between layers
 * and the M-FALCON paragraph of the same section (microbatched candidates
 * reusing cached history keys/values).
 *
 * Readings fixed by this library where the pages are silent:
 *   - phi2 is selectable (SiLU by default; ReLU; identity); attention weights
 *     are divided by N = n_u, the user's own length (candidates: max(n_u, 1));
 *   - no 1/sqrt(d) scale; rab is added before phi2; the causal mask zeroes
 *     weights of later keys after phi2;
 *   - rab_ij = rab_pos[h, min(i-j, P-1)] + rab_time[h, bt(t_i - t_j)],
 *     bt(dt) = clamp(floor(ln(dt + 1) / 0.301), 0, Tb-1), dt < 0 -> 0;
 *   - Norm = LayerNorm over the H*dv concatenated heads of a token, biased
 *     variance, eps from the config, optional affine;
 *   - Y = X + f2(...): the residual stream is fp32.
 *   - bf16 layers compute attention on fp16 Q, K, V and P (f1 writes them in
 *     fp16; values saturate at +-65504), with fp32 accumulation, and f2 on
 *     fp16 operands (Norm(AV) (.) U, and an fp16 copy of W2 made in the
 *     workspace each call).  Inside hstu_forward and mfalcon_score the layers
 *     after the first take an fp16 copy of the fp32 residual stream, with an
 *     fp16 copy of W1.  fp16 runs at the bf16 tensor-core rate with 8x finer
 *     rounding; bf16 weights convert to fp16 exactly inside fp16's normal
 *     range.
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" must point to memory of the current CUDA
 *     device; the caller owns every buffer.  The library never allocates
 *     device memory inside a call and keeps no per-call state.
 *   - All device work is enqueued on `stream` (a cudaStream_t passed as void*,
 *     NULL = legacy default stream) and is asynchronous to the host.
 *   - Argument errors are detected on the host before any launch and return
 *     HSTU_ERR_INVALID_ARGUMENT or HSTU_ERR_UNSUPPORTED without touching
 *     device memory.  A failed launch returns HSTU_ERR_CUDA.  A kernel that
 *     gives up on a bounded wait records HSTU_ERR_DEVICE_TIMEOUT in the
 *     device status word (read with hstu_get_device_status); no kernel traps.
 *   - Layouts are row-major.  Jagged batches: user u owns rows
 *     offsets[u] .. offsets[u+1]-1 of every per-token tensor.
 *   - Timestamps are int64 seconds, non-decreasing inside each user (the
 *     result is unspecified otherwise).
 *   - Supported shapes: dqk = dv = 64; d_model a multiple of 64;
 *     1 <= num_heads with num_heads*64 a multiple of 64; max_len <= 16384;
 *     num_pos_buckets <= 16384; num_time_buckets <= 256.  bf16 and fp32
 *     storage (fp32 runs the fp32 SIMT path, bf16 the tensor-core path).
 */
#ifndef HSTU_H_
#define HSTU_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HSTU_OK = 0,
  HSTU_ERR_INVALID_ARGUMENT = 1,   /* NULL pointer, negative size, inconsistent shapes */
  HSTU_ERR_UNSUPPORTED = 2,        /* valid request outside the supported shapes */
  HSTU_ERR_CUDA = 3,               /* a CUDA runtime call or launch failed */
  HSTU_ERR_WORKSPACE_TOO_SMALL = 4,/* ws_bytes < hstu_*_workspace_bytes(...) */
  HSTU_ERR_DEVICE_TIMEOUT = 5,     /* a kernel gave up on a bounded wait */
  HSTU_ERR_DEVICE_CHECK = 6        /* a device-side input check failed */
} hstu_status_t;

/* Storage types.  Layers run in bf16 (tensor cores) or fp32 (SIMT); FP16 is
 * accepted by the attention-only entry points (hstu_attn_fwd*,
 * mfalcon_attn_fwd) for fp16 Q, K, V, the operand type the bf16 layers use
 * for their attention internally. */
typedef enum { HSTU_BF16 = 0, HSTU_FP32 = 1, HSTU_FP16 = 2 } hstu_dtype_t;

/* Pointwise nonlinearities.  HSTU_ACT_SOFTMAX is accepted for phi2 only: the
 * "HSTU (-rab, Softmax)" ablation of the review's section 六 (HSTU component
 * ablation table), a row-wise softmax over the visible keys of the same
 * pre-activation Q K^T + rab, replacing phi2 and its 1/N (pass zero bias
 * tables for "-rab"). */
typedef enum {
  HSTU_ACT_IDENTITY = 0,
  HSTU_ACT_RELU = 1,
  HSTU_ACT_SILU = 2,
  HSTU_ACT_SOFTMAX = 3
} hstu_act_t;

/* A jagged batch of per-user, time-ordered action sequences (the "unified
 * time series" x_0..x_{n-1} of each user, section 二/三 of the review). */
typedef struct {
  int32_t batch;              /* B >= 0 */
  int64_t total_tokens;       /* T == offsets[B], known to the caller (no device read) */
  int32_t max_len;            /* >= max_u (offsets[u+1] - offsets[u]); >= 1 when T > 0.
                                 Kernels are sized from it: a longer user is reported
                                 as HSTU_ERR_DEVICE_CHECK and its rows are not computed */
  const int64_t* offsets;     /* device [B+1], offsets[0] = 0, non-decreasing */
  const int64_t* timestamps;  /* device [T], int64 seconds */
  /* Generalised masks (the Dynamic Masking of MTGR, RecSysChannel digest of
   * "MTGR: Industrial-Scale Generative Recommendation Framework in Meituan"),
   * or NULL for the plain causal mask.  device int32 [B, 2]: (n_us, n_r) per
   * user, whose tokens are then ordered U+S (n_us: profile and long history),
   * R (n_r: short history), candidates (the rest).  U+S keys are visible to
   * every row and U+S rows see only U+S (both directions); R rows are causal;
   * a candidate sees U+S, the R events at or before its own timestamp and
   * itself, not the other candidates.  The position bucket of a key after
   * the row is min(|i - j|, P - 1); N stays n_u.  Timestamps must be
   * non-decreasing over U+S and R; candidates' timestamps are free.  Not
   * accepted by the M-FALCON entry points. */
  const int32_t* segments;
  int32_t max_static;         /* >= every n_us when segments is given */
} hstu_jagged_t;

typedef struct {
  int32_t d_model;            /* d */
  int32_t num_heads;          /* H */
  int32_t dqk;                /* per-head query/key width (64) */
  int32_t dv;                 /* per-head value width (64) */
  int32_t num_pos_buckets;    /* P */
  int32_t num_time_buckets;   /* Tb */
  int32_t phi1;               /* hstu_act_t, ReLU per Eq. 1 */
  int32_t phi2;               /* hstu_act_t, SiLU by default (or SOFTMAX) */
  float ln_eps;               /* LayerNorm epsilon (1e-5) */
  int32_t dtype;              /* hstu_dtype_t of X, W1, W2 and all bf16 intermediates */
  int32_t flags;              /* HSTU_FLAG_* bits, 0 by default */
} hstu_layer_cfg_t;

/* cfg.flags.  HSTU_FLAG_FUSED_F2: the causal bf16 layer (hstu_layer_fwd,
 * hstu_forward, hstu_layer_fwd_static) runs f2 inside the attention kernel
 * when d_model <= 512 and num_heads * dv <= 512: the last of a query tile
 * pair's H head CTAs to finish builds Norm(AV) (.) U for the pair's 256 rows
 * and computes their Y = X + f2(...), reading AV and U back through L2.  The
 * results are bit-identical to the default form, which runs f2 as its own
 * kernel after the attention kernel; on B200 at d_model 512 the default form
 * is the faster one (the fused tail runs on one SM per tile pair and is bound
 * by that SM's memory latency).  M-FALCON candidate layers always run f2 as
 * its own kernel. */
#define HSTU_FLAG_FUSED_F2 1

/* Weights of one layer (all device pointers). */
typedef struct {
  const void* w1;        /* [2H(dqk+dv), d] in cfg dtype; rows ordered U, V, Q, K */
  const float* b1;       /* [2H(dqk+dv)] fp32 */
  const void* w2;        /* [d, H*dv] in cfg dtype */
  const float* b2;       /* [d] fp32 */
  const float* rab_pos;  /* [H, P] fp32 */
  const float* rab_time; /* [H, Tb] fp32 */
  const float* ln_gamma; /* [H*dv] fp32 or NULL (= 1) */
  const float* ln_beta;  /* [H*dv] fp32 or NULL (= 0) */
} hstu_layer_weights_t;

/* Library version string (static storage). */
const char* hstu_version(void);

/* Human-readable name of a status code (static storage, never NULL). */
const char* hstu_status_string(hstu_status_t status);

/* Number of workspace bytes hstu_layer_fwd / hstu_forward / hstu_attn_fwd need
 * for `total_tokens` rows.  Returns 0 for an invalid cfg. */
size_t hstu_layer_workspace_bytes(const hstu_layer_cfg_t* cfg, int64_t total_tokens);
size_t hstu_forward_workspace_bytes(const hstu_layer_cfg_t* cfg, int32_t num_layers,
                                    int64_t total_tokens);

/* Workspace bytes for mfalcon_score with `num_cand` candidate rows in total. */
size_t hstu_mfalcon_workspace_bytes(const hstu_layer_cfg_t* cfg, int64_t num_cand);

/*
 * Eq. 2 alone: AV = phi2(Q K^T + rab^{p,t}) V / n_u per user and head, causal.
 *   q, k   device [T, H*dqk], v device [T, H*dv], av_out device [T, H*dv],
 *          all in cfg->dtype; head h occupies columns h*64 .. h*64+63.
 *   rab_pos device [H, P] fp32, rab_time device [H, Tb] fp32.
 *   workspace may be NULL when ws_bytes == 0 (this entry needs none).
 * Rows of av_out belonging to users are written; nothing else is touched.
 */
hstu_status_t hstu_attn_fwd(const hstu_layer_cfg_t* cfg, const hstu_jagged_t* jag,
                            const void* q, const void* k, const void* v,
                            const float* rab_pos, const float* rab_time, void* av_out,
                            void* workspace, size_t ws_bytes, void* stream);

/* Gradients of one layer's parameters (all device fp32, overwritten). */
typedef struct {
  float* dw1;        /* [2H(dqk+dv), d] */
  float* db1;        /* [2H(dqk+dv)] */
  float* dw2;        /* [d, H*dv] */
  float* db2;        /* [d] */
  float* drab_pos;   /* [H, P] */
  float* drab_time;  /* [H, Tb] */
  float* dgamma;     /* [H*dv], or NULL (written when the layer has ln_gamma) */
  float* dbeta;      /* [H*dv], or NULL (written when the layer has ln_beta) */
} hstu_layer_grads_t;

/* Backward of the causal attention step (the derivative of hstu_attn_fwd's
 * Eq. 2 of the review, section 三 核心公式; the pages print no backward):
 * given dO = dL/dAV,
 *   dV = A^T dO,  dS = (dO V^T) (.) phi2'(Q K^T + rab) / N on visible pairs,
 *   dQ = dS K,  dK = dS^T Q,
 *   drab_pos[h, min(i-j, P-1)] and drab_time[h, bt(t_i - t_j)] += dS_ij.
 *   cfg         dtype HSTU_FP16 or HSTU_BF16 (operand type of q, k, v, d_o),
 *               phi2 SiLU (SiLU'(s) = sigmoid(s)(1 + s(1 - sigmoid(s)))),
 *               ReLU (ReLU'(0) = 0) or identity; HSTU_ACT_SOFTMAX and
 *               HSTU_FP32 return HSTU_ERR_UNSUPPORTED
 *   jag         causal only (segments must be NULL)
 *   q, k, v, d_o device [T, H*64] in the operand type, 16-byte aligned
 *   dq, dk, dv  device [T, H*64] fp32, written (dq is zeroed, then accumulated
 *               one key tile at a time with TMA reduce-adds: its summation
 *               order, and so its last bits, vary from run to run)
 *   drab_pos    device [H, P] fp32, drab_time device [H, Tb] fp32: overwritten
 *               (zeroed, then accumulated with atomics; the same holds)
 * Timestamps must be non-decreasing within each user.  Runs one tcgen05 kernel
 * (one CTA per head, user and 128-key tile).  HSTU_ERR_UNSUPPORTED when the
 * time-bucket table does not fit the octave lookup (as for the forward). */
hstu_status_t hstu_attn_bwd(const hstu_layer_cfg_t* cfg, const hstu_jagged_t* jag,
                            const void* q, const void* k, const void* v, const void* d_o,
                            const float* rab_pos, const float* rab_time, float* dq, float* dk,
                            float* dv, float* drab_pos, float* drab_time, void* stream);

/*
 * Eq. 2 alone with an fp32 result: the same computation as hstu_attn_fwd, with
 * AV written in fp32 (the precision the layer path hands to Norm(.) of Eq. 3)
 * instead of being rounded to cfg->dtype.
 *   q, k, v  device [T, H*64] in cfg->dtype; av_out device [T, H*64] fp32.
 *   rab_pos device [H, P] fp32, rab_time device [H, Tb] fp32.
 * Needs no workspace.  Rows of av_out belonging to users are written.  A user
 * longer than jag->max_len is reported as HSTU_ERR_DEVICE_CHECK in the device
 * status word and its rows are not written.
 */
hstu_status_t hstu_attn_fwd_f32(const hstu_layer_cfg_t* cfg, const hstu_jagged_t* jag,
                                const void* q, const void* k, const void* v,
                                const float* rab_pos, const float* rab_time, float* av_out,
                                void* stream);

/*
 * Eq. 2 in candidate mode alone (the attention step of M-FALCON, section 三,
 * M-FALCON 推理算法): every candidate row c of user u sits at position n_u with
 * timestamp request_ts[u] and attends to all n_u cached history keys/values of
 * u and to its own key/value (position bucket 0, time bucket 0):
 *   AV_c = ( sum_j phi2(q_c.k_j + rab_pos[h, min(n_u - j, P-1)]
 *                        + rab_time[h, bt(t_req - t_j)]) v_j
 *            + phi2(q_c.k_c + rab_pos[h, 0] + rab_time[h, 0]) v_c ) / max(n_u, 1).
 *   history      jagged history (offsets, timestamps, max_len >= every n_u).
 *   k_hist, v_hist device [T_hist, H*64] in cfg->dtype (cached keys/values).
 *   cand_offsets device [B+1]; num_cand rows in all, max_cand >= each count.
 *   q, k, v      device [num_cand, H*64] in cfg->dtype: the candidates' own rows.
 *   request_ts   device [B] int64.  av_out device [num_cand, H*64] fp32.
 * Needs no workspace.  Lengths beyond max_len / max_cand are reported as
 * HSTU_ERR_DEVICE_CHECK in the device status word.
 */
hstu_status_t mfalcon_attn_fwd(const hstu_layer_cfg_t* cfg, const hstu_jagged_t* history,
                               const void* k_hist, const void* v_hist,
                               const int64_t* cand_offsets, int64_t num_cand, int32_t max_cand,
                               const void* q, const void* k, const void* v,
                               const int64_t* request_ts, const float* rab_pos,
                               const float* rab_time, float* av_out, void* stream);

/*
 * One HSTU layer (Eq. 1-3 and the residual) over a jagged batch.
 *   x_in        device [T, d] in cfg dtype: the layer input fed to f1.  For
 *               bf16 layers it may be NULL when x_res is given: f1 then reads
 *               x_res rounded to fp16 (with an fp16 copy of W1), the way the
 *               layers after the first of hstu_forward run.
 *   x_res       device [T, d] fp32 residual input, or NULL to use x_in.
 *   y_out       device [T, d] fp32: X + f2(Norm(AV) (.) U).
 *   y_out_lp    device [T, d] in cfg dtype (a rounded copy of y_out for the
 *               next layer's f1), or NULL.
 *   kv_cache_out device [T, 2, H, 64] (per row: K of every head,
 *               then V of every head), or NULL.  When given, this layer's K
 *               and V rows are kept there for M-FALCON.  bf16 layers keep
 *               K and V in fp16 (their attention operands are fp16: the
 *               same tensor-core rate as bf16 with 8x finer rounding);
 *               fp32 layers in fp32.
 *   workspace   device, ws_bytes >= hstu_layer_workspace_bytes(cfg, T).
 * x_in, y_out and y_out_lp must not overlap.
 */
hstu_status_t hstu_layer_fwd(const hstu_layer_cfg_t* cfg, const hstu_layer_weights_t* w,
                             const hstu_jagged_t* jag, const void* x_in, const float* x_res,
                             float* y_out, void* y_out_lp, void* kv_cache_out,
                             void* workspace, size_t ws_bytes, void* stream);

/* Workspace bytes of hstu_layer_bwd for T tokens. */
size_t hstu_layer_bwd_workspace_bytes(const hstu_layer_cfg_t* cfg, int64_t total_tokens);

/* Backward of one bf16 layer (the derivative of hstu_layer_fwd; the pages
 * print no backward, so this is the chain rule through Eq. 1-3 of the review
 * and the residual): given dY = dL/dY, writes dX = dL/dX and the parameter
 * gradients.  The forward intermediates are recomputed from X with the
 * forward's own kernels (f1, attention), so only X is kept between the
 * passes.  Then:
 *   dG = dY W2, dW2 = dY^T G, db2 = sum dY                  (GEMMs: cuBLAS, TF32)
 *   dU, dAV, dgamma, dbeta through G = LayerNorm(AV) (.) U  (one warp per row)
 *   dQ, dK, dV, drab_pos, drab_time                         (hstu_attn_bwd's kernel)
 *   dZ = [dU | dV | dQ | dK] (.) phi1', db1 = sum dZ,
 *   dW1 = dZ^T X, dX = dY + dZ W1                           (GEMMs: cuBLAS, TF32)
 *   cfg       dtype HSTU_BF16; phi1 ReLU (ReLU'(0) = 0) or identity; phi2
 *             SiLU, ReLU or identity; HSTU_ERR_UNSUPPORTED otherwise
 *   jag       causal (segments NULL)
 *   x_in      device [T, d] bf16 layer input, or NULL with x_res (as in
 *             hstu_layer_fwd: f1 then read x_res rounded to fp16)
 *   x_res     device [T, d] fp32 or NULL
 *   dy        device [T, d] fp32
 *   dx        device [T, d] fp32, written
 *   grads     parameter gradients, overwritten
 * The first call on a device creates that device's cuBLAS handle; its
 * workspace is carved from `workspace`. */
hstu_status_t hstu_layer_bwd(const hstu_layer_cfg_t* cfg, const hstu_layer_weights_t* w,
                             const hstu_jagged_t* jag, const void* x_in, const float* x_res,
                             const float* dy, float* dx, const hstu_layer_grads_t* grads,
                             void* workspace, size_t ws_bytes, void* stream);

/*
 * A stack of num_layers HSTU layers (the residual stream stays fp32).
 *   weights      host array [num_layers] of per-layer weight structs.
 *   x_in         device [T, d] in cfg dtype.  y_out device [T, d] fp32.
 *   kv_cache_out device [num_layers][T, 2, H, 64] (fp16 for bf16 layers, fp32
 *                for fp32 layers), or NULL.
 *   workspace    ws_bytes >= hstu_forward_workspace_bytes(cfg, num_layers, T).
 */
hstu_status_t hstu_forward(const hstu_layer_cfg_t* cfg, int32_t num_layers,
                           const hstu_layer_weights_t* weights, const hstu_jagged_t* jag,
                           const void* x_in, float* y_out, void* kv_cache_out,
                           void* workspace, size_t ws_bytes, void* stream);

/*
 * M-FALCON scoring (section 三, M-FALCON 推理算法): each candidate c of user u,
 * with embedding e_c, runs through the num_layers layers as a row placed at
 * position n_u with timestamp request_ts[u]; at every layer it attends to the
 * user's cached history keys/values and to itself only.  score_c = <y_c, e_c>
 * where y_c is its final fp32 residual-stream row.
 *   history      jagged history (offsets/timestamps of the cached rows).
 *   kv_cache     device [num_layers][T_hist, 2, H, 64] from hstu_forward (fp16
 *                for bf16 layers, fp32 for fp32 layers).
 *   cand_offsets device [B+1] candidate row ranges per user; num_cand = total
 *                rows, max_cand >= the largest per-user count.
 *   cand_emb     device [num_cand, d] in cfg dtype.  request_ts device [B].
 *   microbatch   b_m >= 1.  Microbatches run concurrently as tiles of one
 *                launch; scores do not depend on b_m.
 *   scores       device [num_cand] fp32.
 *   cand_y_out   device [num_cand, d] fp32, or NULL: receives y_c, each
 *                candidate's final residual-stream row (the vector the score
 *                is taken against).
 *   workspace    ws_bytes >= hstu_mfalcon_workspace_bytes(cfg, num_cand).
 * A history or candidate count beyond max_len / max_cand is reported as
 * HSTU_ERR_DEVICE_CHECK in the device status word.
 */
hstu_status_t mfalcon_score(const hstu_layer_cfg_t* cfg, int32_t num_layers,
                            const hstu_layer_weights_t* weights, const hstu_jagged_t* history,
                            const void* kv_cache, const int64_t* cand_offsets, int64_t num_cand,
                            int32_t max_cand, const void* cand_emb, const int64_t* request_ts,
                            int32_t microbatch, float* scores, float* cand_y_out, void* workspace,
                            size_t ws_bytes, void* stream);

/*
 * Stochastic Length (review section 三, Stochastic Length): every user's n
 * events are shortened to L = min(n, ceil(n u^(1/alpha))), u ~ Uniform(0, 1],
 * keeping a uniformly random subset of L events in time order.
 * Randomness: Philox4x64-10 (Salmon et al., SC 2011) with key (seed, 0);
 * user u's length uses counter (0, u, step, 0) and u = ((x >> 11) + 1) 2^-53
 * from its first output word x; position p's rank key is the first output
 * word of counter (p, u, step, 1); the kept subset is the L smallest rank
 * keys (equal keys: the lower position).  The length is decided in fp64.
 *   full          the input batch (offsets and timestamps on the device;
 *                 max_len <= 16384).
 *   x_full        device [T_full] rows of row_bytes bytes each (any element
 *                 type; row_bytes a multiple of 16), or NULL with x_out NULL.
 *   alpha > 0; seed, step select the random stream (use the training step
 *                 as `step` to draw fresh subsets each step).
 *   offsets_out   device [B+1]: the output batch's offsets; offsets_out[B]
 *                 is its total T_out (read it back to size the next call).
 *   lengths_out   device int32 [B]: L per user.
 *   max_len_out   device int32 [1] or NULL: the largest L.
 *   kept_index_out device int64 [T_full]: for output row r < T_out, the row
 *                 of the input it copies.
 *   timestamps_out device int64 [T_full] or NULL; x_out device [T_full] rows
 *                 or NULL: the kept rows' timestamps and rows.
 * Allocates nothing; four launches on `stream`.
 */
hstu_status_t hstu_stochastic_length(const hstu_jagged_t* full, const void* x_full,
                                     int32_t row_bytes, float alpha, uint64_t seed, uint64_t step,
                                     int64_t* offsets_out, int32_t* lengths_out,
                                     int32_t* max_len_out, int64_t* kept_index_out,
                                     int64_t* timestamps_out, void* x_out, void* stream);

/* Per-kernel timing.  Between hstu_profiler_start() and hstu_profiler_stop()
 * every kernel the library launches is bracketed by CUDA events recorded on
 * its own stream (device time, no host synchronisation while running).
 * stop() waits for the recorded events, writes up to `capacity` entries (one
 * per kernel kind that ran: name, launch count, summed milliseconds) and sets
 * *count.  The profiler is process-wide; calls from several threads are
 * serialised. */
typedef struct {
  const char* name;      /* static string, e.g. "attention", "f1_gemm", "f2_gemm" */
  int32_t launches;
  double total_ms;
} hstu_kernel_time_t;

hstu_status_t hstu_profiler_start(void);
hstu_status_t hstu_profiler_stop(hstu_kernel_time_t* out, int32_t capacity, int32_t* count);

/*
 * hstu_layer_fwd for callers that cannot allocate device memory.  The
 * pages have no counterpart: this is an interface convenience.  Some callers
 * are handed only their input and output buffers: a plugin inside a serving
 * engine that owns every byte of device memory, or a process whose memory is
 * pre-reserved by another allocator.  Others must not call cudaMalloc on a
 * latency-critical path, because it can synchronise the device.  This entry
 * takes the same arguments as hstu_layer_fwd minus the workspace.  Its
 * scratch is one fixed array inside the library,
 * HSTU_STATIC_SCRATCH_BYTES (64 MiB) per GPU, which every GPU that loads the
 * library keeps until the process exits.
 *   - Size limit: hstu_layer_workspace_bytes(cfg, T) must not exceed
 *     HSTU_STATIC_SCRATCH_BYTES (about 9,000 tokens at d_model 512 and 8 heads,
 *     about 18,000 at d_model 256 and 4 heads).  A larger request returns
 *     HSTU_ERR_WORKSPACE_TOO_SMALL before any launch.
 *   - No call allocates: no cudaMalloc, no cudaFree, no allocating library.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current).  Make that first call
 *     before capturing any stream.
 *   - Every call on a device shares the same array and leaves its contents
 *     behind.  The layer writes every scratch byte it reads, so nothing needs
 *     clearing, but two calls whose work overlaps on the GPU (different
 *     streams, or different host threads) race on the array: order them.
 */
#define HSTU_STATIC_SCRATCH_BYTES (64ull << 20)
hstu_status_t hstu_layer_fwd_static(const hstu_layer_cfg_t* cfg, const hstu_layer_weights_t* w,
                                    const hstu_jagged_t* jag, const void* x_in,
                                    const float* x_res, float* y_out, void* y_out_lp,
                                    void* kv_cache_out, void* stream);

/* Synchronises `stream`, returns the first error a kernel recorded in the
 * device status word since the last call (HSTU_OK if none) and clears it. */
hstu_status_t hstu_get_device_status(void* stream);

/* Host only: writes thr[0..Tb-1], the smallest int64 dt reaching each time
 * bucket under bt(dt) above (thr[0] = 0).  Tb in [1, 256]. */
hstu_status_t hstu_time_bucket_thresholds(int32_t num_time_buckets, int64_t* thr_out);

/* Test support: for every user writes the n_u x n_u row-major block of
 * position buckets min(i-j, P-1) and time buckets bt(t_i - t_j) for j <= i
 * (-1 for j > i), using the same device code as the attention kernels.
 * pos_idx / time_idx: device int32 [sum_u n_u^2], blocks in user order;
 * block_offsets: device int64 [B+1] prefix sums of n_u^2. */
hstu_status_t hstu_debug_rab_index(const hstu_jagged_t* jag, int32_t num_pos_buckets,
                                   int32_t num_time_buckets, const int64_t* block_offsets,
                                   int32_t* pos_idx, int32_t* time_idx, void* stream);

/* Test support: launches one CTA that waits on an mbarrier nothing completes,
 * bounded by timeout_ns; it records HSTU_ERR_DEVICE_TIMEOUT and returns. */
hstu_status_t hstu_debug_wait_timeout(uint64_t timeout_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_H_ */
