// Pointwise aggregated attention (Eq. 2 of the review of "Actions Speak Louder
// than Words", section 三 核心公式): AV = phi2(Q K^T + rab^{p,t}) V / N over
// jagged per-user sequences, with no softmax (hence no row max, no row sum,
// no rescaling of the running output).
//
// One CTA owns a pair of 128-row query tiles (A = rows q0..q0+127, B = the
// next 128) of one user and one head, and walks that user's key tiles in
// order.  Causal mode (the layer forward) stops at the diagonal and masks
// inside it; candidate mode (M-FALCON) lets candidate rows see every cached
// history key and adds each candidate's own key/value in the epilogue.
//
// Warp roles (608 threads):
//   warps 0-7   element group A (query tile A): warps 0-3 own key columns
//               0-31 of every S tile, warps 4-7 columns 32-63; within each
//               warpgroup thread t owns query row t
//   warps 8-15  element group B, the same for tile B
//   warp 16     producer: TMA loads of the two Q tiles and of the K, V tiles
//               (128B swizzle, no multicast) and the per-key side data
//               (int32 times, or the whole candidate-mode bias)
//   warp 17     MMA issuer of tile A and TMEM owner
//   warp 18     MMA issuer of tile B
// Each issuing warp runs its loop together (waits are warp votes) and one
// lane, elected once, issues every MMA and commit: issued that way the MMA
// operands stay warp-uniform, and one warp per query tile keeps the tensor
// pipe fed.  The two issuers touch disjoint tensor memory; a K/V stage is
// released by one commit from each.
// Two warpgroups per query tile halve the elements each thread handles per
// key tile and double the warps that hide tensor-memory, shared-memory and
// MUFU latency; the work per element is one row-thread's arithmetic either way.
// Key tiles are 64 keys.  Tensor memory (all 512 columns): three S buffers
// per group (64 fp32 columns each; each half writes its 32 keys of P, bf16
// pairs, over the first 16 columns of its own 32-column half once they are
// read) and O_A, O_B (64 fp32 columns each).  S of tile k+3 reuses the buffer
// of tile k, so it is issued right after P V of tile k: the MMAs for a tile
// are issued two tiles before the group needs them, which covers the
// issue-to-completion latency of the tensor pipe.  Q_A, Q_B live in shared
// memory.
// Per key tile: S = Q K^T (tcgen05, both operands in shared memory), the
// element group reads S row by row, adds the gathered bias, applies phi2 and
// the mask, writes P (bf16) back over S, then O += P V (tcgen05 with A from
// tensor memory, V as an MN-major B operand).  The MMAs of one issuing thread
// execute in issue order, so S of tile k+3 is only written after P V of tile
// k has read P.  1/N is applied once to O.
//
// Elementwise work per (query, key, head), SiLU case: x = s + rab, and
// x*sigmoid(x) = h + h*tanh(h) with h = x/2.  The 1/2 is folded into the bias
// tables when they are staged, so h = fma(s, 1/2, rab/2) and only one
// transcendental (tanh) is needed.  The position bias is staged reversed in
// two copies offset by one entry, so every thread reads the biases of two
// adjacent keys with one aligned 8-byte shared load; pairs of keys then go
// through packed fp32x2 adds and FMAs.  The time bucket only decreases along
// a row (keys are time-ordered), so a 32-key chunk whose last visible key
// still lies in each row's current bucket takes the row's cached time bias;
// otherwise the chunk is resolved per key (see causal_chunk).
#pragma once

#include "ptx.cuh"

namespace hstu {

constexpr int ATT_ROWS = 128;
constexpr int ATT_KEYS = 64;
constexpr int ATT_HD = 64;
constexpr int ATT_STAGES = 6;
constexpr int ATT_THREADS = 608;
constexpr int ATT_PRODUCER_WARP = 16;
constexpr int ATT_MMA_WARP = 17;  // + query tile (A: 17, B: 18)
constexpr int MAX_TIME_BUCKETS = 256;

constexpr uint32_t ATT_TILE_BYTES = ATT_KEYS * ATT_HD * 2;  // one K or V tile: 8 KB
constexpr uint32_t ATT_Q_BYTES = ATT_ROWS * ATT_HD * 2;     // one Q tile: 16 KB
constexpr int ATT_SBUF = 3;                                 // S buffers per query tile

// Layer-fused f2 (causal layer path): the last of the H head CTAs of a query
// tile pair to finish builds Norm(AV) (.) U of the pair's rows and runs
// Y = X + (Norm(AV) (.) U) W2^T + b2 for them before it exits.
struct TailParams {
  int32_t* count;              // [B * num_qpairs] arrivals per tile pair, zero before the launch
  const float* u;              // [T, ld_u] U (fp32)
  int64_t ld_u;
  const float* x_res;          // [T, ld_x] fp32 residual, or nullptr:
  const __nv_bfloat16* x_lp;   //   bf16 residual
  int64_t ld_x;
  const float* b2;             // [N]
  const float* gamma;          // [K] or nullptr (1)
  const float* beta;           // [K] or nullptr (0)
  float eps;
  float* y;                    // [T, ld_y] fp32
  void* y_lp;                  // [T, ld_y] fp16 (ylp_f16) or bf16 copy, or nullptr
  int32_t ylp_f16;
  int64_t ld_y;
  int32_t N;                   // d_model (<= 512)
  int32_t K;                   // H * 64 (<= 512)
};

struct AttnParams {
  const int64_t* kv_offsets;   // [B+1] key/value rows per user (query rows too in causal mode)
  const int64_t* q_offsets;    // [B+1] candidate rows per user (candidate mode)
  const int64_t* timestamps;   // [T_kv]
  const int64_t* request_ts;   // [B] (candidate mode)
  const float* rab_pos;        // [H, P]
  const float* rab_time;       // [H, Tb]
  const void* q_self;          // rows' own Q, K, V for the self term (candidate mode,
  const void* k_self;          // and candidate rows of the generalised masks), in the
  const void* v_self;          // kernel's operand type (bf16 or fp16)
  int64_t ld_qs, ld_ks, ld_vs; // their row strides (elements)
  const int32_t* segments;     // [B, 2] (n_us, n_r) per user: generalised masks, or nullptr
  int32_t max_static;          // bound on n_us (staged position range)
  void* av;                    // [T_q, ld_av] output in the operand type, or
  float* av_f32;               // [T_q, ld_av] fp32 output (the layer path feeds LayerNorm)
  int64_t ld_av;
  float* ln_part;              // [T_q, H, 2] (sum, centred sum of squares) or nullptr
  int32_t B, H, P, Tb;
  int32_t max_q, max_kv;       // host-declared length bounds the launch is sized for
  int32_t num_qpairs;
  int32_t pos_len;             // entries per staged copy of the position table
  int32_t phi2;
  uint64_t timeout_ns;
  int64_t thr[MAX_TIME_BUCKETS];  // time-bucket thresholds (thr[0] = 0)
  int4 oct[32];                   // per octave k of dt+1: {t1, t2, t3, bucket(2^k - 1)}
  TailParams tail;                // FUSED kernels only
};

// ---------------------------------------------------------------- time buckets

// Largest b in [0, Tb) with thr[b] <= dt (dt < 0 -> 0): the bucket of dt.
__device__ __forceinline__ int time_bucket_search(int64_t dt, const int64_t* thr, int Tb) {
  if (dt <= 0) return 0;
  int lo = 0, hi = Tb - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (thr[mid] <= dt) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Bucket of t_i - t_j for one query row as j walks forward through keys with
// non-decreasing timestamps: the bucket can only go down, so each step is a
// compare against the current lower edge and an occasional decrement.
// T is int64_t (absolute seconds, with the int64 threshold table) or int32_t
// (seconds since the user's first event, used when the user's whole span
// fits, with the threshold table clamped to int32: every bucket the walk
// visits has a threshold at most t_i < 2^31, so the clamp changes no bound).
template <typename T>
struct BucketWalk {
  using TT = T;  // threshold table entry type
  int b;
  T ti;
  T bound;  // keys with t_j <= bound are still in bucket >= b

  __device__ __forceinline__ void init(T t_row, T t_first_key, const int64_t* thr64, const TT* thr,
                                       int Tb) {
    ti = t_row;
    b = time_bucket_search(static_cast<int64_t>(t_row) - static_cast<int64_t>(t_first_key), thr64,
                           Tb);
    set_bound(thr);
  }
  __device__ __forceinline__ void set_bound(const TT* thr) {
    if constexpr (sizeof(T) == 8) {
      bound = (b == 0) ? INT64_MAX : ti - thr[b];
    } else {
      bound = (b == 0) ? INT32_MAX : ti - thr[b];  // ti >= 0, thr[b] in [0, INT32_MAX]
    }
  }
  // Advance to a key with timestamp tj; returns true when the bucket changed.
  __device__ __forceinline__ bool step(T tj, const TT* thr) {
    bool changed = false;
    while (tj > bound) {
      --b;
      set_bound(thr);
      changed = true;
    }
    return changed;
  }
};

// Time bucket of 0 <= dt < 2^31 - 1 without a walk.  For dt + 1 in the octave
// [2^k, 2^(k+1)) the bucket is oct[k].w plus the number of the next three
// bucket edges oct[k].x/y/z it reaches (edges are ~1.35x apart, so at most
// three fall inside one octave; INT32_MAX pads missing edges).
__device__ __forceinline__ int time_bucket_octave(int32_t dt, const int4* oct) {
  const int32_t d = dt > 0 ? dt : 0;
  const int k = 31 - __clz(d + 1);
  const int4 o = oct[k];
  return o.w + (d >= o.x ? 1 : 0) + (d >= o.y ? 1 : 0) + (d >= o.z ? 1 : 0);
}

// Time bias of 0 <= dt < 2^31 - 1 straight from the octave: `ort[k]` holds the
// (scaled) biases of the octave's base bucket and of the three buckets after
// it, so the bias is three compares and selects, with no dependent lookup.
__device__ __forceinline__ float time_bias_octave(int32_t dt, const int4* oct, const float4* ort) {
  const int32_t d = dt > 0 ? dt : 0;
  const int k = 31 - __clz(d + 1);
  const int4 o = oct[k];
  const float4 r = ort[k];
  float v = r.x;
  v = d >= o.x ? r.y : v;
  v = d >= o.y ? r.z : v;
  v = d >= o.z ? r.w : v;
  return v;
}

// phi2 applied to a pair given h = (scaled) pre-activation, in fp32; returns
// the pair of P values as bf16x2, or as fp16x2 when F16.
// SiLU: tables carry x/2, so p = h + h*tanh(h); ReLU / identity: h = x.
template <int PHI, bool F16>
__device__ __forceinline__ uint32_t phi_pair(uint64_t h2) {
  auto to16 = [](uint64_t v) -> uint32_t {
    if constexpr (F16) return f2_to_h2(v);
    else return f2_to_bf16x2(v);
  };
  if constexpr (PHI == HSTU_ACT_SILU) {
    float h0, h1;
    f2_unpack(h2, h0, h1);
    const uint64_t t2 = f2_pack(tanh_approx(h0), tanh_approx(h1));
    return to16(f2_fma(h2, t2, h2));
  } else if constexpr (PHI == HSTU_ACT_RELU) {
    float h0, h1;
    f2_unpack(h2, h0, h1);
    return to16(f2_pack(fmaxf(h0, 0.0f), fmaxf(h1, 0.0f)));
  } else {
    return to16(h2);
  }
}

// phi2 of an fp16x2 pair of (scaled) pre-activations; SiLU: p = h + h*tanh(h).
template <int PHI>
__device__ __forceinline__ uint32_t phi_h2(uint32_t h) {
  if constexpr (PHI == HSTU_ACT_SILU) {
    return h2_fma(h, h2_tanh(h), h);
  } else if constexpr (PHI == HSTU_ACT_RELU) {
    return h2_max(h, 0u);
  } else {
    return h;
  }
}

template <int PHI>
__device__ __forceinline__ float apply_phi(float x) {
  if constexpr (PHI == HSTU_ACT_SILU) {
    const float h = 0.5f * x;
    return fmaf(h, tanh_approx(h), h);
  } else if constexpr (PHI == HSTU_ACT_RELU) {
    return fmaxf(x, 0.0f);
  } else {
    return x;
  }
}

// Scale folded into the staged bias tables and applied to S: SiLU works on
// x/2 (x sigmoid(x) = h + h tanh(h), h = x/2); softmax on x log2(e), so that
// exp(x - m) = 2^(h - m') with the MUFU's exp2.
template <int PHI>
__host__ __device__ constexpr float phi_scale() {
  return PHI == HSTU_ACT_SILU ? 0.5f : (PHI == HSTU_ACT_SOFTMAX ? 1.4426950408889634f : 1.0f);
}

// Zero the keys of a bf16 pair at columns c, c+1 that are above `last`.
__device__ __forceinline__ uint32_t mask_pair(uint32_t w, int c, int last) {
  const uint32_t lo = (c <= last) ? 0x0000FFFFu : 0u;
  const uint32_t hi = (c + 1 <= last) ? 0xFFFF0000u : 0u;
  return w & (lo | hi);
}

// ---------------------------------------------------------------- shared memory

struct AttnSmem {
  static constexpr uint32_t kQ = 0;                                   // 2 x 16 KB
  static constexpr uint32_t kK = kQ + 2 * ATT_Q_BYTES;                // stages x 8 KB
  static constexpr uint32_t kV = kK + ATT_STAGES * ATT_TILE_BYTES;    // stages x 8 KB
  static constexpr uint32_t kKeyInfo = kV + ATT_STAGES * ATT_TILE_BYTES;  // stages x 256 B
  static constexpr uint32_t kKeyStride = ATT_KEYS * 4;                // bytes per stage
  static constexpr uint32_t kTimeTab = kKeyInfo + ATT_STAGES * kKeyStride;
  static constexpr uint32_t kThr = kTimeTab + MAX_TIME_BUCKETS * 4;
  static constexpr uint32_t kThr32 = kThr + MAX_TIME_BUCKETS * 8;   // int32 copy, clamped
  static constexpr uint32_t kOct = kThr32 + MAX_TIME_BUCKETS * 4;    // 32 x int4
  static constexpr uint32_t kOrt = kOct + 32 * 16;                   // 32 x float4
  static constexpr uint32_t kBars = kOrt + 32 * 16;
  static constexpr uint32_t kMisc = kBars + 48 * 8;
  static constexpr uint32_t kLnX = kMisc + 64;                        // 2 x 128 float2
  static constexpr uint32_t kML = kLnX + 2 * ATT_ROWS * 8;           // 4 x 128 float2
  static constexpr uint32_t kPos = kML + 4 * ATT_ROWS * 8;
  // pos_len entries per copy of `elt` bytes each (fp32, or fp16 for the
  // causal fp16-operand kernel), two copies with paired reads
  // fused f2 tail, after the attention is done: a ring of four 32 KB W2 boxes
  // (256 rows x 64 columns, fp16) over Q, K and V, and a ring of three 16 KB
  // A blocks (128 rows x 64 columns of Norm(AV) (.) U, fp16) after the side data
  static constexpr uint32_t kTailBox = 256 * 64 * 2;
  static constexpr int kTailWStages = 4;
  static constexpr uint32_t kTailW = 0;
  static constexpr uint32_t kTailABlock = ATT_ROWS * 128;
  static constexpr int kTailAStages = 3;
  static constexpr uint32_t kTailA = (kPos + 1023u) & ~1023u;
  // epilogue staging, per element warp 32 rows x 32 fp32 (4 KB), over the A
  // ring (idle between a tile's last MMA and the next tile's A build)
  static constexpr uint32_t kTailStage = kTailA;
  static constexpr uint32_t kTailBytes = kTailA + 16 * 4096 + 1024u;  // + align slack
  static_assert(16 * 4096 >= kTailAStages * kTailABlock, "staging covers the A ring");
  static_assert(kTailW + kTailWStages * kTailBox <= kKeyInfo, "tail W2 ring overlaps the side data");
  static constexpr uint32_t bytes(int pos_len, bool pairs, uint32_t elt = 4u) {
    return kPos + static_cast<uint32_t>(pos_len) * elt * (pairs ? 2u : 1u) + 1024u;  // + align slack
  }
};

// barrier slots
enum : int {
  BAR_Q_FULL = 0,
  BAR_KV_FULL = 1,                     // + stage
  BAR_KV_EMPTY = BAR_KV_FULL + ATT_STAGES,
  BAR_S_FULL = BAR_KV_EMPTY + ATT_STAGES,  // + ATT_SBUF * group + buffer
  BAR_P_FULL = BAR_S_FULL + 2 * ATT_SBUF,  // + ATT_SBUF * group + buffer
  BAR_O_FULL = BAR_P_FULL + 2 * ATT_SBUF,  // + group
  BAR_DONE = BAR_O_FULL + 2,               // + group
  // fused f2 tail
  BAR_T_A_FULL = BAR_DONE + 2,             // + stage: an A block is built
  BAR_T_A_EMPTY = BAR_T_A_FULL + 3,        // + stage: its MMAs completed
  BAR_T_W_FULL = BAR_T_A_EMPTY + 3,        // + stage: a W2 box landed
  BAR_T_W_EMPTY = BAR_T_W_FULL + 4,        // + stage: its MMAs completed
  BAR_T_ACC_FULL = BAR_T_W_EMPTY + 4,      // the tile's accumulator is complete
  BAR_T_DONE = BAR_T_ACC_FULL + 1,
  BAR_COUNT = BAR_T_DONE + 1
};
static_assert(BAR_COUNT <= 48, "barrier slots");

// ---------------------------------------------------------------- causal chunk

// One 32-key chunk of one causal row: the pre-activations h = scale * (s + rab)
// of its key pairs are handed to `sink(c, h2)` (columns c, c + 1 as an fp32
// pair) in live lanes only.  `rvx` points at the staged position table entry
// of column 0 (entries for consecutive columns are consecutive; with PAIRS the
// entry pair of an even column is one aligned 8-byte load), `kts` at the
// chunk's key times (seconds since the user's first event, 16-byte aligned).
// Columns above `lim` are masked by the caller and never move the time-bucket
// walk; lim < 0 marks a lane with no visible key in the chunk (the sink is not
// called).  The walk `w` enters at the bucket of the previous key and leaves
// at the bucket of the last visible key.  Per warp the chunk falls in one of
// three cases:
//   every row keeps its bucket      -> one time bias per row, `rt_cur`, kept
//                                      in a register (one compare of the last
//                                      visible key against the bucket edge);
//   two buckets B, B+1 in the warp  -> per key: B+1 iff t_j <= t_i - thr[B+1];
//   more (near the diagonal)        -> per key bias from the octave tables.
template <bool PAIRS, class Sink>
__device__ __forceinline__ void causal_chunk(const uint32_t (&sv)[32], Sink&& sink,
                                             const float* rvx, const int32_t* kts, int lim,
                                             BucketWalk<int32_t>& w, const float* sTime,
                                             const int32_t* sThr, const int4* sOct,
                                             const float4* sOrt, uint64_t scale2, float& rt_cur) {
  const unsigned full = 0xffffffffu;
  const bool live = lim >= 0;
  const int last = lim < 31 ? lim : 31;
  // key times of a pair of columns (broadcast shared loads, only off the
  // one-bucket path)
  auto kt_pair = [&](int c) -> int2 { return *reinterpret_cast<const int2*>(kts + c); };
  auto pos_pair = [&](int c) -> uint64_t {
    if constexpr (PAIRS) return lds_b64(rvx + c);
    else return f2_pack(rvx[c], rvx[c + 1]);
  };
  auto s_pair = [&](int c) -> uint64_t {
    return f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1]));
  };
  // every visible key of every lane still in the lane's current bucket
  if (__all_sync(full, !live || kts[last] <= w.bound)) {
    if (live) {
      const uint64_t rt2 = f2_pack(rt_cur, rt_cur);
#pragma unroll
      for (int c = 0; c < 32; c += 2) sink(c, f2_fma(s_pair(c), scale2, f2_add(pos_pair(c), rt2)));
    }
    return;
  }
  int b_first = -1, b_last = 1 << 30;
  bool lane_steady = true;
  if (live) {
    w.step(kts[0], sThr);
    b_first = w.b;
    const int32_t k_last = kts[last];
    lane_steady = k_last <= w.bound;
    if (!lane_steady) w.step(k_last, sThr);
    b_last = w.b;
    rt_cur = sTime[b_last];
  }
  if (__all_sync(full, lane_steady)) {
    if (live) {
      const float rt = sTime[b_first];
      const uint64_t rt2 = f2_pack(rt, rt);
#pragma unroll
      for (int c = 0; c < 32; c += 2) sink(c, f2_fma(s_pair(c), scale2, f2_add(pos_pair(c), rt2)));
    }
  } else {
    const int B_hi = __reduce_max_sync(full, b_first);
    const int B_lo = __reduce_min_sync(full, b_last);
    if (B_hi - B_lo == 1) {
      if (live) {
        const float rt_hi = sTime[B_hi], rt_lo = sTime[B_lo];
        // keys with t_j <= edge are in bucket B_hi (ti >= 0 and the clamped
        // threshold <= INT32_MAX, so the difference does not overflow)
        const int32_t edge = w.ti - sThr[B_hi];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const int2 k2 = kt_pair(c);
          const float r0 = (k2.x <= edge) ? rt_hi : rt_lo;
          const float r1 = (k2.y <= edge) ? rt_hi : rt_lo;
          sink(c, f2_fma(s_pair(c), scale2, f2_add(pos_pair(c), f2_pack(r0, r1))));
        }
      }
    } else if (live) {
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const int2 k2 = kt_pair(c);
        const float r0 = time_bias_octave(w.ti - k2.x, sOct, sOrt);
        const float r1 = time_bias_octave(w.ti - k2.y, sOct, sOrt);
        sink(c, f2_fma(s_pair(c), scale2, f2_add(pos_pair(c), f2_pack(r0, r1))));
      }
    }
  }
}

// Pointwise phi2 of one causal chunk: packed 16-bit P (bf16, or fp16 when F16)
// in `pk`, masked above `lim`.
template <int PHI, bool PAIRS, bool F16>
__device__ __forceinline__ void causal_chunk_pointwise(const uint32_t (&sv)[32], uint32_t (&pk)[16],
                                                       const float* rvx, const int32_t* kts, int lim,
                                                       BucketWalk<int32_t>& w, const float* sTime,
                                                       const int32_t* sThr, const int4* sOct,
                                                       const float4* sOrt, uint64_t scale2,
                                                       float& rt_cur) {
  causal_chunk<PAIRS>(
      sv, [&](int c, uint64_t h) { pk[c >> 1] = phi_pair<PHI, F16>(h); }, rvx, kts, lim, w, sTime,
      sThr, sOct, sOrt, scale2, rt_cur);
  if (lim < 0) {
#pragma unroll
    for (int q = 0; q < 16; ++q) pk[q] = 0u;
  } else if (lim < 31) {
#pragma unroll
    for (int c = 0; c < 32; c += 2) pk[c >> 1] = mask_pair(pk[c >> 1], c, lim);
  }
}

// ---------------------------------------------------------------- fused f2 tail

// Y = X + (Norm(AV) (.) U) W2^T + b2 for the query rows [q0, q0 + 256) of user
// u (rows at or past n_q are skipped), run by the whole CTA after its
// attention, one 128-row tile after the other:
//   element warps (threads 0..511) build the fp16 A operand one 64-column
//     block at a time into a ring of three (all loads of a block are issued
//     before its slot is awaited), then run the epilogue from tensor memory;
//   the producer warp streams the fp16 W2 boxes (256 output columns x 64) by
//     TMA through a ring of four;
//   the first MMA warp issues, per block, the MMAs of both 256-column halves
//     into tensor memory columns 0..N-1.
// AV and the LayerNorm partial sums of the other heads were written by other
// CTAs of this launch and are read through L2 (ld.global.cg).
__device__ __forceinline__ void attn_f2_tail(const CUtensorMap* tm_w2, const AttnParams& p,
                                             uint8_t* smem, uint64_t* bars, uint32_t tmem,
                                             int64_t q_start, int q0, int n_q,
                                             const WaitCtl& ctl) {
  const TailParams& t = p.tail;
  const int warp = warp_id(), lane = lane_id(), tid = threadIdx.x;
  uint8_t* sA = smem + AttnSmem::kTailA;
  uint8_t* sW = smem + AttnSmem::kTailW;
  float2* sStats = reinterpret_cast<float2*>(smem + AttnSmem::kLnX);
  constexpr int kWS = AttnSmem::kTailWStages, kAS = AttnSmem::kTailAStages;
  constexpr uint32_t kBox = AttnSmem::kTailBox, kABlk = AttnSmem::kTailABlock;
  const int n_mt = (q0 + ATT_ROWS < n_q) ? 2 : 1;
  const int k_blocks = t.K / 64;
  const int halves = (t.N + 255) / 256;

  if (warp == ATT_PRODUCER_WARP) {
    if (lane == 0) {
      tma_prefetch_desc(tm_w2);
      int st = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int mt = 0; ok && mt < n_mt; ++mt)
        for (int kb = 0; ok && kb < k_blocks; ++kb)
          for (int hf = 0; hf < halves; ++hf) {
            ok = mbar_wait(&bars[BAR_T_W_EMPTY + st], ph ^ 1u, ctl);
            if (!ok) break;
            mbar_arrive_expect_tx(&bars[BAR_T_W_FULL + st], kBox);
            tma_load_2d(sW + st * kBox, tm_w2, &bars[BAR_T_W_FULL + st], kb * 64, hf * 256);
            ++issued;
            if (++st == kWS) { st = 0; ph ^= 1u; }
          }
      // the boxes still in flight land before shared memory is released
      for (int k = max(0, issued - kWS); k < issued; ++k)
        mbar_wait_drain(&bars[BAR_T_W_FULL + (k % kWS)], static_cast<uint32_t>(k / kWS) & 1u,
                        ctl.limit_ns);
    }
    __syncwarp();
  } else if (warp == ATT_MMA_WARP) {
    const bool leader = elect_one();
    auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, par, ctl));
    };
    int ws = 0, as = 0;
    uint32_t wph = 0, aph = 0;
    bool ok = true;
    for (int mt = 0; ok && mt < n_mt; ++mt) {
      for (int kb = 0; ok && kb < k_blocks; ++kb) {
        ok = wait_all(&bars[BAR_T_A_FULL + as], aph);
        if (!ok) break;
        tc_fence_after();
        const uint64_t da = smem_desc_sw128(smem_u32(sA + as * kABlk), 16, 1024);
        for (int hf = 0; hf < halves; ++hf) {
          ok = wait_all(&bars[BAR_T_W_FULL + ws], wph);
          if (!ok) break;
          tc_fence_after();
          const uint64_t dw = smem_desc_sw128(smem_u32(sW + ws * kBox), 16, 1024);
          const int n = min(256, t.N - hf * 256);
          const uint32_t idesc = idesc_16_f32(ATT_ROWS, n, false, false, true);
          if (leader) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ss(tmem + static_cast<uint32_t>(hf * 256), da + 2 * kk, dw + 2 * kk, idesc,
                          (kb > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&bars[BAR_T_W_EMPTY + ws]);
          }
          __syncwarp();
          if (++ws == kWS) { ws = 0; wph ^= 1u; }
        }
        if (leader) mma_commit(&bars[BAR_T_A_EMPTY + as]);
        __syncwarp();
        if (++as == kAS) { as = 0; aph ^= 1u; }
      }
      if (ok && leader) mma_commit(&bars[BAR_T_ACC_FULL]);
      __syncwarp();
    }
    if (leader) mma_commit(&bars[BAR_T_DONE]);
    __syncwarp();
    mbar_wait_drain(&bars[BAR_T_DONE], 0, ctl.limit_ns);
  } else if (tid < 16 * 32) {
    const float inv_k = 1.0f / static_cast<float>(t.K);
    const int q4 = warp & 3;    // tensor-memory lane quarter
    const int cg = warp >> 2;   // 128-column group of the epilogue
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    int as = 0;
    uint32_t aph = 0;
    bool ok = true;
    for (int mt = 0; mt < n_mt; ++mt) {
      const int base = q0 + mt * ATT_ROWS;
      // per-row LayerNorm statistics from the heads' partial sums
      if (tid < ATT_ROWS) {
        float mean = 0.0f, rstd = 0.0f;
        if (base + tid < n_q) {
          const float2* lp = reinterpret_cast<const float2*>(p.ln_part) + (q_start + base + tid) * p.H;
          float tot = 0.0f;
          for (int hh = 0; hh < p.H; ++hh) tot += __ldcg(&lp[hh].x);
          mean = tot * inv_k;
          float m2 = 0.0f;
          for (int hh = 0; hh < p.H; ++hh) {
            const float2 v = __ldcg(&lp[hh]);
            const float dm = v.x * (1.0f / 64.0f) - mean;
            m2 += v.y + 64.0f * dm * dm;
          }
          rstd = rsqrtf(m2 * inv_k + t.eps);
        }
        sStats[tid] = make_float2(mean, rstd);
      }
      named_barrier_sync(3, 16 * 32);
      // A blocks: 128 rows x 8 chunks of 8 columns; this thread's two chunks
      // (rows tid/8 and tid/8 + 64, chunk tid%8) of every block
      // lane j of each group of 8 takes columns 4j .. 4j + 3 and 32 + 4j .. + 3
      // of the block: each load instruction reads whole 128-byte rows; the
      // results go to the two 8-byte halves of their swizzled 16-byte chunks
      const int j = tid & 7;
      for (int kb = 0; kb < k_blocks; ++kb) {
        const int colA = kb * 64 + 4 * j, colB = colA + 32;
        float4 av[2][2], uv[2][2];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int r = (tid >> 3) + h2 * 64;
          if (base + r < n_q) {
            const int64_t row = q_start + base + r;
            const float* ap = p.av_f32 + row * p.ld_av;
            const float* up = t.u + row * t.ld_u;
            av[h2][0] = __ldcg(reinterpret_cast<const float4*>(ap + colA));
            av[h2][1] = __ldcg(reinterpret_cast<const float4*>(ap + colB));
            uv[h2][0] = *reinterpret_cast<const float4*>(up + colA);
            uv[h2][1] = *reinterpret_cast<const float4*>(up + colB);
          } else {
            av[h2][0] = av[h2][1] = uv[h2][0] = uv[h2][1] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        float gm[8], bt[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int c = (e < 4 ? colA : colB - 4) + e;
          gm[e] = t.gamma != nullptr ? __ldg(t.gamma + c) : 1.0f;
          bt[e] = t.beta != nullptr ? __ldg(t.beta + c) : 0.0f;
        }
        if (ok) ok = mbar_wait(&bars[BAR_T_A_EMPTY + as], aph ^ 1u, ctl);
        uint8_t* blk = sA + as * kABlk;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int r = (tid >> 3) + h2 * 64;
          const float2 sr = sStats[r];
          const float af[8] = {av[h2][0].x, av[h2][0].y, av[h2][0].z, av[h2][0].w,
                               av[h2][1].x, av[h2][1].y, av[h2][1].z, av[h2][1].w};
          const float uf[8] = {uv[h2][0].x, uv[h2][0].y, uv[h2][0].z, uv[h2][0].w,
                               uv[h2][1].x, uv[h2][1].y, uv[h2][1].z, uv[h2][1].w};
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float g0 = fmaf((af[2 * e] - sr.x) * sr.y, gm[2 * e], bt[2 * e]) * uf[2 * e];
            const float g1 =
                fmaf((af[2 * e + 1] - sr.x) * sr.y, gm[2 * e + 1], bt[2 * e + 1]) * uf[2 * e + 1];
            w[e] = pack_h2(g0, g1);
          }
          // rows past the end carry zeros (their statistics and data are zero);
          // columns 4j.. sit in chunk j / 2, 32 + 4j.. in chunk 4 + j / 2
          if (ok) {
            const int half8 = (j & 1) * 8;
            *reinterpret_cast<uint2*>(blk + r * 128 + (((j >> 1) ^ (r & 7)) << 4) + half8) =
                make_uint2(w[0], w[1]);
            *reinterpret_cast<uint2*>(blk + r * 128 + (((4 + (j >> 1)) ^ (r & 7)) << 4) + half8) =
                make_uint2(w[2], w[3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();  // the previous tile's tensor-memory reads, before the MMAs reuse it
        mbar_arrive(&bars[BAR_T_A_FULL + as]);
        if (++as == kAS) { as = 0; aph ^= 1u; }
      }
      // epilogue: + b2 + residual -> Y (fp32) and its 16-bit copy
      if (ok) ok = mbar_wait(&bars[BAR_T_ACC_FULL], static_cast<uint32_t>(mt) & 1u, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) continue;  // keep arriving: the other threads' barriers stay consistent
      tc_fence_after();
      // Each warp owns rows base + 32 q4 .. + 31 (its tensor-memory lane
      // quarter) and 128 columns.  Per 32-column chunk the accumulators go
      // through a 128B-swizzled 32 x 32 staging block, so that the residual
      // loads and the Y stores run along rows: lane l takes row 4k + l / 8 and
      // columns 4 (l % 8) .. + 3 of the chunk, one 128-byte row segment per 8
      // lanes.  Y = (accumulator + b2) + residual, the unfused epilogue's order.
      uint8_t* stg = smem + AttnSmem::kTailStage + warp * 4096;
      const int r0 = base + q4 * 32;          // first row of this warp (within the user)
      const int rsub = lane >> 3, j4 = lane & 7;
      const bool h16 = t.ylp_f16 != 0;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        const int col = cg * 128 + ch * 32;
        if (col >= t.N) break;  // warp-uniform
        uint32_t v[32];
        __syncwarp();
        tmem_ld32(tmem + lane_off + static_cast<uint32_t>(col), v);
        tmem_ld_wait(v);
        // row `lane` of the block: 16-byte chunk q at (q ^ (lane & 7))
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<uint4*>(stg + lane * 128 + ((q ^ (lane & 7)) << 4)) =
              make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        __syncwarp();
        const float4 bb = __ldg(reinterpret_cast<const float4*>(t.b2 + col) + j4);
#pragma unroll 2
        for (int k = 0; k < 8; ++k) {
          const int rr = 4 * k + rsub;
          if (r0 + rr < n_q) {
            const int64_t grow = q_start + r0 + rr;
            const float4 a = *reinterpret_cast<const float4*>(stg + rr * 128 + ((j4 ^ (rr & 7)) << 4));
            float4 xx;
            if (t.x_res != nullptr) {
              xx = *reinterpret_cast<const float4*>(t.x_res + grow * t.ld_x + col + 4 * j4);
            } else {
              const uint2 xb = *reinterpret_cast<const uint2*>(t.x_lp + grow * t.ld_x + col + 4 * j4);
              const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xb.x));
              const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xb.y));
              xx = make_float4(f0.x, f0.y, f1.x, f1.y);
            }
            float4 y;
            y.x = a.x + bb.x + xx.x;
            y.y = a.y + bb.y + xx.y;
            y.z = a.z + bb.z + xx.z;
            y.w = a.w + bb.w + xx.w;
            *reinterpret_cast<float4*>(t.y + grow * t.ld_y + col + 4 * j4) = y;
            if (t.y_lp != nullptr) {
              auto pk2 = [h16](float a0, float a1) { return h16 ? pack_h2(a0, a1) : pack_bf16x2(a0, a1); };
              *reinterpret_cast<uint2*>(static_cast<uint16_t*>(t.y_lp) + grow * t.ld_y + col + 4 * j4) =
                  make_uint2(pk2(y.x, y.y), pk2(y.z, y.w));
            }
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------- kernel

// F16: Q, K, V (and so P) are fp16 instead of bf16.  The causal element math
// is fp32 either way; candidate mode with fp16 operands runs it on packed fp16
// pairs (its per-key bias is precomputed, so the chain is short).
// FUSED (causal mode only): the last head CTA of each query tile pair runs
// the layer's f2 for the pair's rows (attn_f2_tail; tm_w2 maps the fp16 W2).
template <bool CAND, int PHI, bool PAIRS, bool F16, bool FUSED>
__global__ void __launch_bounds__(ATT_THREADS, 1)
hstu_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w2,
                 const __grid_constant__ AttnParams p) {
  static_assert(!(CAND && FUSED), "the fused f2 tail is for the causal layer path");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));

  const int h = blockIdx.x;
  const int u = blockIdx.y;
  const int qp = p.num_qpairs - 1 - static_cast<int>(blockIdx.z);  // longest work first
  const int64_t kv_start = p.kv_offsets[u];
  const int n_kv = static_cast<int>(p.kv_offsets[u + 1] - kv_start);
  int64_t q_start;
  int n_q;
  if constexpr (CAND) {
    q_start = p.q_offsets[u];
    n_q = static_cast<int>(p.q_offsets[u + 1] - q_start);
  } else {
    q_start = kv_start;
    n_q = n_kv;
  }
  // The grid and the staged position table are sized from the host-declared
  // maximum lengths; a user longer than declared would leave rows unwritten
  // or read past the staged table, so it is reported and nothing runs.
  if (n_q > p.max_q || n_kv > p.max_kv || n_q < 0 || n_kv < 0) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0) record_status(HSTU_ERR_DEVICE_CHECK);
    return;  // uniform across the CTA, before any allocation
  }
  // Generalised (MTGR-style) masks: the user's tokens are U+S (n_us), R (n_r),
  // then candidates.  Every row sees a prefix of the keys (U+S rows: the U+S
  // block; R rows: up to themselves; candidate rows: U+S and the R events up
  // to their own time) and candidate rows also themselves, added like the
  // candidate-mode self term.
  const bool masked = !CAND && p.segments != nullptr;
  int n_us = 0, r_end = n_kv;  // plain causal: every row is an R row
  if (masked) {
    n_us = p.segments[2 * u];
    const int n_r = p.segments[2 * u + 1];
    if (n_us < 0 || n_r < 0 || n_us + n_r > n_kv || n_us > p.max_static) {
      if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0) record_status(HSTU_ERR_DEVICE_CHECK);
      return;  // uniform across the CTA, before any allocation
    }
    r_end = n_us + n_r;
  }
  const int q0 = qp * 2 * ATT_ROWS;
  if (q0 >= n_q) return;  // uniform across the CTA, before any allocation
  const bool has_b = (q0 + ATT_ROWS) < n_q;

  // The softmax ablation takes two passes over the key tiles: the first finds
  // each row's max and sum, the second writes P and runs P V.  Stage index
  // si = pass * nk_total + tile.
  constexpr bool kSoftmax = PHI == HSTU_ACT_SOFTMAX;
  constexpr int kPasses = kSoftmax ? 2 : 1;

  // number of key tiles each query tile consumes
  int nA, nB;
  if constexpr (CAND) {
    const int nk = (n_kv + ATT_KEYS - 1) / ATT_KEYS;
    nA = nk;
    nB = has_b ? nk : 0;
  } else if (!masked) {
    nA = (q0 + ATT_ROWS) / ATT_KEYS;      // keys 0 .. q0 + 127
    nB = has_b ? (q0 + 2 * ATT_ROWS) / ATT_KEYS : 0;
  } else {
    // exclusive end of the keys any row in [r0, r0 + 128) sees
    auto tile_end = [&](int r0) -> int {
      if (r0 >= n_q) return 0;
      const int r1 = min(r0 + ATT_ROWS, n_q);
      int e = 0;
      if (r0 < n_us) e = n_us;                                   // U+S rows
      if (r1 > n_us && r0 < r_end) e = max(e, min(r1, r_end));   // R rows
      if (r1 > r_end) e = max(e, r_end);                         // candidate rows
      return e;
    };
    nA = (tile_end(q0) + ATT_KEYS - 1) / ATT_KEYS;
    nB = (tile_end(q0 + ATT_ROWS) + ATT_KEYS - 1) / ATT_KEYS;
    // two passes look three items ahead across the pass boundary; the ring
    // of stages holds that only while tile A takes at most two fewer key
    // tiles than tile B, so tile A then walks tile B's (masked) tiles too
    if (kSoftmax && has_b && nB - nA > 2) nA = nB;
    if (kSoftmax && has_b && nA - nB > 2) nB = nA;
  }
  const int nk_total = nA > nB ? nA : nB;
  const int n_stages = kPasses * nk_total;

  // causal rows read position offsets i - j in [-127, q0 + 255]; candidates
  // read n_kv - j in [1, n_kv].  The staged table holds scale * rab_pos at
  // index x = D - (i - j).
  const int D = CAND ? n_kv : q0 + 2 * ATT_ROWS;
  constexpr float kScale = phi_scale<PHI>();

  uint8_t* sQ = smem + AttnSmem::kQ;
  uint8_t* sK = smem + AttnSmem::kK;
  uint8_t* sV = smem + AttnSmem::kV;
  uint8_t* sKey = smem + AttnSmem::kKeyInfo;
  float* sTime = reinterpret_cast<float*>(smem + AttnSmem::kTimeTab);
  int64_t* sThr = reinterpret_cast<int64_t*>(smem + AttnSmem::kThr);
  int32_t* sThr32 = reinterpret_cast<int32_t*>(smem + AttnSmem::kThr32);
  int4* sOct = reinterpret_cast<int4*>(smem + AttnSmem::kOct);
  float4* sOrt = reinterpret_cast<float4*>(smem + AttnSmem::kOrt);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AttnSmem::kBars);
  uint32_t* sTmemBase = reinterpret_cast<uint32_t*>(smem + AttnSmem::kMisc);
  float2* sLnX = reinterpret_cast<float2*>(smem + AttnSmem::kLnX);
  float2* sML = reinterpret_cast<float2*>(smem + AttnSmem::kML);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + AttnSmem::kMisc + 4);
  float* sRv = reinterpret_cast<float*>(smem + AttnSmem::kPos);

  const int warp = warp_id();
  const int lane = lane_id();
  const int tid = threadIdx.x;

  // key times are kept as int32 seconds since the user's first event; a user
  // spanning 2^31 - 1 seconds (68 years) or more is outside the contract and
  // is reported through the device status word (times are then clamped)
  const int64_t t_first = n_kv > 0 ? p.timestamps[kv_start] : 0;
  if (!CAND && n_kv > 0 && tid == 0 &&
      p.timestamps[kv_start + n_kv - 1] - t_first >= static_cast<int64_t>(INT32_MAX) - 1)
    record_status(HSTU_ERR_DEVICE_CHECK);

  // ---------------- setup
  if (tid == 0) {
    mbar_init(&bars[BAR_Q_FULL], 1);  // the producer's expect-tx arrival + the Q bytes
    for (int s = 0; s < ATT_STAGES; ++s) {
      mbar_init(&bars[BAR_KV_FULL + s], 2);
      mbar_init(&bars[BAR_KV_EMPTY + s], 2);  // one commit per issuer
    }
    for (int g = 0; g < 2; ++g) {
      // one S-ready and one P-ready barrier per S buffer: S of tile k+3 is
      // only issued once P of tile k has been seen, so no barrier can run a
      // phase ahead of its waiters
      for (int b = 0; b < ATT_SBUF; ++b) {
        mbar_init(&bars[BAR_S_FULL + ATT_SBUF * g + b], 1);
        mbar_init(&bars[BAR_P_FULL + ATT_SBUF * g + b], 2 * ATT_ROWS);  // both column halves
      }
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&bars[BAR_O_FULL + g], 1);
      mbar_init(&bars[BAR_DONE + g], 1);
    }
    if constexpr (FUSED) {
      for (int st = 0; st < AttnSmem::kTailAStages; ++st) {
        mbar_init(&bars[BAR_T_A_FULL + st], 16 * 32);  // every element thread
        mbar_init(&bars[BAR_T_A_EMPTY + st], 1);
      }
      for (int st = 0; st < AttnSmem::kTailWStages; ++st) {
        mbar_init(&bars[BAR_T_W_FULL + st], 1);
        mbar_init(&bars[BAR_T_W_EMPTY + st], 1);
      }
      mbar_init(&bars[BAR_T_ACC_FULL], 1);
      mbar_init(&bars[BAR_T_DONE], 1);
    }
    *sAbort = 0;
    fence_mbar_init();
  }
  if (warp == ATT_MMA_WARP) {
    tmem_alloc(sTmemBase, 512);
    tmem_relinquish();
  }
  {
    const float* rp = p.rab_pos + static_cast<int64_t>(h) * p.P;
    // offsets i - j down to -(keys after the row a chunk reads): 127 + 2 in
    // causal mode, up to the U+S block (+ a chunk) with the generalised masks;
    // the bucket of an offset d is min(|d|, P - 1)
    const int xend = min(p.pos_len, D + (masked ? max(ATT_ROWS, p.max_static + 2 * 32) : ATT_ROWS) + 2);
    for (int x = tid; x < xend; x += ATT_THREADS) {
      const int d0 = D - x;  // copy 0 holds offset D - x
      sRv[x] = kScale * rp[min(abs(d0), p.P - 1)];
      if constexpr (PAIRS) {
        const int d1 = D + 1 - x;  // copy 1 holds offset D + 1 - x
        sRv[p.pos_len + x] = kScale * rp[min(abs(d1), p.P - 1)];
      }
    }
  }
  for (int k = tid; k < p.Tb; k += ATT_THREADS) {
    sTime[k] = kScale * p.rab_time[static_cast<int64_t>(h) * p.Tb + k];
    sThr[k] = p.thr[k];
    sThr32[k] = p.thr[k] < static_cast<int64_t>(INT32_MAX) ? static_cast<int32_t>(p.thr[k]) : INT32_MAX;
  }
  if (tid < 32) {
    const int4 o = p.oct[tid];
    sOct[tid] = o;
    const float* rt = p.rab_time + static_cast<int64_t>(h) * p.Tb;
    auto tb = [&](int b) { return kScale * rt[min(max(b, 0), p.Tb - 1)]; };
    sOrt[tid] = make_float4(tb(o.w), tb(o.w + 1), tb(o.w + 2), tb(o.w + 3));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmemBase;
  const WaitCtl ctl{sAbort, p.timeout_ns};

  if (warp == ATT_PRODUCER_WARP) {
    // ---------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      // both query tiles (rows past the tensor's end read as zeros; rows of
      // the next user are loaded but their results are never stored)
      mbar_arrive_expect_tx(&bars[BAR_Q_FULL], 2 * ATT_Q_BYTES);
      const int64_t qrow = q_start + q0;  // < 2^31 (row counts are checked on the host)
      const int64_t qrow_b = min(qrow + ATT_ROWS, static_cast<int64_t>(INT32_MAX));
      tma_load_2d(sQ, &tm_q, &bars[BAR_Q_FULL], h * ATT_HD, static_cast<int32_t>(qrow));
      tma_load_2d(sQ + ATT_Q_BYTES, &tm_q, &bars[BAR_Q_FULL], h * ATT_HD,
                  static_cast<int32_t>(qrow_b));
    }
    int64_t t_req = 0;
    if constexpr (CAND) t_req = p.request_ts[u];
    int issued = 0;
    // the key timestamps of the next tile are loaded one tile ahead, so that
    // their global-memory latency overlaps the wait for a free stage and the
    // current tile's work
    constexpr int KPL = ATT_KEYS / 32;  // keys per lane per tile
    int64_t ts_next[KPL];
    auto load_ts = [&](int kt, int64_t (&t)[KPL]) {
#pragma unroll
      for (int e = 0; e < KPL; ++e) {
        const int j = kt * ATT_KEYS + lane + 32 * e;
        t[e] = j < n_kv ? p.timestamps[kv_start + j] : 0;
      }
    };
    if (n_stages > 0) load_ts(0, ts_next);
    for (int si = 0; si < n_stages; ++si) {
      const int kt = si % nk_total;                // key tile
      const bool last_pass = si >= (kPasses - 1) * nk_total;
      const int s = si % ATT_STAGES;
      int64_t ts[KPL];
#pragma unroll
      for (int e = 0; e < KPL; ++e) ts[e] = ts_next[e];
      if (si + 1 < n_stages) load_ts((si + 1) % nk_total, ts_next);
      const uint32_t par = (static_cast<uint32_t>(si / ATT_STAGES) & 1u) ^ 1u;
      int ok = 0;
      if (lane == 0) ok = mbar_wait(&bars[BAR_KV_EMPTY + s], par, ctl) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (lane == 0) {
        // V is only read by P V, in the last pass
        mbar_arrive_expect_tx(&bars[BAR_KV_FULL + s], (last_pass ? 2 : 1) * ATT_TILE_BYTES);
        const int32_t row = static_cast<int32_t>(kv_start + kt * ATT_KEYS);
        tma_load_2d(sK + s * ATT_TILE_BYTES, &tm_k, &bars[BAR_KV_FULL + s], h * ATT_HD, row);
        if (last_pass)
          tma_load_2d(sV + s * ATT_TILE_BYTES, &tm_v, &bars[BAR_KV_FULL + s], h * ATT_HD, row);
      }
      ++issued;
      uint8_t* key = sKey + s * AttnSmem::kKeyStride;
#pragma unroll
      for (int e = 0; e < KPL; ++e) {
        const int c = lane + 32 * e;
        const int j = kt * ATT_KEYS + c;
        if constexpr (CAND) {
          // the whole per-key bias: candidates share position n_kv and time t_req
          float r = 0.0f;
          if (j < n_kv) {
            const int64_t dt = t_req - ts[e];
            const int b = (dt >= 0 && dt < static_cast<int64_t>(INT32_MAX) - 1)
                              ? time_bucket_octave(static_cast<int32_t>(dt), sOct)
                              : time_bucket_search(dt, sThr, p.Tb);
            r = sRv[j] + sTime[b];
          }
          if constexpr (F16) reinterpret_cast<__half*>(key)[c] = __float2half_rn(r);
          else reinterpret_cast<float*>(key)[c] = r;
        } else {
          int32_t rel = INT32_MAX;
          if (j < n_kv) {
            const int64_t d = ts[e] - t_first;
            rel = d >= static_cast<int64_t>(INT32_MAX) - 1 ? INT32_MAX - 1 : static_cast<int32_t>(d);
          }
          reinterpret_cast<int32_t*>(key)[c] = rel;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[BAR_KV_FULL + s]);
    }
    // drain: every issued load must land before shared memory is released
    if (lane == 0) {
      mbar_wait_drain(&bars[BAR_Q_FULL], 0, p.timeout_ns);
      for (int kt = max(0, issued - ATT_STAGES); kt < issued; ++kt)
        mbar_wait_drain(&bars[BAR_KV_FULL + kt % ATT_STAGES],
                        static_cast<uint32_t>(kt / ATT_STAGES) & 1u, p.timeout_ns);
    }
  } else if (warp >= ATT_MMA_WARP) {
    // ---------------- MMA issuers, one warp per query tile: the whole warp
    // runs the loop (waits are warp votes), one elected lane issues
    const int g = warp - ATT_MMA_WARP;
    {
      const bool leader = elect_one();
      constexpr uint32_t idesc_qk = idesc_16_f32(ATT_ROWS, ATT_KEYS, false, false, F16);
      constexpr uint32_t idesc_pv = idesc_16_f32(ATT_ROWS, ATT_HD, false, true, F16);
      const int nWg = g == 0 ? nA : nB;
      // tensor memory: S buffers (P over them) and O of this tile
      const uint32_t tS = tmem + static_cast<uint32_t>(g * ATT_SBUF * 64);
      const uint32_t tOg = tmem + static_cast<uint32_t>(2 * ATT_SBUF * 64 + g * 64);
      // this tile's Q, and the K/V descriptors of stage 0; stage s adds
      // s * 8 KB (s * 512 in 16-byte units) to the start-address field
      const uint64_t dQ = smem_desc_sw128(smem_u32(sQ + g * ATT_Q_BYTES), 16, 1024);
      const uint64_t dK0 = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(smem_u32(sV), 8192, 1024);
      constexpr uint64_t kStageDesc = ATT_TILE_BYTES >> 4;
      auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, par, ctl));
      };
      bool ok = wait_all(&bars[BAR_Q_FULL], 0);
      tc_fence_after();
      int kv_ready = 0;  // key tiles whose K/V this warp has seen land
      auto await_kv = [&](int kt) -> bool {
        while (kv_ready <= kt) {
          if (!wait_all(&bars[BAR_KV_FULL + kv_ready % ATT_STAGES],
                        static_cast<uint32_t>(kv_ready / ATT_STAGES) & 1u))
            return false;
          tc_fence_after();
          ++kv_ready;
        }
        return true;
      };
      // S of tile kt into buffer b = kt mod 3
      auto issue_s = [&](int kt, int b) {
        const uint64_t dk = dK0 + static_cast<uint64_t>(kt % ATT_STAGES) * kStageDesc;
        const uint32_t d = tS + static_cast<uint32_t>(b * 64);
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < ATT_HD / 16; ++kk)
            mma_bf16_ss(d, dQ + 2 * kk, dk + 2 * kk, idesc_qk, kk > 0 ? 1u : 0u);
          mma_commit(&bars[BAR_S_FULL + ATT_SBUF * g + b]);
        }
        __syncwarp();
      };
      // O += P(kt) V(kt) from stage si; P of keys 0-31 sits at columns 0-15
      // of the S buffer, P of keys 32-63 at columns 32-47
      auto issue_pv = [&](int kt, int si, int b) {
        const uint64_t dv = dV0 + static_cast<uint64_t>(si % ATT_STAGES) * kStageDesc;
        const uint32_t a = tS + static_cast<uint32_t>(b * 64);
        const uint32_t acc0 = kt > 0 ? 1u : 0u;
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < ATT_KEYS / 16; ++kk)
            mma_bf16_ts(tOg, a + (kk >> 1) * 32 + (kk & 1) * 8, dv + 128 * kk, idesc_pv,
                        kk > 0 ? 1u : acc0);
        }
        __syncwarp();
      };
      // This tile's items: its nWg key tiles, once per pass; item gi reads
      // stage stage_of(gi).  (With two passes the look-ahead of three items
      // reaches at most nB - nA + 3 = 5 stages past the current one, inside
      // the ring of ATT_STAGES.)
      const int n_items = kPasses * nWg;
      auto stage_of = [&](int gi) -> int {
        return gi < nWg ? gi : nk_total + (gi - nWg);
      };
      // three items ahead: S of items 0, 1, 2 before any P exists
      for (int t = 0; ok && t < ATT_SBUF && t < n_items; ++t) {
        ok = await_kv(stage_of(t));
        if (ok) issue_s(stage_of(t), t);
      }
      int b = 0;         // buffer of item gi
      uint32_t ph = 0;   // phase parity of that buffer's barriers at item gi
      int gi = 0;
      for (int si = 0; ok && si < n_stages; ++si) {
        const int kt = si % nk_total;
        if (kt < nWg) {
          ok = wait_all(&bars[BAR_P_FULL + ATT_SBUF * g + b], ph);
          if (!ok) break;
          tc_fence_after();
          if (si >= (kPasses - 1) * nk_total) issue_pv(kt, si, b);  // last pass: P V
          if (gi + ATT_SBUF < n_items) {
            const int sn = stage_of(gi + ATT_SBUF);
            ok = await_kv(sn);
            if (!ok) break;
            issue_s(sn, b);  // into the buffer P V(kt) has just been issued to read
          }
          ++gi;
          if (++b == ATT_SBUF) {
            b = 0;
            ph ^= 1u;
          }
        } else {
          // past this tile's last key tile: the release below must still
          // follow the stage's load, so it counts toward this tile's phase
          ok = await_kv(si);
          if (!ok) break;
        }
        if (leader) mma_commit(&bars[BAR_KV_EMPTY + si % ATT_STAGES]);
        __syncwarp();
      }
      if (leader) {
        mma_commit(&bars[BAR_O_FULL + g]);
        // every MMA of this warp must be complete before TMEM is released
        mma_commit(&bars[BAR_DONE + g]);
      }
      __syncwarp();
      mbar_wait_drain(&bars[BAR_DONE + g], 0, p.timeout_ns);
    }
    __syncwarp();
  } else {
    // ---------------- element groups
    const int g = warp >> 3;               // 0 = tile A, 1 = tile B
    const int half = (warp >> 2) & 1;      // key columns 32*half .. 32*half + 31 of each tile
    const int r = tid & (ATT_ROWS - 1);    // row within the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    // this half's 32 columns of S buffer 0 (+64 per buffer)
    const uint32_t tS0 = tmem + lane_off + static_cast<uint32_t>(g * ATT_SBUF * 64 + half * 32);
    const uint32_t tO =
        tmem + lane_off + static_cast<uint32_t>(2 * ATT_SBUF * 64 + g * 64 + half * 32);
    const int i = q0 + g * ATT_ROWS + r;   // query index within the user
    const bool valid = i < n_q;
    const int nW = g == 0 ? nA : nB;
    bool ok = true;
    const uint64_t scale2 = f2_pack(kScale, kScale);
    const uint32_t scale_h2 = h2_splat(kScale);

    // causal: per-row time-bucket walk and staged position-table copy
    BucketWalk<int32_t> w32;
    float rt_cur = 0.0f;  // time bias of the walk's current bucket
    int copy = 0;
    const float* rv = sRv;
    // keys this row sees: the prefix [0, vis_end), and itself when self_row
    int vis_end = i + 1;
    bool self_row = false;
    if constexpr (!CAND) {
      const int64_t d = (valid ? p.timestamps[kv_start + i] : t_first) - t_first;
      if (valid && d >= static_cast<int64_t>(INT32_MAX) - 1) record_status(HSTU_ERR_DEVICE_CHECK);
      w32.init(d >= static_cast<int64_t>(INT32_MAX) - 1 ? INT32_MAX - 1 : static_cast<int32_t>(d), 0,
               sThr, sThr32, p.Tb);
      if constexpr (PAIRS) copy = (D - i) & 1;
      rv = sRv + copy * p.pos_len;
      rt_cur = sTime[w32.b];
      if (masked && valid) {
        if (i < n_us) {
          vis_end = n_us;
        } else if (i >= r_end) {
          // a candidate: the R events at or before its own time (R is time-ordered)
          const int64_t t_i = p.timestamps[kv_start + i];
          int lo = n_us, hi = r_end;
          while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (p.timestamps[kv_start + mid] <= t_i) lo = mid + 1;
            else hi = mid;
          }
          vis_end = lo;
          self_row = true;
        }
      }
    }

    // this half's 32 keys of tile kt: S values in `sv`, packed 16-bit P pairs to `pk`
    auto chunk = [&](const uint32_t (&sv)[32], uint32_t (&pk)[16], int kt, int s) {
      const uint8_t* key = sKey + s * AttnSmem::kKeyStride;
      const int j0 = kt * ATT_KEYS + half * 32;  // key index of column 0
      if constexpr (CAND) {
        if constexpr (F16) {
          const __half* kr = reinterpret_cast<const __half*>(key) + half * 32;
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const uint32_t s16 =
                f2_to_h2(f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])));
            pk[c >> 1] = phi_h2<PHI>(h2_fma(s16, scale_h2, lds_b32(kr + c)));
          }
        } else {
          const float* kr = reinterpret_cast<const float*>(key) + half * 32;
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const uint64_t h2 = f2_fma(f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])),
                                       scale2, lds_b64(kr + c));
            pk[c >> 1] = phi_pair<PHI, false>(h2);
          }
        }
        const int last = n_kv - 1 - j0;  // last live column
        if (last < 31) {
#pragma unroll
          for (int c = 0; c < 32; c += 2) pk[c >> 1] = mask_pair(pk[c >> 1], c, last);
        }
      } else {
        // last visible column: keys past the row's visible prefix are masked;
        // rows past the user's end are not stored and skip the work
        const int lim = !valid ? -1 : vis_end - 1 - j0;
        const int32_t* kts = reinterpret_cast<const int32_t*>(key) + half * 32;
        const int xc = D - i + j0 + copy;  // table index at column 0
        causal_chunk_pointwise<PHI, PAIRS, F16>(sv, pk, rv + xc, kts, lim, w32, sTime, sThr32,
                                                sOct, sOrt, scale2, rt_cur);
      }
    };

    // candidate mode: the candidate's own key/value enters with position
    // bucket 0 and time bucket 0
    const int64_t row = q_start + i;
    auto to_f2 = [](uint32_t w) -> float2 {  // a packed pair of the operand type
      if constexpr (F16) return __half22float2(*reinterpret_cast<const __half2*>(&w));
      else return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
    };
    auto self_dot = [&]() -> float {
      const uint16_t* qs = static_cast<const uint16_t*>(p.q_self) + row * p.ld_qs + h * ATT_HD;
      const uint16_t* ks = static_cast<const uint16_t*>(p.k_self) + row * p.ld_ks + h * ATT_HD;
      float dot = 0.0f;
#pragma unroll
      for (int c = 0; c < ATT_HD; c += 8) {
        const uint4 qa = *reinterpret_cast<const uint4*>(qs + c);
        const uint4 ka = *reinterpret_cast<const uint4*>(ks + c);
        const uint32_t qw[4] = {qa.x, qa.y, qa.z, qa.w};
        const uint32_t kw[4] = {ka.x, ka.y, ka.z, ka.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float2 qf = to_f2(qw[t]);
          const float2 kf = to_f2(kw[t]);
          dot = fmaf(qf.x, kf.x, dot);
          dot = fmaf(qf.y, kf.y, dot);
        }
      }
      return dot;
    };
    auto self_rab = [&]() -> float {
      return p.rab_pos[static_cast<int64_t>(h) * p.P] + p.rab_time[static_cast<int64_t>(h) * p.Tb];
    };

    // ---- softmax ablation: running max and sum of 2^h over this half's keys
    // (h = (s + rab) log2 e); the first pass only reads S, the second writes
    // P = 2^(h - m - log2 l)
    float sm_m = -INFINITY, sm_l = 0.0f;
    float h_self = -INFINITY;  // candidate mode: the own key's pre-activation
    if (kSoftmax && (CAND || self_row)) {
      if (valid) h_self = kScale * (self_dot() + self_rab());
      if (half == 0 && valid) {
        sm_m = h_self;
        sm_l = 1.0f;
      }
    }
    // fold the scaled pre-activations of one chunk (pairs in hh, columns
    // above `last` invisible) into (sm_m, sm_l)
    auto softmax_accumulate = [&](const uint64_t (&hh)[16], int last) {
      if (last < 0) return;
      float cm = -INFINITY;
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        float a, bb;
        f2_unpack(hh[q], a, bb);
        if (2 * q <= last) cm = fmaxf(cm, a);
        if (2 * q + 1 <= last) cm = fmaxf(cm, bb);
      }
      if (cm > sm_m) {
        sm_l *= ex2_approx(sm_m - cm);
        sm_m = cm;
      }
      const uint64_t neg = f2_pack(-sm_m, -sm_m);
      float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        float a, bb;
        f2_unpack(f2_add(hh[q], neg), a, bb);
        const float e0 = ex2_approx(a), e1 = ex2_approx(bb);
        acc0 += (2 * q <= last) ? e0 : 0.0f;
        acc1 += (2 * q + 1 <= last) ? e1 : 0.0f;
      }
      sm_l += acc0 + acc1;
    };
    // pre-activations of keys 32*half .. 32*half + 31 of tile kt (fp32 pairs)
    // and the last visible column
    auto chunk_h = [&](const uint32_t (&sv)[32], uint64_t (&hh)[16], int kt, int s) -> int {
      const uint8_t* key = sKey + s * AttnSmem::kKeyStride;
      const int j0 = kt * ATT_KEYS + half * 32;
      if constexpr (CAND) {
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          uint64_t bias;
          if constexpr (F16) {
            const float2 bf = __half22float2(
                *reinterpret_cast<const __half2*>(reinterpret_cast<const __half*>(key) + half * 32 + c));
            bias = f2_pack(bf.x, bf.y);
          } else {
            bias = lds_b64(reinterpret_cast<const float*>(key) + half * 32 + c);
          }
          hh[c >> 1] = f2_fma(f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), scale2, bias);
        }
        return valid ? min(31, n_kv - 1 - j0) : -1;
      } else {
        const int lim = !valid ? -1 : vis_end - 1 - j0;
        causal_chunk<PAIRS>(
            sv, [&](int c, uint64_t hv) { hh[c >> 1] = hv; }, rv + (D - i + j0 + copy),
            reinterpret_cast<const int32_t*>(key) + half * 32, lim, w32, sTime, sThr32, sOct,
            sOrt, scale2, rt_cur);
        return lim < 31 ? lim : 31;
      }
    };

    int buf = 0;        // S buffer of the current item (item index mod 3)
    uint32_t ph = 0;    // its barriers' phase parity
    // one pass over this tile's nW key tiles; stage of tile kt in pass `pass`
    // is pass * nk_total + kt
    auto run_pass = [&](int pass) {
      for (int kt = 0; kt < nW; ++kt) {
        const int si = pass * nk_total + kt;
        const int s = si % ATT_STAGES;
        ok = mbar_wait(&bars[BAR_S_FULL + ATT_SBUF * g + buf], ph, ctl);
        // the producer's per-key side data for this stage (already complete)
        if (ok)
          ok = mbar_wait(&bars[BAR_KV_FULL + s], static_cast<uint32_t>(si / ATT_STAGES) & 1u, ctl);
        ok = __all_sync(0xffffffffu, ok);  // TMEM loads below are warp-collective
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = tS0 + static_cast<uint32_t>(buf * 64);
        // 32 keys: TMEM -> registers -> bias, phi2, mask -> P over this half's S
        uint32_t sa[32];
        tmem_ld32(tS, sa);
        tmem_ld_wait(sa);
        if (kSoftmax && pass == 0) {
          uint64_t hh[16];
          const int last = chunk_h(sa, hh, kt, s);
          softmax_accumulate(hh, last);
        } else if constexpr (kSoftmax) {
          uint64_t hh[16];
          const int last = chunk_h(sa, hh, kt, s);
          uint32_t pk[16];
          const uint64_t neg = f2_pack(-sm_m, -sm_m);
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            float a, bb;
            f2_unpack(f2_add(hh[q], neg), a, bb);
            const uint64_t e2 = f2_pack(ex2_approx(a), ex2_approx(bb));
            if constexpr (F16) pk[q] = f2_to_h2(e2);
            else pk[q] = f2_to_bf16x2(e2);
          }
          if (last < 0) {
#pragma unroll
            for (int q = 0; q < 16; ++q) pk[q] = 0u;
          } else if (last < 31) {
#pragma unroll
            for (int c = 0; c < 32; c += 2) pk[c >> 1] = mask_pair(pk[c >> 1], c, last);
          }
          __syncwarp();
          tmem_st16(tS, pk);
          tmem_st_wait();
        } else {
          uint32_t pk[16];
          chunk(sa, pk, kt, s);
          __syncwarp();
          tmem_st16(tS, pk);
          tmem_st_wait();
        }
        tc_fence_before();
        mbar_arrive(&bars[BAR_P_FULL + ATT_SBUF * g + buf]);
        if (++buf == ATT_SBUF) {
          buf = 0;
          ph ^= 1u;
        }
      }
    };
    if constexpr (kSoftmax) {
      run_pass(0);
      // merge the two halves' (max, sum) of each row; every thread of the
      // group's 256 reaches this barrier (a failed wait only skips work)
      sML[(g * 2 + half) * ATT_ROWS + r] = make_float2(sm_m, sm_l);
      named_barrier_sync(1 + g, 2 * ATT_ROWS);
      const float2 other = sML[(g * 2 + (half ^ 1)) * ATT_ROWS + r];
      const float m = fmaxf(sm_m, other.x);
      float l = 0.0f;
      if (m > -INFINITY) l = sm_l * ex2_approx(sm_m - m) + other.y * ex2_approx(other.x - m);
      // P = 2^(h - m) / l = 2^(h - (m + log2 l)); rows with no visible key keep P = 0
      sm_m = l > 0.0f ? m + lg2_approx(l) : INFINITY;
      named_barrier_sync(1 + g, 2 * ATT_ROWS);  // both halves have read before reuse
      if constexpr (!CAND) {
        // the second pass walks the time buckets from the first key again
        const int64_t d = (valid ? p.timestamps[kv_start + i] : t_first) - t_first;
        w32.init(d >= static_cast<int64_t>(INT32_MAX) - 1 ? INT32_MAX - 1 : static_cast<int32_t>(d),
                 0, sThr, sThr32, p.Tb);
        rt_cur = sTime[w32.b];
      }
      if (ok) run_pass(1);
    } else {
      run_pass(0);
    }

    // ---------------- epilogue: O / N, LayerNorm partial sums, store
    // Each half finishes its 32 columns of O; the two halves' (sum, centred
    // sum of squares) merge by the pairwise update for equal counts:
    // M2 = M2_0 + M2_1 + (mean_0 - mean_1)^2 * 32 * 32 / 64.
    constexpr int HC = ATT_HD / 2;
    float o[HC];
    if (ok && nW > 0) ok = mbar_wait(&bars[BAR_O_FULL + g], 0, ctl);
    ok = __all_sync(0xffffffffu, ok);
    float hsum = 0.0f, hm2 = 0.0f;
    if (ok) {
      if (nW > 0) {
        tc_fence_after();
        uint32_t ov[32];
        tmem_ld32(tO, ov);
        tmem_ld_wait(ov);
#pragma unroll
        for (int c = 0; c < HC; ++c) o[c] = __uint_as_float(ov[c]);
      } else {
#pragma unroll
        for (int c = 0; c < HC; ++c) o[c] = 0.0f;
      }
      if (valid) {
        if (CAND || self_row) {
          // the candidate's own key/value: position bucket 0, time bucket 0
          const uint16_t* vs =
              static_cast<const uint16_t*>(p.v_self) + row * p.ld_vs + h * ATT_HD + half * HC;
          float ps;
          if constexpr (kSoftmax) ps = ex2_approx(h_self - sm_m);  // already divided by the sum
          else ps = apply_phi<PHI>(self_dot() + self_rab());
#pragma unroll
          for (int c = 0; c < HC; c += 8) {
            const uint4 va = *reinterpret_cast<const uint4*>(vs + c);
            const uint32_t vw[4] = {va.x, va.y, va.z, va.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const float2 vf = to_f2(vw[t]);
              o[c + 2 * t] = fmaf(ps, vf.x, o[c + 2 * t]);
              o[c + 2 * t + 1] = fmaf(ps, vf.y, o[c + 2 * t + 1]);
            }
          }
        }
        // pointwise phi2 divides by N = n_u; softmax weights are normalised already
        const float inv_n =
            kSoftmax ? 1.0f : 1.0f / static_cast<float>(CAND ? max(n_kv, 1) : n_kv);
#pragma unroll
        for (int c = 0; c < HC; ++c) {
          o[c] *= inv_n;
          hsum += o[c];
        }
        const float mean = hsum * (1.0f / HC);
#pragma unroll
        for (int c = 0; c < HC; ++c) {
          const float dlt = o[c] - mean;
          hm2 = fmaf(dlt, dlt, hm2);
        }
        if (p.av_f32 != nullptr) {
          float4* dst = reinterpret_cast<float4*>(p.av_f32 + row * p.ld_av + h * ATT_HD + half * HC);
#pragma unroll
          for (int c = 0; c < HC; c += 4)
            dst[c >> 2] = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
        } else {
          uint16_t* dst = static_cast<uint16_t*>(p.av) + row * p.ld_av + h * ATT_HD + half * HC;
          auto pack = [](float a, float b) -> uint32_t {
            if constexpr (F16) return pack_h2(a, b);
            else return pack_bf16x2(a, b);
          };
#pragma unroll
          for (int c = 0; c < HC; c += 8) {
            uint4 pkt;
            pkt.x = pack(o[c + 0], o[c + 1]);
            pkt.y = pack(o[c + 2], o[c + 3]);
            pkt.z = pack(o[c + 4], o[c + 5]);
            pkt.w = pack(o[c + 6], o[c + 7]);
            *reinterpret_cast<uint4*>(dst + c) = pkt;
          }
        }
      }
    }
    // every thread of the group's 256 reaches this barrier (no early exit)
    if (half == 1) sLnX[g * ATT_ROWS + r] = make_float2(hsum, hm2);
    named_barrier_sync(1 + g, 2 * ATT_ROWS);
    if (half == 0 && ok && valid && p.ln_part != nullptr) {
      const float2 other = sLnX[g * ATT_ROWS + r];
      const float dm = (hsum - other.x) * (1.0f / HC);
      float2* lp = reinterpret_cast<float2*>(p.ln_part + (row * p.H + h) * 2);
      *lp = make_float2(hsum + other.x, hm2 + other.y + dm * dm * (HC * HC / (2.0f * HC)));
    }
  }

  if constexpr (FUSED) {
    // The pair's AV rows and LayerNorm partial sums of this head are written;
    // the CTA that completes the pair's H arrivals runs f2 for its rows.
    __threadfence();
    tc_fence_before();
    __syncthreads();
    volatile int* sLast = reinterpret_cast<volatile int*>(smem + AttnSmem::kMisc + 8);
    if (tid == 0) {
      // one counter per query tile pair, indexed by the pair's first row (< T)
      const int old = atomicAdd(&p.tail.count[q_start + q0], 1);
      *sLast = (old == p.H - 1) ? 1 : 0;
    }
    __syncthreads();
    if (*sLast) {
      __threadfence();
      tc_fence_after();
      attn_f2_tail(&tm_w2, p, smem, bars, tmem, q_start, q0, n_q, ctl);
    }
  }

  // ---------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == ATT_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- debug: bucket indices

// Writes, per user, the n x n blocks of position and time bucket indices the
// attention kernel uses (the int32 and int64 BucketWalk for the time buckets,
// min(i-j, P-1) for positions; -1 above the diagonal).  One thread per query row.
__global__ void hstu_debug_rab_index_kernel(const int64_t* offsets, const int64_t* timestamps,
                                            const int64_t* block_offsets, int B, int P, int Tb,
                                            int max_len, int32_t* pos_idx, int32_t* time_idx,
                                            const __grid_constant__ AttnParams p) {
  __shared__ int64_t sThr[MAX_TIME_BUCKETS];
  __shared__ int32_t sThr32[MAX_TIME_BUCKETS];
  __shared__ int4 sOct[32];
  for (int k = threadIdx.x; k < Tb; k += blockDim.x) {
    sThr[k] = p.thr[k];
    sThr32[k] = p.thr[k] < static_cast<int64_t>(INT32_MAX) ? static_cast<int32_t>(p.thr[k]) : INT32_MAX;
  }
  if (threadIdx.x < 32) sOct[threadIdx.x] = p.oct[threadIdx.x];
  __syncthreads();
  const int u = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= B) return;
  const int64_t s = offsets[u];
  const int n = static_cast<int>(offsets[u + 1] - s);
  if (i >= n) return;
  const int64_t base = block_offsets[u] + static_cast<int64_t>(i) * n;
  const int64_t t0 = timestamps[s];
  const bool ts32 = timestamps[s + n - 1] - t0 < static_cast<int64_t>(INT32_MAX) - 1;
  BucketWalk<int32_t> w32;
  BucketWalk<int64_t> w64;
  if (ts32) w32.init(static_cast<int32_t>(timestamps[s + i] - t0), 0, sThr, sThr32, Tb);
  else w64.init(timestamps[s + i], t0, sThr, sThr, Tb);
  for (int j = 0; j < n; ++j) {
    if (j <= i) {
      int b;
      if (ts32) {
        w32.step(static_cast<int32_t>(timestamps[s + j] - t0), sThr32);
        b = w32.b;
      } else {
        w64.step(timestamps[s + j], sThr);
        b = w64.b;
      }
      // the attention kernels use both the walk and the octave table; a
      // disagreement between them is reported as -2
      if (ts32 && b != time_bucket_octave(static_cast<int32_t>(timestamps[s + i] - timestamps[s + j]), sOct))
        b = -2;
      pos_idx[base + j] = min(i - j, P - 1);
      time_idx[base + j] = b;
    } else {
      pos_idx[base + j] = -1;
      time_idx[base + j] = -1;
    }
  }
}

// One CTA waits on a barrier that nothing completes; the bounded wait records
// HSTU_ERR_DEVICE_TIMEOUT and the kernel returns.
__global__ void hstu_debug_wait_timeout_kernel(uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitCtl ctl{&abort_flag, timeout_ns};
  mbar_wait(&bar, 0, ctl);
  __syncthreads();
}

}  // namespace hstu
