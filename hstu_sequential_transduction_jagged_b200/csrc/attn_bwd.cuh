// Backward of the causal pointwise attention (Eq. 2 of the review of "Actions
// Speak Louder than Words", section 三 核心公式, differentiated):
//   S = Q K^T + rab,  A = phi2(S) / N (visible pairs j <= i),  O = A V
//   dV = A^T dO,  dS = (dO V^T) (.) phi2'(S) / N,  dQ = dS K,  dK = dS^T Q,
//   drab_pos[h, min(i-j, P-1)] += dS_ij,  drab_time[h, bt(t_i - t_j)] += dS_ij.
//
// One tcgen05 kernel over fp16 (or bf16) Q, K, V, dO with fp32 accumulation
// in tensor memory and fp32 outputs.  A CTA owns one (head, user, 128-key
// tile) and walks the query tiles at and after its keys.  For each tile pair:
//   S^T = K Q^T and dP^T = V dO^T go to tensor memory; the element warps read
//   them into registers (after which the next pair's S^T / dP^T may be issued,
//   so they run during this pair's element work), form P^T and dS^T and write
//   both, 16-bit, to shared memory; then
//   dQ_part = dS K (A = dS^T read transposed) goes to one of two tensor-memory
//   buffers, and dV += P^T dO, dK += dS^T Q accumulate in tensor memory.
// While the tensor core runs the next pair the element warps stage the
// previous dQ_part in shared memory and add it to dQ with TMA reduce-adds (the
// caller's dQ is zeroed first; the order of the additions is not fixed).  dK
// and dV rows belong to one CTA and are stored once at the end.
// Table gradients: the position-table gradient goes through per-warp buffers
// of the 63 diagonals of each 32 x 32 block and then straight to drab_pos
// (coalesced reductions); the time-table gradient is a running sum per lane,
// flushed when its bucket changes (per warp aggregated into shared memory, or
// to global memory in the general path), and the shared sums go to drab_time
// at the end.
// Warp roles (576 threads): warps 0-15 element work (thread = one key row:
// lane quarter warp & 3; 32 of the query tile's 128 rows: column group
// warp >> 2), warp 16 TMA producer, warp 17 MMA issue (one elected lane).
// The time bias of a block comes from the lane's current bucket ("steady"),
// its current bucket or the next one (a compare per element), or, in the
// general path, the octave table per element; the position bias from the tile
// pair's 255-entry band staged in shared memory.  Timestamps are
// non-decreasing within a user.  Every wait is bounded.
#pragma once

#include "attn.cuh"

namespace hstu {

constexpr int BW_ROWS = 128;          // rows of the tile the CTA owns
constexpr int BW_COLS = 128;          // rows of each streamed tile
constexpr int BW_ELEM_WARPS = 16;
constexpr int BW_THREADS = (BW_ELEM_WARPS + 2) * 32;
constexpr int BW_PRODUCER_WARP = BW_ELEM_WARPS;
constexpr int BW_MMA_WARP = BW_ELEM_WARPS + 1;
constexpr uint32_t BW_TILE_BYTES = 128 * ATT_HD * 2;  // one 128 x 64 fp16 tile: 16 KB

struct AttnBwdParams {
  const int64_t* offsets;      // [B+1]
  const int64_t* timestamps;   // [T]
  const float* rab_pos;        // [H, P]
  const float* rab_time;       // [H, Tb]
  float* dq;                   // [T, ld_g] fp32 (head h at columns h*64), accumulated into (caller zeroes)
  float* dk;
  float* dv;
  int64_t ld_g;
  float* drab_pos;             // [H, P] fp32, accumulated into (caller zeroes)
  float* drab_time;            // [H, Tb]
  int32_t B, H, P, Tb, max_len;
  int32_t phi2;
  uint64_t timeout_ns;
  int32_t thr[MAX_TIME_BUCKETS];  // time-bucket thresholds (thr[0] = 0), clamped to int32
  int4 oct[32];                   // per octave k of dt+1: {t1, t2, t3, bucket(2^k - 1)}
};

struct BwSmem {
  static constexpr uint32_t kOwn0 = 0;                      // K tile
  static constexpr uint32_t kOwn1 = kOwn0 + BW_TILE_BYTES;  // V tile
  static constexpr uint32_t kStg = kOwn1 + BW_TILE_BYTES;   // 2 stages x (Q, dO tiles)
  static constexpr uint32_t kStgBytes = 2 * BW_TILE_BYTES;
  // dS^T of the current tile pair, 16-bit, 128B-swizzled rows of 64 queries:
  // queries 0-63 at kDs, 64-127 at kDs + BW_TILE_BYTES (row = key, 128 B)
  static constexpr uint32_t kDs = kStg + 2 * kStgBytes;
  static constexpr uint32_t kPt = kDs + 2 * BW_TILE_BYTES;     // P^T, the same layout
  static constexpr uint32_t kTimes = kPt + 2 * BW_TILE_BYTES;  // 2 x 128 int32 (query rows)
  // 2 x 256 float pairs: entry e of the rab_pos band with its successor
  static constexpr uint32_t kBand = kTimes + 2 * 128 * 4;
  static constexpr uint32_t kThr = kBand + 2 * 256 * 8;     // Tb int32 thresholds
  static constexpr uint32_t kRt = kThr + MAX_TIME_BUCKETS * 4;  // Tb floats (rab_time row)
  static constexpr uint32_t kTg = kRt + MAX_TIME_BUCKETS * 4;   // Tb floats (time gradient)
  static constexpr uint32_t kOct = kTg + MAX_TIME_BUCKETS * 4;  // 32 int4 octave entries
  static constexpr uint32_t kBars = kOct + 32 * 16;             // 16 barriers
  static constexpr uint32_t kMisc = kBars + 16 * 8;
  // per element warp two 64-float diagonal buffers (odd lanes, even lanes)
  static constexpr uint32_t kDiag = kMisc + 64;
  // dQ_part of one tile pair in fp32 for the TMA reduce-add: two 32-column
  // boxes of 128 rows (128B-swizzled rows of 128 bytes), 16 KB each
  static constexpr uint32_t kDqs = (kDiag + BW_ELEM_WARPS * 128 * 4 + 1023u) & ~1023u;
  static constexpr uint32_t kBytes = kDqs + 2 * BW_TILE_BYTES + 1024u;
};

enum : int {
  BWB_OWN = 0,          // the CTA's own two tiles landed
  BWB_FULL = 1,         // + stage
  BWB_EMPTY = 3,        // + stage
  BWB_S = 5,            // S^T and dP^T of the current tile pair are in tensor memory
  BWB_P = 6,            // the element warps wrote P^T / dS^T
  BWB_DONE = 7,         // every MMA completed
  BWB_S3 = 8,           // dQ_part, dV and dK MMAs of the tile pair done (P^T, dS^T read)
  BWB_XYF = 9,          // the element warps read S^T / dP^T: tensor memory X / Y free
  BWB_COUNT = 10
};

// phi2 and its derivative at s (pointwise modes)
template <int PHI>
__device__ __forceinline__ void phi_and_grad(float s, float& p, float& g) {
  if constexpr (PHI == HSTU_ACT_SILU) {
    const float sg = fmaf(0.5f, tanh_approx(0.5f * s), 0.5f);  // sigmoid(s)
    p = s * sg;
    g = sg * fmaf(s, 1.0f - sg, 1.0f);
  } else if constexpr (PHI == HSTU_ACT_RELU) {
    p = fmaxf(s, 0.0f);
    g = s > 0.0f ? 1.0f : 0.0f;
  } else {
    p = s;
    g = 1.0f;
  }
}

// phi2 / N and phi2' / N of a packed pair of pre-activations
template <int PHI>
__device__ __forceinline__ void phi_grad_pair(uint64_t s2, float inv_n, uint64_t& p2, uint64_t& g2) {
  if constexpr (PHI == HSTU_ACT_SILU) {
    // sigmoid(s) = 0.5 + 0.5 tanh(s / 2);  SiLU' = sigmoid(s) (1 + s (1 - sigmoid(s)))
    float a, b;
    f2_unpack(f2_mul(s2, f2_pack(0.5f, 0.5f)), a, b);
    const uint64_t t = f2_pack(tanh_approx(a), tanh_approx(b));
    const float hn = 0.5f * inv_n;
    const uint64_t sgn = f2_fma(t, f2_pack(hn, hn), f2_pack(hn, hn));              // sigmoid / N
    const uint64_t om = f2_fma(t, f2_pack(-0.5f, -0.5f), f2_pack(0.5f, 0.5f));     // 1 - sigmoid
    p2 = f2_mul(s2, sgn);
    g2 = f2_mul(sgn, f2_fma(s2, om, f2_pack(1.0f, 1.0f)));
  } else {
    float a, b;
    f2_unpack(s2, a, b);
    if constexpr (PHI == HSTU_ACT_RELU) {
      p2 = f2_pack(fmaxf(a, 0.0f) * inv_n, fmaxf(b, 0.0f) * inv_n);
      g2 = f2_pack(a > 0.0f ? inv_n : 0.0f, b > 0.0f ? inv_n : 0.0f);
    } else {
      p2 = f2_pack(a * inv_n, b * inv_n);
      g2 = f2_pack(inv_n, inv_n);
    }
  }
}

// sTg[b] += v for every lane with `act`, as one shared-memory atomic per
// distinct b (a shared fp32 atomic is a compare-and-swap loop, so 32 lanes on
// one address would retry one after the other).  Warp-converged callers only.
__device__ __forceinline__ void warp_bucket_add(float* sTg, bool act, int b, float v) {
  const unsigned full = 0xffffffffu;
  unsigned m = __ballot_sync(full, act);
  while (m != 0u) {
    const int leader = __ffs(m) - 1;
    const int bb = __shfl_sync(full, b, leader);
    const bool mine = act && b == bb;
    float sum = mine ? v : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(full, sum, o);
    if (lane_id() == leader) atomicAdd(&sTg[bb], sum);
    m &= ~__ballot_sync(full, mine);
  }
}

// Seconds since the user's first event (int32, clamped; the span check is
// made once per CTA).
__device__ __forceinline__ int32_t bw_rel_time(const int64_t* ts, int64_t row, int64_t t_first) {
  const int64_t d = ts[row] - t_first;
  return d >= static_cast<int64_t>(INT32_MAX) - 1 ? INT32_MAX - 1 : static_cast<int32_t>(d);
}

// F16: fp16 operands (else bf16); P and dS are packed in the operand type.
template <int PHI, bool F16>
__global__ void __launch_bounds__(BW_THREADS, 1)
hstu_attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ AttnBwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int h = blockIdx.x, u = blockIdx.y;
  // longest work first: key tile 0 meets every query tile
  const int ot = static_cast<int>(blockIdx.z);
  const int64_t start = p.offsets[u];
  const int n = static_cast<int>(p.offsets[u + 1] - start);
  if (n > p.max_len || n < 0) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0) record_status(HSTU_ERR_DEVICE_CHECK);
    return;
  }
  const int o0 = ot * BW_ROWS;  // first key (within the user) of the own tile
  if (o0 >= n) return;          // uniform, before any allocation
  const int n_tiles = (n + BW_COLS - 1) / BW_COLS;
  const int n_st = n_tiles - ot;  // query tiles ot .. n_tiles - 1

  uint8_t* sOwn0 = smem + BwSmem::kOwn0;
  uint8_t* sOwn1 = smem + BwSmem::kOwn1;
  uint8_t* sStg = smem + BwSmem::kStg;
  uint8_t* sDs = smem + BwSmem::kDs;
  uint8_t* sPt = smem + BwSmem::kPt;
  int32_t* sTimes = reinterpret_cast<int32_t*>(smem + BwSmem::kTimes);
  float* sBand = reinterpret_cast<float*>(smem + BwSmem::kBand);
  int32_t* sThr = reinterpret_cast<int32_t*>(smem + BwSmem::kThr);
  float* sRt = reinterpret_cast<float*>(smem + BwSmem::kRt);
  float* sTg = reinterpret_cast<float*>(smem + BwSmem::kTg);
  int4* sOct = reinterpret_cast<int4*>(smem + BwSmem::kOct);
  uint8_t* sDqs = smem + BwSmem::kDqs;
  float* sDiag = reinterpret_cast<float*>(smem + BwSmem::kDiag);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BwSmem::kBars);
  uint32_t* sTmemBase = reinterpret_cast<uint32_t*>(smem + BwSmem::kMisc);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + BwSmem::kMisc + 4);
  const int warp = warp_id(), lane = lane_id(), tid = threadIdx.x;
  const int64_t t_first = p.timestamps[start];
  if (tid == 0 && p.timestamps[start + n - 1] - t_first >= static_cast<int64_t>(INT32_MAX) - 1)
    record_status(HSTU_ERR_DEVICE_CHECK);

  if (tid == 0) {
    mbar_init(&bars[BWB_OWN], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[BWB_FULL + s], 1);
      mbar_init(&bars[BWB_EMPTY + s], 1);
    }
    mbar_init(&bars[BWB_S], 1);
    mbar_init(&bars[BWB_P], BW_ELEM_WARPS * 32);
    mbar_init(&bars[BWB_DONE], 1);
    mbar_init(&bars[BWB_S3], 1);
    mbar_init(&bars[BWB_XYF], BW_ELEM_WARPS * 32);
    *sAbort = 0;
    fence_mbar_init();
  }
  if (warp == BW_MMA_WARP) {
    tmem_alloc(sTmemBase, 512);
    tmem_relinquish();
  }
  for (int k = tid; k < p.Tb; k += BW_THREADS) {
    sThr[k] = p.thr[k];
    sRt[k] = p.rab_time[static_cast<int64_t>(h) * p.Tb + k];
    sTg[k] = 0.0f;
  }
  if (tid < 32) sOct[tid] = p.oct[tid];
  for (int k = tid; k < BW_ELEM_WARPS * 128; k += BW_THREADS) sDiag[k] = 0.0f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmemBase;
  const WaitCtl ctl{sAbort, p.timeout_ns};
  // tensor memory: X = S^T (columns 0-127), Y = dP^T (128-255), dV (256-319),
  // dK (320-383), dQ_part of even / odd tile pairs (384-447 / 448-511)
  constexpr uint32_t kX = 0, kY = 128, kAcc0 = 256, kAcc1 = 320, kDq = 384;

  if (warp == BW_PRODUCER_WARP) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      const int32_t orow = static_cast<int32_t>(start + o0);
      mbar_arrive_expect_tx(&bars[BWB_OWN], 2 * BW_TILE_BYTES);
      tma_load_2d(sOwn0, &tm_k, &bars[BWB_OWN], h * ATT_HD, orow);
      tma_load_2d(sOwn1, &tm_v, &bars[BWB_OWN], h * ATT_HD, orow);
      int issued = 0;
      for (int it = 0; it < n_st; ++it) {
        const int s = it & 1;
        if (!mbar_wait(&bars[BWB_EMPTY + s], ((it >> 1) & 1) ^ 1u, ctl)) break;
        const int32_t row = static_cast<int32_t>(start + (ot + it) * BW_COLS);
        uint8_t* dst = sStg + s * BwSmem::kStgBytes;
        mbar_arrive_expect_tx(&bars[BWB_FULL + s], 2 * BW_TILE_BYTES);
        tma_load_2d(dst, &tm_q, &bars[BWB_FULL + s], h * ATT_HD, row);
        tma_load_2d(dst + BW_TILE_BYTES, &tm_do, &bars[BWB_FULL + s], h * ATT_HD, row);
        ++issued;
      }
      // every load lands before shared memory is released
      mbar_wait_drain(&bars[BWB_OWN], 0, p.timeout_ns);
      for (int it = max(0, issued - 2); it < issued; ++it)
        mbar_wait_drain(&bars[BWB_FULL + (it & 1)], static_cast<uint32_t>(it >> 1) & 1u, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == BW_MMA_WARP) {
    const bool leader = elect_one();
    auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, par, ctl));
    };
    constexpr uint32_t idesc_ss = idesc_16_f32(BW_ROWS, BW_COLS, false, false, F16);
    constexpr uint32_t idesc_acc = idesc_16_f32(BW_ROWS, ATT_HD, false, true, F16);
    constexpr uint32_t idesc_dq = idesc_16_f32(BW_COLS, ATT_HD, true, true, F16);
    const uint64_t dOwn0 = smem_desc_sw128(smem_u32(sOwn0), 16, 1024);   // K, K-major A
    const uint64_t dOwn1 = smem_desc_sw128(smem_u32(sOwn1), 16, 1024);   // V, K-major A
    const uint64_t dOwn0m = smem_desc_sw128(smem_u32(sOwn0), 8192, 1024);  // K, MN-major B
    // dS as an MN-major A (M = 128 queries: two 64-query halves BW_TILE_BYTES
    // apart; K = keys: 8-row groups 1024 bytes apart)
    const uint64_t dDsm = smem_desc_sw128(smem_u32(sDs), BW_TILE_BYTES, 1024);
    // dS^T and P^T as K-major A (M = 128 keys, K = queries: 16-query steps of
    // 32 bytes inside a 64-query half, the second half BW_TILE_BYTES further)
    const uint64_t dDsk = smem_desc_sw128(smem_u32(sDs), 16, 1024);
    const uint64_t dPtk = smem_desc_sw128(smem_u32(sPt), 16, 1024);
    // S^T = K Q^T, dP^T = V dO^T of tile pair j (K = 64: four steps)
    auto issue_sdp = [&](int j) -> bool {
      const int s = j & 1;
      if (!wait_all(&bars[BWB_FULL + s], (j >> 1) & 1)) return false;
      tc_fence_after();
      const uint32_t sa = smem_u32(sStg + s * BwSmem::kStgBytes);
      const uint64_t dS0k = smem_desc_sw128(sa, 16, 1024);                  // Q, K-major
      const uint64_t dS1k = smem_desc_sw128(sa + BW_TILE_BYTES, 16, 1024);  // dO, K-major
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < ATT_HD / 16; ++kk)
          mma_bf16_ss(tmem + kX, dOwn0 + 2 * kk, dS0k + 2 * kk, idesc_ss, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < ATT_HD / 16; ++kk)
          mma_bf16_ss(tmem + kY, dOwn1 + 2 * kk, dS1k + 2 * kk, idesc_ss, kk > 0 ? 1u : 0u);
        mma_commit(&bars[BWB_S]);
      }
      __syncwarp();
      return true;
    };
    bool ok = wait_all(&bars[BWB_OWN], 0);
    tc_fence_after();
    if (ok) ok = issue_sdp(0);
    for (int it = 0; ok && it < n_st; ++it) {
      // the next tile pair's S^T / dP^T as soon as this pair's are read, so
      // they run while the element warps work on this pair
      if (it + 1 < n_st) {
        ok = wait_all(&bars[BWB_XYF], static_cast<uint32_t>(it) & 1u);
        if (!ok) break;
        tc_fence_after();
        ok = issue_sdp(it + 1);
        if (!ok) break;
      }
      ok = wait_all(&bars[BWB_P], static_cast<uint32_t>(it) & 1u);
      if (!ok) break;
      tc_fence_after();
      const int s = it & 1;
      const uint32_t sa = smem_u32(sStg + s * BwSmem::kStgBytes);
      const uint64_t dS0m = smem_desc_sw128(sa, 8192, 1024);                  // Q, MN-major B
      const uint64_t dS1m = smem_desc_sw128(sa + BW_TILE_BYTES, 8192, 1024);  // dO, MN-major B
      if (leader) {
        // dQ_part = dS K over the 128 keys (eight steps of 16 keys, 2 KB each)
        const uint32_t dq_acc = tmem + kDq + 64u * static_cast<uint32_t>(it & 1);
#pragma unroll
        for (int kk = 0; kk < BW_ROWS / 16; ++kk)
          mma_bf16_ss(dq_acc, dDsm + 128 * kk, dOwn0m + 128 * kk, idesc_dq, kk > 0 ? 1u : 0u);
        // dV += P^T dO ; dK += dS^T Q over the 128 queries (eight steps)
#pragma unroll
        for (int kk = 0; kk < BW_COLS / 16; ++kk) {
          const uint64_t ak = static_cast<uint64_t>((kk >> 2) * (BW_TILE_BYTES >> 4) + (kk & 3) * 2);
          mma_bf16_ss(tmem + kAcc0, dPtk + ak, dS1m + 128 * kk, idesc_acc,
                      (it > 0 || kk > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < BW_COLS / 16; ++kk) {
          const uint64_t ak = static_cast<uint64_t>((kk >> 2) * (BW_TILE_BYTES >> 4) + (kk & 3) * 2);
          mma_bf16_ss(tmem + kAcc1, dDsk + ak, dS0m + 128 * kk, idesc_acc,
                      (it > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bars[BWB_S3]);
        mma_commit(&bars[BWB_EMPTY + s]);
      }
      __syncwarp();
    }
    if (leader) mma_commit(&bars[BWB_DONE]);
    __syncwarp();
    mbar_wait_drain(&bars[BWB_DONE], 0, p.timeout_ns);
  } else {
    // ---------------- element warps
    const int q4 = warp & 3, cg = warp >> 2;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const int r = q4 * 32 + lane;        // key row of the own tile
    const int orow = o0 + r;             // its index within the user
    const bool own_ok = orow < n;
    const int32_t t_own = own_ok ? bw_rel_time(p.timestamps, start + orow, t_first) : 0;
    const float inv_n = 1.0f / static_cast<float>(n);
    const float* rp = p.rab_pos + static_cast<int64_t>(h) * p.P;
    const int c0 = cg * 32;              // this warp's 32 queries of each tile
    // this thread's 64-byte slice of the dS^T rows in shared memory (four
    // 16-byte chunks of 8 queries, 128B swizzle: chunk index ^ (row & 7))
    uint8_t* ds_row = sDs + (cg >> 1) * BW_TILE_BYTES + r * 128;
    uint8_t* pt_row = ds_row + (BwSmem::kPt - BwSmem::kDs);  // the same slice of P^T
    const int ds_chunk0 = (cg & 1) * 4;
    // Tile pair j's dQ_part (rows = its queries) into global dQ.  Each lane
    // quarter (32 query rows; the four warps of 16 columns that share it)
    // stages its rows in the two swizzled fp32 boxes, then one thread of the
    // quarter adds them to dQ with two TMA reduce-adds.  The quarter's barrier
    // is taken on every call, `live` or not, so that no warp waits on one that
    // gave up; the staging rows are rewritten only after the issuing thread has
    // seen its previous reduce read them (bulk_wait_read0 before the CTA
    // barrier at the top of each iteration, or before the last call).
    const bool dq_issuer = cg == 0 && lane == 0;
    uint8_t* dq_stage = sDqs + (cg >> 1) * BW_TILE_BYTES + q4 * 4096 + lane * 128;
    auto drain_dq = [&](int j, bool live) {
      if (live) {
        uint32_t v[16];
        tmem_ld16(tmem + lane_off + kDq + 64u * static_cast<uint32_t>(j & 1) +
                      static_cast<uint32_t>(cg * 16), v);
        tmem_ld_wait(v);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          *reinterpret_cast<uint4*>(dq_stage + ((((cg & 1) * 4 + k) ^ (lane & 7)) << 4)) =
              make_uint4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
        fence_proxy_async_smem();
      }
      named_barrier_sync(2 + q4, 4 * 32);
      const int qrow0 = (ot + j) * BW_COLS + q4 * 32;
      if (live && dq_issuer && qrow0 < n) {
        // rows past the user's end hold exact zeros (no visible key)
#pragma unroll
        for (int b = 0; b < 2; ++b)
          tma_reduce_add_2d(&tm_dq, sDqs + b * BW_TILE_BYTES + q4 * 4096, h * ATT_HD + 32 * b,
                            static_cast<int32_t>(start + qrow0));
        bulk_commit();
      }
    };
    // Time-bucket walk over this thread's visible pairs in the order visited:
    // dt = t_i - t_own grows with the query i, so the bucket goes up from 0.
    // The bucket of dt is the largest b with thr[b] <= dt (thr[0] = 0).
    int tb = 0;
    float rt_cur = sRt[0];
    // the edge the walk compares against: thr[tb + 1] (INT32_MAX past the last bucket)
    int32_t edge = p.Tb > 1 ? sThr[1] : INT32_MAX;
    float tg_acc = 0.0f;    // time-gradient running sum of the current bucket
    float pg_clamp = 0.0f;  // position gradient of the clamped bucket P - 1
    // moves every lane's walk to the bucket of its dt (dt < edge: no move),
    // flushing the running sums that change bucket; warp-converged callers
    const unsigned full = 0xffffffffu;
    auto advance = [&](int32_t dt) {
      tg_acc = 0.0f;
      do {
        ++tb;
        edge = tb + 1 < p.Tb ? sThr[tb + 1] : INT32_MAX;
      } while (dt >= edge);
      rt_cur = sRt[tb];
    };
    auto walk_to = [&](int32_t dt) {
      const bool mv = dt >= edge;
      if (__any_sync(full, mv)) {
        warp_bucket_add(sTg, mv && tg_acc != 0.0f, tb, tg_acc);
        if (mv) advance(dt);
      }
    };
    // the general path, where lanes sit in many different buckets, takes each
    // element's bucket straight from the octave table; a lane's running sum
    // goes to global memory (a reduction that does not return) when its
    // bucket changes
    float* drt = p.drab_time + static_cast<int64_t>(h) * p.Tb;
    float* drp = p.drab_pos + static_cast<int64_t>(h) * p.P;
    // position-table gradient: this warp's 32 x 32 block adds dS to its 63
    // diagonals k = cc - lane + 31 (D = i - j = dg0 + k - 31).  Odd lanes add
    // into diagB[k], even lanes into diagA[k + 1], so that the two diagonals of
    // a column pair are one aligned 8-byte entry for every lane.  The 32 lanes
    // of one column touch 32 different diagonals, so the adds are plain
    // read-modify-writes (a __syncwarp before each keeps the lanes in step);
    // the block's diagonals go to the CTA histogram afterwards.
    float* diagB = sDiag + warp * 128;
    float* diagA = diagB + 64;
    float* dlp = ((lane & 1) ? diagB : diagA + 1) + 31 - lane;  // dlp[cc]: this lane's entry
    // Staging of tile pair j's 128 query times and 255-entry position-bias
    // band (entry e: rab_pos[min(D, P - 1)] for D = i - j = (j's first query -
    // o0) + e - 127, 0 for D < 0, paired with entry e + 1), written for the
    // next pair once this pair's element work is done.
    int64_t pf_t = 0;
    float pf_b0 = 0.0f, pf_b1 = 0.0f;
    auto stage_load = [&](int j) {
      const int sb = (ot + j) * BW_COLS;
      if (tid < 128) {
        const int row = sb + tid;
        pf_t = row < n ? p.timestamps[start + row] : t_first;
      } else if (tid < 128 + 255) {
        const int dd = sb - o0 + (tid - 128) - 127;
        pf_b0 = dd >= 0 ? __ldg(rp + min(dd, p.P - 1)) : 0.0f;
        pf_b1 = dd + 1 >= 0 ? __ldg(rp + min(dd + 1, p.P - 1)) : 0.0f;
      }
    };
    auto stage_store = [&](int j) {
      if (tid < 128) {
        const int64_t d = pf_t - t_first;
        sTimes[(j & 1) * 128 + tid] =
            d >= static_cast<int64_t>(INT32_MAX) - 1 ? INT32_MAX - 1 : static_cast<int32_t>(d);
      } else if (tid < 128 + 255) {
        reinterpret_cast<uint64_t*>(sBand)[(j & 1) * 256 + tid - 128] = f2_pack(pf_b0, pf_b1);
      }
    };
    stage_load(0);
    stage_store(0);
    bool ok = true;
    for (int it = 0; it < n_st; ++it) {
      const int sbase = (ot + it) * BW_COLS;  // first query of the tile
      const int32_t* tt = sTimes + (it & 1) * 128;
      const uint64_t* bandp = reinterpret_cast<const uint64_t*>(sBand) + (it & 1) * 256;
      if (dq_issuer) bulk_wait_read0();
      named_barrier_sync(1, BW_ELEM_WARPS * 32);
      if (ok) ok = mbar_wait(&bars[BWB_S], static_cast<uint32_t>(it) & 1u, ctl);
      ok = __all_sync(full, ok);
      bool xy_read = false;  // this thread arrived on BWB_XYF for the pair
      // the previous pair's dQ / dV / dK MMAs read P^T and dS^T from shared memory
      auto wait_s3 = [&]() {
        if (it > 0) {
          ok = __all_sync(full, mbar_wait(&bars[BWB_S3], static_cast<uint32_t>(it - 1) & 1u, ctl));
          tc_fence_after();
        }
      };
      if (ok) {
        tc_fence_after();
        // band pair of column cc: bp[cc]
        const uint64_t* bp = bandp + (c0 - r + 127);
        // every column of the block visible (not the diagonal tile, not past
        // the user's end) and no pair in the clamped position bucket
        const bool interior = it > 0 && sbase + c0 + 32 <= n &&
                              sbase + c0 + 31 - (o0 + q4 * 32) < p.P - 1;
        // General path: per element visibility, bucket and clamp.  A rolled loop
        // over four 8-column groups (the rare blocks keep their code small)
        // that reads S^T / dP^T from tensor memory and writes each group's
        // packed P^T / dS^T to shared memory.
        auto general = [&]() {
          wait_s3();
          int c_lo = 0, c_hi = 31;
          if (!own_ok) {
            c_lo = 32;
          } else {
            c_lo = max(0, orow - (sbase + c0));
            c_hi = min(31, n - 1 - (sbase + c0));
          }
#pragma unroll 1
          for (int g = 0; g < 4; ++g) {
            uint32_t x8[8], y8[8];
            tmem_ld8(tmem + lane_off + kX + static_cast<uint32_t>(c0 + 8 * g), x8);
            tmem_ld8(tmem + lane_off + kY + static_cast<uint32_t>(c0 + 8 * g), y8);
            tmem_ld_wait(x8, y8);
            uint32_t pk[4], dk[4];
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
              float pv[2], dsv[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int cc = 8 * g + c + e;
                float pp = 0.0f, ds = 0.0f, dsp = 0.0f;
                if (cc >= c_lo && cc <= c_hi) {
                  const int b = time_bucket_octave(tt[c0 + cc] - t_own, sOct);
                  if (b != tb) {
                    if (tg_acc != 0.0f) atomicAdd(&drt[tb], tg_acc);
                    tg_acc = 0.0f;
                    tb = b;
                    rt_cur = sRt[b];
                  }
                  const int dpos = (sbase + c0 + cc) - orow;  // D = i - j
                  float b0, b1;
                  f2_unpack(bp[cc], b0, b1);
                  const float sv = __uint_as_float(x8[c + e]) + b0 + rt_cur;
                  float ph, pg;
                  phi_and_grad<PHI>(sv, ph, pg);
                  pp = ph * inv_n;
                  ds = __uint_as_float(y8[c + e]) * pg * inv_n;
                  if (dpos >= p.P - 1) pg_clamp += ds;
                  else dsp = ds;
                  tg_acc += ds;
                }
                __syncwarp();
                dlp[cc] += dsp;
                pv[e] = pp;
                dsv[e] = ds;
              }
              if constexpr (F16) {
                pk[c >> 1] = pack_h2(pv[0], pv[1]);
                dk[c >> 1] = pack_h2(dsv[0], dsv[1]);
              } else {
                pk[c >> 1] = pack_bf16x2(pv[0], pv[1]);
                dk[c >> 1] = pack_bf16x2(dsv[0], dsv[1]);
              }
            }
            const int off = ((ds_chunk0 + g) ^ (r & 7)) << 4;
            *reinterpret_cast<uint4*>(pt_row + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            *reinterpret_cast<uint4*>(ds_row + off) = make_uint4(dk[0], dk[1], dk[2], dk[3]);
          }
          edge = tb + 1 < p.Tb ? sThr[tb + 1] : INT32_MAX;
          tc_fence_before();
          mbar_arrive(&bars[BWB_XYF]);
          xy_read = true;
        };
        // interior blocks: the time bias of each column pair comes from the
        // lane's current bucket (every lane stays in it: "steady") or from the
        // lane's current bucket and the next one (hi iff dt >= thr_hi)
        int path = 2;  // 0 steady, 1 two buckets, 2 general
        int32_t dt_last = 0, thr_hi = INT32_MAX;
        float rt_lo = 0.0f, rt_hi = 0.0f;
        if (interior) {
          const int32_t dt_first = tt[c0] - t_own;
          dt_last = tt[c0 + 31] - t_own;
          if (__all_sync(full, dt_last < edge)) {
            path = 0;
          } else {
            walk_to(dt_first);
            // every lane spans at most two buckets (its current one and the
            // next): per element, bucket tb + 1 iff dt >= edge
            if (__all_sync(full, tb + 2 >= p.Tb || dt_last < sThr[tb + 2])) {
              path = 1;
              rt_lo = rt_cur;
              rt_hi = tb + 1 < p.Tb ? sRt[tb + 1] : rt_cur;
              thr_hi = edge;
            }
          }
        }
        if (path == 2) {
          general();
        } else {
          uint32_t xs[32], ys[32];
          tmem_ld32(tmem + lane_off + kX + static_cast<uint32_t>(c0), xs);
          tmem_ld32(tmem + lane_off + kY + static_cast<uint32_t>(c0), ys);
          tmem_ld_wait(xs);
          tmem_ld_wait(ys);
          // S^T / dP^T are in registers: the next pair's MMAs may overwrite them
          tc_fence_before();
          mbar_arrive(&bars[BWB_XYF]);
          xy_read = true;
          uint32_t px[16], py[16];
          // rt_pair(c) gives the pair's time bias, ds_sink(c, ds2) sees its dS
          auto interior_pairs = [&](auto rt_pair, auto ds_sink) {
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              const uint64_t s2 = f2_add(f2_pack(__uint_as_float(xs[c]), __uint_as_float(xs[c + 1])),
                                         f2_add(bp[c], rt_pair(c)));
              uint64_t p2, g2;
              phi_grad_pair<PHI>(s2, inv_n, p2, g2);
              const uint64_t ds2 =
                  f2_mul(f2_pack(__uint_as_float(ys[c]), __uint_as_float(ys[c + 1])), g2);
              ds_sink(c, ds2);
              __syncwarp();
              uint64_t* dd = reinterpret_cast<uint64_t*>(dlp + c);
              *dd = f2_add(*dd, ds2);
              if constexpr (F16) {
                px[c >> 1] = f2_to_h2(p2);
                py[c >> 1] = f2_to_h2(ds2);
              } else {
                px[c >> 1] = f2_to_bf16x2(p2);
                py[c >> 1] = f2_to_bf16x2(ds2);
              }
            }
          };
          if (path == 0) {
            const uint64_t rt2 = f2_pack(rt_cur, rt_cur);
            uint64_t tg2 = f2_pack(0.0f, 0.0f);
            interior_pairs([&](int) { return rt2; },
                           [&](int, uint64_t d) { tg2 = f2_add(tg2, d); });
            float a0, a1;
            f2_unpack(tg2, a0, a1);
            tg_acc += a0 + a1;
          } else {
            uint64_t tg2 = f2_pack(0.0f, 0.0f), hi2 = f2_pack(0.0f, 0.0f);
            interior_pairs(
                [&](int c) {
                  const int2 t2 = *reinterpret_cast<const int2*>(tt + c0 + c);
                  return f2_pack(t2.x - t_own >= thr_hi ? rt_hi : rt_lo,
                                 t2.y - t_own >= thr_hi ? rt_hi : rt_lo);
                },
                [&](int c, uint64_t d) {
                  const int2 t2 = *reinterpret_cast<const int2*>(tt + c0 + c);
                  float d0, d1;
                  f2_unpack(d, d0, d1);
                  hi2 = f2_add(hi2, f2_pack(t2.x - t_own >= thr_hi ? d0 : 0.0f,
                                            t2.y - t_own >= thr_hi ? d1 : 0.0f));
                  tg2 = f2_add(tg2, d);
                });
            float a0, a1, h0, h1;
            f2_unpack(tg2, a0, a1);
            f2_unpack(hi2, h0, h1);
            const float hsum = h0 + h1;
            // the lane's elements below thr_hi belong to its current bucket
            tg_acc += (a0 + a1) - hsum;
            walk_to(dt_last);
            tg_acc += hsum;
          }
          // P^T and dS^T rows to shared memory for the dQ / dV / dK MMAs
          wait_s3();
          if (ok) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int off = ((ds_chunk0 + k) ^ (r & 7)) << 4;
              *reinterpret_cast<uint4*>(pt_row + off) =
                  make_uint4(px[4 * k], px[4 * k + 1], px[4 * k + 2], px[4 * k + 3]);
              *reinterpret_cast<uint4*>(ds_row + off) =
                  make_uint4(py[4 * k], py[4 * k + 1], py[4 * k + 2], py[4 * k + 3]);
            }
          }
        }
        fence_proxy_async_smem();
        // this block's diagonals into drab_pos (0 <= D < P - 1 there: clamped
        // pairs went to pg_clamp; consecutive lanes add to consecutive entries,
        // with reductions that do not return), and the buffers cleared
        __syncwarp();
        const int dg0 = (sbase + c0) - (o0 + q4 * 32);
#pragma unroll
        for (int k = lane; k < 63; k += 32) {
          const float v = diagB[k] + diagA[k + 1];
          const int dd = dg0 + k - 31;
          if (v != 0.0f && dd >= 0 && dd < p.P - 1) atomicAdd(&drp[dd], v);
          diagB[k] = 0.0f;
          diagA[k + 1] = 0.0f;
        }
      }
      if (!xy_read) mbar_arrive(&bars[BWB_XYF]);  // error path: keep the count
      tc_fence_before();
      mbar_arrive(&bars[BWB_P]);
      if (it + 1 < n_st) {
        stage_load(it + 1);
        stage_store(it + 1);
      }
      // the previous tile pair's dQ_part, while this pair's MMAs run
      if (it > 0) drain_dq(it - 1, ok);
    }
    warp_bucket_add(sTg, tg_acc != 0.0f, tb, tg_acc);
    if (ok) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[BWB_S3], static_cast<uint32_t>(n_st - 1) & 1u, ctl));
      tc_fence_after();
    }
    if (dq_issuer) bulk_wait_read0();
    named_barrier_sync(2 + q4, 4 * 32);
    drain_dq(n_st - 1, ok);
    if (dq_issuer) bulk_wait_all();
    // ---------------- epilogue: the accumulators (rows of the own tile); the
    // four column groups take 16 of the 64 accumulator columns each
    if (ok) ok = mbar_wait(&bars[BWB_DONE], 0, ctl);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const int64_t grow = start + orow;
      for (int a = 0; a < 2; ++a) {
        uint32_t v[16];
        tmem_ld16(tmem + lane_off + (a == 0 ? kAcc0 : kAcc1) + static_cast<uint32_t>(cg * 16), v);
        tmem_ld_wait(v);
        float* dst = a == 0 ? p.dv : p.dk;
        if (own_ok) {
          float4* d4 = reinterpret_cast<float4*>(dst + grow * p.ld_g + h * ATT_HD + cg * 16);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            d4[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
        }
      }
    }
    if (pg_clamp != 0.0f) atomicAdd(&p.drab_pos[static_cast<int64_t>(h) * p.P + p.P - 1], pg_clamp);
  }

  // ---------------- time-table gradient and teardown
  tc_fence_before();
  __syncthreads();
  for (int k = tid; k < p.Tb; k += BW_THREADS) {
    const float g = sTg[k];
    if (g != 0.0f) atomicAdd(&p.drab_time[static_cast<int64_t>(h) * p.Tb + k], g);
  }
  if (warp == BW_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace hstu
