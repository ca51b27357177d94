// Stochastic Length (SL) subsampling of jagged user sequences on the GPU
// (review of "Actions Speak Louder than Words", section 三 技术架构,
// Stochastic Length): user u's n events are shortened to
// L = min(n, ceil(n u^(1/alpha))), u ~ Uniform(0, 1], keeping a uniformly
// random subset of L events in time order.
//
// Randomness: Philox4x64-10 (Salmon, Moraes, Dror and Shaw, "Parallel
// Random Numbers: As Easy as 1, 2, 3", SC 2011), key (seed, 0):
//   length draw of user u     counter (0, u, step, 0), first output word x,
//                             u = ((x >> 11) + 1) 2^-53;
//   rank key of position p    counter (p, u, step, 1), first output word.
// The kept subset is the L positions with the smallest rank keys (equal keys
// go to the lower position).
//
// Four launches: per-user lengths (one thread per user), an exclusive scan
// into the output offsets (one CTA), the per-user selection (one CTA per
// user: rank keys in shared memory, a most-significant-digit-first radix
// select of the L-th smallest key, then a compaction in time order), and the
// gather of the kept rows (all SMs, one warp per row, 16-byte copies).
#pragma once

#include "ptx.cuh"

namespace hstu {

constexpr int SL_MAX_LEN = 16384;       // rank keys of one user fit in shared memory
constexpr int SL_SELECT_THREADS = 512;
constexpr int SL_SCAN_THREADS = 1024;

struct Philox4x64 {
  uint64_t w[4];
};

__device__ __forceinline__ Philox4x64 philox4x64_10(uint64_t c0, uint64_t c1, uint64_t c2,
                                                    uint64_t c3, uint64_t k0, uint64_t k1) {
  constexpr uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
  constexpr uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t lo0 = M0 * c0, hi0 = __umul64hi(M0, c0);
    const uint64_t lo1 = M1 * c2, hi1 = __umul64hi(M1, c2);
    const uint64_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
    k0 += W0;
    k1 += W1;
  }
  return Philox4x64{{c0, c1, c2, c3}};
}

// L_u for every user (one thread per user); the decision is taken in fp64.
__global__ void hstu_sl_lengths_kernel(const int64_t* offsets, int32_t B, double inv_alpha,
                                       uint64_t seed, uint64_t step, int32_t* lengths) {
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= B) return;
  const int64_t n = offsets[u + 1] - offsets[u];
  int32_t L = 0;
  if (n > 0) {
    const uint64_t x = philox4x64_10(0, static_cast<uint64_t>(u), step, 0, seed, 0).w[0];
    const double uu = static_cast<double>((x >> 11) + 1) * 0x1.0p-53;
    const double len = ceil(static_cast<double>(n) * pow(uu, inv_alpha));
    L = static_cast<int32_t>(len < static_cast<double>(n) ? len : static_cast<double>(n));
  }
  lengths[u] = L;
}

// offsets_out[u] = sum of lengths[v < u] (offsets_out[B] = total), and the
// largest length; one CTA.
__global__ void __launch_bounds__(SL_SCAN_THREADS) hstu_sl_scan_kernel(
    const int32_t* lengths, int32_t B, int64_t* offsets_out, int32_t* max_len_out) {
  __shared__ int64_t s_part[SL_SCAN_THREADS / 32];
  __shared__ int32_t s_max[SL_SCAN_THREADS / 32];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int per = (B + SL_SCAN_THREADS - 1) / SL_SCAN_THREADS;
  const int b0 = tid * per;
  const int b1 = min(B, b0 + per);
  int64_t sum = 0;
  int32_t mx = 0;
  for (int b = b0; b < b1; ++b) {
    sum += lengths[b];
    mx = max(mx, lengths[b]);
  }
  // inclusive scan of the per-thread sums across the warp, then the warps
  int64_t inc = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t v = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += v;
  }
  int32_t wmx = mx;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wmx = max(wmx, __shfl_xor_sync(0xffffffffu, wmx, o));
  if (lane == 31) s_part[wid] = inc;
  if (lane == 0) s_max[wid] = wmx;
  __syncthreads();
  if (wid == 0) {
    int64_t v = lane < SL_SCAN_THREADS / 32 ? s_part[lane] : 0;
    int32_t m = lane < SL_SCAN_THREADS / 32 ? s_max[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t t = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += t;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane < SL_SCAN_THREADS / 32) s_part[lane] = v;  // inclusive warp totals
    if (lane == 0 && max_len_out != nullptr) *max_len_out = m;
  }
  __syncthreads();
  int64_t run = (wid > 0 ? s_part[wid - 1] : 0) + inc - sum;  // exclusive prefix of this thread
  for (int b = b0; b < b1; ++b) {
    offsets_out[b] = run;
    run += lengths[b];
  }
  if (tid == SL_SCAN_THREADS - 1) offsets_out[B] = s_part[SL_SCAN_THREADS / 32 - 1];
}

// Block-wide exclusive count of a per-thread flag (512 threads): returns the
// number of set flags at lower thread indices; *total receives the count.
__device__ __forceinline__ int sl_block_count(bool flag, int* s_warp, int* total) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(bal & ((1u << lane) - 1u));
  __syncthreads();  // s_warp of the previous call has been read
  if (lane == 0) s_warp[wid] = __popc(bal);
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < SL_SELECT_THREADS / 32; ++w) {
    const int c = s_warp[w];
    before += (w < wid) ? c : 0;
    all += c;
  }
  *total = all;
  return before + in_warp;
}

// One CTA per user: rank keys of the n positions, the L-th smallest by a
// radix select over 8-bit digits (most significant first), then the kept
// positions in time order.  Dynamic shared memory: n_max 64-bit keys.
// A user longer than max_len (the shared-memory size of the launch) or rows
// outside the declared T_full are reported as a device-side check failure and
// that user is skipped.
__global__ void __launch_bounds__(SL_SELECT_THREADS) hstu_sl_select_kernel(
    const int64_t* offsets, const int64_t* timestamps, const int32_t* lengths,
    const int64_t* offsets_out, int32_t max_len, int64_t T_full, uint64_t seed, uint64_t step,
    int64_t* kept_index, int64_t* timestamps_out) {
  extern __shared__ __align__(16) uint64_t s_key[];
  __shared__ int s_hist[256];
  __shared__ int s_warp[SL_SELECT_THREADS / 32];
  __shared__ uint64_t s_prefix;
  __shared__ int s_rank;
  const int u = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t base = offsets[u];
  const int n = static_cast<int>(offsets[u + 1] - base);
  const int L = lengths[u];
  const int64_t out0 = offsets_out[u];
  if (n < 0 || n > max_len || base < 0 || base + n > T_full || out0 + L > T_full) {
    if (threadIdx.x == 0) record_status(HSTU_ERR_DEVICE_CHECK);
    return;  // uniform across the CTA
  }
  if (L <= 0) return;  // uniform across the CTA
  if (L < n) {
    for (int pos = tid; pos < n; pos += SL_SELECT_THREADS)
      s_key[pos] =
          philox4x64_10(static_cast<uint64_t>(pos), static_cast<uint64_t>(u), step, 1, seed, 0).w[0];
  }
  if (tid == 0) {
    s_prefix = 0;
    s_rank = L;  // 1-based rank of the threshold key among the candidates
  }
  __syncthreads();
  uint64_t thr = ~0ull;  // keys below thr are kept; `take` keys equal to thr too
  int take = 0;
  if (L < n) {
    // after the pass over digit `shift`, s_prefix holds the threshold's bits
    // above and at that digit, and s_rank its rank among keys sharing them
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int b = tid; b < 256; b += SL_SELECT_THREADS) s_hist[b] = 0;
      __syncthreads();
      const uint64_t pre = s_prefix;
      const uint64_t hi_mask = shift == 56 ? 0ull : (~0ull << (shift + 8));
      for (int pos = tid; pos < n; pos += SL_SELECT_THREADS) {
        const uint64_t k = s_key[pos];
        if ((k & hi_mask) == pre) atomicAdd(&s_hist[(k >> shift) & 255u], 1);
      }
      __syncthreads();
      if (tid == 0) {
        int rank = s_rank, d = 0;
        while (d < 255 && rank > s_hist[d]) {
          rank -= s_hist[d];
          ++d;
        }
        s_prefix = pre | (static_cast<uint64_t>(d) << shift);
        s_rank = rank;
      }
      __syncthreads();
    }
    thr = s_prefix;
    take = s_rank;  // how many keys equal to thr are kept (the lowest positions)
  }
  // compaction in position order, 512 positions per round
  int kept_before = 0, eq_before = 0;
  for (int p0 = 0; p0 < n; p0 += SL_SELECT_THREADS) {
    const int pos = p0 + tid;
    const bool in = pos < n;
    const uint64_t k = (in && L < n) ? s_key[pos] : ~0ull;
    const bool eq = in && L < n && k == thr;
    int eq_total = 0;
    const int eq_rank = sl_block_count(eq, s_warp, &eq_total);
    const bool keep = in && (L >= n || k < thr || (eq && eq_before + eq_rank < take));
    int kept_total = 0;
    const int idx = sl_block_count(keep, s_warp, &kept_total);
    if (keep) {
      const int64_t o = out0 + kept_before + idx;
      kept_index[o] = base + pos;
      if (timestamps_out != nullptr) timestamps_out[o] = timestamps[base + pos];
    }
    kept_before += kept_total;
    eq_before += eq_total;
  }
}

// x_out[r] = x[kept_index[r]] for r < offsets_out[B]: a warp copies four rows
// at a time (16-byte accesses, every load of the four rows issued before the
// first store, so enough bytes are in flight to cover the memory latency),
// grid-strided over the rows.
constexpr int SL_GATHER_ROWS = 4;

__global__ void __launch_bounds__(256) hstu_sl_gather_kernel(const int64_t* offsets_out, int32_t B,
                                                             int64_t T_full,
                                                             const int64_t* kept_index,
                                                             const uint4* x, uint4* x_out,
                                                             int32_t row_vec) {
  const int64_t total = offsets_out[B];
  if (total > T_full) {  // inconsistent input offsets (reported by the selection)
    if (blockIdx.x == 0 && threadIdx.x == 0) record_status(HSTU_ERR_DEVICE_CHECK);
    return;
  }
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  for (int64_t r0 = w0 * SL_GATHER_ROWS; r0 < total; r0 += warps * SL_GATHER_ROWS) {
    int64_t src[SL_GATHER_ROWS];
#pragma unroll
    for (int q = 0; q < SL_GATHER_ROWS; ++q) {
      const int64_t r = r0 + q;
      const int64_t k = r < total ? kept_index[r] : -1;
      src[q] = (k >= 0 && k < T_full) ? k : -1;  // -1: past the end, or a user the selection skipped
    }
    for (int c0 = 0; c0 < row_vec; c0 += 64) {
      uint4 v[SL_GATHER_ROWS][2];
#pragma unroll
      for (int q = 0; q < SL_GATHER_ROWS; ++q)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = c0 + e * 32 + lane;
          if (src[q] >= 0 && c < row_vec) v[q][e] = x[src[q] * row_vec + c];
        }
#pragma unroll
      for (int q = 0; q < SL_GATHER_ROWS; ++q)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = c0 + e * 32 + lane;
          if (src[q] >= 0 && c < row_vec) x_out[(r0 + q) * row_vec + c] = v[q][e];
        }
    }
  }
}

}  // namespace hstu
