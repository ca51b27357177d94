// The two linear layers of an HSTU block (review of "Actions Speak Louder
// than Words", section 三 核心公式, Eq. 1 and Eq. 3; the efficiency table of
// section 五 counts exactly two linear layers per block):
//
//   f1:  Z = phi1(X W1^T + b1), written straight into the U, V, Q, K blocks
//        (Eq. 1's Split is only a choice of destination per column block).
//   f2:  Y = X + (Norm(AV) (.) U) W2^T + b2 (Eq. 3 plus the residual), with the
//        LayerNorm-and-gate computed by producer warps directly into the
//        swizzled shared-memory A tile, so Norm(AV) (.) U never reaches HBM.
//
// Both are persistent tcgen05 GEMMs with 64-wide K steps through a shared-
// memory ring fed by TMA (128B swizzle), an MMA warp that issues from one
// elected lane, and epilogue warps that stage 128-byte output row segments in
// swizzled shared memory for TMA tensor stores.  f1 uses 128 x 256 tiles, 4
// stages and two tensor-memory accumulators (2 x 256 columns), so the
// epilogue of one tile overlaps the main loop of the next.  f2 uses 128-row
// tiles covering up to 512 output columns (two 256-column halves side by side
// in tensor memory), so its A operand is built once per row tile, with 2
// stages and a single accumulator.
#pragma once

#include "ptx.cuh"

namespace hstu {

constexpr int G_BM = 128;
constexpr int G_BN = 256;
constexpr int G_BK = 64;
constexpr int G_STAGES = 4;
constexpr uint32_t G_A_BYTES = G_BM * G_BK * 2;  // 16 KB
constexpr uint32_t G_B_BYTES = G_BN * G_BK * 2;  // 32 KB
constexpr uint32_t G_STAGE_BYTES = G_A_BYTES + G_B_BYTES;

struct GemmSmem {
  static constexpr uint32_t kA = 0;
  static constexpr uint32_t kB = G_STAGES * G_A_BYTES;
  static constexpr uint32_t kBars = kB + G_STAGES * G_B_BYTES;  // 16 barriers
  static constexpr uint32_t kMisc = kBars + 16 * 8;
  static constexpr uint32_t kRowStats = kMisc + 64;             // 128 x (mean, rstd)
  static constexpr uint32_t kBytes = kRowStats + G_BM * 8 + 1024;
};

enum : int {
  GB_FULL = 0,                       // + stage
  GB_EMPTY = GB_FULL + G_STAGES,     // + stage
  GB_ACC_FULL = GB_EMPTY + G_STAGES, // + buffer
  GB_ACC_EMPTY = GB_ACC_FULL + 2,    // + buffer
  GB_DONE = GB_ACC_EMPTY + 2,
  GB_COUNT = GB_DONE + 1
};

template <int ACT>
__device__ __forceinline__ float apply_act(float x) {
  if constexpr (ACT == HSTU_ACT_RELU) {
    return fmaxf(x, 0.0f);
  } else if constexpr (ACT == HSTU_ACT_SILU) {
    return x / (1.0f + __expf(-x));
  } else {
    return x;
  }
}

// f1's extra shared memory: per epilogue warp two 4 KB staging buffers of 32
// rows x 128 bytes (128B-swizzled) for the tensor stores of the output.
struct F1Smem {
  static constexpr uint32_t kOut = (GemmSmem::kMisc + 64 + 1023) / 1024 * 1024;
  static constexpr uint32_t kBufBytes = 32 * 128;
  static constexpr uint32_t kBytes = kOut + 4 * 2 * kBufBytes + 1024;
};
static_assert(F1Smem::kBytes <= 227u * 1024u, "f1 shared memory");

// Tensor maps of the four output column blocks (U, V, Q, K): rows of the
// block, 128-byte boxes (32 fp32 or 64 bf16 columns) x 32 rows, 128B swizzle.
struct F1OutMaps {
  CUtensorMap m[4];
};

struct F1Params {
  void* dst[4];           // destination of column block b (U, V, Q, K)
  int64_t ld_dst[4];      // row stride of each destination (elements)
  uint32_t f32_mask;      // bit b set: block b is stored as fp32
  uint32_t f16_mask;      // bit b set: block b is stored as fp16 (else bf16)
  int32_t ab_f16;         // X and W1 are fp16 (else bf16)
  const float* bias;      // [N]
  int64_t M;
  int32_t N, K;
  int32_t blk_w;          // width of one column block (H*64)
  int32_t num_m_tiles, num_n_tiles;
  uint64_t timeout_ns;
};

// f2 works on 128-row tiles that cover up to F2_NW = 512 output columns: two
// 256-column MMA halves accumulate side by side in tensor memory, so each
// k-block of the A operand, LayerNorm(AV) (.) U, is built once per row tile
// (a 256-column tiling builds it once per column tile).  A stage holds the
// A tile and both W2 halves; the single accumulator uses all 512 columns.
constexpr int F2_STAGES = 2;
constexpr int F2_NW = 2 * G_BN;
constexpr uint32_t F2_B_BYTES = 2 * G_B_BYTES;  // both W2 halves of a k-block: 64 KB

struct F2Smem {
  static constexpr uint32_t kA = 0;                                // stages x 16 KB
  static constexpr uint32_t kB = F2_STAGES * G_A_BYTES;            // stages x 64 KB
  static constexpr uint32_t kBars = kB + F2_STAGES * F2_B_BYTES;   // 16 barriers
  static constexpr uint32_t kMisc = kBars + 16 * 8;
  static constexpr uint32_t kRowStats = kMisc + 64;                // 128 x (mean, rstd)
  // per epilogue warp one 4 KB staging buffer for Y (32 rows x 32 fp32) and one
  // for its bf16 copy (32 rows x 64 bf16), both 128B-swizzled, for tensor stores
  static constexpr uint32_t kOut = (kRowStats + G_BM * 8 + 1023) / 1024 * 1024;
  static constexpr uint32_t kBufBytes = 32 * 128;
  static constexpr uint32_t kBytes = kOut + 4 * 2 * kBufBytes + 1024;
};
static_assert(F2Smem::kBytes <= 227u * 1024u, "f2 shared memory");

enum : int {
  F2B_FULL = 0,                          // + stage: W2 bytes + every A-producer warp
  F2B_EMPTY = F2B_FULL + F2_STAGES,      // + stage
  F2B_ACC_FULL = F2B_EMPTY + F2_STAGES,
  F2B_ACC_EMPTY = F2B_ACC_FULL + 1,
  F2B_DONE = F2B_ACC_EMPTY + 1,
};

// Tensor maps of Y (fp32) and of its bf16 copy: 128-byte boxes x 32 rows.
struct F2OutMaps {
  CUtensorMap y, y_lp;
};

struct F2Params {
  const float* av;          // [M, ld_av] fp32 attention output
  const float* u;           // [M, ld_u] fp32 gate
  int64_t ld_av, ld_u;
  const float* ln_part;     // [M, H, 2] per-head (sum, centred sum of squares) of AV rows
  const float* gamma;       // [K] or nullptr
  const float* beta;        // [K] or nullptr
  float eps;
  const float* bias;        // [N]
  const float* x_res;       // [M, ld_x] fp32 residual, or nullptr -> x_lp
  const __nv_bfloat16* x_lp;
  int64_t ld_x;
  float* y;                 // [M, ld_y] fp32
  void* y_lp;               // [M, ld_y] bf16 (fp16 when ylp_f16), or nullptr
  int32_t ylp_f16;
  int32_t ab_f16;           // the A tile (Norm(AV) (.) U) and W2 are fp16 (else bf16)
  int64_t ld_y;
  int64_t M;
  int32_t N, K, H;
  int32_t num_m_tiles, num_n_tiles;  // f2: num_n_tiles counts groups of F2_NW columns
  uint64_t timeout_ns;
};

// ------------------------------------------------------------------ shared pieces

struct TileIter {
  int t, step, total, n_tiles;
  __device__ __forceinline__ int m() const { return t / n_tiles; }
  __device__ __forceinline__ int n() const { return t % n_tiles; }
};

// Run by a whole warp (waits are warp votes); one elected lane issues every
// MMA and commit.
__device__ __forceinline__ void gemm_mma_loop(uint64_t* bars, const uint8_t* sA, const uint8_t* sB,
                                              uint32_t tmem, int total_tiles, int k_blocks,
                                              const WaitCtl& ctl, uint64_t drain_ns, bool f16) {
  const uint32_t idesc = idesc_16_f32(G_BM, G_BN, false, false, f16);
  const bool leader = elect_one();
  auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
    return __all_sync(0xffffffffu, mbar_wait(bar, par, ctl));
  };
  int stage = 0;
  uint32_t phase = 0;
  int lt = 0;
  bool ok = true;
  for (int t = blockIdx.x; ok && t < total_tiles; t += gridDim.x, ++lt) {
    const int acc = lt & 1;
    const uint32_t acc_par = (static_cast<uint32_t>(lt >> 1) & 1u) ^ 1u;
    ok = wait_all(&bars[GB_ACC_EMPTY + acc], acc_par);
    if (!ok) break;
    tc_fence_after();
    const uint32_t d = tmem + static_cast<uint32_t>(acc * G_BN);
    for (int kb = 0; kb < k_blocks; ++kb) {
      ok = wait_all(&bars[GB_FULL + stage], phase);
      if (!ok) break;
      tc_fence_after();
      const uint64_t da = smem_desc_sw128(smem_u32(sA + stage * G_A_BYTES), 16, 1024);
      const uint64_t db = smem_desc_sw128(smem_u32(sB + stage * G_B_BYTES), 16, 1024);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < G_BK / 16; ++kk)
          mma_bf16_ss(d, da + 2 * kk, db + 2 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars[GB_EMPTY + stage]);
      }
      __syncwarp();
      if (++stage == G_STAGES) { stage = 0; phase ^= 1u; }
    }
    if (ok && leader) mma_commit(&bars[GB_ACC_FULL + acc]);
    __syncwarp();
  }
  if (leader) mma_commit(&bars[GB_DONE]);
  __syncwarp();
  mbar_wait_drain(&bars[GB_DONE], 0, drain_ns);
}

// ------------------------------------------------------------------ f1

template <int ACT>
__global__ void __launch_bounds__(192, 1)
hstu_f1_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
               const __grid_constant__ F1OutMaps out,
               const __grid_constant__ F1Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem + GemmSmem::kA;
  uint8_t* sB = smem + GemmSmem::kB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + GemmSmem::kBars);
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + GemmSmem::kMisc);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + GemmSmem::kMisc + 4);
  const int warp = warp_id(), lane = lane_id();
  const int total = p.num_m_tiles * p.num_n_tiles;
  const int k_blocks = p.K / G_BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < G_STAGES; ++s) {
      mbar_init(&bars[GB_FULL + s], 1);
      mbar_init(&bars[GB_EMPTY + s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[GB_ACC_FULL + b], 1);
      mbar_init(&bars[GB_ACC_EMPTY + b], 128);
    }
    mbar_init(&bars[GB_DONE], 1);
    *sAbort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sTmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;
  const WaitCtl ctl{sAbort, p.timeout_ns};

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      tma_prefetch_desc(&tm_w);
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
        const int mt = t / p.num_n_tiles, nt = t % p.num_n_tiles;
        for (int kb = 0; kb < k_blocks; ++kb) {
          ok = mbar_wait(&bars[GB_EMPTY + stage], phase ^ 1u, ctl);
          if (!ok) break;
          mbar_arrive_expect_tx(&bars[GB_FULL + stage], G_STAGE_BYTES);
          tma_load_2d(sA + stage * G_A_BYTES, &tm_x, &bars[GB_FULL + stage], kb * G_BK, mt * G_BM);
          tma_load_2d(sB + stage * G_B_BYTES, &tm_w, &bars[GB_FULL + stage], kb * G_BK, nt * G_BN);
          ++issued;
          if (++stage == G_STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // drain the loads still in flight
      for (int k = max(0, issued - G_STAGES); k < issued; ++k)
        mbar_wait_drain(&bars[GB_FULL + (k % G_STAGES)], static_cast<uint32_t>(k / G_STAGES) & 1u,
                          p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    gemm_mma_loop(bars, sA, sB, tmem, total, k_blocks, ctl, p.timeout_ns, p.ab_f16 != 0);
    __syncwarp();
  } else {
    // epilogue warps 2..5: TMEM lane quarter = warp % 4.  Each warp turns its
    // 32 rows into 128-byte row segments (32 fp32 or 64 bf16 columns) in a
    // 128B-swizzled staging buffer and writes them with tensor stores; two
    // buffers alternate, a buffer is refilled once its store has read it.
    const int q4 = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    uint8_t* stage_base = smem + F1Smem::kOut + q4 * 2 * F1Smem::kBufBytes;
    uint8_t* my_row = nullptr;  // this lane's row in the current buffer
    const int sw = lane & 7;    // 16-byte chunk j of row r sits at chunk j ^ (r % 8)
    int nseg = 0;               // segments this warp has stored
    int lt = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++lt) {
      const int mt = t / p.num_n_tiles, nt = t % p.num_n_tiles;
      const int acc = lt & 1;
      bool ok = mbar_wait(&bars[GB_ACC_FULL + acc], static_cast<uint32_t>(lt >> 1) & 1u, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int32_t row0 = static_cast<int32_t>(static_cast<int64_t>(mt) * G_BM + q4 * 32);
#pragma unroll 1
      for (int ch = 0; ch < G_BN / 32; ++ch) {
        uint32_t v[32];
        __syncwarp();
        tmem_ld32(tmem + lane_off + static_cast<uint32_t>(acc * G_BN + ch * 32), v);
        tmem_ld_wait();
        const int col = nt * G_BN + ch * 32;
        const int blk = col / p.blk_w;
        const int cb = col - blk * p.blk_w;
        const bool f32 = (p.f32_mask >> blk) & 1u;
        const bool h16 = (p.f16_mask >> blk) & 1u;
        const float4* b4 = reinterpret_cast<const float4*>(p.bias + col);
        float z[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 bb = __ldg(b4 + q);
          z[4 * q + 0] = apply_act<ACT>(__uint_as_float(v[4 * q + 0]) + bb.x);
          z[4 * q + 1] = apply_act<ACT>(__uint_as_float(v[4 * q + 1]) + bb.y);
          z[4 * q + 2] = apply_act<ACT>(__uint_as_float(v[4 * q + 2]) + bb.z);
          z[4 * q + 3] = apply_act<ACT>(__uint_as_float(v[4 * q + 3]) + bb.w);
        }
        // a bf16 segment takes two 32-column chunks; blocks are 64-column aligned
        if (f32 || (ch & 1) == 0) {
          if (lane == 0) bulk_wait_read1();  // the store that used this buffer has read it
          __syncwarp();
          my_row = stage_base + (nseg & 1) * F1Smem::kBufBytes + lane * 128;
        }
        if (f32) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<float4*>(my_row + ((j ^ sw) << 4)) =
                make_float4(z[4 * j], z[4 * j + 1], z[4 * j + 2], z[4 * j + 3]);
        } else {
          const int j0 = (ch & 1) * 4;
          auto pk2 = [h16](float a, float b) { return h16 ? pack_h2(a, b) : pack_bf16x2(a, b); };
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(my_row + (((j0 + j) ^ sw) << 4)) =
                make_uint4(pk2(z[8 * j], z[8 * j + 1]), pk2(z[8 * j + 2], z[8 * j + 3]),
                           pk2(z[8 * j + 4], z[8 * j + 5]), pk2(z[8 * j + 6], z[8 * j + 7]));
        }
        if (f32 || (ch & 1) == 1) {
          fence_proxy_async_smem();  // this lane's writes, before the tensor store reads them
          __syncwarp();
          if (lane == 0) {
            // rows at or past M lie outside the tensor and are not written
            tma_store_2d(&out.m[blk], stage_base + (nseg & 1) * F1Smem::kBufBytes,
                         f32 ? cb : cb - 32, row0);
            bulk_commit();
          }
          ++nseg;
        }
      }
      tc_fence_before();
      mbar_arrive(&bars[GB_ACC_EMPTY + acc]);
    }
    // every store must have completed before shared memory is released
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ f2

constexpr int F2_PRODUCER_WARPS = 8;
constexpr int F2_THREADS = (6 + F2_PRODUCER_WARPS) * 32;

__global__ void __launch_bounds__(F2_THREADS, 1)
hstu_f2_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ F2OutMaps out,
               const __grid_constant__ F2Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem + F2Smem::kA;
  uint8_t* sB = smem + F2Smem::kB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + F2Smem::kBars);
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + F2Smem::kMisc);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + F2Smem::kMisc + 4);
  float2* sStats = reinterpret_cast<float2*>(smem + F2Smem::kRowStats);
  const int warp = warp_id(), lane = lane_id();
  const int total = p.num_m_tiles * p.num_n_tiles;
  const int k_blocks = p.K / G_BK;
  // 256-column MMA halves in column group ng (the last group may have one)
  auto halves_of = [&](int ng) { return min(2, (p.N - ng * F2_NW + G_BN - 1) / G_BN); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < F2_STAGES; ++s) {
      mbar_init(&bars[F2B_FULL + s], 1 + F2_PRODUCER_WARPS);  // TMA of W2 + A-tile producer warps
      mbar_init(&bars[F2B_EMPTY + s], 1);
    }
    mbar_init(&bars[F2B_ACC_FULL], 1);
    mbar_init(&bars[F2B_ACC_EMPTY], 128);
    mbar_init(&bars[F2B_DONE], 1);
    *sAbort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sTmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;
  const WaitCtl ctl{sAbort, p.timeout_ns};

  if (warp == 0) {
    // W2 tiles by TMA
    if (lane == 0) {
      tma_prefetch_desc(&tm_w);
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
        const int ng = t % p.num_n_tiles;
        const int nh = halves_of(ng);
        for (int kb = 0; kb < k_blocks; ++kb) {
          ok = mbar_wait(&bars[F2B_EMPTY + stage], phase ^ 1u, ctl);
          if (!ok) break;
          mbar_arrive_expect_tx(&bars[F2B_FULL + stage], nh * G_B_BYTES);
          for (int hf = 0; hf < nh; ++hf)
            tma_load_2d(sB + stage * F2_B_BYTES + hf * G_B_BYTES, &tm_w, &bars[F2B_FULL + stage],
                        kb * G_BK, ng * F2_NW + hf * G_BN);
          ++issued;
          if (++stage == F2_STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      for (int k = max(0, issued - F2_STAGES); k < issued; ++k)
        mbar_wait_drain(&bars[F2B_FULL + (k % F2_STAGES)], static_cast<uint32_t>(k / F2_STAGES) & 1u,
                          p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // MMA warp: whole-warp loop, one elected lane issues.  Per k-block both
    // 256-column halves (tensor-memory columns 0-255 and 256-511).
    const uint32_t idesc = idesc_16_f32(G_BM, G_BN, false, false, p.ab_f16 != 0);
    constexpr uint64_t kHalfDesc = G_B_BYTES >> 4;  // start-address step of the second W2 half
    const bool leader = elect_one();
    auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, par, ctl));
    };
    int stage = 0;
    uint32_t phase = 0;
    int lt = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < total; t += gridDim.x, ++lt) {
      const int nh = halves_of(t % p.num_n_tiles);
      // the epilogue has drained the previous tile's accumulator
      ok = wait_all(&bars[F2B_ACC_EMPTY], (static_cast<uint32_t>(lt) & 1u) ^ 1u);
      if (!ok) break;
      tc_fence_after();
      for (int kb = 0; kb < k_blocks; ++kb) {
        ok = wait_all(&bars[F2B_FULL + stage], phase);
        if (!ok) break;
        tc_fence_after();
        const uint64_t da = smem_desc_sw128(smem_u32(sA + stage * G_A_BYTES), 16, 1024);
        const uint64_t db = smem_desc_sw128(smem_u32(sB + stage * F2_B_BYTES), 16, 1024);
        if (leader) {
          for (int hf = 0; hf < nh; ++hf) {
#pragma unroll
            for (int kk = 0; kk < G_BK / 16; ++kk)
              mma_bf16_ss(tmem + static_cast<uint32_t>(hf * G_BN), da + 2 * kk,
                          db + hf * kHalfDesc + 2 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bars[F2B_EMPTY + stage]);
        }
        __syncwarp();
        if (++stage == F2_STAGES) { stage = 0; phase ^= 1u; }
      }
      if (ok && leader) mma_commit(&bars[F2B_ACC_FULL]);
      __syncwarp();
    }
    if (leader) mma_commit(&bars[F2B_DONE]);
    __syncwarp();
    mbar_wait_drain(&bars[F2B_DONE], 0, p.timeout_ns);
  } else if (warp >= 6) {
    // A-tile producers: Norm(AV) (.) U, bf16, 128B-swizzled K-major layout.
    // Each warp owns 16 rows of the tile; all of a k-block's loads (4 rows x
    // 8 fp32 of AV and of U per thread) are issued before the smem stage is
    // awaited, so a whole k-block (64 KB per CTA) is in flight at once.
    const int aw = warp - 6;                 // 0..F2_PRODUCER_WARPS-1
    const int tp = threadIdx.x - 6 * 32;     // 0..255
    const int sub = lane >> 3;               // row within a group of 4
    const int c16 = lane & 7;                // 16-byte chunk within a 128-byte row
    constexpr int kRowsPerWarp = G_BM / F2_PRODUCER_WARPS;  // 16
    constexpr int kIters = kRowsPerWarp / 4;                // 4
    const float inv_cnt = 1.0f / static_cast<float>(p.K);
    const float inv_hd = 1.0f / 64.0f;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    // every producer warp runs every iteration (the named barriers below must
    // match); after a failed wait a warp only skips the work
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const int mt = t / p.num_n_tiles;
      const int64_t m0 = static_cast<int64_t>(mt) * G_BM;
      // per-row LayerNorm statistics combined from per-head partial sums
      {
        named_barrier_sync(1, 32 * F2_PRODUCER_WARPS);  // previous tile's readers are done
        if (tp < G_BM) {
          const int64_t row = m0 + tp;
          float mean = 0.0f, rstd = 0.0f;
          if (row < p.M) {
            const float2* lp = reinterpret_cast<const float2*>(p.ln_part + row * p.H * 2);
            float tot = 0.0f;
            for (int hh = 0; hh < p.H; ++hh) tot += lp[hh].x;
            mean = tot * inv_cnt;
            float m2 = 0.0f;
            for (int hh = 0; hh < p.H; ++hh) {
              const float2 v = lp[hh];
              const float dm = v.x * inv_hd - mean;
              m2 += v.y + 64.0f * dm * dm;
            }
            rstd = rsqrtf(m2 * inv_cnt + p.eps);
          }
          sStats[tp] = make_float2(mean, rstd);
        }
        named_barrier_sync(1, 32 * F2_PRODUCER_WARPS);
      }
      for (int kb = 0; kb < k_blocks && ok; ++kb) {
        const int col = kb * G_BK + c16 * 8;
        float4 av[kIters][2], uv[kIters][2];
#pragma unroll
        for (int it = 0; it < kIters; ++it) {
          const int64_t row = m0 + aw * kRowsPerWarp + it * 4 + sub;
          if (row < p.M) {
            const float4* ap = reinterpret_cast<const float4*>(p.av + row * p.ld_av + col);
            const float4* up = reinterpret_cast<const float4*>(p.u + row * p.ld_u + col);
            av[it][0] = ap[0]; av[it][1] = ap[1];
            uv[it][0] = up[0]; uv[it][1] = up[1];
          } else {
            av[it][0] = av[it][1] = uv[it][0] = uv[it][1] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        float gm[8], bt[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) { gm[e] = 1.0f; bt[e] = 0.0f; }
        if (p.gamma != nullptr) {
          const float4 g0 = __ldg(reinterpret_cast<const float4*>(p.gamma + col));
          const float4 g1 = __ldg(reinterpret_cast<const float4*>(p.gamma + col) + 1);
          gm[0] = g0.x; gm[1] = g0.y; gm[2] = g0.z; gm[3] = g0.w;
          gm[4] = g1.x; gm[5] = g1.y; gm[6] = g1.z; gm[7] = g1.w;
        }
        if (p.beta != nullptr) {
          const float4 b0 = __ldg(reinterpret_cast<const float4*>(p.beta + col));
          const float4 b1 = __ldg(reinterpret_cast<const float4*>(p.beta + col) + 1);
          bt[0] = b0.x; bt[1] = b0.y; bt[2] = b0.z; bt[3] = b0.w;
          bt[4] = b1.x; bt[5] = b1.y; bt[6] = b1.z; bt[7] = b1.w;
        }
        int wok = 0;
        if (lane == 0) wok = mbar_wait(&bars[F2B_EMPTY + stage], phase ^ 1u, ctl) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, wok, 0) != 0;
        if (!ok) break;
        uint8_t* a_tile = sA + stage * G_A_BYTES;
#pragma unroll
        for (int it = 0; it < kIters; ++it) {
          const int r = aw * kRowsPerWarp + it * 4 + sub;
          const float2 st = sStats[r];
          const float af[8] = {av[it][0].x, av[it][0].y, av[it][0].z, av[it][0].w,
                               av[it][1].x, av[it][1].y, av[it][1].z, av[it][1].w};
          const float uf[8] = {uv[it][0].x, uv[it][0].y, uv[it][0].z, uv[it][0].w,
                               uv[it][1].x, uv[it][1].y, uv[it][1].z, uv[it][1].w};
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float g0 = fmaf((af[2 * e] - st.x) * st.y, gm[2 * e], bt[2 * e]) * uf[2 * e];
            const float g1 =
                fmaf((af[2 * e + 1] - st.x) * st.y, gm[2 * e + 1], bt[2 * e + 1]) * uf[2 * e + 1];
            w4[e] = p.ab_f16 ? pack_h2(g0, g1) : pack_bf16x2(g0, g1);
          }
          // rows past the end carry zeros (their stats are zero and the data too)
          *reinterpret_cast<uint4*>(a_tile + r * 128 + ((c16 ^ (r & 7)) << 4)) =
              make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[F2B_FULL + stage]);
        if (++stage == F2_STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  } else {
    // epilogue warps 2..5: + b2 + residual; Y (fp32, 32-column segments) and
    // its optional bf16 copy (64-column segments) go out through 128B-swizzled
    // staging buffers and tensor stores
    const int q4 = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const int row_in_tile = q4 * 32 + lane;
    uint8_t* buf_y = smem + F2Smem::kOut + q4 * 2 * F2Smem::kBufBytes;
    uint8_t* buf_l = buf_y + F2Smem::kBufBytes;
    const int sw = lane & 7;  // 16-byte chunk j of row r sits at chunk j ^ (r % 8)
    int lt = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++lt) {
      const int mt = t / p.num_n_tiles, ng = t % p.num_n_tiles;
      bool ok = mbar_wait(&bars[F2B_ACC_FULL], static_cast<uint32_t>(lt) & 1u, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int64_t row = static_cast<int64_t>(mt) * G_BM + row_in_tile;
      const bool row_ok = row < p.M;
      const int32_t row0 = static_cast<int32_t>(static_cast<int64_t>(mt) * G_BM + q4 * 32);
#pragma unroll 1
      for (int ch = 0; ch < F2_NW / 32; ++ch) {
        const int col = ng * F2_NW + ch * 32;
        if (col >= p.N) break;  // warp-uniform: the last column group may be partial
        uint32_t v[32];
        __syncwarp();
        tmem_ld32(tmem + lane_off + static_cast<uint32_t>(ch * 32), v);
        tmem_ld_wait();
        float y[32];
        const float4* b4 = reinterpret_cast<const float4*>(p.bias + col);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 bb = __ldg(b4 + q);
          y[4 * q + 0] = __uint_as_float(v[4 * q + 0]) + bb.x;
          y[4 * q + 1] = __uint_as_float(v[4 * q + 1]) + bb.y;
          y[4 * q + 2] = __uint_as_float(v[4 * q + 2]) + bb.z;
          y[4 * q + 3] = __uint_as_float(v[4 * q + 3]) + bb.w;
        }
        if (row_ok) {
          if (p.x_res != nullptr) {
            const float4* xr = reinterpret_cast<const float4*>(p.x_res + row * p.ld_x + col);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 xx = xr[q];
              y[4 * q + 0] += xx.x;
              y[4 * q + 1] += xx.y;
              y[4 * q + 2] += xx.z;
              y[4 * q + 3] += xx.w;
            }
          } else {
            const uint4* xr = reinterpret_cast<const uint4*>(p.x_lp + row * p.ld_x + col);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 xx = xr[q];
              const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&xx);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(x2[e]);
                y[8 * q + 2 * e] += f.x;
                y[8 * q + 2 * e + 1] += f.y;
              }
            }
          }
        }
        // both staging buffers are free once the earlier stores have read them
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
        uint8_t* ry = buf_y + lane * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<float4*>(ry + ((j ^ sw) << 4)) =
              make_float4(y[4 * j], y[4 * j + 1], y[4 * j + 2], y[4 * j + 3]);
        const bool lp = p.y_lp != nullptr;
        const bool lp16 = p.ylp_f16 != 0;
        auto pk2 = [lp16](float a, float b) { return lp16 ? pack_h2(a, b) : pack_bf16x2(a, b); };
        if (lp) {
          // this chunk is one half of a 64-column bf16 segment
          uint8_t* rl = buf_l + lane * 128;
          const int j0 = (ch & 1) * 4;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(rl + (((j0 + j) ^ sw) << 4)) =
                make_uint4(pk2(y[8 * j], y[8 * j + 1]), pk2(y[8 * j + 2], y[8 * j + 3]),
                           pk2(y[8 * j + 4], y[8 * j + 5]), pk2(y[8 * j + 6], y[8 * j + 7]));
        }
        fence_proxy_async_smem();  // this lane's writes, before the tensor stores read them
        __syncwarp();
        if (lane == 0) {
          // rows at or past M lie outside the tensor and are not written
          tma_store_2d(&out.y, buf_y, col, row0);
          if (lp && ((ch & 1) == 1 || col + 32 >= p.N)) tma_store_2d(&out.y_lp, buf_l, col & ~63, row0);
          bulk_commit();
        }
      }
      tc_fence_before();
      mbar_arrive(&bars[F2B_ACC_EMPTY]);
    }
    // every store must have completed before shared memory is released
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ weight conversion

// dst[i] = fp16(src[i]) for bf16 src: exact for every bf16 value inside the
// fp16 normal range (both carry 8 bits of significand or more); values below
// 2^-14 keep fp16's subnormal spacing of 2^-24.  n is a multiple of 8 and
// both pointers are 16-byte aligned.
__global__ void hstu_bf16_to_f16_kernel(const uint4* src, uint4* dst, int64_t n8) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const uint4 v = src[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
      o[e] = pack_h2(f.x, f.y);
    }
    dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// dst[i] = fp16(src[i]) for fp32 src (round to nearest, saturating at
// +-65504); n is a multiple of 8, both pointers 16-byte aligned.
__global__ void hstu_f32_to_f16_kernel(const float4* src, uint4* dst, int64_t n8) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const float4 a = src[2 * i], b = src[2 * i + 1];
    dst[i] = make_uint4(pack_h2(a.x, a.y), pack_h2(a.z, a.w), pack_h2(b.x, b.y), pack_h2(b.z, b.w));
  }
}

// ------------------------------------------------------------------ M-FALCON score

// score[r] = <y[r, :], e[r, :]>, one warp per candidate row.
template <typename TE>
__global__ void hstu_score_kernel(const float* y, int64_t ld_y, const TE* e, int64_t ld_e,
                                  int64_t M, int d, float* scores) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  float acc = 0.0f;
  for (int c = lane; c < d; c += 32) {
    float ev;
    if constexpr (sizeof(TE) == 2) ev = __bfloat162float(e[row * ld_e + c]);
    else ev = static_cast<float>(e[row * ld_e + c]);
    acc = fmaf(y[row * ld_y + c], ev, acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) scores[row] = acc;
}

}  // namespace hstu
