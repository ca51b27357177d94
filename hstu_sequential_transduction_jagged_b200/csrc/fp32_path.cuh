// fp32 storage path of the HSTU layer (Eq. 1-3 of the review of "Actions
// Speak Louder than Words", section 三 核心公式), SIMT FFMA arithmetic in fp32.
// It serves layers configured with fp32 storage, which are small (the fp32
// workload has d = 64, one head, tens of tokens per user), so plain tiled
// kernels are used: a 64x64-tile linear layer with a fused bias, activation,
// column-block split and residual; a per-(user, head, 32-row) attention
// kernel; and a one-warp-per-row LayerNorm-and-gate.
#pragma once

#include "attn.cuh"

namespace hstu {

struct F32LinParams {
  const float* a;        // [M, lda]
  int64_t lda;
  const float* w;        // [N, K]
  const float* bias;     // [N]
  const float* res;      // [M, ld_res] or nullptr
  int64_t ld_res;
  float* dst[4];         // destination of column block b
  int64_t ld_dst[4];
  int32_t blk_w;
  int64_t M;
  int32_t N, K;
  int32_t act;
};

__global__ void __launch_bounds__(256) hstu_f32_linear_kernel(const __grid_constant__ F32LinParams p) {
  __shared__ float sa[16][65];
  __shared__ float sw[16][65];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * 64;
  const int n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < p.K; k0 += 16) {
    for (int e = threadIdx.x; e < 64 * 16; e += 256) {
      const int r = e >> 4, kk = e & 15;
      const int64_t gm = m0 + r;
      const int gk = k0 + kk;
      sa[kk][r] = (gm < p.M && gk < p.K) ? p.a[gm * p.lda + gk] : 0.0f;
      const int gn = n0 + r;
      sw[kk][r] = (gn < p.N && gk < p.K) ? p.w[static_cast<int64_t>(gn) * p.K + gk] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float av[4], wv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = sa[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) wv[j] = sw[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], wv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t gm = m0 + ty * 4 + i;
    if (gm >= p.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn >= p.N) continue;
      float z = acc[i][j] + p.bias[gn];
      if (p.act == HSTU_ACT_RELU) z = fmaxf(z, 0.0f);
      else if (p.act == HSTU_ACT_SILU) z = z / (1.0f + expf(-z));
      if (p.res != nullptr) z += p.res[gm * p.ld_res + gn];
      const int blk = gn / p.blk_w;
      p.dst[blk][gm * p.ld_dst[blk] + (gn - blk * p.blk_w)] = z;
    }
  }
}

struct F32AttnParams {
  const float* q; const float* k; const float* v;
  int64_t ldq, ldk, ldv;
  const int64_t* kv_offsets;
  const int64_t* q_offsets;    // candidate mode
  const int64_t* timestamps;
  const int64_t* request_ts;   // candidate mode
  const float* rab_pos;
  const float* rab_time;
  const float* q_self; const float* k_self; const float* v_self;  // candidate mode
  int64_t ld_self;
  float* av;
  int64_t ld_av;
  int32_t B, H, P, Tb, phi2;
  int32_t cand;
  int32_t max_q, max_kv;  // host-declared length bounds the grid is sized for
  const int32_t* segments;  // [B, 2] (n_us, n_r): generalised masks, or nullptr
  int64_t thr[MAX_TIME_BUCKETS];
};

__device__ __forceinline__ float phi_runtime(float x, int kind) {
  if (kind == HSTU_ACT_SILU) return x / (1.0f + expf(-x));
  if (kind == HSTU_ACT_RELU) return fmaxf(x, 0.0f);
  return x;
}

// grid (ceil(max_rows/32), H, B), 128 threads; thread (r = t/4, quarter = t%4)
__global__ void __launch_bounds__(128) hstu_f32_attn_kernel(const __grid_constant__ F32AttnParams p) {
  __shared__ float sq[32][65];
  __shared__ float sk[32][65];
  __shared__ float sv[32][65];
  __shared__ float sp[32][33];
  __shared__ int64_t sthr[MAX_TIME_BUCKETS];
  const int u = blockIdx.z, h = blockIdx.y;
  const int64_t kv0 = p.kv_offsets[u];
  const int n_kv = static_cast<int>(p.kv_offsets[u + 1] - kv0);
  const int64_t q0g = p.cand ? p.q_offsets[u] : kv0;
  const int n_q = p.cand ? static_cast<int>(p.q_offsets[u + 1] - q0g) : n_kv;
  if (n_q > p.max_q || n_kv > p.max_kv || n_q < 0 || n_kv < 0) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) record_status(HSTU_ERR_DEVICE_CHECK);
    return;
  }
  const int r0 = blockIdx.x * 32;
  if (r0 >= n_q) return;
  for (int e = threadIdx.x; e < p.Tb; e += blockDim.x) sthr[e] = p.thr[e];
  const int r = threadIdx.x >> 2, qt = threadIdx.x & 3;
  for (int e = threadIdx.x; e < 32 * 64; e += 128) {
    const int rr = e >> 6, c = e & 63;
    sq[rr][c] = (r0 + rr < n_q) ? p.q[(q0g + r0 + rr) * p.ldq + h * 64 + c] : 0.0f;
  }
  const int i = r0 + r;  // query index within the user
  const int64_t t_row = p.cand ? p.request_ts[u] : ((i < n_q) ? p.timestamps[kv0 + i] : 0);
  const int pos_row = p.cand ? n_kv : i;
  // keys this row sees: the prefix [0, vis_end), and itself when self_row
  // (candidate mode, or a candidate row of the generalised masks)
  int vis_end = i + 1;
  bool self_row = p.cand != 0;
  const bool masked = !p.cand && p.segments != nullptr;
  if (masked) {
    const int n_us = p.segments[2 * u], n_r = p.segments[2 * u + 1];
    if (n_us < 0 || n_r < 0 || n_us + n_r > n_kv) {
      if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) record_status(HSTU_ERR_DEVICE_CHECK);
      return;
    }
    const int r_end = n_us + n_r;
    if (i < n_us) {
      vis_end = n_us;
    } else if (i >= r_end && i < n_q) {
      int lo = n_us, hi = r_end;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (p.timestamps[kv0 + mid] <= t_row) lo = mid + 1;
        else hi = mid;
      }
      vis_end = lo;
      self_row = true;
    }
  }
  float o[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) o[c] = 0.0f;
  const int key_end = (p.cand || masked) ? n_kv : min(n_kv, r0 + 32);
  const float* rp = p.rab_pos + static_cast<int64_t>(h) * p.P;
  const float* rt = p.rab_time + static_cast<int64_t>(h) * p.Tb;
  // The softmax ablation takes two passes: the first finds the row's max m
  // and sum l of exp(x - m) over its visible keys (the candidate's own key
  // included), the second accumulates exp(x - m) / l times V.
  const bool softmax = p.phi2 == HSTU_ACT_SOFTMAX;
  float sm_m = -INFINITY, sm_l = 0.0f, x_self = 0.0f;
  // the row's own query and key (self term)
  const int64_t row_s = q0g + i;
  const float* qs = p.cand ? p.q_self + row_s * p.ld_self : p.q + row_s * p.ldq;
  const float* ks = p.cand ? p.k_self + row_s * p.ld_self : p.k + row_s * p.ldk;
  const float* vs = p.cand ? p.v_self + row_s * p.ld_self : p.v + row_s * p.ldv;
  if (softmax && self_row && i < n_q) {
    float s = 0.0f;
    for (int c = 0; c < 64; ++c) s = fmaf(qs[h * 64 + c], ks[h * 64 + c], s);
    x_self = s + rp[0] + rt[0];
    if (qt == 0) {
      sm_m = x_self;
      sm_l = 1.0f;
    }
  }
  for (int pass = softmax ? 0 : 1; pass < 2; ++pass) {
  if (pass == 1 && softmax) {
    // merge the four threads of the row
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
      const float om = __shfl_xor_sync(0xffffffffu, sm_m, o);
      const float ol = __shfl_xor_sync(0xffffffffu, sm_l, o);
      const float m = fmaxf(sm_m, om);
      sm_l = (m == -INFINITY) ? 0.0f : sm_l * expf(sm_m - m) + ol * expf(om - m);
      sm_m = m;
    }
  }
  for (int j0 = 0; j0 < key_end; j0 += 32) {
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * 64; e += 128) {
      const int rr = e >> 6, c = e & 63;
      const bool in = j0 + rr < n_kv;
      sk[rr][c] = in ? p.k[(kv0 + j0 + rr) * p.ldk + h * 64 + c] : 0.0f;
      sv[rr][c] = in ? p.v[(kv0 + j0 + rr) * p.ldv + h * 64 + c] : 0.0f;
    }
    __syncthreads();
#pragma unroll 1
    for (int kk = 0; kk < 8; ++kk) {
      const int jj = qt * 8 + kk;
      const int j = j0 + jj;
      float pval = 0.0f;
      const bool live = (j < n_kv) && (p.cand || j < vis_end) && (i < n_q);
      if (live) {
        float s = 0.0f;
        for (int c = 0; c < 64; ++c) s = fmaf(sq[r][c], sk[jj][c], s);
        const int bp = min(abs(pos_row - j), p.P - 1);
        const int bt = time_bucket_search(t_row - p.timestamps[kv0 + j], sthr, p.Tb);
        const float x = s + rp[bp] + rt[bt];
        if (!softmax) {
          pval = phi_runtime(x, p.phi2);
        } else if (pass == 0) {
          if (x > sm_m) {
            sm_l = sm_l * expf(sm_m - x) + 1.0f;
            sm_m = x;
          } else {
            sm_l += expf(x - sm_m);
          }
        } else {
          pval = expf(x - sm_m) / sm_l;
        }
      }
      sp[r][jj] = pval;
    }
    __syncthreads();
    if (pass == 1) {
      for (int jj = 0; jj < 32; ++jj) {
        const float pv = sp[r][jj];
#pragma unroll
        for (int c = 0; c < 16; ++c) o[c] = fmaf(pv, sv[jj][qt * 16 + c], o[c]);
      }
    }
  }
  }
  if (i >= n_q) return;
  const int64_t row = q0g + i;
  if (self_row) {
    float ps;
    if (softmax) {
      ps = expf(x_self - sm_m) / sm_l;
    } else {
      float s = 0.0f;
      for (int c = 0; c < 64; ++c) s = fmaf(qs[h * 64 + c], ks[h * 64 + c], s);
      ps = phi_runtime(s + rp[0] + rt[0], p.phi2);
    }
#pragma unroll
    for (int c = 0; c < 16; ++c) o[c] = fmaf(ps, vs[h * 64 + qt * 16 + c], o[c]);
  }
  const float inv_n = softmax ? 1.0f : 1.0f / static_cast<float>(p.cand ? max(n_kv, 1) : n_kv);
#pragma unroll
  for (int c = 0; c < 16; ++c) p.av[row * p.ld_av + h * 64 + qt * 16 + c] = o[c] * inv_n;
}

// g[row] = (LayerNorm(av[row]) * gamma + beta) (.) u[row]; one warp per row.
__global__ void hstu_f32_ln_gate_kernel(const float* av, int64_t ld_av, const float* u, int64_t ld_u,
                                        const float* gamma, const float* beta, float eps,
                                        int64_t M, int width, float* g, int64_t ld_g) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const float* a = av + row * ld_av;
  float s = 0.0f;
  for (int c = lane; c < width; c += 32) s += a[c];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s / static_cast<float>(width);
  float m2 = 0.0f;
  for (int c = lane; c < width; c += 32) {
    const float d = a[c] - mean;
    m2 = fmaf(d, d, m2);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m2 += __shfl_xor_sync(0xffffffffu, m2, o);
  const float rstd = rsqrtf(m2 / static_cast<float>(width) + eps);
  for (int c = lane; c < width; c += 32) {
    float nv = (a[c] - mean) * rstd;
    if (gamma != nullptr) nv *= gamma[c];
    if (beta != nullptr) nv += beta[c];
    g[row * ld_g + c] = nv * u[row * ld_u + c];
  }
}

}  // namespace hstu
