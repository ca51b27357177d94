// Elementwise and row kernels of the HSTU layer backward (the derivative of
// Eq. 1-3 of the review of "Actions Speak Louder than Words", section 三
// 核心公式, with the residual):
//   G = Ln (.) U,  Ln = n gamma + beta,  n = (AV - mean) rstd  (LayerNorm over H*64)
//   dU = dG (.) Ln,  dLn = dG (.) U,  dgamma += dLn (.) n,  dbeta += dLn,
//   dAV = rstd (dn - mean(dn) - n mean(dn (.) n)),  dn = dLn (.) gamma,
//   dZpre = dZ (.) phi1'(Z pre-activation)  (ReLU: Z > 0; identity: 1).
// The GEMMs of the backward (dG = dY W2, dW2 = dY^T G, dW1 = dZ^T X,
// dX = dY + dZ W1) are plain library GEMMs; the attention backward is
// attn_bwd.cuh.
#pragma once

#include "ptx.cuh"

namespace hstu {

// One warp per row (grid-stride): recomputes the LayerNorm of AV from the
// per-head partial sums (the same merge as the f2 kernel), then writes
//   dav16 [T, K]  dAV in the attention operand type (fp16 or bf16),
//   dz    [T, ld_dz] columns 0..K-1: dU masked by phi1' of U,
//   g     [T, K]  G = Ln (.) U (fp32) for dW2,
// and accumulates dgamma / dbeta (per-warp partials, one atomic per column).
// K = H * 64 <= 1024 (each lane owns K / 32 columns, at most 32).
template <int KPL>  // columns per lane: K / 32
__global__ void __launch_bounds__(256) hstu_gate_bwd_kernel(
    const float* av, const float* ln_part, const float* u, const float* dg, const float* gamma,
    const float* beta, float eps, int H, int64_t T, void* dav16, int dav_f16, float* dz,
    int64_t ld_dz, float* g, float* dgamma, float* dbeta, int relu) {
  constexpr int K = KPL * 32;
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  float gm[KPL], bt[KPL], dgam[KPL], dbet[KPL];
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const int c = lane + 32 * e;
    gm[e] = gamma != nullptr ? gamma[c] : 1.0f;
    bt[e] = beta != nullptr ? beta[c] : 0.0f;
    dgam[e] = 0.0f;
    dbet[e] = 0.0f;
  }
  const float inv_k = 1.0f / static_cast<float>(K);
  for (int64_t r = w0; r < T; r += warps) {
    // LayerNorm statistics from the heads' (sum, centred sum of squares)
    const float2* lp = reinterpret_cast<const float2*>(ln_part) + r * H;
    float tot = 0.0f;
    for (int hh = 0; hh < H; ++hh) tot += lp[hh].x;
    const float mean = tot * inv_k;
    float m2 = 0.0f;
    for (int hh = 0; hh < H; ++hh) {
      const float2 v = lp[hh];
      const float dm = v.x * (1.0f / 64.0f) - mean;
      m2 += v.y + 64.0f * dm * dm;
    }
    const float rstd = rsqrtf(m2 * inv_k + eps);
    float n[KPL], dn[KPL];
    float s1 = 0.0f, s2 = 0.0f;
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
      const int64_t idx = r * K + lane + 32 * e;
      const float nv = (av[idx] - mean) * rstd;
      const float ln = fmaf(nv, gm[e], bt[e]);
      const float uv = u[idx];
      const float dgv = dg[idx];
      const float dln = dgv * uv;
      g[idx] = ln * uv;
      float du = dgv * ln;
      if (relu && !(uv > 0.0f)) du = 0.0f;
      dz[r * ld_dz + lane + 32 * e] = du;
      dgam[e] = fmaf(dln, nv, dgam[e]);
      dbet[e] += dln;
      n[e] = nv;
      dn[e] = dln * gm[e];
      s1 += dn[e];
      s2 = fmaf(dn[e], nv, s2);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s1 += __shfl_xor_sync(0xffffffffu, s1, o);
      s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    }
    const float m1 = s1 * inv_k, mn = s2 * inv_k;
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
      const float d = rstd * (dn[e] - m1 - n[e] * mn);
      const int64_t idx = r * K + lane + 32 * e;
      if (dav_f16) reinterpret_cast<__half*>(dav16)[idx] = __float2half_rn(d);
      else reinterpret_cast<__nv_bfloat16*>(dav16)[idx] = __float2bfloat16_rn(d);
    }
  }
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const int c = lane + 32 * e;
    if (dgamma != nullptr && dgam[e] != 0.0f) atomicAdd(&dgamma[c], dgam[e]);
    if (dbeta != nullptr && dbet[e] != 0.0f) atomicAdd(&dbeta[c], dbet[e]);
  }
}

// dz[r, c] *= (z[r, c - c0] > 0) for the columns c0 .. c0 + width - 1 of dz
// (V, Q, K blocks: dz holds their gradients, z the fp16 values the forward
// produced, ReLU so z > 0 exactly where the pre-activation is positive).
__global__ void hstu_relu_mask_kernel(float* dz, int64_t ld_dz, int c0, const __half* z,
                                      int64_t ld_z, int width, int64_t T) {
  const int64_t total = T * width;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += stride) {
    const int64_t r = i / width;
    const int c = static_cast<int>(i - r * width);
    if (!(__half2float(z[r * ld_z + c]) > 0.0f)) dz[r * ld_dz + c0 + c] = 0.0f;
  }
}

// out[c] = sum over rows of a[r, c] (out zeroed before; one atomic per column
// per block of rows).
__global__ void __launch_bounds__(256) hstu_colsum_kernel(const float* a, int64_t lda, int64_t M,
                                                          int N, int rows_per_block, float* out) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= N) return;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_block;
  const int64_t r1 = min(M, r0 + rows_per_block);
  float s = 0.0f;
  for (int64_t r = r0; r < r1; ++r) s += a[r * lda + c];
  atomicAdd(&out[c], s);
}

// dst[i] = float(src[i]) for bf16 src.
__global__ void hstu_bf16_to_f32_kernel(const __nv_bfloat16* src, float* dst, int64_t n) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
    dst[i] = __bfloat162float(src[i]);
}

}  // namespace hstu
