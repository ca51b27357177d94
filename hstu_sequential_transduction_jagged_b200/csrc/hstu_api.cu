// libhstu: the C ABI declared in include/hstu.h.
//
// Host side of every entry point: argument validation (no launch on error),
// workspace carving, TMA tensor-map encoding and kernel launches on the
// caller's stream.  The library is one translation unit so the device status
// word in status.cuh is shared by all kernels.
#include <cublas_v2.h>
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/hstu.h"
#include "attn.cuh"
#include "attn_bwd.cuh"
#include "fp32_path.cuh"
#include "gemm.cuh"
#include "layer_bwd.cuh"
#include "sl.cuh"

using namespace hstu;

namespace {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per bounded wait
constexpr int kMaxLen = 16384;
constexpr int kMaxPos = 16384;
constexpr int kMaxDevices = 64;

#define HSTU_CHECK_CUDA(expr)                      \
  do {                                             \
    cudaError_t err__ = (expr);                    \
    if (err__ != cudaSuccess) return HSTU_ERR_CUDA; \
  } while (0)

// ------------------------------------------------------------------ time buckets

// The unclamped bucket formula of rab^{p,t}: floor(ln(dt + 1) / 0.301), dt < 0 -> 0.
int64_t time_bucket_formula(int64_t dt) {
  if (dt < 0) return 0;
  return static_cast<int64_t>(std::floor(std::log(static_cast<double>(dt) + 1.0) / 0.301));
}

// thr[k] = min { dt >= 0 : formula(dt) >= k } for k = 1..Tb-1, thr[0] = 0.
// The formula is non-decreasing in dt, so a doubling search plus bisection
// finds each edge exactly; the kernels then compare integers only.
// Buckets that no dt below 2^62 reaches get INT64_MAX.
void compute_thresholds(int Tb, int64_t* thr) {
  const int64_t cap = int64_t(1) << 62;
  thr[0] = 0;
  for (int k = 1; k < Tb; ++k) {
    if (time_bucket_formula(cap) < k) {
      thr[k] = INT64_MAX;
      continue;
    }
    int64_t hi = 1;
    while (time_bucket_formula(hi) < k) hi = (hi < cap / 2) ? hi * 2 : cap;
    int64_t lo = 0;
    while (lo < hi) {
      const int64_t mid = lo + (hi - lo) / 2;
      if (time_bucket_formula(mid) >= k) hi = mid; else lo = mid + 1;
    }
    thr[k] = lo;
  }
}

// Octave table for dt < 2^31 - 1: for dt + 1 in [2^k, 2^(k+1)), {t1, t2, t3}
// are the next three bucket edges after bucket(2^k - 1) (INT32_MAX when the
// bucket index would reach Tb or the edge does not fit), w = bucket(2^k - 1).
// Returns false if some octave holds more than three edges.
bool compute_octaves(int Tb, const int64_t* thr, int4* oct) {
  for (int k = 0; k < 32; ++k) {
    const int64_t lo = (int64_t(1) << k) - 1;
    const int64_t hi = (int64_t(2) << k) - 2;  // largest dt with dt + 1 < 2^(k+1)
    int b = 0;
    while (b + 1 < Tb && thr[b + 1] <= lo) ++b;
    int32_t t[4];
    for (int e = 0; e < 4; ++e) {
      const int idx = b + 1 + e;
      t[e] = (idx < Tb && thr[idx] < INT32_MAX) ? static_cast<int32_t>(thr[idx]) : INT32_MAX;
    }
    if (static_cast<int64_t>(t[3]) <= hi && t[3] != INT32_MAX) return false;
    oct[k] = make_int4(t[0], t[1], t[2], b);
  }
  return true;
}

const int64_t* thresholds_for(int Tb) {
  static std::mutex mu;
  static int64_t table[MAX_TIME_BUCKETS + 1][MAX_TIME_BUCKETS];
  static bool ready[MAX_TIME_BUCKETS + 1] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (!ready[Tb]) {
    compute_thresholds(Tb, table[Tb]);
    ready[Tb] = true;
  }
  return table[Tb];
}

// ------------------------------------------------------------------ profiler

enum KernelKind : int {
  K_F1 = 0, K_ATTN, K_F2, K_CAND_ATTN, K_SCORE, K_F32_LINEAR, K_F32_ATTN, K_F32_LN, K_CVT,
  K_SL, K_SL_GATHER, K_ATTN_FUSED, K_ATTN_BWD, K_BWD_GEMM, K_GATE_BWD,
  K_BWD_ELT, K_COUNT
};
const char* const kKernelNames[K_COUNT] = {"f1_gemm",     "attention",      "f2_gemm",
                                           "mfalcon_attention", "score",    "fp32_linear",
                                           "fp32_attention",    "fp32_ln_gate", "weight_cvt",
                                           "sl_select",         "sl_gather",
                                           "attention_f2_fused", "attention_bwd",
                                           "bwd_gemm_cublas", "gate_bwd", "bwd_elementwise"};

struct Profiler {
  std::mutex mu;
  bool on = false;
  struct Rec { int kind; cudaEvent_t a, b; };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
};

Profiler& profiler() {
  static Profiler p;
  return p;
}

// Brackets one kernel launch with events while the profiler is on.
class ProfScope {
 public:
  ProfScope(int kind, cudaStream_t st) : kind_(kind), st_(st) {
    Profiler& p = profiler();
    std::lock_guard<std::mutex> lock(p.mu);
    if (!p.on) return;
    a_ = p.get();
    b_ = p.get();
    if (a_ != nullptr) cudaEventRecord(a_, st_);
  }
  ~ProfScope() {
    if (a_ == nullptr || b_ == nullptr) return;
    cudaEventRecord(b_, st_);
    Profiler& p = profiler();
    std::lock_guard<std::mutex> lock(p.mu);
    p.recs.push_back({kind_, a_, b_});
  }

 private:
  int kind_;
  cudaStream_t st_;
  cudaEvent_t a_ = nullptr, b_ = nullptr;
};

// ------------------------------------------------------------------ device info

using AttnKernelFn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                             const CUtensorMap, const AttnParams);

template <bool CAND, bool PAIRS, bool F16, bool FUSED>
AttnKernelFn attn_kernel_for(int phi) {
  switch (phi) {
    case HSTU_ACT_SILU: return hstu_attn_kernel<CAND, HSTU_ACT_SILU, PAIRS, F16, FUSED>;
    case HSTU_ACT_RELU: return hstu_attn_kernel<CAND, HSTU_ACT_RELU, PAIRS, F16, FUSED>;
    case HSTU_ACT_SOFTMAX: return hstu_attn_kernel<CAND, HSTU_ACT_SOFTMAX, PAIRS, F16, FUSED>;
    default: return hstu_attn_kernel<CAND, HSTU_ACT_IDENTITY, PAIRS, F16, FUSED>;
  }
}

template <bool F16>
AttnKernelFn attn_kernel_ptr_t(bool cand, int phi, bool pairs) {
  if (cand)
    return pairs ? attn_kernel_for<true, true, F16, false>(phi)
                 : attn_kernel_for<true, false, F16, false>(phi);
  return pairs ? attn_kernel_for<false, true, F16, false>(phi)
               : attn_kernel_for<false, false, F16, false>(phi);
}

// The layer-fused form exists for the causal kernel with fp16 operands (the
// bf16 layer path).
AttnKernelFn attn_kernel_ptr(bool cand, int phi, bool pairs, bool f16, bool fused = false) {
  if (fused)
    return pairs ? attn_kernel_for<false, true, true, true>(phi)
                 : attn_kernel_for<false, false, true, true>(phi);
  return f16 ? attn_kernel_ptr_t<true>(cand, phi, pairs) : attn_kernel_ptr_t<false>(cand, phi, pairs);
}

using AttnBwdFn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                          const CUtensorMap, const CUtensorMap, const AttnBwdParams);

template <bool F16>
AttnBwdFn attn_bwd_kernel_for(int phi) {
  switch (phi) {
    case HSTU_ACT_SILU: return hstu_attn_bwd_kernel<HSTU_ACT_SILU, F16>;
    case HSTU_ACT_RELU: return hstu_attn_bwd_kernel<HSTU_ACT_RELU, F16>;
    default: return hstu_attn_bwd_kernel<HSTU_ACT_IDENTITY, F16>;
  }
}

AttnBwdFn attn_bwd_kernel_ptr(int phi, bool f16) {
  return f16 ? attn_bwd_kernel_for<true>(phi) : attn_bwd_kernel_for<false>(phi);
}

struct DeviceInfo {
  int sm_count = 0;
  bool smem_set = false;
};

hstu_status_t device_info(DeviceInfo** out) {
  static std::mutex mu;
  static DeviceInfo info[kMaxDevices];
  int dev = 0;
  HSTU_CHECK_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return HSTU_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  DeviceInfo& d = info[dev];
  if (d.sm_count == 0) {
    HSTU_CHECK_CUDA(cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev));
  }
  if (!d.smem_set) {
    const int att_max = 227 * 1024;
    for (int cand = 0; cand < 2; ++cand)
      for (int phi = 0; phi < 4; ++phi)
        for (int pairs = 0; pairs < 2; ++pairs)
          for (int f16 = 0; f16 < 2; ++f16)
            HSTU_CHECK_CUDA(cudaFuncSetAttribute(
                attn_kernel_ptr(cand != 0, phi, pairs != 0, f16 != 0),
                cudaFuncAttributeMaxDynamicSharedMemorySize, att_max));
    for (int phi = 0; phi < 4; ++phi)
      for (int pairs = 0; pairs < 2; ++pairs)
        HSTU_CHECK_CUDA(cudaFuncSetAttribute(attn_kernel_ptr(false, phi, pairs != 0, true, true),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, att_max));
    for (int phi = 0; phi < 3; ++phi)
      for (int f16 = 0; f16 < 2; ++f16)
        HSTU_CHECK_CUDA(cudaFuncSetAttribute(attn_bwd_kernel_ptr(phi, f16 != 0),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, att_max));
    const int g1 = static_cast<int>(F1Smem::kBytes);
    HSTU_CHECK_CUDA(cudaFuncSetAttribute(hstu_f1_kernel<HSTU_ACT_RELU>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, g1));
    HSTU_CHECK_CUDA(cudaFuncSetAttribute(hstu_f1_kernel<HSTU_ACT_SILU>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, g1));
    HSTU_CHECK_CUDA(cudaFuncSetAttribute(hstu_f1_kernel<HSTU_ACT_IDENTITY>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, g1));
    HSTU_CHECK_CUDA(cudaFuncSetAttribute(hstu_f2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(F2Smem::kBytes)));
    HSTU_CHECK_CUDA(cudaFuncSetAttribute(hstu_sl_select_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SL_MAX_LEN * static_cast<int>(sizeof(uint64_t))));
    d.smem_set = true;
  }
  *out = &d;
  return HSTU_OK;
}

// ------------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D map over a row-major [rows, cols] matrix of 16-bit elements (bf16, or
// fp16 when f16) with row stride `ld` elements; box = box_cols x box_rows;
// 128-byte swizzle.
hstu_status_t make_map_16(CUtensorMap* map, const void* base, int64_t rows, int64_t cols,
                          int64_t ld, int box_cols, int box_rows, bool f16 = false) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return HSTU_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? HSTU_OK : HSTU_ERR_CUDA;
}

// 2-D map for tensor stores of f1's output blocks: fp32, bf16 or fp16
// [rows, cols] with row stride `ld` elements; box = one 128-byte row segment x
// 32 rows.
hstu_status_t make_out_map(CUtensorMap* map, void* base, bool f32, int64_t rows, int64_t cols,
                           int64_t ld, bool f16 = false) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return HSTU_ERR_CUDA;
  const int elt = f32 ? 4 : 2;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * elt};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elt), 32};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt = f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                     : (f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                            : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
  CUresult r = fn(map, dt, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? HSTU_OK : HSTU_ERR_CUDA;
}

// ------------------------------------------------------------------ validation

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

hstu_status_t check_cfg(const hstu_layer_cfg_t* c) {
  if (c == nullptr) return HSTU_ERR_INVALID_ARGUMENT;
  if (c->d_model <= 0 || c->num_heads <= 0 || c->dqk <= 0 || c->dv <= 0 ||
      c->num_pos_buckets <= 0 || c->num_time_buckets <= 0)
    return HSTU_ERR_INVALID_ARGUMENT;
  if (c->phi1 < HSTU_ACT_IDENTITY || c->phi1 > HSTU_ACT_SILU || c->phi2 < HSTU_ACT_IDENTITY ||
      c->phi2 > HSTU_ACT_SOFTMAX)
    return HSTU_ERR_INVALID_ARGUMENT;
  if (c->dtype != HSTU_BF16 && c->dtype != HSTU_FP32 && c->dtype != HSTU_FP16)
    return HSTU_ERR_INVALID_ARGUMENT;
  if (!(c->ln_eps >= 0.0f)) return HSTU_ERR_INVALID_ARGUMENT;
  if ((c->flags & ~HSTU_FLAG_FUSED_F2) != 0) return HSTU_ERR_INVALID_ARGUMENT;
  if (c->dqk != ATT_HD || c->dv != ATT_HD) return HSTU_ERR_UNSUPPORTED;
  if (c->d_model % 64 != 0) return HSTU_ERR_UNSUPPORTED;
  if (c->num_pos_buckets > kMaxPos || c->num_time_buckets > MAX_TIME_BUCKETS)
    return HSTU_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(c->num_heads) * ATT_HD > 8192) return HSTU_ERR_UNSUPPORTED;
  return HSTU_OK;
}

// Layer entry points: bf16 or fp32 storage (fp16 is an attention-operand type only).
hstu_status_t check_layer_cfg(const hstu_layer_cfg_t* c) {
  hstu_status_t s = check_cfg(c);
  if (s != HSTU_OK) return s;
  return c->dtype == HSTU_FP16 ? HSTU_ERR_UNSUPPORTED : HSTU_OK;
}

hstu_status_t check_jag(const hstu_jagged_t* j) {
  if (j == nullptr) return HSTU_ERR_INVALID_ARGUMENT;
  if (j->batch < 0 || j->total_tokens < 0 || j->max_len < 0) return HSTU_ERR_INVALID_ARGUMENT;
  if (j->batch > 0 && j->offsets == nullptr) return HSTU_ERR_INVALID_ARGUMENT;
  if (j->total_tokens > 0 && (j->timestamps == nullptr || j->batch == 0))
    return HSTU_ERR_INVALID_ARGUMENT;
  // a batch with rows has a user of length >= 1; the kernels are sized from max_len
  if (j->total_tokens > 0 && j->max_len == 0) return HSTU_ERR_INVALID_ARGUMENT;
  if (j->max_len > kMaxLen || j->batch > 65535) return HSTU_ERR_UNSUPPORTED;
  if (j->segments != nullptr && (j->max_static < 0 || j->max_static > kMaxLen))
    return HSTU_ERR_INVALID_ARGUMENT;
  if (j->total_tokens > (int64_t(1) << 31) - 1) return HSTU_ERR_UNSUPPORTED;
  return HSTU_OK;
}

size_t elt(const hstu_layer_cfg_t* c) { return c->dtype == HSTU_BF16 ? 2 : 4; }

int n1_of(const hstu_layer_cfg_t* c) { return 2 * c->num_heads * (c->dqk + c->dv); }

// Workspace of one layer.
//   bf16 path: VQK [T, 3*H*dv] bf16 (V, Q, K blocks; K/V may go to a cache
//              instead), U [T, H*dv] fp32, AV [T, H*dv] fp32, LN partials
//              [T, H, 2] fp32.  AV and U stay fp32 because LayerNorm removes the
//              large common mean of AV and would magnify bf16 rounding there.
//   fp32 path: Z [T, n1] fp32, AV [T, H*dv] fp32, G [T, H*dv] fp32.
//   bf16 path, also: fp16 copies of W1 [n1, d] and W2 [d, H*dv] (the GEMM
//              operands paired with fp16 activations).
struct LayerWs {
  void* z;      // bf16: VQK; fp32: Z
  float* u;     // bf16 path: U fp32
  void* av;
  void* extra;  // bf16: LN partials; fp32: G
  __half* w1h;  // bf16 path: fp16 W1
  __half* w2h;  // bf16 path: fp16 W2
  __half* x16;  // bf16 path: fp16 copy of the fp32 layer input (x_in = NULL)
  int32_t* count;  // bf16 path: [T] arrivals per query tile pair of the fused f2 tail
};

size_t weights_f16_bytes(const hstu_layer_cfg_t* c) {
  const size_t hv = static_cast<size_t>(c->num_heads) * c->dv;
  const size_t d = static_cast<size_t>(c->d_model);
  return align_up(static_cast<size_t>(n1_of(c)) * d * 2, 256) + align_up(d * hv * 2, 256);
}

size_t layer_ws_bytes(const hstu_layer_cfg_t* c, int64_t T) {
  const size_t t = static_cast<size_t>(T);
  const size_t hv = static_cast<size_t>(c->num_heads) * c->dv;
  if (c->dtype == HSTU_BF16)
    return align_up(t * 3 * hv * 2, 256) + 2 * align_up(t * hv * 4, 256) +
           align_up(t * c->num_heads * 2 * sizeof(float), 256) + weights_f16_bytes(c) +
           align_up(t * static_cast<size_t>(c->d_model) * 2, 256) + align_up(t * 4, 256);
  return align_up(t * n1_of(c) * 4, 256) + 2 * align_up(t * hv * 4, 256);
}

LayerWs carve_layer(const hstu_layer_cfg_t* c, int64_t T, void* ws) {
  const size_t t = static_cast<size_t>(T);
  const size_t hv = static_cast<size_t>(c->num_heads) * c->dv;
  uint8_t* p = static_cast<uint8_t*>(ws);
  LayerWs w;
  w.z = p;
  if (c->dtype == HSTU_BF16) {
    p += align_up(t * 3 * hv * 2, 256);
    w.u = reinterpret_cast<float*>(p);
    p += align_up(t * hv * 4, 256);
  } else {
    p += align_up(t * n1_of(c) * 4, 256);
    w.u = nullptr;
  }
  w.av = p;
  p += align_up(t * hv * 4, 256);
  w.extra = p;
  w.w1h = w.w2h = w.x16 = nullptr;
  w.count = nullptr;
  if (c->dtype == HSTU_BF16) {
    p += align_up(t * c->num_heads * 2 * sizeof(float), 256);
    w.w1h = reinterpret_cast<__half*>(p);
    p += align_up(static_cast<size_t>(n1_of(c)) * c->d_model * 2, 256);
    w.w2h = reinterpret_cast<__half*>(p);
    p += align_up(static_cast<size_t>(c->d_model) * hv * 2, 256);
    w.x16 = reinterpret_cast<__half*>(p);
    p += align_up(t * static_cast<size_t>(c->d_model) * 2, 256);
    w.count = reinterpret_cast<int32_t*>(p);
  }
  return w;
}

hstu_status_t convert_f32_to_f16(const float* src, __half* dst, int64_t n, cudaStream_t st) {
  const int64_t n8 = n / 8;  // n = T * d_model, d_model a multiple of 64
  const int blocks = static_cast<int>(std::min<int64_t>((n8 + 255) / 256, 4096));
  ProfScope prof(K_CVT, st);
  hstu_f32_to_f16_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<const float4*>(src),
                                                  reinterpret_cast<uint4*>(dst), n8);
  HSTU_CHECK_CUDA(cudaGetLastError());
  return HSTU_OK;
}

hstu_status_t convert_bf16_to_f16(const void* src, __half* dst, int64_t n, cudaStream_t st) {
  // n is a multiple of 64 for every weight matrix here (d and H*64 are)
  const int64_t n8 = n / 8;
  const int blocks = static_cast<int>(std::min<int64_t>((n8 + 255) / 256, 1024));
  ProfScope prof(K_CVT, st);
  hstu_bf16_to_f16_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint4*>(src),
                                                   reinterpret_cast<uint4*>(dst), n8);
  HSTU_CHECK_CUDA(cudaGetLastError());
  return HSTU_OK;
}

// residual-stream buffers of a multi-layer pass: 2 x fp32 [T, d] + 2 x low-precision [T, d]
size_t stream_ws_bytes(const hstu_layer_cfg_t* c, int64_t T) {
  const size_t d = static_cast<size_t>(c->d_model);
  return 2 * align_up(static_cast<size_t>(T) * d * 4, 256) +
         2 * align_up(static_cast<size_t>(T) * d * elt(c), 256);
}

// ------------------------------------------------------------------ launches

struct AttnJob {
  const hstu_layer_cfg_t* cfg;
  const int64_t* kv_offsets;
  const int64_t* q_offsets;   // nullptr in causal mode
  const int64_t* timestamps;
  const int64_t* request_ts;
  int32_t batch;
  int32_t max_q_len;
  int32_t max_kv_len;
  int64_t T_q, T_kv;
  const void* q; int64_t ldq;
  const void* k; int64_t ldk;
  const void* v; int64_t ldv;
  const void* q_self; const void* k_self; const void* v_self; int64_t ld_self;
  const int32_t* segments;      // generalised masks (causal mode), or nullptr
  int32_t max_static;
  const float* rab_pos;
  const float* rab_time;
  void* av; int64_t ld_av;      // bf16 [.., ld_av] output (attention alone)
  float* av_f32;                // fp32 output (layer path)
  float* ln_part;
  uint64_t timeout_ns;
  bool f16;                     // Q, K, V (and P) in fp16 instead of bf16
  // layer-fused f2 (causal, f16): tail.count is [T_q] and zeroed here; w2h is
  // the fp16 W2 [d, H*64]
  const TailParams* tail = nullptr;
  const void* w2h = nullptr;
};

// Tensor-core attention over 16-bit operands (bf16, or fp16 when j.f16).
template <bool CAND>
hstu_status_t launch_attn_tc(const AttnJob& j, cudaStream_t st) {
  const hstu_layer_cfg_t* c = j.cfg;
  if (j.batch == 0 || j.T_q == 0 || j.max_q_len == 0) return HSTU_OK;
  DeviceInfo* di = nullptr;
  hstu_status_t s = device_info(&di);
  if (s != HSTU_OK) return s;
  CUtensorMap mq, mk, mv, mw;
  const int64_t hc = static_cast<int64_t>(c->num_heads) * ATT_HD;
  if ((s = make_map_16(&mq, j.q, j.T_q, hc, j.ldq, ATT_HD, ATT_ROWS, j.f16)) != HSTU_OK) return s;
  // with no key rows at all (every history empty) no K/V tile is ever loaded;
  // the maps then describe the query rows so that they stay valid
  const bool no_kv = j.T_kv == 0;
  if ((s = make_map_16(&mk, no_kv ? j.q : j.k, no_kv ? j.T_q : j.T_kv, hc,
                       no_kv ? j.ldq : j.ldk, ATT_HD, ATT_KEYS, j.f16)) != HSTU_OK)
    return s;
  if ((s = make_map_16(&mv, no_kv ? j.q : j.v, no_kv ? j.T_q : j.T_kv, hc,
                       no_kv ? j.ldq : j.ldv, ATT_HD, ATT_KEYS, j.f16)) != HSTU_OK)
    return s;
  const bool fused = !CAND && j.tail != nullptr;
  if (fused) {
    if (!j.f16 || j.av_f32 == nullptr || j.ln_part == nullptr || j.w2h == nullptr ||
        j.tail->N > 512 || j.tail->K != hc || hc > 512)
      return HSTU_ERR_UNSUPPORTED;
    if ((s = make_map_16(&mw, j.w2h, j.tail->N, hc, hc, 64, 256, true)) != HSTU_OK) return s;
    // one arrival counter per query tile pair, indexed by the pair's first row
    HSTU_CHECK_CUDA(cudaMemsetAsync(j.tail->count, 0, static_cast<size_t>(j.T_q) * sizeof(int32_t), st));
  } else {
    mw = mq;  // unused
  }
  AttnParams p;
  std::memset(&p, 0, sizeof(p));
  if (fused) p.tail = *j.tail;
  p.kv_offsets = j.kv_offsets;
  p.q_offsets = j.q_offsets;
  p.timestamps = j.timestamps;
  p.request_ts = j.request_ts;
  p.rab_pos = j.rab_pos;
  p.rab_time = j.rab_time;
  if (!CAND && j.segments != nullptr) {
    // candidate rows of the generalised masks add their own key/value: read
    // from the tensors being attended
    p.q_self = j.q; p.ld_qs = j.ldq;
    p.k_self = j.k; p.ld_ks = j.ldk;
    p.v_self = j.v; p.ld_vs = j.ldv;
    p.segments = j.segments;
    p.max_static = j.max_static;
  } else {
    p.q_self = j.q_self;
    p.k_self = j.k_self;
    p.v_self = j.v_self;
    p.ld_qs = p.ld_ks = p.ld_vs = j.ld_self;
  }
  p.av = j.av;
  p.av_f32 = j.av_f32;
  p.ld_av = j.ld_av;
  p.ln_part = j.ln_part;
  p.B = j.batch;
  p.H = c->num_heads;
  p.P = c->num_pos_buckets;
  p.Tb = c->num_time_buckets;
  p.max_q = j.max_q_len;
  p.max_kv = j.max_kv_len;
  p.num_qpairs = (j.max_q_len + 2 * ATT_ROWS - 1) / (2 * ATT_ROWS);
  // largest staged-table origin D over the CTAs, plus the diagonal overhang
  const size_t dmax = CAND ? static_cast<size_t>(j.max_kv_len)
                           : align_up(static_cast<size_t>(j.max_q_len), 2 * ATT_ROWS);
  // per-copy length = 16 (mod 32) floats: the two copies' 8-byte pair reads
  // by neighbouring lanes then fall in disjoint shared-memory banks
  // the staged offsets reach 127 + 2 past a row (causal), or the U+S block
  // plus two chunks (generalised masks)
  const size_t extra = (!CAND && j.segments != nullptr)
                           ? std::max<size_t>(ATT_ROWS, static_cast<size_t>(j.max_static) + 64)
                           : ATT_ROWS;
  p.pos_len = static_cast<int32_t>(align_up(dmax + extra + 2, 32) + 16);
  const uint32_t pos_elt = 4u;
  p.phi2 = c->phi2;
  p.timeout_ns = j.timeout_ns;
  std::memcpy(p.thr, thresholds_for(c->num_time_buckets), sizeof(int64_t) * c->num_time_buckets);
  if (!compute_octaves(c->num_time_buckets, p.thr, p.oct)) return HSTU_ERR_UNSUPPORTED;
  dim3 grid(c->num_heads, j.batch, p.num_qpairs);
  const bool pairs = AttnSmem::bytes(p.pos_len, true, pos_elt) <= 227u * 1024u;
  size_t smem = AttnSmem::bytes(p.pos_len, pairs, pos_elt);
  if (fused) smem = std::max<size_t>(smem, AttnSmem::kTailBytes);
  if (smem > 227u * 1024u) return HSTU_ERR_UNSUPPORTED;
  ProfScope prof(CAND ? K_CAND_ATTN : (fused ? K_ATTN_FUSED : K_ATTN), st);
  attn_kernel_ptr(CAND, c->phi2, pairs, j.f16, fused)<<<grid, ATT_THREADS, smem, st>>>(mq, mk, mv,
                                                                                       mw, p);
  HSTU_CHECK_CUDA(cudaGetLastError());
  return HSTU_OK;
}

// Backward of the causal pointwise attention: dQ, dK, dV (fp32, [T, ld_g]) and
// the table gradients (overwritten).  q, k, v, d_o are 16-bit [T, H*64] with
// row strides ldq, ldk, ldv, ld_do.
hstu_status_t launch_attn_bwd(const hstu_layer_cfg_t* c, const hstu_jagged_t* jag, const void* q,
                              int64_t ldq, const void* k, int64_t ldk, const void* v, int64_t ldv,
                              const void* d_o, int64_t ld_do, const float* rab_pos,
                              const float* rab_time, float* dq, float* dk, float* dv, int64_t ld_g,
                              float* drab_pos, float* drab_time, bool f16, cudaStream_t st) {
  const int H = c->num_heads, P = c->num_pos_buckets, Tb = c->num_time_buckets;
  HSTU_CHECK_CUDA(cudaMemsetAsync(drab_pos, 0, sizeof(float) * H * P, st));
  HSTU_CHECK_CUDA(cudaMemsetAsync(drab_time, 0, sizeof(float) * H * Tb, st));
  if (jag->batch == 0 || jag->total_tokens == 0 || jag->max_len == 0) return HSTU_OK;
  DeviceInfo* di = nullptr;
  hstu_status_t s = device_info(&di);
  if (s != HSTU_OK) return s;
  const int64_t T = jag->total_tokens, hv = static_cast<int64_t>(H) * ATT_HD;
  CUtensorMap mq, mk, mv, mo;
  if ((s = make_map_16(&mq, q, T, hv, ldq, ATT_HD, BW_COLS, f16)) != HSTU_OK) return s;
  if ((s = make_map_16(&mk, k, T, hv, ldk, ATT_HD, BW_COLS, f16)) != HSTU_OK) return s;
  if ((s = make_map_16(&mv, v, T, hv, ldv, ATT_HD, BW_COLS, f16)) != HSTU_OK) return s;
  if ((s = make_map_16(&mo, d_o, T, hv, ld_do, ATT_HD, BW_COLS, f16)) != HSTU_OK) return s;
  AttnBwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.offsets = jag->offsets;
  p.timestamps = jag->timestamps;
  p.rab_pos = rab_pos;
  p.rab_time = rab_time;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.ld_g = ld_g;
  p.drab_pos = drab_pos;
  p.drab_time = drab_time;
  p.B = jag->batch;
  p.H = H;
  p.P = P;
  p.Tb = Tb;
  p.max_len = jag->max_len;
  p.phi2 = c->phi2;
  p.timeout_ns = kDefaultTimeoutNs;
  const int64_t* thr = thresholds_for(Tb);
  for (int b = 0; b < Tb; ++b)
    p.thr[b] = thr[b] < static_cast<int64_t>(INT32_MAX) ? static_cast<int32_t>(thr[b]) : INT32_MAX;
  if (!compute_octaves(Tb, thr, p.oct)) return HSTU_ERR_UNSUPPORTED;
  const size_t smem = BwSmem::kBytes;
  static_assert(BwSmem::kBytes <= 227u * 1024u, "backward shared memory");
  // dQ is accumulated into (a TMA reduce-add per tile pair)
  CUtensorMap mdq;
  if ((s = make_out_map(&mdq, dq, true, T, hv, ld_g)) != HSTU_OK) return s;
  HSTU_CHECK_CUDA(cudaMemset2DAsync(dq, sizeof(float) * ld_g, 0, sizeof(float) * hv, T, st));
  dim3 grid(H, jag->batch, (jag->max_len + BW_ROWS - 1) / BW_ROWS);
  {
    ProfScope prof(K_ATTN_BWD, st);
    attn_bwd_kernel_ptr(c->phi2, f16)<<<grid, BW_THREADS, smem, st>>>(mq, mk, mv, mo, mdq, p);
    HSTU_CHECK_CUDA(cudaGetLastError());
  }
  return HSTU_OK;
}

// f32_mask / f16_mask bit b: column block b (U, V, Q, K) is stored as fp32 /
// fp16; otherwise bf16.
hstu_status_t launch_f1_bf16(const hstu_layer_cfg_t* c, const void* x, int64_t ldx, int64_t M,
                             const void* w1, const float* b1, void* const dst[4],
                             const int64_t ld_dst[4], uint32_t f32_mask, uint32_t f16_mask,
                             bool ab_f16, cudaStream_t st) {
  if (M == 0) return HSTU_OK;
  DeviceInfo* di = nullptr;
  hstu_status_t s = device_info(&di);
  if (s != HSTU_OK) return s;
  const int N = n1_of(c), K = c->d_model;
  CUtensorMap mx, mw;
  if ((s = make_map_16(&mx, x, M, K, ldx, G_BK, G_BM, ab_f16)) != HSTU_OK) return s;
  if ((s = make_map_16(&mw, w1, N, K, K, G_BK, G_BN, ab_f16)) != HSTU_OK) return s;
  F1Params p;
  std::memset(&p, 0, sizeof(p));
  F1OutMaps om;
  std::memset(&om, 0, sizeof(om));
  const int64_t blk_w = static_cast<int64_t>(c->num_heads) * ATT_HD;
  for (int b = 0; b < 4; ++b) {
    p.dst[b] = dst[b];
    p.ld_dst[b] = ld_dst[b];
    if ((s = make_out_map(&om.m[b], dst[b], (f32_mask >> b) & 1u, M, blk_w, ld_dst[b],
                          (f16_mask >> b) & 1u)) != HSTU_OK)
      return s;
  }
  p.f32_mask = f32_mask;
  p.f16_mask = f16_mask;
  p.ab_f16 = ab_f16 ? 1 : 0;
  p.bias = b1;
  p.M = M;
  p.N = N;
  p.K = K;
  p.blk_w = c->num_heads * ATT_HD;
  p.num_m_tiles = static_cast<int32_t>((M + G_BM - 1) / G_BM);
  p.num_n_tiles = N / G_BN;
  p.timeout_ns = kDefaultTimeoutNs;
  const int total = p.num_m_tiles * p.num_n_tiles;
  const int grid = total < di->sm_count ? total : di->sm_count;
  ProfScope prof(K_F1, st);
  switch (c->phi1) {
    case HSTU_ACT_RELU:
      hstu_f1_kernel<HSTU_ACT_RELU><<<grid, 192, F1Smem::kBytes, st>>>(mx, mw, om, p);
      break;
    case HSTU_ACT_SILU:
      hstu_f1_kernel<HSTU_ACT_SILU><<<grid, 192, F1Smem::kBytes, st>>>(mx, mw, om, p);
      break;
    default:
      hstu_f1_kernel<HSTU_ACT_IDENTITY><<<grid, 192, F1Smem::kBytes, st>>>(mx, mw, om, p);
      break;
  }
  HSTU_CHECK_CUDA(cudaGetLastError());
  return HSTU_OK;
}

// w2 is bf16 as given, or its fp16 copy (ab_f16: the A tile is then built in
// fp16 too); y_lp is written in fp16 when ylp_f16.
hstu_status_t launch_f2_bf16(const hstu_layer_cfg_t* c, const hstu_layer_weights_t* w,
                             const void* w2, bool ab_f16, const float* av, int64_t ld_av,
                             const float* u, int64_t ld_u, const float* ln_part,
                             const float* x_res, const void* x_lp, int64_t ld_x, float* y,
                             void* y_lp, bool ylp_f16, int64_t ld_y, int64_t M, cudaStream_t st) {
  if (M == 0) return HSTU_OK;
  DeviceInfo* di = nullptr;
  hstu_status_t s = device_info(&di);
  if (s != HSTU_OK) return s;
  const int N = c->d_model, K = c->num_heads * c->dv;
  CUtensorMap mw;
  if ((s = make_map_16(&mw, w2, N, K, K, G_BK, G_BN, ab_f16)) != HSTU_OK) return s;
  F2OutMaps om;
  std::memset(&om, 0, sizeof(om));
  if ((s = make_out_map(&om.y, y, true, M, N, ld_y)) != HSTU_OK) return s;
  if (y_lp != nullptr &&
      (s = make_out_map(&om.y_lp, y_lp, false, M, N, ld_y, ylp_f16)) != HSTU_OK)
    return s;
  F2Params p;
  std::memset(&p, 0, sizeof(p));
  p.av = av;
  p.u = u;
  p.ld_av = ld_av;
  p.ld_u = ld_u;
  p.ln_part = ln_part;
  p.gamma = w->ln_gamma;
  p.beta = w->ln_beta;
  p.eps = c->ln_eps;
  p.bias = w->b2;
  p.x_res = x_res;
  p.x_lp = static_cast<const __nv_bfloat16*>(x_lp);
  p.ld_x = ld_x;
  p.y = y;
  p.y_lp = y_lp;
  p.ylp_f16 = ylp_f16 ? 1 : 0;
  p.ab_f16 = ab_f16 ? 1 : 0;
  p.ld_y = ld_y;
  p.M = M;
  p.N = N;
  p.K = K;
  p.H = c->num_heads;
  p.num_m_tiles = static_cast<int32_t>((M + G_BM - 1) / G_BM);
  p.num_n_tiles = (N + F2_NW - 1) / F2_NW;  // column groups of up to 512
  p.timeout_ns = kDefaultTimeoutNs;
  const int total = p.num_m_tiles * p.num_n_tiles;
  const int grid = total < di->sm_count ? total : di->sm_count;
  ProfScope prof(K_F2, st);
  hstu_f2_kernel<<<grid, F2_THREADS, F2Smem::kBytes, st>>>(mw, om, p);
  HSTU_CHECK_CUDA(cudaGetLastError());
  return HSTU_OK;
}

// ------------------------------------------------------------------ fp32 path

hstu_status_t launch_f32_linear(const float* a, int64_t lda, int64_t M, int N, int K,
                                const float* w, const float* bias, const float* res,
                                int64_t ld_res, float* const dst[4], const int64_t ld_dst[4],
                                int blk_w, int act, cudaStream_t st) {
  if (M == 0) return HSTU_OK;
  F32LinParams p;
  std::memset(&p, 0, sizeof(p));
  p.a = a;
  p.lda = lda;
  p.w = w;
  p.bias = bias;
  p.res = res;
  p.ld_res = ld_res;
  for (int b = 0; b < 4; ++b) {
    p.dst[b] = dst[b];
    p.ld_dst[b] = ld_dst[b];
  }
  p.blk_w = blk_w;
  p.M = M;
  p.N = N;
  p.K = K;
  p.act = act;
  dim3 grid((N + 63) / 64, static_cast<unsigned>((M + 63) / 64));
  ProfScope prof(K_F32_LINEAR, st);
  hstu_f32_linear_kernel<<<grid, 256, 0, st>>>(p);
  HSTU_CHECK_CUDA(cudaGetLastError());
  return HSTU_OK;
}

hstu_status_t launch_f32_attn(const AttnJob& j, cudaStream_t st) {
  const hstu_layer_cfg_t* c = j.cfg;
  if (j.batch == 0 || j.T_q == 0 || j.max_q_len == 0) return HSTU_OK;
  F32AttnParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = static_cast<const float*>(j.q);
  p.k = static_cast<const float*>(j.k);
  p.v = static_cast<const float*>(j.v);
  p.ldq = j.ldq;
  p.ldk = j.ldk;
  p.ldv = j.ldv;
  p.kv_offsets = j.kv_offsets;
  p.q_offsets = j.q_offsets;
  p.timestamps = j.timestamps;
  p.request_ts = j.request_ts;
  p.rab_pos = j.rab_pos;
  p.rab_time = j.rab_time;
  p.q_self = static_cast<const float*>(j.q_self);
  p.k_self = static_cast<const float*>(j.k_self);
  p.v_self = static_cast<const float*>(j.v_self);
  p.ld_self = j.ld_self;
  p.av = static_cast<float*>(j.av);
  p.ld_av = j.ld_av;
  p.B = j.batch;
  p.H = c->num_heads;
  p.P = c->num_pos_buckets;
  p.Tb = c->num_time_buckets;
  p.phi2 = c->phi2;
  p.cand = j.q_offsets != nullptr ? 1 : 0;
  p.segments = p.cand ? nullptr : j.segments;
  p.max_q = j.max_q_len;
  p.max_kv = j.max_kv_len;
  std::memcpy(p.thr, thresholds_for(c->num_time_buckets), sizeof(int64_t) * c->num_time_buckets);
  dim3 grid((j.max_q_len + 31) / 32, c->num_heads, j.batch);
  ProfScope prof(K_F32_ATTN, st);
  hstu_f32_attn_kernel<<<grid, 128, 0, st>>>(p);
  HSTU_CHECK_CUDA(cudaGetLastError());
  return HSTU_OK;
}

// One layer on the fp32 path.
hstu_status_t layer_fp32(const hstu_layer_cfg_t* c, const hstu_layer_weights_t* w,
                         const AttnJob& base, const float* x_in, const float* x_res, int64_t T,
                         float* y_out, float* kv_cache, const LayerWs& ws, bool cand,
                         cudaStream_t st) {
  const int H = c->num_heads, hv = H * ATT_HD, n1 = n1_of(c), d = c->d_model;
  float* z = static_cast<float*>(ws.z);
  float* dst[4] = {z, z + hv, z + 2 * hv, z + 2 * hv + hv};
  int64_t ldd[4] = {n1, n1, n1, n1};
  if (kv_cache != nullptr) {
    dst[1] = kv_cache + hv;  // V
    dst[3] = kv_cache;       // K
    ldd[1] = ldd[3] = 2 * hv;
  }
  hstu_status_t s = launch_f32_linear(x_in, d, T, n1, d, static_cast<const float*>(w->w1), w->b1,
                                      nullptr, 0, dst, ldd, hv, c->phi1, st);
  if (s != HSTU_OK) return s;
  AttnJob j = base;
  if (!cand) {
    j.q = dst[2]; j.ldq = ldd[2];
    j.k = dst[3]; j.ldk = ldd[3];
    j.v = dst[1]; j.ldv = ldd[1];
  } else {
    j.q_self = dst[2]; j.k_self = dst[3]; j.v_self = dst[1]; j.ld_self = n1;
    j.q = dst[2]; j.ldq = n1;
  }
  j.rab_pos = w->rab_pos;
  j.rab_time = w->rab_time;
  j.av = ws.av;
  j.ld_av = hv;
  if ((s = launch_f32_attn(j, st)) != HSTU_OK) return s;
  float* g = static_cast<float*>(ws.extra);
  const unsigned blocks = static_cast<unsigned>((T * 32 + 255) / 256);
  ProfScope prof(K_F32_LN, st);
  hstu_f32_ln_gate_kernel<<<blocks, 256, 0, st>>>(static_cast<const float*>(ws.av), hv, z, n1,
                                                  w->ln_gamma, w->ln_beta, c->ln_eps, T, hv, g, hv);
  HSTU_CHECK_CUDA(cudaGetLastError());
  float* ydst[4] = {y_out, y_out, y_out, y_out};
  int64_t ydl[4] = {d, d, d, d};
  return launch_f32_linear(g, hv, T, d, hv, static_cast<const float*>(w->w2), w->b2,
                           x_res != nullptr ? x_res : x_in, d, ydst, ydl, d, HSTU_ACT_IDENTITY, st);
}

// One layer on the bf16 tensor-core path.
//   x_f16   x_in is fp16 (a residual-stream copy handed over by the previous
//           layer of a stack; then x_res must be given): f1 runs on fp16 X and
//           an fp16 copy of W1.  Otherwise x_in is the caller's bf16 and f1 runs
//           on bf16 X and W1 as given.
//   ylp_f16 the rounded copy of Y (y_lp) is fp16, else bf16.
// f2 always runs on fp16: its A tile Norm(AV) (.) U is built in fp16 and W2 is
// converted.  fp16 has the same tensor-core rate as bf16 and 8x finer
// rounding; bf16 weights convert to fp16 exactly inside fp16's normal range.
hstu_status_t layer_bf16(const hstu_layer_cfg_t* c, const hstu_layer_weights_t* w,
                         const AttnJob& base, const void* x_in, bool x_f16, const float* x_res,
                         int64_t T, float* y_out, void* y_lp, bool ylp_f16, void* kv_cache,
                         const LayerWs& ws, bool cand, cudaStream_t st) {
  const int hv = c->num_heads * ATT_HD, d = c->d_model;
  if (x_f16 && x_res == nullptr) return HSTU_ERR_INVALID_ARGUMENT;
  hstu_status_t s;
  if (x_f16 && (s = convert_bf16_to_f16(w->w1, ws.w1h, static_cast<int64_t>(n1_of(c)) * d, st)) !=
                   HSTU_OK)
    return s;
  if ((s = convert_bf16_to_f16(w->w2, ws.w2h, static_cast<int64_t>(d) * hv, st)) != HSTU_OK)
    return s;
  __half* vqk = static_cast<__half*>(ws.z);
  // f1 column blocks U, V, Q, K -> U (fp32), V, Q, K (fp16; K/V into the cache
  // if given).  The attention operands are fp16: the same tensor-core rate as
  // bf16 with 8x finer rounding of Q, K, V and P.
  void* dst[4] = {ws.u, vqk, vqk + hv, vqk + 2 * hv};
  int64_t ldd[4] = {hv, 3 * hv, 3 * hv, 3 * hv};
  if (kv_cache != nullptr) {
    __half* kv = static_cast<__half*>(kv_cache);
    dst[1] = kv + hv;  // V
    dst[3] = kv;       // K
    ldd[1] = ldd[3] = 2 * hv;
  }
  s = launch_f1_bf16(c, x_in, d, T, x_f16 ? static_cast<const void*>(ws.w1h) : w->w1, w->b1, dst,
                     ldd, 1u, 0xEu, x_f16, st);
  if (s != HSTU_OK) return s;
  AttnJob j = base;
  j.q = dst[2];
  j.ldq = ldd[2];
  if (!cand) {
    j.k = dst[3]; j.ldk = ldd[3];
    j.v = dst[1]; j.ldv = ldd[1];
  } else {
    j.q_self = dst[2]; j.k_self = dst[3]; j.v_self = dst[1]; j.ld_self = 3 * hv;
  }
  j.rab_pos = w->rab_pos;
  j.rab_time = w->rab_time;
  j.av = nullptr;
  j.av_f32 = static_cast<float*>(ws.av);
  j.ld_av = hv;
  j.ln_part = static_cast<float*>(ws.extra);
  j.f16 = true;
  // on request, causal layers with d <= 512 and H * 64 <= 512 run f2 inside
  // the attention kernel (the tail of the last head CTA of each query tile pair)
  const bool fused = !cand && (c->flags & HSTU_FLAG_FUSED_F2) != 0 && c->d_model <= 512 &&
                     hv <= 512;
  if (fused) {
    TailParams tp;
    std::memset(&tp, 0, sizeof(tp));
    tp.count = ws.count;
    tp.u = ws.u;
    tp.ld_u = hv;
    tp.x_res = x_res;
    tp.x_lp = static_cast<const __nv_bfloat16*>(x_in);
    tp.ld_x = d;
    tp.b2 = w->b2;
    tp.gamma = w->ln_gamma;
    tp.beta = w->ln_beta;
    tp.eps = c->ln_eps;
    tp.y = y_out;
    tp.y_lp = y_lp;
    tp.ylp_f16 = ylp_f16 ? 1 : 0;
    tp.ld_y = d;
    tp.N = c->d_model;
    tp.K = static_cast<int32_t>(hv);
    j.tail = &tp;
    j.w2h = ws.w2h;
    return launch_attn_tc<false>(j, st);
  }
  s = cand ? launch_attn_tc<true>(j, st) : launch_attn_tc<false>(j, st);
  if (s != HSTU_OK) return s;
  return launch_f2_bf16(c, w, ws.w2h, true, static_cast<const float*>(ws.av), hv, ws.u, hv,
                        static_cast<const float*>(ws.extra), x_res, x_in, d, y_out, y_lp,
                        ylp_f16, d, T, st);
}

// ------------------------------------------------------------------ layer backward

// Workspace of hstu_layer_bwd: the forward's (recomputed intermediates), then
// dG, G [T, H*64] fp32, dZ [T, n1] fp32, dAV [T, H*64] 16-bit, X [T, d] fp32,
// fp32 copies of W1 and W2, and the cuBLAS workspace.
constexpr size_t kCublasWsBytes = size_t(32) << 20;

struct BwdWs {
  LayerWs fwd;
  float* dg;
  float* g;
  float* dz;
  void* dav16;
  float* x32;
  float* w1f;
  float* w2f;
  void* cublas_ws;
};

size_t layer_bwd_ws_bytes(const hstu_layer_cfg_t* c, int64_t T) {
  const size_t t = static_cast<size_t>(T);
  const size_t hv = static_cast<size_t>(c->num_heads) * ATT_HD;
  const size_t d = static_cast<size_t>(c->d_model), n1 = static_cast<size_t>(n1_of(c));
  return layer_ws_bytes(c, T) + 2 * align_up(t * hv * 4, 256) + align_up(t * n1 * 4, 256) +
         align_up(t * hv * 2, 256) + align_up(t * d * 4, 256) + align_up(n1 * d * 4, 256) +
         align_up(d * hv * 4, 256) + kCublasWsBytes;
}

BwdWs carve_bwd(const hstu_layer_cfg_t* c, int64_t T, void* ws) {
  const size_t t = static_cast<size_t>(T);
  const size_t hv = static_cast<size_t>(c->num_heads) * ATT_HD;
  const size_t d = static_cast<size_t>(c->d_model), n1 = static_cast<size_t>(n1_of(c));
  BwdWs b;
  b.fwd = carve_layer(c, T, ws);
  uint8_t* p = static_cast<uint8_t*>(ws) + layer_ws_bytes(c, T);
  auto take = [&](size_t bytes) { uint8_t* q = p; p += align_up(bytes, 256); return q; };
  b.dg = reinterpret_cast<float*>(take(t * hv * 4));
  b.g = reinterpret_cast<float*>(take(t * hv * 4));
  b.dz = reinterpret_cast<float*>(take(t * n1 * 4));
  b.dav16 = take(t * hv * 2);
  b.x32 = reinterpret_cast<float*>(take(t * d * 4));
  b.w1f = reinterpret_cast<float*>(take(n1 * d * 4));
  b.w2f = reinterpret_cast<float*>(take(d * hv * 4));
  b.cublas_ws = take(kCublasWsBytes);
  return b;
}

// One cuBLAS handle per device, created on first use; calls on it are
// serialised by the mutex (the stream and workspace are set per call).
struct CublasSlot {
  std::mutex mu;
  cublasHandle_t h = nullptr;
};

CublasSlot* cublas_slot() {
  static CublasSlot slots[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  return &slots[dev];
}

// Row-major C[M, N] = op(A) op(B) + beta C in fp32 storage with TF32 tensor
// cores (op(A) is [M, K]: A is [M, K] or, transposed, [K, M]).  Through the
// column-major library: C^T = op(B)^T op(A)^T.
hstu_status_t gemm_rm(cublasHandle_t h, bool ta, bool tb, int64_t M, int64_t N, int64_t K,
                      const float* A, int64_t lda, const float* B, int64_t ldb, float* C,
                      int64_t ldc, float beta) {
  if (M == 0 || N == 0) return HSTU_OK;
  const float alpha = 1.0f;
  const cublasStatus_t r = cublasGemmEx(
      h, tb ? CUBLAS_OP_T : CUBLAS_OP_N, ta ? CUBLAS_OP_T : CUBLAS_OP_N, static_cast<int>(N),
      static_cast<int>(M), static_cast<int>(K), &alpha, B, CUDA_R_32F, static_cast<int>(ldb), A,
      CUDA_R_32F, static_cast<int>(lda), &beta, C, CUDA_R_32F, static_cast<int>(ldc),
      CUBLAS_COMPUTE_32F_FAST_TF32, CUBLAS_GEMM_DEFAULT);
  return r == CUBLAS_STATUS_SUCCESS ? HSTU_OK : HSTU_ERR_CUDA;
}

hstu_status_t convert_bf16_to_f32(const void* src, float* dst, int64_t n, cudaStream_t st) {
  if (n == 0) return HSTU_OK;
  ProfScope prof(K_BWD_ELT, st);
  hstu_bf16_to_f32_kernel<<<std::min<int64_t>((n + 255) / 256, 148 * 16), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(src), dst, n);
  HSTU_CHECK_CUDA(cudaGetLastError());
  return HSTU_OK;
}

hstu_status_t colsum(const float* a, int64_t lda, int64_t M, int N, float* out, cudaStream_t st) {
  HSTU_CHECK_CUDA(cudaMemsetAsync(out, 0, sizeof(float) * N, st));
  if (M == 0) return HSTU_OK;
  const int rows = 512;
  dim3 grid((N + 255) / 256, static_cast<unsigned>((M + rows - 1) / rows));
  ProfScope prof(K_BWD_ELT, st);
  hstu_colsum_kernel<<<grid, 256, 0, st>>>(a, lda, M, N, rows, out);
  HSTU_CHECK_CUDA(cudaGetLastError());
  return HSTU_OK;
}

template <int KPL>
void launch_gate_bwd_k(const float* av, const float* ln_part, const float* u, const float* dg,
                       const hstu_layer_cfg_t* c, const hstu_layer_weights_t* w, int64_t T,
                       void* dav16, float* dz, int64_t ld_dz, float* g, float* dgamma,
                       float* dbeta, cudaStream_t st) {
  const int64_t blocks = std::min<int64_t>((T + 7) / 8, 148 * 8);
  hstu_gate_bwd_kernel<KPL><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      av, ln_part, u, dg, w->ln_gamma, w->ln_beta, c->ln_eps, c->num_heads, T, dav16, 1, dz,
      ld_dz, g, dgamma, dbeta, c->phi1 == HSTU_ACT_RELU ? 1 : 0);
}

hstu_status_t launch_gate_bwd(const float* av, const float* ln_part, const float* u,
                              const float* dg, const hstu_layer_cfg_t* c,
                              const hstu_layer_weights_t* w, int64_t T, void* dav16, float* dz,
                              int64_t ld_dz, float* g, float* dgamma, float* dbeta,
                              cudaStream_t st) {
  ProfScope prof(K_GATE_BWD, st);
  switch (c->num_heads) {
#define HSTU_GATE_CASE(HH) \
    case HH: launch_gate_bwd_k<2 * HH>(av, ln_part, u, dg, c, w, T, dav16, dz, ld_dz, g, dgamma, dbeta, st); break;
    HSTU_GATE_CASE(1) HSTU_GATE_CASE(2) HSTU_GATE_CASE(3) HSTU_GATE_CASE(4)
    HSTU_GATE_CASE(5) HSTU_GATE_CASE(6) HSTU_GATE_CASE(7) HSTU_GATE_CASE(8)
    HSTU_GATE_CASE(10) HSTU_GATE_CASE(12) HSTU_GATE_CASE(16)
#undef HSTU_GATE_CASE
    default: return HSTU_ERR_UNSUPPORTED;
  }
  HSTU_CHECK_CUDA(cudaGetLastError());
  return HSTU_OK;
}

// The backward of one bf16 layer: recompute f1 and the attention (the same
// kernels as the forward), then the chain rule through Eq. 3, the attention
// and Eq. 1.
hstu_status_t layer_bwd_bf16(const hstu_layer_cfg_t* c, const hstu_layer_weights_t* w,
                             const hstu_jagged_t* jag, const void* x_in, const float* x_res,
                             const float* dy, float* dx, const hstu_layer_grads_t* gr,
                             const BwdWs& b, cudaStream_t st) {
  const int64_t T = jag->total_tokens;
  const int hv = c->num_heads * ATT_HD, d = c->d_model, n1 = n1_of(c);
  const LayerWs& ws = b.fwd;
  hstu_status_t s;
  // ---- forward recompute: f1 (U fp32; V, Q, K fp16) and the attention (AV, LN partials)
  const bool x_f16 = x_in == nullptr;
  if (x_f16 && (s = convert_f32_to_f16(x_res, ws.x16, T * d, st)) != HSTU_OK) return s;
  if (x_f16 && (s = convert_bf16_to_f16(w->w1, ws.w1h, static_cast<int64_t>(n1) * d, st)) != HSTU_OK)
    return s;
  __half* vqk = static_cast<__half*>(ws.z);
  void* dst[4] = {ws.u, vqk, vqk + hv, vqk + 2 * hv};
  int64_t ldd[4] = {hv, 3 * hv, 3 * hv, 3 * hv};
  s = launch_f1_bf16(c, x_f16 ? static_cast<const void*>(ws.x16) : x_in, d, T,
                     x_f16 ? static_cast<const void*>(ws.w1h) : w->w1, w->b1, dst, ldd, 1u, 0xEu,
                     x_f16, st);
  if (s != HSTU_OK) return s;
  AttnJob j;
  std::memset(&j, 0, sizeof(j));
  j.cfg = c;
  j.kv_offsets = jag->offsets;
  j.timestamps = jag->timestamps;
  j.batch = jag->batch;
  j.max_q_len = j.max_kv_len = jag->max_len;
  j.T_q = j.T_kv = T;
  j.q = vqk + hv; j.ldq = 3 * hv;
  j.k = vqk + 2 * hv; j.ldk = 3 * hv;
  j.v = vqk; j.ldv = 3 * hv;
  j.rab_pos = w->rab_pos;
  j.rab_time = w->rab_time;
  j.av_f32 = static_cast<float*>(ws.av);
  j.ld_av = hv;
  j.ln_part = static_cast<float*>(ws.extra);
  j.timeout_ns = kDefaultTimeoutNs;
  j.f16 = true;
  if ((s = launch_attn_tc<false>(j, st)) != HSTU_OK) return s;
  // ---- fp32 operands of the library GEMMs
  if ((s = convert_bf16_to_f32(w->w1, b.w1f, static_cast<int64_t>(n1) * d, st)) != HSTU_OK) return s;
  if ((s = convert_bf16_to_f32(w->w2, b.w2f, static_cast<int64_t>(d) * hv, st)) != HSTU_OK) return s;
  const float* x32 = x_res;
  if (!x_f16) {
    if ((s = convert_bf16_to_f32(x_in, b.x32, T * d, st)) != HSTU_OK) return s;
    x32 = b.x32;
  }
  CublasSlot* cs = cublas_slot();
  if (cs == nullptr) return HSTU_ERR_CUDA;
  std::lock_guard<std::mutex> lock(cs->mu);
  if (cs->h == nullptr && cublasCreate(&cs->h) != CUBLAS_STATUS_SUCCESS) {
    cs->h = nullptr;
    return HSTU_ERR_CUDA;
  }
  if (cublasSetStream(cs->h, st) != CUBLAS_STATUS_SUCCESS ||
      cublasSetWorkspace(cs->h, b.cublas_ws, kCublasWsBytes) != CUBLAS_STATUS_SUCCESS)
    return HSTU_ERR_CUDA;
  // ---- Y = X + G W2^T + b2:  dG = dY W2,  dW2 = dY^T G,  db2 = colsum(dY)
  {
    ProfScope prof(K_BWD_GEMM, st);
    if ((s = gemm_rm(cs->h, false, false, T, hv, d, dy, d, b.w2f, hv, b.dg, hv, 0.0f)) != HSTU_OK)
      return s;
  }
  // ---- G = Ln(AV) (.) U: dU (masked), G, dAV (fp16), dgamma / dbeta
  if (gr->dgamma != nullptr) HSTU_CHECK_CUDA(cudaMemsetAsync(gr->dgamma, 0, sizeof(float) * hv, st));
  if (gr->dbeta != nullptr) HSTU_CHECK_CUDA(cudaMemsetAsync(gr->dbeta, 0, sizeof(float) * hv, st));
  if ((s = launch_gate_bwd(static_cast<const float*>(ws.av), static_cast<const float*>(ws.extra),
                           ws.u, b.dg, c, w, T, b.dav16, b.dz, n1, b.g,
                           w->ln_gamma != nullptr ? gr->dgamma : nullptr,
                           w->ln_beta != nullptr ? gr->dbeta : nullptr, st)) != HSTU_OK)
    return s;
  {
    ProfScope prof(K_BWD_GEMM, st);
    if ((s = gemm_rm(cs->h, true, false, d, hv, T, dy, d, b.g, hv, gr->dw2, hv, 0.0f)) != HSTU_OK)
      return s;
  }
  if ((s = colsum(dy, d, T, d, gr->db2, st)) != HSTU_OK) return s;
  // ---- attention: dV, dQ, dK straight into their dZ column blocks, table gradients
  if ((s = launch_attn_bwd(c, jag, vqk + hv, 3 * hv, vqk + 2 * hv, 3 * hv, vqk, 3 * hv, b.dav16, hv,
                           w->rab_pos, w->rab_time, b.dz + 2 * hv, b.dz + 3 * hv, b.dz + hv, n1,
                           gr->drab_pos, gr->drab_time, true, st)) != HSTU_OK)
    return s;
  // ---- Z = phi1(X W1^T + b1): mask, db1, dW1 = dZ^T X, dX = dY + dZ W1
  if (c->phi1 == HSTU_ACT_RELU) {
    ProfScope prof(K_BWD_ELT, st);
    const int64_t total = T * 3 * hv;
    hstu_relu_mask_kernel<<<std::min<int64_t>((total + 255) / 256, 148 * 16), 256, 0, st>>>(
        b.dz, n1, hv, vqk, 3 * hv, 3 * hv, T);
    HSTU_CHECK_CUDA(cudaGetLastError());
  }
  if ((s = colsum(b.dz, n1, T, n1, gr->db1, st)) != HSTU_OK) return s;
  {
    ProfScope prof(K_BWD_GEMM, st);
    if ((s = gemm_rm(cs->h, true, false, n1, d, T, b.dz, n1, x32, d, gr->dw1, d, 0.0f)) != HSTU_OK)
      return s;
    HSTU_CHECK_CUDA(cudaMemcpyAsync(dx, dy, sizeof(float) * T * d, cudaMemcpyDeviceToDevice, st));
    if ((s = gemm_rm(cs->h, false, false, T, d, n1, b.dz, n1, b.w1f, d, dx, d, 1.0f)) != HSTU_OK)
      return s;
  }
  return HSTU_OK;
}

hstu_status_t check_weights(const hstu_layer_cfg_t* c, const hstu_layer_weights_t* w) {
  if (w == nullptr || w->w1 == nullptr || w->b1 == nullptr || w->w2 == nullptr ||
      w->b2 == nullptr || w->rab_pos == nullptr || w->rab_time == nullptr)
    return HSTU_ERR_INVALID_ARGUMENT;
  if (!aligned16(w->w1) || !aligned16(w->b1) || !aligned16(w->w2) || !aligned16(w->b2) ||
      !aligned16(w->ln_gamma) || !aligned16(w->ln_beta))
    return HSTU_ERR_INVALID_ARGUMENT;
  (void)c;
  return HSTU_OK;
}

// Scratch for hstu_layer_fwd_static: a fixed block in the library's own device
// memory, for callers that cannot allocate.  Host code may not use the symbol
// as an address; static_scratch() looks the device address up once per device.
static __device__ __align__(256) unsigned char g_static_scratch[HSTU_STATIC_SCRATCH_BYTES];

hstu_status_t static_scratch(void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  HSTU_CHECK_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return HSTU_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    HSTU_CHECK_CUDA(cudaGetSymbolAddress(&p, g_static_scratch));
    if (p == nullptr) return HSTU_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return HSTU_OK;
}

}  // namespace

// ====================================================================== C ABI

extern "C" {

const char* hstu_version(void) { return "libhstu 0.1 (sm_100a)"; }

const char* hstu_status_string(hstu_status_t s) {
  switch (s) {
    case HSTU_OK: return "ok";
    case HSTU_ERR_INVALID_ARGUMENT: return "invalid argument";
    case HSTU_ERR_UNSUPPORTED: return "unsupported shape or option";
    case HSTU_ERR_CUDA: return "CUDA error";
    case HSTU_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case HSTU_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case HSTU_ERR_DEVICE_CHECK: return "device-side input check failed";
  }
  return "unknown status";
}

size_t hstu_layer_workspace_bytes(const hstu_layer_cfg_t* cfg, int64_t total_tokens) {
  if (check_layer_cfg(cfg) != HSTU_OK || total_tokens < 0) return 0;
  return layer_ws_bytes(cfg, total_tokens);
}

size_t hstu_forward_workspace_bytes(const hstu_layer_cfg_t* cfg, int32_t num_layers,
                                    int64_t total_tokens) {
  if (check_layer_cfg(cfg) != HSTU_OK || total_tokens < 0 || num_layers < 1) return 0;
  return layer_ws_bytes(cfg, total_tokens) + stream_ws_bytes(cfg, total_tokens);
}

size_t hstu_mfalcon_workspace_bytes(const hstu_layer_cfg_t* cfg, int64_t num_cand) {
  if (check_layer_cfg(cfg) != HSTU_OK || num_cand < 0) return 0;
  return layer_ws_bytes(cfg, num_cand) + stream_ws_bytes(cfg, num_cand);
}

hstu_status_t hstu_time_bucket_thresholds(int32_t num_time_buckets, int64_t* thr_out) {
  if (thr_out == nullptr || num_time_buckets < 1 || num_time_buckets > MAX_TIME_BUCKETS)
    return HSTU_ERR_INVALID_ARGUMENT;
  std::memcpy(thr_out, thresholds_for(num_time_buckets), sizeof(int64_t) * num_time_buckets);
  return HSTU_OK;
}

hstu_status_t hstu_attn_fwd(const hstu_layer_cfg_t* cfg, const hstu_jagged_t* jag, const void* q,
                            const void* k, const void* v, const float* rab_pos,
                            const float* rab_time, void* av_out, void* workspace,
                            size_t ws_bytes, void* stream) {
  (void)workspace;
  (void)ws_bytes;
  hstu_status_t s;
  if ((s = check_cfg(cfg)) != HSTU_OK) return s;
  if ((s = check_jag(jag)) != HSTU_OK) return s;
  if (jag->total_tokens == 0 || jag->batch == 0) return HSTU_OK;
  if (q == nullptr || k == nullptr || v == nullptr || rab_pos == nullptr ||
      rab_time == nullptr || av_out == nullptr)
    return HSTU_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(av_out))
    return HSTU_ERR_INVALID_ARGUMENT;
  const int64_t hv = static_cast<int64_t>(cfg->num_heads) * ATT_HD;
  AttnJob j;
  std::memset(&j, 0, sizeof(j));
  j.cfg = cfg;
  j.kv_offsets = jag->offsets;
  j.segments = jag->segments;
  j.max_static = jag->max_static;
  j.timestamps = jag->timestamps;
  j.batch = jag->batch;
  j.max_q_len = j.max_kv_len = jag->max_len;
  j.T_q = j.T_kv = jag->total_tokens;
  j.q = q; j.ldq = hv;
  j.k = k; j.ldk = hv;
  j.v = v; j.ldv = hv;
  j.rab_pos = rab_pos;
  j.rab_time = rab_time;
  j.av = av_out;
  j.ld_av = hv;
  j.timeout_ns = kDefaultTimeoutNs;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cfg->dtype == HSTU_FP32) return launch_f32_attn(j, st);
  j.f16 = cfg->dtype == HSTU_FP16;
  return launch_attn_tc<false>(j, st);
}

size_t hstu_layer_bwd_workspace_bytes(const hstu_layer_cfg_t* cfg, int64_t total_tokens) {
  if (check_layer_cfg(cfg) != HSTU_OK || total_tokens < 0 || cfg->dtype != HSTU_BF16) return 0;
  return layer_bwd_ws_bytes(cfg, total_tokens);
}

hstu_status_t hstu_layer_bwd(const hstu_layer_cfg_t* cfg, const hstu_layer_weights_t* w,
                             const hstu_jagged_t* jag, const void* x_in, const float* x_res,
                             const float* dy, float* dx, const hstu_layer_grads_t* grads,
                             void* workspace, size_t ws_bytes, void* stream) {
  hstu_status_t s;
  if ((s = check_layer_cfg(cfg)) != HSTU_OK) return s;
  if ((s = check_jag(jag)) != HSTU_OK) return s;
  if ((s = check_weights(cfg, w)) != HSTU_OK) return s;
  if (cfg->dtype != HSTU_BF16 || jag->segments != nullptr || cfg->phi2 == HSTU_ACT_SOFTMAX ||
      (cfg->phi1 != HSTU_ACT_RELU && cfg->phi1 != HSTU_ACT_IDENTITY) || cfg->num_heads > 16)
    return HSTU_ERR_UNSUPPORTED;
  if (grads == nullptr || grads->dw1 == nullptr || grads->db1 == nullptr || grads->dw2 == nullptr ||
      grads->db2 == nullptr || grads->drab_pos == nullptr || grads->drab_time == nullptr)
    return HSTU_ERR_INVALID_ARGUMENT;
  const int64_t T = jag->total_tokens;
  const int hv = cfg->num_heads * ATT_HD, d = cfg->d_model, n1 = n1_of(cfg);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0 || jag->batch == 0) {
    // no tokens: every gradient is zero
    HSTU_CHECK_CUDA(cudaMemsetAsync(grads->dw1, 0, sizeof(float) * n1 * d, st));
    HSTU_CHECK_CUDA(cudaMemsetAsync(grads->db1, 0, sizeof(float) * n1, st));
    HSTU_CHECK_CUDA(cudaMemsetAsync(grads->dw2, 0, sizeof(float) * d * hv, st));
    HSTU_CHECK_CUDA(cudaMemsetAsync(grads->db2, 0, sizeof(float) * d, st));
    HSTU_CHECK_CUDA(cudaMemsetAsync(grads->drab_pos, 0, sizeof(float) * cfg->num_heads * cfg->num_pos_buckets, st));
    HSTU_CHECK_CUDA(cudaMemsetAsync(grads->drab_time, 0, sizeof(float) * cfg->num_heads * cfg->num_time_buckets, st));
    if (grads->dgamma != nullptr) HSTU_CHECK_CUDA(cudaMemsetAsync(grads->dgamma, 0, sizeof(float) * hv, st));
    if (grads->dbeta != nullptr) HSTU_CHECK_CUDA(cudaMemsetAsync(grads->dbeta, 0, sizeof(float) * hv, st));
    return HSTU_OK;
  }
  if ((x_in == nullptr && x_res == nullptr) || dy == nullptr || dx == nullptr)
    return HSTU_ERR_INVALID_ARGUMENT;
  if (!aligned16(x_in) || !aligned16(x_res) || !aligned16(dy) || !aligned16(dx) ||
      !aligned16(workspace))
    return HSTU_ERR_INVALID_ARGUMENT;
  if (workspace == nullptr || ws_bytes < layer_bwd_ws_bytes(cfg, T)) return HSTU_ERR_WORKSPACE_TOO_SMALL;
  return layer_bwd_bf16(cfg, w, jag, x_in, x_res, dy, dx, grads, carve_bwd(cfg, T, workspace), st);
}

hstu_status_t hstu_attn_bwd(const hstu_layer_cfg_t* cfg, const hstu_jagged_t* jag, const void* q,
                            const void* k, const void* v, const void* d_o, const float* rab_pos,
                            const float* rab_time, float* dq, float* dk, float* dv,
                            float* drab_pos, float* drab_time, void* stream) {
  hstu_status_t s;
  if ((s = check_cfg(cfg)) != HSTU_OK) return s;
  if ((s = check_jag(jag)) != HSTU_OK) return s;
  if (cfg->dtype == HSTU_FP32 || cfg->phi2 == HSTU_ACT_SOFTMAX || jag->segments != nullptr)
    return HSTU_ERR_UNSUPPORTED;
  if (rab_pos == nullptr || rab_time == nullptr || drab_pos == nullptr || drab_time == nullptr)
    return HSTU_ERR_INVALID_ARGUMENT;
  if (jag->total_tokens > 0 &&
      (q == nullptr || k == nullptr || v == nullptr || d_o == nullptr || dq == nullptr ||
       dk == nullptr || dv == nullptr))
    return HSTU_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(d_o) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv))
    return HSTU_ERR_INVALID_ARGUMENT;
  const int64_t hv = static_cast<int64_t>(cfg->num_heads) * ATT_HD;
  return launch_attn_bwd(cfg, jag, q, hv, k, hv, v, hv, d_o, hv, rab_pos, rab_time, dq, dk, dv,
                         hv, drab_pos, drab_time, cfg->dtype == HSTU_FP16,
                         static_cast<cudaStream_t>(stream));
}

hstu_status_t hstu_attn_fwd_f32(const hstu_layer_cfg_t* cfg, const hstu_jagged_t* jag,
                                const void* q, const void* k, const void* v, const float* rab_pos,
                                const float* rab_time, float* av_out, void* stream) {
  hstu_status_t s;
  if ((s = check_cfg(cfg)) != HSTU_OK) return s;
  if ((s = check_jag(jag)) != HSTU_OK) return s;
  if (jag->total_tokens == 0 || jag->batch == 0) return HSTU_OK;
  if (q == nullptr || k == nullptr || v == nullptr || rab_pos == nullptr ||
      rab_time == nullptr || av_out == nullptr)
    return HSTU_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(av_out))
    return HSTU_ERR_INVALID_ARGUMENT;
  const int64_t hv = static_cast<int64_t>(cfg->num_heads) * ATT_HD;
  AttnJob j;
  std::memset(&j, 0, sizeof(j));
  j.cfg = cfg;
  j.kv_offsets = jag->offsets;
  j.segments = jag->segments;
  j.max_static = jag->max_static;
  j.timestamps = jag->timestamps;
  j.batch = jag->batch;
  j.max_q_len = j.max_kv_len = jag->max_len;
  j.T_q = j.T_kv = jag->total_tokens;
  j.q = q; j.ldq = hv;
  j.k = k; j.ldk = hv;
  j.v = v; j.ldv = hv;
  j.rab_pos = rab_pos;
  j.rab_time = rab_time;
  j.ld_av = hv;
  j.timeout_ns = kDefaultTimeoutNs;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cfg->dtype == HSTU_FP32) {
    j.av = av_out;
    return launch_f32_attn(j, st);
  }
  j.av_f32 = av_out;
  j.f16 = cfg->dtype == HSTU_FP16;
  return launch_attn_tc<false>(j, st);
}

hstu_status_t mfalcon_attn_fwd(const hstu_layer_cfg_t* cfg, const hstu_jagged_t* history,
                               const void* k_hist, const void* v_hist,
                               const int64_t* cand_offsets, int64_t num_cand, int32_t max_cand,
                               const void* q, const void* k, const void* v,
                               const int64_t* request_ts, const float* rab_pos,
                               const float* rab_time, float* av_out, void* stream) {
  hstu_status_t s;
  if ((s = check_cfg(cfg)) != HSTU_OK) return s;
  if ((s = check_jag(history)) != HSTU_OK) return s;
  if (num_cand < 0 || max_cand < 0) return HSTU_ERR_INVALID_ARGUMENT;
  if (history->segments != nullptr) return HSTU_ERR_UNSUPPORTED;
  if (num_cand == 0 || history->batch == 0) return HSTU_OK;
  if (max_cand == 0) return HSTU_ERR_INVALID_ARGUMENT;
  if (max_cand > kMaxLen || num_cand > (int64_t(1) << 31) - 1) return HSTU_ERR_UNSUPPORTED;
  if (cand_offsets == nullptr || q == nullptr || k == nullptr || v == nullptr ||
      request_ts == nullptr || rab_pos == nullptr || rab_time == nullptr || av_out == nullptr ||
      (history->total_tokens > 0 && (k_hist == nullptr || v_hist == nullptr)))
    return HSTU_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(k_hist) ||
      !aligned16(v_hist) || !aligned16(av_out))
    return HSTU_ERR_INVALID_ARGUMENT;
  const int64_t hv = static_cast<int64_t>(cfg->num_heads) * ATT_HD;
  AttnJob j;
  std::memset(&j, 0, sizeof(j));
  j.cfg = cfg;
  j.kv_offsets = history->offsets;
  j.q_offsets = cand_offsets;
  j.timestamps = history->timestamps;
  j.request_ts = request_ts;
  j.batch = history->batch;
  j.max_q_len = max_cand;
  j.max_kv_len = history->max_len;
  j.T_q = num_cand;
  j.T_kv = history->total_tokens;
  j.q = q; j.ldq = hv;
  j.k = k_hist; j.ldk = hv;
  j.v = v_hist; j.ldv = hv;
  j.q_self = q; j.k_self = k; j.v_self = v; j.ld_self = hv;
  j.rab_pos = rab_pos;
  j.rab_time = rab_time;
  j.ld_av = hv;
  j.timeout_ns = kDefaultTimeoutNs;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cfg->dtype == HSTU_FP32) {
    j.av = av_out;
    return launch_f32_attn(j, st);
  }
  j.av_f32 = av_out;
  j.f16 = cfg->dtype == HSTU_FP16;
  return launch_attn_tc<true>(j, st);
}

hstu_status_t hstu_layer_fwd(const hstu_layer_cfg_t* cfg, const hstu_layer_weights_t* w,
                             const hstu_jagged_t* jag, const void* x_in, const float* x_res,
                             float* y_out, void* y_out_lp, void* kv_cache_out, void* workspace,
                             size_t ws_bytes, void* stream) {
  hstu_status_t s;
  if ((s = check_layer_cfg(cfg)) != HSTU_OK) return s;
  if ((s = check_jag(jag)) != HSTU_OK) return s;
  if ((s = check_weights(cfg, w)) != HSTU_OK) return s;
  const int64_t T = jag->total_tokens;
  if (T == 0 || jag->batch == 0) return HSTU_OK;
  // x_in may be NULL when the fp32 residual x_res is given (bf16 layers)
  if ((x_in == nullptr && (x_res == nullptr || cfg->dtype != HSTU_BF16)) || y_out == nullptr)
    return HSTU_ERR_INVALID_ARGUMENT;
  if (!aligned16(x_in) || !aligned16(x_res) || !aligned16(y_out) || !aligned16(y_out_lp) ||
      !aligned16(kv_cache_out) || !aligned16(workspace))
    return HSTU_ERR_INVALID_ARGUMENT;
  if (workspace == nullptr || ws_bytes < layer_ws_bytes(cfg, T)) return HSTU_ERR_WORKSPACE_TOO_SMALL;
  AttnJob base;
  std::memset(&base, 0, sizeof(base));
  base.cfg = cfg;
  base.kv_offsets = jag->offsets;
  base.segments = jag->segments;
  base.max_static = jag->max_static;
  base.timestamps = jag->timestamps;
  base.batch = jag->batch;
  base.max_q_len = base.max_kv_len = jag->max_len;
  base.T_q = base.T_kv = T;
  base.timeout_ns = kDefaultTimeoutNs;
  const LayerWs ws = carve_layer(cfg, T, workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cfg->dtype == HSTU_FP32) {
    s = layer_fp32(cfg, w, base, static_cast<const float*>(x_in), x_res, T, y_out,
                   static_cast<float*>(kv_cache_out), ws, false, st);
    if (s == HSTU_OK && y_out_lp != nullptr && y_out_lp != y_out)
      HSTU_CHECK_CUDA(cudaMemcpyAsync(y_out_lp, y_out, sizeof(float) * T * cfg->d_model,
                                      cudaMemcpyDeviceToDevice, st));
    return s;
  }
  if (x_in == nullptr) {
    // f1 reads the fp32 residual input rounded to fp16 (as between the layers of a stack)
    if ((s = convert_f32_to_f16(x_res, ws.x16, T * cfg->d_model, st)) != HSTU_OK) return s;
    return layer_bf16(cfg, w, base, ws.x16, true, x_res, T, y_out, y_out_lp, false, kv_cache_out,
                      ws, false, st);
  }
  return layer_bf16(cfg, w, base, x_in, false, x_res, T, y_out, y_out_lp, false, kv_cache_out, ws,
                    false, st);
}

hstu_status_t hstu_layer_fwd_static(const hstu_layer_cfg_t* cfg, const hstu_layer_weights_t* w,
                                    const hstu_jagged_t* jag, const void* x_in,
                                    const float* x_res, float* y_out, void* y_out_lp,
                                    void* kv_cache_out, void* stream) {
  hstu_status_t s;
  if ((s = check_layer_cfg(cfg)) != HSTU_OK) return s;
  if ((s = check_jag(jag)) != HSTU_OK) return s;
  if (layer_ws_bytes(cfg, jag->total_tokens) > HSTU_STATIC_SCRATCH_BYTES)
    return HSTU_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  if ((s = static_scratch(&scratch)) != HSTU_OK) return s;
  return hstu_layer_fwd(cfg, w, jag, x_in, x_res, y_out, y_out_lp, kv_cache_out, scratch,
                        HSTU_STATIC_SCRATCH_BYTES, stream);
}

hstu_status_t hstu_forward(const hstu_layer_cfg_t* cfg, int32_t num_layers,
                           const hstu_layer_weights_t* weights, const hstu_jagged_t* jag,
                           const void* x_in, float* y_out, void* kv_cache_out, void* workspace,
                           size_t ws_bytes, void* stream) {
  hstu_status_t s;
  if ((s = check_layer_cfg(cfg)) != HSTU_OK) return s;
  if ((s = check_jag(jag)) != HSTU_OK) return s;
  if (num_layers < 1 || weights == nullptr) return HSTU_ERR_INVALID_ARGUMENT;
  for (int l = 0; l < num_layers; ++l)
    if ((s = check_weights(cfg, &weights[l])) != HSTU_OK) return s;
  const int64_t T = jag->total_tokens;
  if (T == 0 || jag->batch == 0) return HSTU_OK;
  if (x_in == nullptr || y_out == nullptr) return HSTU_ERR_INVALID_ARGUMENT;
  if (!aligned16(x_in) || !aligned16(y_out) || !aligned16(kv_cache_out) || !aligned16(workspace))
    return HSTU_ERR_INVALID_ARGUMENT;
  if (workspace == nullptr || ws_bytes < hstu_forward_workspace_bytes(cfg, num_layers, T))
    return HSTU_ERR_WORKSPACE_TOO_SMALL;
  const int d = cfg->d_model;
  const size_t lw = layer_ws_bytes(cfg, T);
  uint8_t* sp = static_cast<uint8_t*>(workspace) + lw;
  const size_t fbytes = align_up(static_cast<size_t>(T) * d * 4, 256);
  const size_t lbytes = align_up(static_cast<size_t>(T) * d * elt(cfg), 256);
  float* yf[2] = {reinterpret_cast<float*>(sp), reinterpret_cast<float*>(sp + fbytes)};
  void* yl[2] = {sp + 2 * fbytes, sp + 2 * fbytes + lbytes};
  const size_t cache_layer = static_cast<size_t>(T) * 2 * cfg->num_heads * ATT_HD * elt(cfg);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  AttnJob base;
  std::memset(&base, 0, sizeof(base));
  base.cfg = cfg;
  base.kv_offsets = jag->offsets;
  base.segments = jag->segments;
  base.max_static = jag->max_static;
  base.timestamps = jag->timestamps;
  base.batch = jag->batch;
  base.max_q_len = base.max_kv_len = jag->max_len;
  base.T_q = base.T_kv = T;
  base.timeout_ns = kDefaultTimeoutNs;
  const LayerWs ws = carve_layer(cfg, T, workspace);
  for (int l = 0; l < num_layers; ++l) {
    const bool last = (l == num_layers - 1);
    const float* xres = (l == 0) ? nullptr : yf[(l - 1) & 1];
    float* yo = last ? y_out : yf[l & 1];
    void* kv = kv_cache_out == nullptr ? nullptr
                                       : static_cast<uint8_t*>(kv_cache_out) + cache_layer * l;
    if (cfg->dtype == HSTU_BF16) {
      // between layers the residual stream's rounded copy is fp16
      const void* xin = (l == 0) ? x_in : yl[(l - 1) & 1];
      s = layer_bf16(cfg, &weights[l], base, xin, l > 0, xres, T, yo, last ? nullptr : yl[l & 1],
                     true, kv, ws, false, st);
    } else {
      const float* xin = (l == 0) ? static_cast<const float*>(x_in) : yf[(l - 1) & 1];
      s = layer_fp32(cfg, &weights[l], base, xin, xres, T, yo, static_cast<float*>(kv), ws, false,
                     st);
    }
    if (s != HSTU_OK) return s;
  }
  return HSTU_OK;
}

hstu_status_t mfalcon_score(const hstu_layer_cfg_t* cfg, int32_t num_layers,
                            const hstu_layer_weights_t* weights, const hstu_jagged_t* history,
                            const void* kv_cache, const int64_t* cand_offsets, int64_t num_cand,
                            int32_t max_cand, const void* cand_emb, const int64_t* request_ts,
                            int32_t microbatch, float* scores, float* cand_y_out, void* workspace,
                            size_t ws_bytes, void* stream) {
  hstu_status_t s;
  if ((s = check_layer_cfg(cfg)) != HSTU_OK) return s;
  if ((s = check_jag(history)) != HSTU_OK) return s;
  if (num_layers < 1 || weights == nullptr || microbatch < 1 || num_cand < 0 || max_cand < 0)
    return HSTU_ERR_INVALID_ARGUMENT;
  if (history->segments != nullptr) return HSTU_ERR_UNSUPPORTED;
  for (int l = 0; l < num_layers; ++l)
    if ((s = check_weights(cfg, &weights[l])) != HSTU_OK) return s;
  if (num_cand == 0 || history->batch == 0) return HSTU_OK;
  if (max_cand > kMaxLen) return HSTU_ERR_UNSUPPORTED;
  if (max_cand == 0) return HSTU_ERR_INVALID_ARGUMENT;  // num_cand > 0 here
  if (num_cand > (int64_t(1) << 31) - 1) return HSTU_ERR_UNSUPPORTED;
  if (cand_offsets == nullptr || cand_emb == nullptr || request_ts == nullptr ||
      scores == nullptr || (history->total_tokens > 0 && kv_cache == nullptr))
    return HSTU_ERR_INVALID_ARGUMENT;
  if (!aligned16(cand_emb) || !aligned16(kv_cache) || !aligned16(workspace) ||
      !aligned16(cand_y_out))
    return HSTU_ERR_INVALID_ARGUMENT;
  if (workspace == nullptr || ws_bytes < hstu_mfalcon_workspace_bytes(cfg, num_cand))
    return HSTU_ERR_WORKSPACE_TOO_SMALL;
  const int64_t M = num_cand;
  const int d = cfg->d_model;
  const int hv = cfg->num_heads * ATT_HD;
  const size_t lw = layer_ws_bytes(cfg, M);
  const LayerWs ws = carve_layer(cfg, M, workspace);
  uint8_t* sp = static_cast<uint8_t*>(workspace) + lw;
  const size_t fbytes = align_up(static_cast<size_t>(M) * d * 4, 256);
  const size_t lbytes = align_up(static_cast<size_t>(M) * d * elt(cfg), 256);
  float* yf[2] = {reinterpret_cast<float*>(sp), reinterpret_cast<float*>(sp + fbytes)};
  void* yl[2] = {sp + 2 * fbytes, sp + 2 * fbytes + lbytes};
  const size_t cache_layer =
      static_cast<size_t>(history->total_tokens) * 2 * hv * elt(cfg);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  AttnJob base;
  std::memset(&base, 0, sizeof(base));
  base.cfg = cfg;
  base.kv_offsets = history->offsets;
  base.q_offsets = cand_offsets;
  base.timestamps = history->timestamps;
  base.request_ts = request_ts;
  base.batch = history->batch;
  base.max_q_len = max_cand;
  base.max_kv_len = history->max_len;
  base.T_q = M;
  base.T_kv = history->total_tokens;
  base.timeout_ns = kDefaultTimeoutNs;
  base.f16 = true;  // bf16 layers keep their cached K/V in fp16
  for (int l = 0; l < num_layers; ++l) {
    const uint8_t* cache_l = static_cast<const uint8_t*>(kv_cache) + cache_layer * l;
    AttnJob j = base;
    const size_t e = elt(cfg);
    j.k = cache_l;
    j.ldk = 2 * hv;
    j.v = cache_l + static_cast<size_t>(hv) * e;
    j.ldv = 2 * hv;
    const float* xres = (l == 0) ? nullptr : yf[(l - 1) & 1];
    // the last layer writes the caller's buffer when one is given
    float* yo = (l == num_layers - 1 && cand_y_out != nullptr) ? cand_y_out : yf[l & 1];
    if (cfg->dtype == HSTU_FP32) {
      const float* xin = (l == 0) ? static_cast<const float*>(cand_emb) : yf[(l - 1) & 1];
      s = layer_fp32(cfg, &weights[l], j, xin, xres, M, yo, nullptr, ws, true, st);
    } else {
      const void* xin = (l == 0) ? cand_emb : yl[(l - 1) & 1];
      s = layer_bf16(cfg, &weights[l], j, xin, l > 0, xres, M, yo, yl[l & 1], true, nullptr, ws,
                     true, st);
    }
    if (s != HSTU_OK) return s;
  }
  const float* yfin = cand_y_out != nullptr ? cand_y_out : yf[(num_layers - 1) & 1];
  const unsigned blocks = static_cast<unsigned>((M * 32 + 255) / 256);
  ProfScope prof(K_SCORE, st);
  if (cfg->dtype == HSTU_FP32)
    hstu_score_kernel<float><<<blocks, 256, 0, st>>>(yfin, d, static_cast<const float*>(cand_emb),
                                                     d, M, d, scores);
  else
    hstu_score_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(
        yfin, d, static_cast<const __nv_bfloat16*>(cand_emb), d, M, d, scores);
  HSTU_CHECK_CUDA(cudaGetLastError());
  return HSTU_OK;
}

hstu_status_t hstu_stochastic_length(const hstu_jagged_t* full, const void* x_full,
                                     int32_t row_bytes, float alpha, uint64_t seed, uint64_t step,
                                     int64_t* offsets_out, int32_t* lengths_out,
                                     int32_t* max_len_out, int64_t* kept_index_out,
                                     int64_t* timestamps_out, void* x_out, void* stream) {
  hstu_status_t s;
  if ((s = check_jag(full)) != HSTU_OK) return s;
  if (!(alpha > 0.0f) || !std::isfinite(alpha)) return HSTU_ERR_INVALID_ARGUMENT;
  if (offsets_out == nullptr || lengths_out == nullptr || kept_index_out == nullptr)
    return HSTU_ERR_INVALID_ARGUMENT;
  if (timestamps_out != nullptr && full->total_tokens > 0 && full->timestamps == nullptr)
    return HSTU_ERR_INVALID_ARGUMENT;
  if ((x_full == nullptr) != (x_out == nullptr)) return HSTU_ERR_INVALID_ARGUMENT;
  if (x_full != nullptr &&
      (row_bytes <= 0 || row_bytes % 16 != 0 || !aligned16(x_full) || !aligned16(x_out)))
    return HSTU_ERR_INVALID_ARGUMENT;
  if (full->max_len > SL_MAX_LEN) return HSTU_ERR_UNSUPPORTED;
  DeviceInfo* di = nullptr;
  if ((s = device_info(&di)) != HSTU_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int32_t B = full->batch;
  {
    ProfScope prof(K_SL, st);
    if (B > 0)
      hstu_sl_lengths_kernel<<<(B + 255) / 256, 256, 0, st>>>(full->offsets, B, 1.0 / alpha, seed,
                                                             step, lengths_out);
    hstu_sl_scan_kernel<<<1, SL_SCAN_THREADS, 0, st>>>(lengths_out, B, offsets_out, max_len_out);
    if (B > 0 && full->max_len > 0)
      hstu_sl_select_kernel<<<B, SL_SELECT_THREADS, full->max_len * sizeof(uint64_t), st>>>(
          full->offsets, full->timestamps, lengths_out, offsets_out, full->max_len,
          full->total_tokens, seed, step, kept_index_out, timestamps_out);
    HSTU_CHECK_CUDA(cudaGetLastError());
  }
  if (x_full != nullptr && B > 0 && full->total_tokens > 0) {
    ProfScope prof(K_SL_GATHER, st);
    hstu_sl_gather_kernel<<<di->sm_count * 8, 256, 0, st>>>(
        offsets_out, B, full->total_tokens, kept_index_out, static_cast<const uint4*>(x_full),
        static_cast<uint4*>(x_out), row_bytes / 16);
    HSTU_CHECK_CUDA(cudaGetLastError());
  }
  return HSTU_OK;
}

hstu_status_t hstu_profiler_start(void) {
  Profiler& p = profiler();
  std::lock_guard<std::mutex> lock(p.mu);
  for (auto& r : p.recs) {
    p.pool.push_back(r.a);
    p.pool.push_back(r.b);
  }
  p.recs.clear();
  p.on = true;
  return HSTU_OK;
}

hstu_status_t hstu_profiler_stop(hstu_kernel_time_t* out, int32_t capacity, int32_t* count) {
  if (count == nullptr || capacity < 0 || (capacity > 0 && out == nullptr))
    return HSTU_ERR_INVALID_ARGUMENT;
  Profiler& p = profiler();
  std::lock_guard<std::mutex> lock(p.mu);
  p.on = false;
  double total[K_COUNT] = {};
  int32_t n[K_COUNT] = {};
  hstu_status_t st = HSTU_OK;
  for (auto& r : p.recs) {
    float ms = 0.0f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
      st = HSTU_ERR_CUDA;
    total[r.kind] += ms;
    n[r.kind] += 1;
    p.pool.push_back(r.a);
    p.pool.push_back(r.b);
  }
  p.recs.clear();
  int32_t k = 0;
  for (int i = 0; i < K_COUNT; ++i) {
    if (n[i] == 0) continue;
    if (k < capacity) out[k] = hstu_kernel_time_t{kKernelNames[i], n[i], total[i]};
    ++k;
  }
  *count = k;
  return st;
}

hstu_status_t hstu_get_device_status(void* stream) {
  HSTU_CHECK_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  unsigned int v = 0;
  HSTU_CHECK_CUDA(cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)));
  const unsigned int zero = 0;
  HSTU_CHECK_CUDA(cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)));
  return static_cast<hstu_status_t>(v);
}

hstu_status_t hstu_debug_rab_index(const hstu_jagged_t* jag, int32_t num_pos_buckets,
                                   int32_t num_time_buckets, const int64_t* block_offsets,
                                   int32_t* pos_idx, int32_t* time_idx, void* stream) {
  hstu_status_t s;
  if ((s = check_jag(jag)) != HSTU_OK) return s;
  if (num_pos_buckets < 1 || num_time_buckets < 1 || num_time_buckets > MAX_TIME_BUCKETS)
    return HSTU_ERR_INVALID_ARGUMENT;
  if (jag->total_tokens == 0 || jag->batch == 0 || jag->max_len == 0) return HSTU_OK;
  if (block_offsets == nullptr || pos_idx == nullptr || time_idx == nullptr)
    return HSTU_ERR_INVALID_ARGUMENT;
  AttnParams p;
  std::memset(&p, 0, sizeof(p));
  std::memcpy(p.thr, thresholds_for(num_time_buckets), sizeof(int64_t) * num_time_buckets);
  if (!compute_octaves(num_time_buckets, p.thr, p.oct)) return HSTU_ERR_UNSUPPORTED;
  dim3 grid((jag->max_len + 127) / 128, jag->batch);
  hstu_debug_rab_index_kernel<<<grid, 128, 0, static_cast<cudaStream_t>(stream)>>>(
      jag->offsets, jag->timestamps, block_offsets, jag->batch, num_pos_buckets,
      num_time_buckets, jag->max_len, pos_idx, time_idx, p);
  HSTU_CHECK_CUDA(cudaGetLastError());
  return HSTU_OK;
}

hstu_status_t hstu_debug_wait_timeout(uint64_t timeout_ns, void* stream) {
  hstu_debug_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
  HSTU_CHECK_CUDA(cudaGetLastError());
  return HSTU_OK;
}

}  // extern "C"
