// C ABI of the jagged HSTU layer forward: argument checks, workspace, tensor
// maps and the launch sequence of one layer / one stack.  Every step of the
// forward runs in this library's kernels; nothing here computes layer math on
// the host except the integer threshold table of the time-bucket rule.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <new>
#include <utility>
#include <vector>

#include "internal.h"

using hstu::Workspace;

namespace hstu {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// bucket index of gap dt under the fp64 rule floor(ln(1 + dt) / div)
int64_t fp64_bucket(int64_t dt, double div) {
  if (dt <= 0) return 0;
  return static_cast<int64_t>(floor(log(1.0 + static_cast<double>(dt)) / div));
}

// Candidate-bucket table for 32-bit gaps: bin (e, m) holds v = dt + 1 with
// floor(log2 v) = e and the two bits after the leading one equal to m, so a
// bin spans at most a factor 1.25 in v (0.223 in ln v), less than one bucket
// (0.301 for the layer's divisor; the table is only used when div > 0.223).
// The bucket of any gap in a bin is therefore the bin's low-edge bucket or the
// next one, and one compare against the next threshold decides.
void build_time_lut(const int64_t* thr, int nb, uint8_t* lut, int32_t* thr32) {
  for (int e = 0; e < 32; ++e)
    for (int m = 0; m < 4; ++m) {
      int64_t vlow;
      if (e == 0) vlow = 1;
      else if (e == 1) vlow = m < 2 ? 2 : 3;
      else vlow = (int64_t(1) << e) + int64_t(m) * (int64_t(1) << (e - 2));
      const int64_t dt = vlow - 1;
      int b = 0;
      for (int k = 1; k < nb; ++k)
        if (dt >= thr[k]) b = k;
      lut[e * 4 + m] = uint8_t(b);
    }
  for (int k = 0; k < 257; ++k) {
    const int64_t t = k < nb ? thr[k] : int64_t(0x7FFFFFFF);
    thr32[k] = t > 0x7FFFFFFF ? 0x7FFFFFFF : int32_t(t);
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <typename T>
cudaError_t alloc(T** p, size_t bytes) {
  if (bytes == 0) bytes = 16;
  return cudaMalloc(reinterpret_cast<void**>(p), bytes);
}

size_t elem_size(hstu_dtype t) { return t == HSTU_DTYPE_BF16 ? 2 : 4; }

}  // namespace

bool make_tmap_2d_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (fn == nullptr || outer == 0 || inner == 0) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_2d_bf16_sw64(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                            uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (fn == nullptr || outer == 0 || inner == 0) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_2d_f32_sw128(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                            uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (fn == nullptr || outer == 0 || inner == 0) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_1d_i64(CUtensorMap* m, const void* base, uint64_t n, uint32_t box) {
  auto fn = encode_fn();
  if (fn == nullptr || n == 0) return false;
  cuuint64_t dims[1] = {n};
  cuuint64_t strides[1] = {n * 8};
  cuuint32_t boxd[1] = {box};
  cuuint32_t estr[1] = {1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_INT64, 1, const_cast<void*>(base), dims, strides, boxd,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace hstu

extern "C" {

const char* hstu_status_string(hstu_status s) {
  switch (s) {
    case HSTU_OK: return "HSTU_OK";
    case HSTU_ERR_INVALID_ARG: return "HSTU_ERR_INVALID_ARG";
    case HSTU_ERR_UNSUPPORTED: return "HSTU_ERR_UNSUPPORTED";
    case HSTU_ERR_WORKSPACE: return "HSTU_ERR_WORKSPACE";
    case HSTU_ERR_CUDA: return "HSTU_ERR_CUDA";
    case HSTU_ERR_DEVICE_CHECK: return "HSTU_ERR_DEVICE_CHECK";
    case HSTU_ERR_TIMEOUT: return "HSTU_ERR_TIMEOUT";
  }
  return "HSTU_ERR_UNKNOWN";
}

hstu_status hstu_time_bucket_thresholds(double div, int32_t nb, int64_t* out) {
  if (out == nullptr || !(div > 0.0) || nb < 1 || nb > 256) return HSTU_ERR_INVALID_ARG;
  out[0] = 0;
  for (int32_t k = 1; k < nb; ++k) {
    // smallest dt in [0, 2^62] with bucket(dt) >= k; the rule is monotone in dt
    int64_t lo = 0, hi = hstu::kMaxTimestamp;
    if (hstu::fp64_bucket(hi, div) < k) {
      out[k] = hstu::kMaxTimestamp;
      continue;
    }
    while (lo < hi) {
      const int64_t mid = lo + (hi - lo) / 2;
      if (hstu::fp64_bucket(mid, div) >= k) hi = mid; else lo = mid + 1;
    }
    out[k] = lo;
  }
  return HSTU_OK;
}

hstu_status hstu_create(const hstu_config* cfg, int32_t device, hstu_handle** out) {
  if (out == nullptr || cfg == nullptr) return HSTU_ERR_INVALID_ARG;
  *out = nullptr;
  const hstu_config& c = *cfg;
  if (c.d_model <= 0 || c.num_heads <= 0 || c.head_dim <= 0 ||
      c.d_model != c.num_heads * c.head_dim)
    return HSTU_ERR_INVALID_ARG;
  if ((c.io_dtype != HSTU_DTYPE_BF16 && c.io_dtype != HSTU_DTYPE_FP32) ||
      (c.compute_dtype != HSTU_DTYPE_BF16 && c.compute_dtype != HSTU_DTYPE_FP32))
    return HSTU_ERR_INVALID_ARG;
  if (c.pos_buckets < 1 || c.pos_clamp < 0 || c.pos_clamp >= c.pos_buckets) return HSTU_ERR_INVALID_ARG;
  if (c.time_buckets < 1 || c.time_buckets > 256 || !(c.time_log_div > 0.0)) return HSTU_ERR_INVALID_ARG;
  if (!(c.ln_eps >= 0.0f) || c.max_tokens < 0 || c.max_tokens > hstu::kMaxTokensLimit ||
      c.max_users < 0)
    return HSTU_ERR_INVALID_ARG;
  if (c.pos_clamp > 4096) return HSTU_ERR_UNSUPPORTED;
  const int d = c.d_model;
  const bool d_ok = d == 64 || (d % 128 == 0 && d <= 1024 && d != 896 && d != 640);
  if (!d_ok) return HSTU_ERR_UNSUPPORTED;
  if (c.compute_dtype == HSTU_DTYPE_BF16) {
    if (c.head_dim != 64 && c.head_dim != 128) return HSTU_ERR_UNSUPPORTED;
    if (d % 128 != 0) return HSTU_ERR_UNSUPPORTED;
  } else {
    if (c.io_dtype != HSTU_DTYPE_FP32) return HSTU_ERR_UNSUPPORTED;
    if (c.head_dim % 32 != 0 || c.head_dim > 128) return HSTU_ERR_UNSUPPORTED;
  }
  if (cudaSetDevice(device) != cudaSuccess) return HSTU_ERR_CUDA;
  hstu_handle* h = new (std::nothrow) hstu_handle_s();
  if (h == nullptr) return HSTU_ERR_CUDA;
  h->cfg = c;
  h->device = device;
  cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, device);
  if (hstu_time_bucket_thresholds(c.time_log_div, c.time_buckets, h->thresholds_host) != HSTU_OK) {
    delete h;
    return HSTU_ERR_INVALID_ARG;
  }
  hstu::build_time_lut(h->thresholds_host, c.time_buckets, h->time_lut_host, h->thr32_host);
  const size_t T = size_t(c.max_tokens);
  const size_t cs = hstu::elem_size(c.compute_dtype);
  const size_t nqt = (T + hstu::kTile - 1) / hstu::kTile + 1;
  Workspace& ws = h->ws;
  cudaError_t e = cudaSuccess;
  if (c.compute_dtype == HSTU_DTYPE_BF16 && c.io_dtype == HSTU_DTYPE_FP32)
    e = hstu::alloc(&ws.xb, T * d * 2);
  if (e == cudaSuccess) e = hstu::alloc(&ws.uvqk, T * 4 * d * cs);
  if (e == cudaSuccess) e = hstu::alloc(&ws.av, T * d * 4);
  if (e == cudaSuccess) e = hstu::alloc(&ws.g, T * d * cs);
  if (e == cudaSuccess) e = hstu::alloc(&ws.rows, T * sizeof(hstu::RowInfo));
  if (e == cudaSuccess) e = hstu::alloc(&ws.qtile_order, nqt * 4);
  if (e == cudaSuccess) e = hstu::alloc(&ws.qtile_cost, nqt * 4);
  if (e == cudaSuccess) e = hstu::alloc(&ws.ktile_order, nqt * 4);
  if (e == cudaSuccess) e = hstu::alloc(&ws.ktile_cost, nqt * 4);
  if (e == cudaSuccess) e = hstu::alloc(&ws.counters, 16);
  if (e == cudaSuccess) e = hstu::alloc(&ws.error, 16);
  if (e == cudaSuccess) e = hstu::alloc(&ws.thresholds, 256 * 8);
  if (e == cudaSuccess) e = hstu::alloc(&ws.time_lut, 128);
  if (e == cudaSuccess) e = hstu::alloc(&ws.thr32, 257 * 4);
  if (e == cudaSuccess) e = cudaMemcpy(ws.time_lut, h->time_lut_host, 128, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(ws.thr32, h->thr32_host, 257 * 4, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemset(ws.error, 0, 16);
  if (e == cudaSuccess)
    e = cudaMemcpy(ws.thresholds, h->thresholds_host, size_t(c.time_buckets) * 8,
                   cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    hstu_destroy(h);
    return HSTU_ERR_CUDA;
  }
  *out = h;
  return HSTU_OK;
}

hstu_status hstu_destroy(hstu_handle* h) {
  if (h == nullptr) return HSTU_OK;
  cudaSetDevice(h->device);
  cudaDeviceSynchronize();
  Workspace& ws = h->ws;
  void* ptrs[] = {ws.xb, ws.uvqk, ws.av, ws.g, ws.rows, ws.qtile_order, ws.qtile_cost,
                  ws.ktile_order, ws.ktile_cost, ws.counters, ws.error, ws.thresholds,
                  ws.time_lut, ws.thr32};
  for (void* p : ptrs)
    if (p != nullptr) cudaFree(p);
  hstu::BwdWorkspace& bw = h->bwd;
  void* bptrs[] = {bw.xb, bw.dyb, bw.w1t, bw.w2t, bw.dg, bw.du, bw.dO, bw.g, bw.dq, bw.dk,
                   bw.dv, bw.h1, bw.dh1, bw.dh1t, bw.xt, bw.dyt, bw.gt, bw.zeros};
  for (void* p : bptrs)
    if (p != nullptr) cudaFree(p);
  if (h->timer.created)
    for (int i = 0; i < 2 * hstu::KernelTimer::kMax; ++i) cudaEventDestroy(h->timer.ev[i]);
  delete h;
  return HSTU_OK;
}

}  // extern "C"

namespace {

enum Kind { kSchedule = 0, kCast = 1, kF1 = 2, kAttention = 3, kLnGate = 4, kF2 = 5, kBlock = 6 };

// Brackets one launch with a pair of events when the handle's timer is on.
struct Timed {
  hstu::KernelTimer* t;
  cudaStream_t st;
  int idx = -1;
  Timed(hstu_handle* h, int kind, cudaStream_t s) : t(&h->timer), st(s) {
    if (t->enabled && t->count < hstu::KernelTimer::kMax) {
      idx = t->count++;
      t->kind[idx] = kind;
      cudaEventRecord(t->ev[2 * idx], st);
    }
  }
  ~Timed() {
    if (idx >= 0) cudaEventRecord(t->ev[2 * idx + 1], st);
  }
};

hstu_status check_common(hstu_handle* h, const void* values, int64_t T, const int32_t* offsets,
                         int32_t B, const int64_t* ts, hstu_mask_mode mode,
                         const int32_t* ncand, const void* out) {
  if (h == nullptr) return HSTU_ERR_INVALID_ARG;
  if (T < 0 || B < 0) return HSTU_ERR_INVALID_ARG;
  if (T > h->cfg.max_tokens || B > h->cfg.max_users) return HSTU_ERR_WORKSPACE;
  if (mode != HSTU_MASK_CAUSAL && mode != HSTU_MASK_MFALCON) return HSTU_ERR_INVALID_ARG;
  if (B == 0 && T != 0) return HSTU_ERR_INVALID_ARG;
  if (offsets == nullptr) return HSTU_ERR_INVALID_ARG;
  if (T > 0) {
    if (values == nullptr || out == nullptr || ts == nullptr) return HSTU_ERR_INVALID_ARG;
    if (!hstu::aligned16(values) || !hstu::aligned16(out) || !hstu::aligned16(ts))
      return HSTU_ERR_INVALID_ARG;
  }
  if (mode == HSTU_MASK_MFALCON && B > 0 && ncand == nullptr) return HSTU_ERR_INVALID_ARG;
  return HSTU_OK;
}

hstu_status check_weights(const hstu_layer_weights* w) {
  if (w == nullptr) return HSTU_ERR_INVALID_ARG;
  const void* ps[] = {w->w1, w->b1, w->w2, w->b2, w->ln_gamma, w->ln_beta, w->rab_pos, w->rab_time};
  for (const void* p : ps)
    if (p == nullptr || !hstu::aligned16(p)) return HSTU_ERR_INVALID_ARG;
  return HSTU_OK;
}

// Where the rows of one layer live.  A plain forward: every row of [0, T) is a
// query and SiLU(f1(X)) goes to the workspace.  A history-cache call: the
// buffer is a cache layer's, the layer computes rows [q0, q0 + M) and their
// attention reads keys anywhere in [0, T_attn).
struct LayerRows {
  void* uvqk;              // [T_attn, 4d] compute dtype
  int64_t q0, M, T_attn;
  int num_pairs;           // query-tile pairs listed in `order`
  const int32_t* order;
  const int64_t* ts;       // [T_attn]
};

LayerRows plain_rows(hstu_handle* h, int64_t T, const int64_t* ts) {
  LayerRows r;
  r.uvqk = h->ws.uvqk;
  r.q0 = 0;
  r.M = T;
  r.T_attn = T;
  r.num_pairs = int((T + 2 * hstu::kTile - 1) / (2 * hstu::kTile));
  r.order = h->ws.qtile_order;
  r.ts = ts;
  return r;
}

// One layer after the schedule is built: f1 -> attention -> LN (.) U -> f2, on
// the M query rows; x and out are [M, d].
// xb_ready: ws.xb already holds bf16(x) (written by the previous layer's f2);
// make_xb: f2 also writes bf16(out) to ws.xb for the next layer (fp32 io only).
hstu_status run_layer(hstu_handle* h, const void* x, const LayerRows& R,
                      const hstu_layer_weights* w, void* out, cudaStream_t st, bool xb_ready,
                      bool make_xb) {
  const hstu_config& c = h->cfg;
  Workspace& ws = h->ws;
  const int d = c.d_model;
  const bool f32 = c.compute_dtype == HSTU_DTYPE_FP32;
  const bool io32 = c.io_dtype == HSTU_DTYPE_FP32;
  const int64_t T = R.M;
  const size_t cs = hstu::elem_size(c.compute_dtype);
  void* uvqk_q = static_cast<char*>(R.uvqk) + size_t(R.q0) * 4 * d * cs;   // the query rows
  float* av_q = ws.av + size_t(R.q0) * d;
  if (f32 && R.q0 != 0) return HSTU_ERR_UNSUPPORTED;
  cudaError_t e = cudaSuccess;
  hstu::AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.uvqk = R.uvqk;
  a.av = ws.av;
  a.rows = ws.rows;
  a.order = R.order;
  a.ts = R.ts;
  a.thresholds = ws.thresholds;
  a.time_lut = ws.time_lut;
  a.thr32 = ws.thr32;
  a.lut_exact = c.time_log_div > 0.2232 ? 1 : 0;
  a.rab_pos = w->rab_pos;
  a.rab_time = w->rab_time;
  a.counters = ws.counters;
  a.error = ws.error;
  a.T = R.T_attn;
  a.d = d;
  a.H = c.num_heads;
  a.hd = c.head_dim;
  a.pos_clamp = c.pos_clamp;
  a.time_buckets = c.time_buckets;
  a.n_norm_fixed = c.n_norm;
  a.num_pairs = R.num_pairs;
  a.wait_limit = h->wait_limit;
  a.q_row0 = R.q0;
  if (f32) {
    {
      Timed tm(h, kF1, st);
      e = hstu::launch_gemm_f32(static_cast<const float*>(x), static_cast<const float*>(w->w1), T,
                                4 * d, d, hstu::Epi::kSiluSplit, w->b1,
                                static_cast<float*>(ws.uvqk), nullptr, st);
    }
    if (e == cudaSuccess) {
      Timed tm(h, kAttention, st);
      e = hstu::launch_attention_f32(a, st);
    }
    if (e == cudaSuccess) {
      Timed tm(h, kLnGate, st);
      e = hstu::launch_ln_gate(ws.av, ws.uvqk, ws.g, w->ln_gamma, w->ln_beta, T, d, c.ln_eps, 1, st);
    }
    if (e == cudaSuccess) {
      Timed tm(h, kF2, st);
      e = hstu::launch_gemm_f32(static_cast<const float*>(ws.g), static_cast<const float*>(w->w2),
                                T, d, d, hstu::Epi::kBiasResidual, w->b2, static_cast<float*>(out),
                                static_cast<const float*>(x), st);
    }
    return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
  }
  const void* xa = x;
  if (io32) {
    if (!xb_ready) {
      Timed tm(h, kCast, st);
      e = hstu::launch_cast_bf16(static_cast<const float*>(x), ws.xb, T * d, st);
    }
    xa = ws.xb;
  }
  hstu::GemmArgs g1;
  g1.a = xa;
  g1.b = w->w1;
  g1.M = T;
  g1.N = 4 * d;
  g1.K = d;
  g1.epi = hstu::Epi::kSiluSplit;
  g1.bias = w->b1;
  g1.out = uvqk_q;
  g1.residual = nullptr;
  g1.io_fp32 = 0;
  g1.out_bf16 = nullptr;
  g1.wait_limit = h->wait_limit;
  if (e == cudaSuccess) {
    Timed tm(h, kF1, st);
    e = hstu::launch_gemm_tc(g1, h->num_sms, st, ws.error);
  }
  if (e == cudaSuccess) {
    Timed tm(h, kAttention, st);
    e = hstu::launch_attention_tc(a, st, false);
  }
  if (e == cudaSuccess) {
    Timed tm(h, kLnGate, st);
    e = hstu::launch_ln_gate(av_q, uvqk_q, ws.g, w->ln_gamma, w->ln_beta, T, d, c.ln_eps, 0, st);
  }
  hstu::GemmArgs g2;
  g2.a = ws.g;
  g2.b = w->w2;
  g2.M = T;
  g2.N = d;
  g2.K = d;
  g2.epi = hstu::Epi::kBiasResidual;
  g2.bias = w->b2;
  g2.out = out;
  g2.residual = x;
  g2.io_fp32 = io32 ? 1 : 0;
  g2.out_bf16 = (io32 && make_xb) ? ws.xb : nullptr;
  g2.wait_limit = h->wait_limit;
  if (e == cudaSuccess) {
    Timed tm(h, kF2, st);
    e = hstu::launch_gemm_tc(g2, h->num_sms, st, ws.error);
  }
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

}  // namespace

extern "C" {

hstu_status hstu_layer_forward(hstu_handle* h, const void* values, int64_t T,
                               const int32_t* offsets, int32_t B, const int64_t* ts,
                               const hstu_layer_weights* w, hstu_mask_mode mode,
                               const int32_t* ncand, void* out, void* stream) {
  return hstu_stack_forward(h, values, T, offsets, B, ts, w, 1, mode, ncand, out, stream);
}

hstu_status hstu_stack_forward(hstu_handle* h, const void* values, int64_t T,
                               const int32_t* offsets, int32_t B, const int64_t* ts,
                               const hstu_layer_weights* layers, int32_t num_layers,
                               hstu_mask_mode mode, const int32_t* ncand, void* out,
                               void* stream) {
  hstu_status s = check_common(h, values, T, offsets, B, ts, mode, ncand, out);
  if (s != HSTU_OK) return s;
  if (layers == nullptr || num_layers < 1) return HSTU_ERR_INVALID_ARG;
  for (int32_t l = 0; l < num_layers; ++l) {
    s = check_weights(&layers[l]);
    if (s != HSTU_OK) return s;
  }
  if (T == 0) return HSTU_OK;
  if (cudaSetDevice(h->device) != cudaSuccess) return HSTU_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  {
    Timed tm(h, kSchedule, st);
    if (hstu::launch_schedule(h, T, offsets, B, ts, mode, ncand, st) != cudaSuccess)
      return HSTU_ERR_CUDA;
  }
  h->last_T = T;
  for (int32_t l = 0; l < num_layers; ++l) {
    const void* x = (l == 0) ? values : out;
    s = run_layer(h, x, plain_rows(h, T, ts), &layers[l], out, st, l > 0, l + 1 < num_layers);
    if (s != HSTU_OK) return s;
  }
  return HSTU_OK;
}

hstu_status hstu_get_device_error(hstu_handle* h, int32_t* bits) {
  if (h == nullptr || bits == nullptr) return HSTU_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return HSTU_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return HSTU_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, h->ws.error, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return HSTU_ERR_CUDA;
  if (cudaMemset(h->ws.error, 0, 4) != cudaSuccess) return HSTU_ERR_CUDA;
  *bits = v;
  if (v & HSTU_DEVERR_TIMEOUT) return HSTU_ERR_TIMEOUT;
  return v ? HSTU_ERR_DEVICE_CHECK : HSTU_OK;
}

hstu_status hstu_copy_intermediate(hstu_handle* h, hstu_tensor which, void* dst, size_t bytes,
                                   void* stream) {
  if (h == nullptr || dst == nullptr) return HSTU_ERR_INVALID_ARG;
  const size_t T = size_t(h->cfg.max_tokens), d = size_t(h->cfg.d_model);
  const size_t cs = hstu::elem_size(h->cfg.compute_dtype);
  const void* src = nullptr;
  size_t cap = 0;
  switch (which) {
    case HSTU_TENSOR_UVQK: src = h->ws.uvqk; cap = T * 4 * d * cs; break;
    case HSTU_TENSOR_AV: src = h->ws.av; cap = T * d * 4; break;
    case HSTU_TENSOR_G: src = h->ws.g; cap = T * d * cs; break;
    default: return HSTU_ERR_INVALID_ARG;
  }
  if (bytes > cap) return HSTU_ERR_INVALID_ARG;
  if (bytes == 0) return HSTU_OK;
  if (cudaSetDevice(h->device) != cudaSuccess) return HSTU_ERR_CUDA;
  return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice,
                         static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? HSTU_OK
             : HSTU_ERR_CUDA;
}

hstu_status hstu_debug_attention_buckets(hstu_handle* h, int64_t T, const int32_t* offsets,
                                         int32_t B, const int64_t* ts, hstu_mask_mode mode,
                                         const int32_t* ncand, int32_t* pidx_out,
                                         int32_t* tidx_out, uint8_t* vis_out) {
  hstu_status s = check_common(h, reinterpret_cast<const void*>(16), T, offsets, B, ts, mode, ncand,
                               reinterpret_cast<const void*>(16));
  if (s != HSTU_OK) return s;
  if (h->cfg.compute_dtype != HSTU_DTYPE_BF16) return HSTU_ERR_UNSUPPORTED;
  if (T > 4096 || pidx_out == nullptr || tidx_out == nullptr || vis_out == nullptr)
    return HSTU_ERR_INVALID_ARG;
  if (T == 0) return HSTU_OK;
  if (cudaSetDevice(h->device) != cudaSuccess) return HSTU_ERR_CUDA;
  const hstu_config& c = h->cfg;
  const int d = c.d_model;
  // zero Q/K/V so that the kernel reads defined values; biases from zero tables
  float* zeros = nullptr;
  if (cudaMalloc(&zeros, size_t(c.pos_buckets + c.time_buckets) * 4) != cudaSuccess)
    return HSTU_ERR_CUDA;
  cudaMemset(zeros, 0, size_t(c.pos_buckets + c.time_buckets) * 4);
  cudaMemset(h->ws.uvqk, 0, size_t(T) * 4 * d * 2);
  cudaError_t e = hstu::launch_schedule(h, T, offsets, B, ts, mode, ncand, 0);
  hstu::AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.uvqk = h->ws.uvqk;
  a.av = h->ws.av;
  a.rows = h->ws.rows;
  a.order = h->ws.qtile_order;
  a.ts = ts;
  a.thresholds = h->ws.thresholds;
  a.time_lut = h->ws.time_lut;
  a.thr32 = h->ws.thr32;
  a.lut_exact = c.time_log_div > 0.2232 ? 1 : 0;
  a.rab_pos = zeros;
  a.rab_time = zeros + c.pos_buckets;
  a.counters = h->ws.counters;
  a.error = h->ws.error;
  a.T = T;
  a.d = d;
  a.H = c.num_heads;
  a.hd = c.head_dim;
  a.pos_clamp = c.pos_clamp;
  a.time_buckets = c.time_buckets;
  a.n_norm_fixed = c.n_norm;
  a.num_pairs = int((T + 2 * hstu::kTile - 1) / (2 * hstu::kTile));
  a.dump_pidx = pidx_out;
  a.dump_tidx = tidx_out;
  a.dump_vis = vis_out;
  if (e == cudaSuccess) e = hstu::launch_attention_tc(a, 0, true);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  cudaFree(zeros);
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

hstu_status hstu_set_wait_limit(hstu_handle* h, int64_t cycles) {
  if (h == nullptr || cycles < 0) return HSTU_ERR_INVALID_ARG;
  h->wait_limit = cycles;
  return HSTU_OK;
}

hstu_status hstu_set_kernel_timing(hstu_handle* h, int32_t enabled) {
  if (h == nullptr) return HSTU_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return HSTU_ERR_CUDA;
  hstu::KernelTimer& t = h->timer;
  if (enabled && !t.created) {
    for (int i = 0; i < 2 * hstu::KernelTimer::kMax; ++i)
      if (cudaEventCreate(&t.ev[i]) != cudaSuccess) return HSTU_ERR_CUDA;
    t.created = true;
  }
  t.enabled = enabled != 0;
  if (t.enabled) t.count = 0;
  return HSTU_OK;
}

hstu_status hstu_get_kernel_timing(hstu_handle* h, double* total_ms, int64_t* launches) {
  if (h == nullptr) return HSTU_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return HSTU_ERR_CUDA;
  double ms[HSTU_KERNEL_KINDS] = {0};
  int64_t n[HSTU_KERNEL_KINDS] = {0};
  const hstu::KernelTimer& t = h->timer;
  for (int i = 0; i < t.count; ++i) {
    if (cudaEventSynchronize(t.ev[2 * i + 1]) != cudaSuccess) return HSTU_ERR_CUDA;
    float e = 0.f;
    if (cudaEventElapsedTime(&e, t.ev[2 * i], t.ev[2 * i + 1]) != cudaSuccess) return HSTU_ERR_CUDA;
    ms[t.kind[i]] += e;
    n[t.kind[i]] += 1;
  }
  for (int k = 0; k < HSTU_KERNEL_KINDS; ++k) {
    if (total_ms != nullptr) total_ms[k] = ms[k];
    if (launches != nullptr) launches[k] = n[k];
  }
  return HSTU_OK;
}

hstu_status hstu_debug_umma_tile(int32_t mode, const void* a, const void* b, float* c, int32_t n,
                                 int32_t k) {
  if (a == nullptr || b == nullptr || c == nullptr) return HSTU_ERR_INVALID_ARG;
  if (mode < 0 || mode > 2 || (k != 64 && k != 128)) return HSTU_ERR_INVALID_ARG;
  if (mode == 0 && n != 64 && n != 128 && n != 256) return HSTU_ERR_INVALID_ARG;
  if (mode != 0 && n != 64 && n != 128) return HSTU_ERR_INVALID_ARG;
  const cudaError_t e = hstu::run_umma_tile(mode, a, b, c, n, k);
  if (e == cudaErrorLaunchTimeout) return HSTU_ERR_TIMEOUT;
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Attention without allocation.  Every piece of scratch of the attention step
// (row facts, pair order and cost, counters, error word, bucket tables) lives
// in one file-scope device array; the call allocates nothing.
namespace hstu {
namespace {

constexpr int64_t kNoAllocMaxTokens = HSTU_NOALLOC_MAX_TOKENS;
constexpr size_t kNoAllocPairs = 1024;   // >= kNoAllocMaxTokens / (2 * kTile)
constexpr size_t kOffRows = 0;
constexpr size_t kOffOrder = kOffRows + size_t(kNoAllocMaxTokens) * sizeof(RowInfo);
constexpr size_t kOffCost = kOffOrder + kNoAllocPairs * 4;
constexpr size_t kOffCounters = kOffCost + kNoAllocPairs * 4;
constexpr size_t kOffError = kOffCounters + 256;
constexpr size_t kOffThr = kOffError + 256;
constexpr size_t kOffLut = kOffThr + 256 * 8;
constexpr size_t kOffThr32 = kOffLut + 256;
constexpr size_t kNoAllocScratchBytes = kOffThr32 + 1280;   // 1,060,864 bytes
static_assert(kNoAllocPairs * 2 * kTile >= size_t(kNoAllocMaxTokens), "pair table size");
static_assert(kOffOrder % 256 == 0 && kOffThr % 256 == 0 && kOffThr32 % 256 == 0, "alignment");

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Host cache of the scratch address per device (set on the first call on that device).
constexpr int kNoAllocMaxDevices = 64;
uint8_t* g_noalloc_addr[kNoAllocMaxDevices] = {nullptr};

// Host cache of the bucket tables for the last (divisor, bucket count).
struct NoAllocTables {
  int64_t thr[256];
  int32_t thr32[260];
  uint8_t lut[128];
  int32_t nb;
};
NoAllocTables g_noalloc_tables;
double g_noalloc_div = 0.0;
int32_t g_noalloc_nb = 0;

// Writes the bucket tables (passed by value) into the scratch and clears the
// counters and the error word: the scratch values that must start at zero.
__global__ void noalloc_prepare_kernel(const NoAllocTables t, int64_t* thr, uint8_t* lut,
                                       int32_t* thr32, int32_t* counters, int32_t* err) {
  for (int k = threadIdx.x; k < 257; k += blockDim.x) {
    thr32[k] = t.thr32[k];
    if (k < t.nb) thr[k] = t.thr[k];
    if (k < 128) lut[k] = t.lut[k];
    if (k < 4) {
      counters[k] = 0;
      err[k] = 0;
    }
  }
}

}  // namespace
}  // namespace hstu

extern "C" hstu_status hstu_attention_noalloc(const hstu_config* cfg, const void* uvqk,
                                              int64_t T, const int32_t* offsets, int32_t B,
                                              const int64_t* ts, hstu_mask_mode mode,
                                              const int32_t* ncand, const float* rab_pos,
                                              const float* rab_time, float* av,
                                              int32_t* device_error, void* stream) {
  using namespace hstu;
  if (cfg == nullptr) return HSTU_ERR_INVALID_ARG;
  const hstu_config& c = *cfg;
  if (c.num_heads <= 0 || c.d_model != c.num_heads * c.head_dim) return HSTU_ERR_INVALID_ARG;
  if (c.pos_buckets < 1 || c.pos_clamp < 0 || c.pos_clamp >= c.pos_buckets) return HSTU_ERR_INVALID_ARG;
  if (c.time_buckets < 1 || c.time_buckets > 256 || !(c.time_log_div > 0.0)) return HSTU_ERR_INVALID_ARG;
  if (c.compute_dtype != HSTU_DTYPE_BF16 || (c.head_dim != 64 && c.head_dim != 128) ||
      c.d_model % 128 != 0 || c.d_model > 1024 || c.pos_clamp > 4096)
    return HSTU_ERR_UNSUPPORTED;
  if (T < 0 || B < 0 || (B == 0 && T != 0) || offsets == nullptr) return HSTU_ERR_INVALID_ARG;
  if (mode != HSTU_MASK_CAUSAL && mode != HSTU_MASK_MFALCON) return HSTU_ERR_INVALID_ARG;
  if (mode == HSTU_MASK_MFALCON && B > 0 && ncand == nullptr) return HSTU_ERR_INVALID_ARG;
  if (T > kNoAllocMaxTokens) return HSTU_ERR_WORKSPACE;
  if (T > 0) {
    const void* ps[] = {uvqk, ts, av, rab_pos, rab_time};
    for (const void* p : ps)
      if (p == nullptr || !aligned16(p)) return HSTU_ERR_INVALID_ARG;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HSTU_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return HSTU_ERR_UNSUPPORTED;
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return HSTU_ERR_CUDA;
    g_noalloc_addr[dev] = static_cast<uint8_t*>(p);
  }
  if (g_noalloc_nb != c.time_buckets || g_noalloc_div != c.time_log_div) {
    if (hstu_time_bucket_thresholds(c.time_log_div, c.time_buckets, g_noalloc_tables.thr) != HSTU_OK)
      return HSTU_ERR_INVALID_ARG;
    build_time_lut(g_noalloc_tables.thr, c.time_buckets, g_noalloc_tables.lut,
                   g_noalloc_tables.thr32);
    g_noalloc_tables.nb = c.time_buckets;
    g_noalloc_nb = c.time_buckets;
    g_noalloc_div = c.time_log_div;
  }
  uint8_t* base = g_noalloc_addr[dev];
  RowInfo* rows = reinterpret_cast<RowInfo*>(base + kOffRows);
  int32_t* order = reinterpret_cast<int32_t*>(base + kOffOrder);
  int32_t* cost = reinterpret_cast<int32_t*>(base + kOffCost);
  int32_t* counters = reinterpret_cast<int32_t*>(base + kOffCounters);
  int32_t* err = reinterpret_cast<int32_t*>(base + kOffError);
  int64_t* thr = reinterpret_cast<int64_t*>(base + kOffThr);
  uint8_t* lut = reinterpret_cast<uint8_t*>(base + kOffLut);
  int32_t* thr32 = reinterpret_cast<int32_t*>(base + kOffThr32);
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  noalloc_prepare_kernel<<<1, 256, 0, st>>>(g_noalloc_tables, thr, lut, thr32, counters, err);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess)
    e = launch_schedule_raw(T, offsets, B, ts, mode, ncand, rows, cost, order, counters, err, st);
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.uvqk = uvqk;
  a.av = av;
  a.rows = rows;
  a.order = order;
  a.ts = ts;
  a.thresholds = thr;
  a.time_lut = lut;
  a.thr32 = thr32;
  a.lut_exact = c.time_log_div > 0.2232 ? 1 : 0;
  a.rab_pos = rab_pos;
  a.rab_time = rab_time;
  a.counters = counters;
  a.error = err;
  a.T = T;
  a.d = c.d_model;
  a.H = c.num_heads;
  a.hd = c.head_dim;
  a.pos_clamp = c.pos_clamp;
  a.time_buckets = c.time_buckets;
  a.n_norm_fixed = c.n_norm;
  a.num_pairs = int((T + 2 * kTile - 1) / (2 * kTile));
  if (e == cudaSuccess) e = launch_attention_tc(a, st, false);
  if (e == cudaSuccess && device_error != nullptr)
    e = cudaMemcpyAsync(device_error, err, sizeof(int32_t), cudaMemcpyDeviceToDevice, st);
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// M-FALCON history cache: the candidate-independent history computation of a
// stack, kept across calls that score micro-batches of candidates.
struct hstu_history_cache_s {
  static constexpr int kRing = 4;   // pinned staging slots for the per-call table
  hstu_handle* h = nullptr;    // the handle whose workspace the calls use
  int device = 0;
  int32_t num_layers = 0;
  int64_t max_hist = 0;        // history rows the buffers hold
  int64_t cand_cap = 0;        // candidate block rows (a multiple of 2 * 128)
  int64_t rows_cap = 0;        // round_up(max_hist, 256) + cand_cap
  int32_t max_users = 0;
  int64_t T_h = -1;            // -1 until the first prefill
  int32_t B = 0;
  std::vector<void*> uvqk;     // per layer: device [rows_cap, 4d] bf16
  int64_t* ts = nullptr;       // device [rows_cap]
  int32_t* hoff = nullptr;     // device [max_users + 1]
  // the last call's table: blk [B + 1] | coff [B + 1] | pair order [P / 256]
  int32_t* table = nullptr;    // device
  size_t table_ints = 0;       // capacity, in int32
  int32_t* hoff_host = nullptr;       // pinned [max_users + 1]: history offsets of the prefill
  cudaEvent_t hoff_ready = nullptr;   // recorded behind their copy
  int32_t* ring[kRing] = {nullptr, nullptr, nullptr, nullptr};   // pinned, table_ints each
  cudaEvent_t ring_done[kRing] = {nullptr, nullptr, nullptr, nullptr};
  bool ring_used[kRing] = {false, false, false, false};
  int ring_next = 0;
  void* xblk = nullptr;        // device [cand_cap, d] io dtype: the block's residual stream
};

namespace {

int64_t round_pair(int64_t n) {
  const int64_t p = 2 * hstu::kTile;
  return (n + p - 1) / p * p;
}

}  // namespace

extern "C" {

hstu_status hstu_cache_destroy(hstu_history_cache* c) {
  if (c == nullptr) return HSTU_OK;
  cudaSetDevice(c->device);
  cudaDeviceSynchronize();
  for (void* p : c->uvqk)
    if (p != nullptr) cudaFree(p);
  void* ptrs[] = {c->ts, c->hoff, c->table, c->xblk};
  for (void* p : ptrs)
    if (p != nullptr) cudaFree(p);
  if (c->hoff_host != nullptr) cudaFreeHost(c->hoff_host);
  if (c->hoff_ready != nullptr) cudaEventDestroy(c->hoff_ready);
  for (int k = 0; k < hstu_history_cache_s::kRing; ++k) {
    if (c->ring[k] != nullptr) cudaFreeHost(c->ring[k]);
    if (c->ring_done[k] != nullptr) cudaEventDestroy(c->ring_done[k]);
  }
  delete c;
  return HSTU_OK;
}

hstu_status hstu_cache_create(hstu_handle* h, int32_t num_layers, int64_t max_history_tokens,
                              int64_t max_candidate_rows, hstu_history_cache** out) {
  if (out == nullptr) return HSTU_ERR_INVALID_ARG;
  *out = nullptr;
  if (h == nullptr || num_layers < 1 || max_history_tokens < 0 || max_candidate_rows < 1)
    return HSTU_ERR_INVALID_ARG;
  const hstu_config& cfg = h->cfg;
  if (cfg.compute_dtype != HSTU_DTYPE_BF16 || cfg.n_norm <= 0) return HSTU_ERR_UNSUPPORTED;
  const int64_t cand_cap = round_pair(max_candidate_rows);
  if (cand_cap / (2 * hstu::kTile) > hstu::kMaxCandidatePairs) return HSTU_ERR_UNSUPPORTED;
  const int64_t rows_cap = round_pair(max_history_tokens) + cand_cap;
  if (rows_cap > cfg.max_tokens || max_history_tokens > cfg.max_tokens) return HSTU_ERR_WORKSPACE;
  if (cudaSetDevice(h->device) != cudaSuccess) return HSTU_ERR_CUDA;
  hstu_history_cache* c = new (std::nothrow) hstu_history_cache_s();
  if (c == nullptr) return HSTU_ERR_CUDA;
  c->h = h;
  c->device = h->device;
  c->num_layers = num_layers;
  c->max_hist = max_history_tokens;
  c->cand_cap = cand_cap;
  c->rows_cap = rows_cap;
  c->max_users = cfg.max_users;
  const size_t d = size_t(cfg.d_model);
  const size_t io = hstu::elem_size(cfg.io_dtype);
  c->uvqk.assign(size_t(num_layers), nullptr);
  cudaError_t e = cudaSuccess;
  // Zeroed once: rows never written (the gap before the candidate block, rows
  // past a shorter history) must hold finite values, since a key tile that
  // straddles them is multiplied by zero weights on the tensor cores.
  for (int32_t l = 0; l < num_layers && e == cudaSuccess; ++l) {
    e = hstu::alloc(&c->uvqk[l], size_t(rows_cap) * 4 * d * 2);
    if (e == cudaSuccess) e = cudaMemset(c->uvqk[l], 0, size_t(rows_cap) * 4 * d * 2);
  }
  if (e == cudaSuccess) e = hstu::alloc(&c->ts, size_t(rows_cap) * 8);
  if (e == cudaSuccess) e = cudaMemset(c->ts, 0, size_t(rows_cap) * 8);
  c->table_ints = size_t(2 * (cfg.max_users + 1)) + size_t(cand_cap / (2 * hstu::kTile));
  if (e == cudaSuccess) e = hstu::alloc(&c->hoff, size_t(cfg.max_users + 1) * 4);
  if (e == cudaSuccess) e = hstu::alloc(&c->table, c->table_ints * 4);
  if (e == cudaSuccess) e = hstu::alloc(&c->xblk, size_t(cand_cap) * d * io);
  if (e == cudaSuccess)
    e = cudaMallocHost(reinterpret_cast<void**>(&c->hoff_host), size_t(cfg.max_users + 1) * 4);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->hoff_ready, cudaEventDisableTiming);
  for (int k = 0; e == cudaSuccess && k < hstu_history_cache_s::kRing; ++k) {
    e = cudaMallocHost(reinterpret_cast<void**>(&c->ring[k]), c->table_ints * 4);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ring_done[k], cudaEventDisableTiming);
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    hstu_cache_destroy(c);
    return HSTU_ERR_CUDA;
  }
  *out = c;
  return HSTU_OK;
}

hstu_status hstu_cache_prefill(hstu_handle* h, hstu_history_cache* c, const void* values,
                               int64_t T_h, const int32_t* offsets, int32_t B,
                               const int64_t* ts, const hstu_layer_weights* layers,
                               int32_t num_layers, void* out, void* stream) {
  if (c == nullptr || h == nullptr || c->h != h) return HSTU_ERR_INVALID_ARG;
  hstu_status s = check_common(h, values, T_h, offsets, B, ts, HSTU_MASK_CAUSAL, nullptr, out);
  if (s != HSTU_OK) return s;
  if (T_h > c->max_hist) return HSTU_ERR_WORKSPACE;
  if (layers == nullptr || num_layers != c->num_layers) return HSTU_ERR_INVALID_ARG;
  for (int32_t l = 0; l < num_layers; ++l) {
    s = check_weights(&layers[l]);
    if (s != HSTU_OK) return s;
  }
  if (cudaSetDevice(h->device) != cudaSuccess) return HSTU_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(c->hoff, offsets, size_t(B + 1) * 4, cudaMemcpyDeviceToDevice, st);
  // the history lengths on the host (pinned), for the pair order of later calls
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(c->hoff_host, offsets, size_t(B + 1) * 4, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaEventRecord(c->hoff_ready, st);
  if (e == cudaSuccess && T_h > 0)
    e = cudaMemcpyAsync(c->ts, ts, size_t(T_h) * 8, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  c->T_h = -1;   // stays invalid unless every launch below is enqueued
  if (T_h > 0) {
    {
      Timed tm(h, kSchedule, st);
      if (hstu::launch_schedule(h, T_h, offsets, B, ts, HSTU_MASK_CAUSAL, nullptr, st) !=
          cudaSuccess)
        return HSTU_ERR_CUDA;
    }
    for (int32_t l = 0; l < num_layers; ++l) {
      LayerRows R = plain_rows(h, T_h, c->ts);
      R.uvqk = c->uvqk[l];
      s = run_layer(h, l == 0 ? values : out, R, &layers[l], out, st, l > 0, l + 1 < num_layers);
      if (s != HSTU_OK) return s;
    }
  }
  c->T_h = T_h;
  c->B = B;
  return HSTU_OK;
}

hstu_status hstu_cache_score(hstu_handle* h, hstu_history_cache* c, const void* values,
                             const int32_t* num_candidates_host, const int64_t* timestamps,
                             const hstu_layer_weights* layers, int32_t num_layers, void* out,
                             void* stream) {
  if (c == nullptr || h == nullptr || c->h != h) return HSTU_ERR_INVALID_ARG;
  if (c->T_h < 0) return HSTU_ERR_INVALID_ARG;   // no history yet
  const int32_t B = c->B;
  if (B > 0 && num_candidates_host == nullptr) return HSTU_ERR_INVALID_ARG;
  if (layers == nullptr || num_layers != c->num_layers) return HSTU_ERR_INVALID_ARG;
  for (int32_t l = 0; l < num_layers; ++l) {
    hstu_status s = check_weights(&layers[l]);
    if (s != HSTU_OK) return s;
  }
  // the block layout and the pair order, on the host, in a pinned slot whose
  // previous copy has finished
  const int slot = c->ring_next;
  if (c->ring_used[slot] && cudaEventSynchronize(c->ring_done[slot]) != cudaSuccess)
    return HSTU_ERR_CUDA;
  int32_t* blk = c->ring[slot];
  int32_t* coff = blk + B + 1;
  int64_t P = 0, T_c = 0;
  for (int32_t b = 0; b < B; ++b) {
    const int32_t n = num_candidates_host[b];
    if (n < 0) return HSTU_ERR_INVALID_ARG;
    blk[b] = int32_t(P);
    coff[b] = int32_t(T_c);
    P += round_pair(n);
    T_c += n;
    if (P > c->cand_cap) return HSTU_ERR_WORKSPACE;
  }
  blk[B] = int32_t(P);
  coff[B] = int32_t(T_c);
  if (T_c == 0) return HSTU_OK;
  if (values == nullptr || out == nullptr || timestamps == nullptr || !hstu::aligned16(values) ||
      !hstu::aligned16(out) || !hstu::aligned16(timestamps))
    return HSTU_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return HSTU_ERR_CUDA;
  if (cudaEventSynchronize(c->hoff_ready) != cudaSuccess) return HSTU_ERR_CUDA;
  // pairs by descending history length of their user (ties by pair index):
  // the longest-first order of the attention's work items
  const int64_t q0 = round_pair(c->T_h);
  const int32_t n_pairs = int32_t(P / (2 * hstu::kTile));
  int32_t* order = coff + B + 1;
  {
    std::vector<std::pair<int64_t, int32_t>> key;
    key.reserve(size_t(n_pairs));
    for (int32_t b = 0; b < B; ++b) {
      int64_t hl = int64_t(c->hoff_host[b + 1]) - int64_t(c->hoff_host[b]);
      if (hl < 0) hl = 0;
      for (int32_t k = blk[b] / (2 * hstu::kTile); k < blk[b + 1] / (2 * hstu::kTile); ++k)
        key.emplace_back(-hl, k);
    }
    std::sort(key.begin(), key.end());
    for (int32_t k = 0; k < n_pairs; ++k)
      order[k] = int32_t(q0 / (2 * hstu::kTile)) + key[size_t(k)].second;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const hstu_config& cfg = h->cfg;
  const int64_t row_bytes = int64_t(cfg.d_model) * int64_t(hstu::elem_size(cfg.io_dtype));
  const size_t ints = size_t(2 * (B + 1) + n_pairs);
  cudaError_t e = cudaMemcpyAsync(c->table, blk, ints * 4, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaEventRecord(c->ring_done[slot], st);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  c->ring_used[slot] = true;
  c->ring_next = (slot + 1) % hstu_history_cache_s::kRing;
  {
    Timed tm(h, kBlock, st);
    e = hstu::launch_candidate_block(c->table, c->hoff, B, c->T_h, q0, int32_t(P), timestamps,
                                     c->ts, h->ws.rows, row_bytes, values, c->xblk, st);
  }
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  LayerRows R;
  R.q0 = q0;
  R.M = P;
  R.T_attn = q0 + P;
  R.num_pairs = int(P / (2 * hstu::kTile));
  R.order = c->table + 2 * (B + 1);
  R.ts = c->ts;
  for (int32_t l = 0; l < num_layers; ++l) {
    R.uvqk = c->uvqk[l];
    const hstu_status s = run_layer(h, c->xblk, R, &layers[l], c->xblk, st, l > 0,
                                    l + 1 < num_layers);
    if (s != HSTU_OK) return s;
  }
  {
    Timed tm(h, kBlock, st);
    e = hstu::launch_candidate_copy(c->table, B, int32_t(P), row_bytes, c->xblk, out, false, st);
  }
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Stochastic Length: argument checks and the scratch layout
//   [0, 256)            error word
//   [256, 256 + 4B')    kept counts (B' = B rounded up to 64)
//   then                flags [T]
namespace {

size_t sl_kept_bytes(int32_t B) { return size_t((int64_t(B) + 63) / 64 * 64) * 4; }

}  // namespace

extern "C" {

size_t hstu_stochastic_length_scratch_bytes(int64_t T, int32_t B) {
  if (T < 0 || B < 0) return 0;
  return 256 + sl_kept_bytes(B) + size_t((T + 255) / 256 * 256);
}

hstu_status hstu_stochastic_length(const int32_t* offsets, int32_t B, int64_t T,
                                   const double* u, const uint32_t* keys, int32_t n_c,
                                   double alpha, const void* values, int64_t row_bytes,
                                   const int64_t* ts, int32_t* out_offsets, int64_t* out_index,
                                   void* out_values, int64_t* out_ts, void* scratch,
                                   int32_t* device_error, void* stream) {
  if (B < 0 || T < 0 || T >= (int64_t(1) << 31) || (B == 0 && T != 0)) return HSTU_ERR_INVALID_ARG;
  if (n_c < 1 || !isfinite(alpha)) return HSTU_ERR_INVALID_ARG;
  if (offsets == nullptr || out_offsets == nullptr || scratch == nullptr) return HSTU_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(scratch) % 256 != 0) return HSTU_ERR_INVALID_ARG;
  if (T > 0 && (u == nullptr || keys == nullptr || out_index == nullptr)) return HSTU_ERR_INVALID_ARG;
  if (ts != nullptr && out_ts == nullptr) return HSTU_ERR_INVALID_ARG;
  if (values != nullptr) {
    if (out_values == nullptr || row_bytes <= 0 || row_bytes % 16 != 0 ||
        !hstu::aligned16(values) || !hstu::aligned16(out_values))
      return HSTU_ERR_INVALID_ARG;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HSTU_ERR_CUDA;
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  uint8_t* base = static_cast<uint8_t*>(scratch);
  hstu::SlArgs a;
  a.offs = offsets;
  a.B = B;
  a.T = T;
  a.u = u;
  a.keys = keys;
  a.n_c = n_c;
  a.numerator = pow(double(n_c), alpha);
  a.values = values;
  a.row_bytes = row_bytes;
  a.ts = ts;
  a.out_offs = out_offsets;
  a.out_index = out_index;
  a.out_values = out_values;
  a.out_ts = ts != nullptr ? out_ts : nullptr;
  a.err = reinterpret_cast<int32_t*>(base);
  a.kept = reinterpret_cast<int32_t*>(base + 256);
  a.flags = base + 256 + sl_kept_bytes(B);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = hstu::launch_stochastic_length(a, sms, st);
  if (e == cudaSuccess && device_error != nullptr)
    e = cudaMemcpyAsync(device_error, a.err, sizeof(int32_t), cudaMemcpyDeviceToDevice, st);
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// The attention step alone, on the handle's workspace
extern "C" hstu_status hstu_attention_forward(hstu_handle* h, const void* uvqk, int64_t T,
                                              const int32_t* offsets, int32_t B,
                                              const int64_t* ts, hstu_mask_mode mode,
                                              const int32_t* ncand, const float* rab_pos,
                                              const float* rab_time, float* av, void* stream) {
  hstu_status s = check_common(h, uvqk, T, offsets, B, ts, mode, ncand, av);
  if (s != HSTU_OK) return s;
  if (T > 0 && (rab_pos == nullptr || rab_time == nullptr || !hstu::aligned16(rab_pos) ||
                !hstu::aligned16(rab_time)))
    return HSTU_ERR_INVALID_ARG;
  if (T == 0) return HSTU_OK;
  if (cudaSetDevice(h->device) != cudaSuccess) return HSTU_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  {
    Timed tm(h, kSchedule, st);
    e = hstu::launch_schedule(h, T, offsets, B, ts, mode, ncand, st);
  }
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  const hstu_config& c = h->cfg;
  hstu::AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.uvqk = uvqk;
  a.av = av;
  a.rows = h->ws.rows;
  a.order = h->ws.qtile_order;
  a.ts = ts;
  a.thresholds = h->ws.thresholds;
  a.time_lut = h->ws.time_lut;
  a.thr32 = h->ws.thr32;
  a.lut_exact = c.time_log_div > 0.2232 ? 1 : 0;
  a.rab_pos = rab_pos;
  a.rab_time = rab_time;
  a.counters = h->ws.counters;
  a.error = h->ws.error;
  a.T = T;
  a.d = c.d_model;
  a.H = c.num_heads;
  a.hd = c.head_dim;
  a.pos_clamp = c.pos_clamp;
  a.time_buckets = c.time_buckets;
  a.n_norm_fixed = c.n_norm;
  a.num_pairs = int((T + 2 * hstu::kTile - 1) / (2 * hstu::kTile));
  a.wait_limit = h->wait_limit;
  {
    Timed tm(h, kAttention, st);
    e = c.compute_dtype == HSTU_DTYPE_FP32 ? hstu::launch_attention_f32(a, st)
                                           : hstu::launch_attention_tc(a, st, false);
  }
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Backward of the attention step
namespace {

// The attention backward's arguments on the handle's schedule (launch_schedule
// must have run on the same batch).
hstu::AttnBwdArgs bwd_args(hstu_handle* h, const void* uvqk, const void* d_out, int64_t T,
                           const int32_t* offsets, int32_t B, const int64_t* ts,
                           const float* rab_pos, const float* rab_time, float* dq, float* dk,
                           float* dv, float* d_rab_pos, float* d_rab_time) {
  const hstu_config& c = h->cfg;
  hstu::AttnBwdArgs a;
  memset(&a, 0, sizeof(a));
  a.uvqk = uvqk;
  a.dO = d_out;
  a.rows = h->ws.rows;
  a.order = h->ws.qtile_order;
  a.key_cost = h->ws.ktile_cost;
  a.key_order = h->ws.ktile_order;
  a.offsets = offsets;
  a.B = B;
  a.ts = ts;
  a.thresholds = h->ws.thresholds;
  a.time_lut = h->ws.time_lut;
  a.thr32 = h->ws.thr32;
  a.rab_pos = rab_pos;
  a.rab_time = rab_time;
  a.counters = h->ws.counters;
  a.error = h->ws.error;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.d_rab_pos = d_rab_pos;
  a.d_rab_time = d_rab_time;
  a.T = T;
  a.d = c.d_model;
  a.H = c.num_heads;
  a.hd = c.head_dim;
  a.pos_clamp = c.pos_clamp;
  a.time_buckets = c.time_buckets;
  a.n_norm_fixed = c.n_norm;
  a.lut_exact = c.time_log_div > 0.2232 ? 1 : 0;
  a.wait_limit = h->wait_limit;
  return a;
}

}  // namespace

extern "C" hstu_status hstu_attention_backward(
    hstu_handle* h, const void* uvqk, const void* d_out, int64_t T, const int32_t* offsets,
    int32_t B, const int64_t* ts, hstu_mask_mode mode, const int32_t* ncand, const float* rab_pos,
    const float* rab_time, float* dq, float* dk, float* dv, float* d_rab_pos, float* d_rab_time,
    void* stream) {
  hstu_status s = check_common(h, uvqk, T, offsets, B, ts, mode, ncand, d_out);
  if (s != HSTU_OK) return s;
  if (h->cfg.compute_dtype != HSTU_DTYPE_BF16) return HSTU_ERR_UNSUPPORTED;
  if (T == 0) return HSTU_OK;
  const void* ps[] = {rab_pos, rab_time, dq, dk, dv, d_rab_pos, d_rab_time};
  for (const void* q : ps)
    if (q == nullptr || !hstu::aligned16(q)) return HSTU_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return HSTU_ERR_CUDA;
  const hstu_config& c = h->cfg;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = hstu::launch_schedule(h, T, offsets, B, ts, mode, ncand, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(d_rab_pos, 0, size_t(c.pos_buckets) * 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(d_rab_time, 0, size_t(c.time_buckets) * 4, st);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  const hstu::AttnBwdArgs a = bwd_args(h, uvqk, d_out, T, offsets, B, ts, rab_pos, rab_time, dq,
                                       dk, dv, d_rab_pos, d_rab_time);
  e = hstu::launch_attention_bwd_tc(a, st);
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Backward of one layer
namespace {

cudaError_t bwd_alloc(hstu_handle* h) {
  hstu::BwdWorkspace& b = h->bwd;
  if (b.ready) return cudaSuccess;
  const size_t T = size_t(h->cfg.max_tokens), d = size_t(h->cfg.d_model);
  const size_t T64 = (T + 63) / 64 * 64;
  cudaError_t e = cudaSuccess;
  auto get = [&](void** p, size_t bytes) {
    if (e == cudaSuccess) e = hstu::alloc(p, bytes > 0 ? bytes : 16);
  };
  get(&b.xb, T * d * 2);
  get(&b.dyb, T * d * 2);
  get(&b.w1t, 4 * d * d * 2);
  get(&b.w2t, d * d * 2);
  get(reinterpret_cast<void**>(&b.dg), T * d * 4);
  get(reinterpret_cast<void**>(&b.du), T * d * 4);
  get(&b.dO, T * d * 2);
  get(&b.g, T * d * 2);
  get(reinterpret_cast<void**>(&b.dq), T * d * 4);
  get(reinterpret_cast<void**>(&b.dk), T * d * 4);
  get(reinterpret_cast<void**>(&b.dv), T * d * 4);
  get(reinterpret_cast<void**>(&b.h1), T * 4 * d * 4);
  get(&b.dh1, T * 4 * d * 2);
  get(&b.dh1t, 4 * d * T64 * 2);
  get(&b.xt, d * T64 * 2);
  get(&b.dyt, d * T64 * 2);
  get(&b.gt, d * T64 * 2);
  get(reinterpret_cast<void**>(&b.zeros), 4 * d * 4);
  if (e == cudaSuccess) e = cudaMemset(b.zeros, 0, 4 * d * 4);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) b.ready = true;
  return e;
}

// out (fp32 [M, N], zeroed first) = A [M, K] B[N, K]^T (+ bias), both K-major bf16
cudaError_t gemm_f32(hstu_handle* h, const void* a, const void* b, int64_t M, int N, int K,
                     const float* bias, float* out, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(out, 0, size_t(M) * size_t(N) * 4, st);
  if (e != cudaSuccess) return e;
  hstu::GemmArgs g;
  g.a = a;
  g.b = b;
  g.M = M;
  g.N = N;
  g.K = K;
  g.epi = hstu::Epi::kBiasResidual;
  g.bias = bias;
  g.out = out;
  g.residual = out;   // zero: out = A B^T + bias
  g.io_fp32 = 1;
  g.out_bf16 = nullptr;
  return hstu::launch_gemm_tc(g, h->num_sms, st, h->ws.error);
}

}  // namespace

extern "C" hstu_status hstu_layer_backward(
    hstu_handle* h, const void* values, const void* uvqk, const float* av, const void* d_out,
    int64_t T, const int32_t* offsets, int32_t B, const int64_t* ts,
    const hstu_layer_weights* w, hstu_mask_mode mode, const int32_t* ncand, void* d_values,
    const hstu_layer_grads* gr, void* stream) {
  hstu_status s = check_common(h, values, T, offsets, B, ts, mode, ncand, d_values);
  if (s != HSTU_OK) return s;
  s = check_weights(w);
  if (s != HSTU_OK) return s;
  if (h->cfg.compute_dtype != HSTU_DTYPE_BF16) return HSTU_ERR_UNSUPPORTED;
  if (gr == nullptr) return HSTU_ERR_INVALID_ARG;
  const void* gp[] = {gr->w1, gr->b1, gr->w2, gr->b2, gr->ln_gamma, gr->ln_beta, gr->rab_pos,
                      gr->rab_time};
  for (const void* q : gp)
    if (q == nullptr || !hstu::aligned16(q)) return HSTU_ERR_INVALID_ARG;
  if (T > 0) {
    const void* ip[] = {uvqk, av, d_out};
    for (const void* q : ip)
      if (q == nullptr || !hstu::aligned16(q)) return HSTU_ERR_INVALID_ARG;
  }
  if (cudaSetDevice(h->device) != cudaSuccess) return HSTU_ERR_CUDA;
  if (bwd_alloc(h) != cudaSuccess) return HSTU_ERR_CUDA;
  const hstu_config& c = h->cfg;
  const int d = c.d_model;
  const bool io32 = c.io_dtype == HSTU_DTYPE_FP32;
  hstu::BwdWorkspace& b = h->bwd;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t T64 = (T + 63) / 64 * 64;
  cudaError_t e = cudaSuccess;
  // gradients that are sums start at zero
  e = cudaMemsetAsync(gr->b1, 0, size_t(4 * d) * 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(gr->b2, 0, size_t(d) * 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(gr->ln_gamma, 0, size_t(d) * 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(gr->ln_beta, 0, size_t(d) * 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(gr->rab_pos, 0, size_t(c.pos_buckets) * 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(gr->rab_time, 0, size_t(c.time_buckets) * 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(gr->w1, 0, size_t(4 * d) * size_t(d) * 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(gr->w2, 0, size_t(d) * size_t(d) * 4, st);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  if (T == 0) return HSTU_OK;
  // bf16 operands
  const void* xb = values;
  const void* dyb = d_out;
  if (io32) {
    e = hstu::launch_cast_bf16(static_cast<const float*>(values), b.xb, T * d, st);
    if (e == cudaSuccess) e = hstu::launch_cast_bf16(static_cast<const float*>(d_out), b.dyb, T * d, st);
    xb = b.xb;
    dyb = b.dyb;
  }
  if (e == cudaSuccess) e = hstu::launch_transpose_bf16(w->w2, false, d, d, d, b.w2t, d, st);
  if (e == cudaSuccess) e = hstu::launch_transpose_bf16(w->w1, false, 4 * d, d, d, b.w1t, 4 * d, st);
  // dG = dY W2; everything else that reads dY happens before dX is written,
  // since d_values may alias d_out
  if (e == cudaSuccess) e = gemm_f32(h, dyb, b.w2t, T, d, d, b.zeros, b.dg, st);
  if (e == cudaSuccess) e = hstu::launch_transpose_bf16(dyb, false, T, d, d, b.dyt, T64, st);
  if (e == cudaSuccess) e = hstu::launch_colsum(d_out, io32, T, d, gr->b2, h->num_sms, st);
  // the gate and the LayerNorm
  if (e == cudaSuccess)
    e = hstu::launch_ln_gate_bwd(b.dg, uvqk, av, w->ln_gamma, w->ln_beta, T, d, c.ln_eps, b.du,
                                 b.dO, b.g, gr->ln_gamma, gr->ln_beta, h->num_sms, st);
  // the attention step (its schedule, then the backward kernel)
  if (e == cudaSuccess) e = hstu::launch_schedule(h, T, offsets, B, ts, mode, ncand, st);
  if (e == cudaSuccess) {
    const hstu::AttnBwdArgs a = bwd_args(h, uvqk, b.dO, T, offsets, B, ts, w->rab_pos,
                                         w->rab_time, b.dq, b.dk, b.dv, gr->rab_pos, gr->rab_time);
    e = hstu::launch_attention_bwd_tc(a, st);
  }
  // SiLU: H1 recomputed, dH1 = dZ (.) SiLU'(H1), b1 gradient
  if (e == cudaSuccess) e = gemm_f32(h, xb, w->w1, T, 4 * d, d, w->b1, b.h1, st);
  if (e == cudaSuccess)
    e = hstu::launch_silu_bwd(b.du, b.dv, b.dq, b.dk, b.h1, T, d, b.dh1, gr->b1, h->num_sms, st);
  // dX = dH1 W1 + dY
  if (e == cudaSuccess) {
    hstu::GemmArgs g;
    g.a = b.dh1;
    g.b = b.w1t;
    g.M = T;
    g.N = d;
    g.K = 4 * d;
    g.epi = hstu::Epi::kBiasResidual;
    g.bias = b.zeros;
    g.out = d_values;
    g.residual = d_out;
    g.io_fp32 = io32 ? 1 : 0;
    g.out_bf16 = nullptr;
    e = hstu::launch_gemm_tc(g, h->num_sms, st, h->ws.error);
  }
  // weight gradients over the tokens: dW1 = dH1^T X, dW2 = dY^T G, b2
  if (e == cudaSuccess) e = hstu::launch_transpose_bf16(b.dh1, false, T, 4 * d, 4 * d, b.dh1t, T64, st);
  if (e == cudaSuccess) e = hstu::launch_transpose_bf16(xb, false, T, d, d, b.xt, T64, st);
  if (e == cudaSuccess) e = hstu::launch_transpose_bf16(b.g, false, T, d, d, b.gt, T64, st);
  if (e == cudaSuccess) e = gemm_f32(h, b.dh1t, b.xt, 4 * d, d, int(T64), b.zeros, gr->w1, st);
  if (e == cudaSuccess) e = gemm_f32(h, b.dyt, b.gt, d, d, int(T64), b.zeros, gr->w2, st);
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}
