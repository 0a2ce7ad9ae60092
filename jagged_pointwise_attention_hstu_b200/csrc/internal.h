// Internal declarations shared by the C-ABI implementation and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/hstu.h"

namespace hstu {

constexpr int kTile = 128;            // query / key rows per attention tile, GEMM BM
constexpr int64_t kMaxTimestamp = int64_t(1) << 62;
// Largest max_tokens a handle accepts: the attention kernels index rows with
// 32-bit integers and round query tiles up past T, so T stays well below 2^31.
constexpr int64_t kMaxTokensLimit = int64_t(1) << 30;

// Per-token facts the attention kernels need, built by the scheduler.
//   lo: first row of the token's user; hi: one past the last key the token may
//   aggregate besides itself (i + 1 for history rows, n_h start for candidates);
//   pos: the position anchor (i for history rows, the user's history end for
//   candidates), so the position bucket of key j is clamp(pos - j, 0, clamp).
struct RowInfo {
  int32_t lo, hi, pos, user;
};

// Key tiles visited by the pair of query tiles (2p, 2p+1): the run
// [a_lo, a_lo + n_a) of tiles before query tile 2p, then the diagonal tiles
// 2p and, when it exists, 2p+1.  Every key visible to a row of either query
// tile lies in these tiles: a query tile's earlier keys belong to the user of
// its first row (users starting inside the tile see only the tile itself),
// and a candidate sees only its history and itself.
struct PairTiles {
  int a_lo, n_a, n_diag;
};

__device__ __forceinline__ void range_before(const RowInfo* rows, int64_t r, int& a, int& e) {
  const RowInfo ri = rows[r];
  int64_t lo = ri.lo;
  if (lo < 0 || lo > r) lo = r;
  int64_t ve = ri.hi < r ? int64_t(ri.hi) : r;
  if (ve < lo) ve = lo;
  a = int(lo / kTile);
  e = int((ve + kTile - 1) / kTile);
}

__device__ __forceinline__ PairTiles pair_tiles(const RowInfo* rows, int64_t T, int pr) {
  const int qt0 = 2 * pr;
  const int64_t r0 = int64_t(qt0) * kTile;
  const int64_t r1 = r0 + kTile;
  int a0, e0;
  range_before(rows, r0, a0, e0);
  PairTiles t;
  t.n_diag = 1;
  int a_lo = a0, a_hi = e0;
  if (r1 < T) {
    int a1, e1;
    range_before(rows, r1, a1, e1);
    a_lo = a1 < a0 ? a1 : a0;
    a_hi = e1 > e0 ? e1 : e0;
    t.n_diag = 2;
  }
  if (a_hi > qt0) a_hi = qt0;
  if (a_hi < a_lo) a_hi = a_lo;
  t.a_lo = a_lo;
  t.n_a = a_hi - a_lo;
  return t;
}

struct Workspace {
  void* xb = nullptr;          // [T, d] bf16: X cast for the GEMM when io is fp32
  void* uvqk = nullptr;        // [T, 4d] compute dtype
  float* av = nullptr;         // [T, d] fp32
  void* g = nullptr;           // [T, d] compute dtype
  RowInfo* rows = nullptr;     // [T]
  int32_t* qtile_order = nullptr;  // [ceil(T / 256)] q-tile pairs by descending cost
  int32_t* qtile_cost = nullptr;   // [ceil(T / 256)]
  int32_t* ktile_order = nullptr;  // [ceil(T / 128)] key tiles of the backward, longest first
  int32_t* ktile_cost = nullptr;   // [ceil(T / 128)]
  int32_t* counters = nullptr;     // [4]: n_norm, max cost, scratch
  int32_t* error = nullptr;        // device error word
  int64_t* thresholds = nullptr;   // [time_buckets] time-bucket thresholds
  uint8_t* time_lut = nullptr;     // [128] bucket at the low edge of each log2 quarter-octave bin
  int32_t* thr32 = nullptr;        // [257] thresholds capped to int32, padded with INT32_MAX
};

}  // namespace hstu

namespace hstu {
// CUDA-event pairs around every kernel launch of a handle (off by default).
struct KernelTimer {
  static constexpr int kMax = 4096;
  bool enabled = false;
  int count = 0;
  int kind[kMax];
  cudaEvent_t ev[2 * kMax];
  bool created = false;
};
}  // namespace hstu

namespace hstu {
// Buffers of the layer backward, allocated on its first call (sized by the
// handle's max_tokens).
struct BwdWorkspace {
  void* xb = nullptr;       // [T, d] bf16: X for the products
  void* dyb = nullptr;      // [T, d] bf16: dY for the products
  void* w1t = nullptr;      // [d, 4d] bf16: W1^T
  void* w2t = nullptr;      // [d, d] bf16: W2^T
  float* dg = nullptr;      // [T, d]
  float* du = nullptr;      // [T, d]
  void* dO = nullptr;       // [T, d] bf16
  void* g = nullptr;        // [T, d] bf16: N (.) U
  float* dq = nullptr;      // [T, d]
  float* dk = nullptr;      // [T, d]
  float* dv = nullptr;      // [T, d]
  float* h1 = nullptr;      // [T, 4d]: X W1^T + b1
  void* dh1 = nullptr;      // [T, 4d] bf16
  void* dh1t = nullptr;     // [4d, T64] bf16
  void* xt = nullptr;       // [d, T64] bf16
  void* dyt = nullptr;      // [d, T64] bf16
  void* gt = nullptr;       // [d, T64] bf16
  float* zeros = nullptr;   // [4d]
  bool ready = false;
};
}  // namespace hstu

struct hstu_handle_s {
  hstu_config cfg;
  hstu::BwdWorkspace bwd;
  hstu::KernelTimer timer;
  int device = 0;
  int num_sms = 148;
  hstu::Workspace ws;
  int64_t last_T = 0;
  int64_t wait_limit = 0;     // pipeline wait bound of the tensor-core kernels (0: default)
  int64_t thresholds_host[256];
  uint8_t time_lut_host[128];
  int32_t thr32_host[257];
};

namespace hstu {

// sched.cu
cudaError_t launch_schedule(const hstu_handle_s* h, int64_t T, const int32_t* offsets, int32_t B,
                            const int64_t* ts, int mask_mode, const int32_t* ncand,
                            cudaStream_t st);
// The same schedule into caller-given scratch; counters[0..3] must already be zero.
cudaError_t launch_schedule_raw(int64_t T, const int32_t* offsets, int32_t B, const int64_t* ts,
                                int mask_mode, const int32_t* ncand, RowInfo* rows, int32_t* cost,
                                int32_t* order, int32_t* counters, int32_t* err, cudaStream_t st);
cudaError_t launch_cast_bf16(const float* x, void* xb, int64_t n, cudaStream_t st);

// serve.cu: the candidate block of a history-cache call.  table = blk[0..B]
// (padded block starts, relative to the block, multiples of 2 * kTile) followed
// by coff[0..B] (packed candidate offsets); hoff[0..B]: history offsets.
constexpr int32_t kMaxCandidatePairs = 8192;
// Row facts and timestamps of the block rows, and the packed candidate rows
// [T_c, row_bytes] moved into the block [P, row_bytes] (padding rows zeroed).
cudaError_t launch_candidate_block(const int32_t* table, const int32_t* hoff, int32_t B,
                                   int64_t T_h, int64_t q0, int32_t P, const int64_t* cand_ts,
                                   int64_t* ts, RowInfo* rows, int64_t row_bytes, const void* src,
                                   void* dst, cudaStream_t st);
// Block rows back to packed order (padding dropped); to_block must be false.
cudaError_t launch_candidate_copy(const int32_t* table, int32_t B, int32_t P, int64_t row_bytes,
                                  const void* src, void* dst, bool to_block, cudaStream_t st);

// sl.cu: Stochastic Length over a jagged batch
constexpr int32_t kSlMaxLen = HSTU_SL_MAX_SAMPLED_LEN;   // longest sequence that is sub-sampled
struct SlArgs {
  const int32_t* offs;        // [B + 1]
  int32_t B;
  int64_t T;
  const double* u;            // [B]
  const uint32_t* keys;       // [T]
  int32_t n_c;
  double numerator;           // n_c^alpha
  const void* values;         // [T, row_bytes] or null
  int64_t row_bytes;
  const int64_t* ts;          // [T] or null
  int32_t* out_offs;          // [B + 1]
  int64_t* out_index;         // [T]
  void* out_values;           // [T, row_bytes] or null
  int64_t* out_ts;            // [T] or null
  uint8_t* flags;             // scratch [T]
  int32_t* kept;              // scratch [B]
  int32_t* err;               // scratch word, cleared first
};
cudaError_t launch_stochastic_length(const SlArgs& a, int num_sms, cudaStream_t st);

// gemm_tc.cu
enum class Epi { kSiluSplit = 0, kBiasResidual = 1 };
struct GemmArgs {
  const void* a;        // [M, K] bf16
  const void* b;        // [N, K] bf16
  int64_t M;
  int N, K;
  Epi epi;
  const float* bias;    // [N]
  // kSiluSplit: out bf16 [M, N]
  // kBiasResidual: out = acc + bias + residual (io dtype), residual may alias out
  void* out;
  const void* residual;
  int io_fp32;
  // kBiasResidual with fp32 out only: when set, bf16(out) is written here too
  // (the next layer's f1 operand), rounded to nearest even
  void* out_bf16;
  // bound of the pipeline waits in SM cycles (0: the default, about a second)
  int64_t wait_limit = 0;
};
cudaError_t launch_gemm_tc(const GemmArgs& a, int num_sms, cudaStream_t st, int32_t* error);

// attn_tc.cu
struct AttnArgs {
  const void* uvqk;          // [T, 4d] bf16
  float* av;                 // [T, d] fp32
  const RowInfo* rows;
  const int32_t* order;      // q-tile pair order
  const int64_t* ts;
  const int64_t* thresholds; // [time_buckets]
  const uint8_t* time_lut;   // [128]
  const int32_t* thr32;      // [257]
  const float* rab_pos;
  const float* rab_time;
  const int32_t* counters;   // [0] = n_norm
  int32_t* error;
  int64_t T;
  int d, H, hd;
  int pos_clamp, time_buckets;
  int n_norm_fixed;          // > 0: use it; else counters[0]
  int num_pairs;             // ceil(T / 256)
  int lut_exact;             // time_log_div > ln 1.25: the candidate-bucket table is exact
  int64_t wait_limit;        // bound of the pipeline waits in SM cycles (0: the default)
  int64_t q_row0;            // first row of the listed pairs (rows [q_row0, T) are written)
  // recording variant
  int32_t* dump_pidx;
  int32_t* dump_tidx;
  uint8_t* dump_vis;
};
cudaError_t launch_attention_tc(const AttnArgs& a, cudaStream_t st, bool record);

// attn_bwd_tc.cu: backward of the attention step
struct AttnBwdArgs {
  const void* uvqk;          // [T, 4d] bf16 (the forward's U | V | Q | K)
  const void* dO;            // [T, d] bf16: gradient of the attention output O
  const RowInfo* rows;       // the forward's row facts (the schedule)
  const int32_t* order;      // query-tile pairs, longest first (the schedule)
  int32_t* key_cost;         // [ceil(T / 128)] scratch: query tiles per key tile
  int32_t* key_order;        // [ceil(T / 128)] scratch: key tiles, longest first
  const int32_t* offsets;    // [B + 1]
  int32_t B;
  const int64_t* ts;
  const int64_t* thresholds; // [time_buckets]
  const uint8_t* time_lut;   // [128]
  const int32_t* thr32;      // [257]
  const float* rab_pos;
  const float* rab_time;
  const int32_t* counters;   // [0] = n_norm when not fixed
  int32_t* error;
  float* dq;                 // [T, d] fp32 (written)
  float* dk;                 // [T, d] fp32 (written)
  float* dv;                 // [T, d] fp32 (written)
  float* d_rab_pos;          // [pos_buckets] fp32, zeroed by the caller (accumulated)
  float* d_rab_time;         // [time_buckets] fp32, zeroed by the caller (accumulated)
  int64_t T;
  int d, H, hd;
  int pos_clamp, time_buckets, n_norm_fixed;
  int lut_exact;             // time_log_div > ln 1.25: the bin table of the buckets is exact
  int64_t wait_limit;        // bound of the pipeline waits in SM cycles (0: the default)
};
cudaError_t launch_attention_bwd_tc(const AttnBwdArgs& a, cudaStream_t st);

// bwd_aux.cu: memory-bound steps of the layer backward
cudaError_t launch_ln_gate_bwd(const float* dG, const void* uvqk, const float* av,
                               const float* gamma, const float* beta, int64_t T, int d, float eps,
                               float* dU, void* dO, void* G, float* dgamma, float* dbeta,
                               int num_sms, cudaStream_t st);
cudaError_t launch_silu_bwd(const float* dU, const float* dV, const float* dQ, const float* dK,
                            const float* H1, int64_t T, int d, void* dH1, float* db1, int num_sms,
                            cudaStream_t st);
cudaError_t launch_colsum(const void* src, bool fp32, int64_t T, int n, float* out, int num_sms,
                          cudaStream_t st);
cudaError_t launch_transpose_bf16(const void* src, bool fp32, int64_t R, int C, int64_t lds,
                                  void* dst, int64_t ldd, cudaStream_t st);

// ln_gate.cu
cudaError_t launch_ln_gate(const float* av, const void* uvqk, void* g, const float* gamma,
                           const float* beta, int64_t T, int d, float eps, int compute_fp32,
                           cudaStream_t st);

// simt_fp32.cu
cudaError_t launch_gemm_f32(const float* a, const float* b, int64_t M, int N, int K, Epi epi,
                            const float* bias, float* out, const float* residual,
                            cudaStream_t st);
cudaError_t launch_attention_f32(const AttnArgs& a, cudaStream_t st);

// umma_check.cu
cudaError_t run_umma_tile(int mode, const void* a, const void* b, float* c, int n, int k);

// Raises a kernel's dynamic shared memory limit to `bytes` on the current
// device, once per device: the attribute lives in each device's context, so a
// process that launches on several GPUs must set it on every one of them.
// `done` holds one bit per device below 64 (devices above are set every call);
// two threads racing on the first call both set it, which is harmless.
template <typename Kernel>
cudaError_t smem_opt_in(Kernel* kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev >= 0 && dev < 64) ? uint64_t(1) << dev : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
  return e;
}

// tensor maps (hstu_api.cu)
bool make_tmap_2d_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer);
// fp32 [outer, inner] row-major, 128-byte swizzle (box_inner * 4 <= 128).
bool make_tmap_2d_f32_sw128(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                            uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer);
// bf16 [outer, inner] row-major, 64-byte swizzle (box_inner * 2 <= 64).
bool make_tmap_2d_bf16_sw64(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                            uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer);
bool make_tmap_1d_i64(CUtensorMap* m, const void* base, uint64_t n, uint32_t box);

}  // namespace hstu
