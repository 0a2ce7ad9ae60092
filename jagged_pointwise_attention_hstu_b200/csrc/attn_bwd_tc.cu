// Backward of the fused jagged pointwise attention on the tcgen05 tensor cores.
//
// For equation (2) of the HSTU layer (blog "Generative Recommendation 16:
// HSTU", section "HSTU Layer 到底改了什么"), with s = q.k + rab and
// a = vis * SiLU(s) / n_norm, O = a V, the gradients of sum(dO * O) are
//     dV = a^T dO,  dA = dO V^T,  dS = vis * dA * SiLU'(s) / n_norm,
//     dQ = dS K,    dK = dS^T Q,
// with SiLU'(s) = sig(s) (1 + s (1 - sig(s))), and every entry of rab_pos /
// rab_time collects dS of each visible (query, key, head) that reads it.  SiLU
// acts on each score alone (same blog, section "不对序列做 softmax"): there are
// no row statistics to keep from the forward, so S is recomputed tile by tile.
//
// Two kernels, each owning its outputs, so no gradient is accumulated with
// atomics across CTAs:
//
//   dq kernel   one CTA per (128-query tile, head), the query tiles in the
//               forward's longest-first order.  Per visible key tile j:
//                 S = Q K_j^T and dA = dO V_j^T (SS MMAs into tensor memory),
//                 dS from S and dA (two row groups, one half of the keys each,
//                 dS written as bf16 over the consumed S columns),
//                 dQ += dS K_j (TS MMA: dS read from tensor memory).
//               The row groups also sum dS into the bias-table gradients
//               (shared-memory accumulators, one global add per entry per CTA).
//   dkv kernel  one CTA per (128-key tile, head), longest first.  Per query
//               tile i that can see the keys (the key tile's own tile up to the
//               end of the user owning its last row):
//                 S^T = K Q_i^T and dA^T = V dO_i^T (keys along the tensor-memory
//                 lanes), P^T and dS^T from them (bf16 over the consumed columns),
//                 dV += P^T dO_i and dK += dS^T Q_i (TS MMAs).
//
// Both: 12 warps.  Warp 0 issues the TMA loads (no multicast), warp 1 the MMAs
// (one elected thread), warps 4-7 and 8-11 are two row groups; group g scores
// columns [64 g, 64 g + 64) of every 128 x 128 tile, one tensor-memory lane
// (row) per thread.  Tensor memory: S [0, 128), dA [128, 256), then the
// accumulators (dQ, or dK and dV).  Every wait is bounded; a CTA that gives up
// sets HSTU_DEVERR_TIMEOUT, drains its own copies and MMAs and frees its
// tensor memory.
//
// Per (warp, half tile) the rows are classified: when every pair is visible,
// every position bucket is the clamped one and each row meets one time bucket
// (the common case far from the diagonal), the bias is a per-row constant and
// the bias gradients are per-row sums; otherwise every pair takes the mask,
// the position bucket and the exact time bucket.  Position-bucket gradients of
// rows at their own positions are summed along the tile diagonals in three
// register slots per lane over a half tile; rows at one position (M-FALCON
// candidates) sum the columns with a 16-shuffle butterfly.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "sm100.cuh"

namespace hstu {
namespace {

using namespace sm100;

constexpr int kBwdThreads = 384;
constexpr int kBwdMaxPos = 4097;       // pos_clamp <= 4096
constexpr int kBwdMaxBuckets = 256;

struct BwdParams {
  const RowInfo* rows;
  const int32_t* order;        // query-tile pairs, longest first (the forward's schedule)
  const int32_t* key_order;    // key tiles, longest first
  const int32_t* offsets;
  int32_t B;
  const int64_t* ts;
  const int64_t* thresholds;
  const uint8_t* time_lut;
  const int32_t* thr32;
  const float* rab_pos;
  const float* rab_time;
  const int32_t* counters;
  int32_t* error;
  float* d_rab_pos;
  float* d_rab_time;
  int64_t T;
  int d, H, num_pairs, num_key_tiles;
  int pos_clamp, time_buckets, n_norm_fixed, lut_exact;
  int rp_smem;                 // the padded rab_pos copy is in shared memory
  long long wait_limit;
};

// The shared copy of rab_pos is padded on both sides with its end values, so a
// relative position in [-kPosPad, clamp + kPosPad] reads its clamped entry.
constexpr int kPosPad = 130;
__host__ __device__ constexpr uint32_t rp_bytes(int clamp) {
  return ((uint32_t(clamp + 1 + 2 * kPosPad) * 4 + 15) / 16) * 16;
}

// ---------------------------------------------------------------- shared helpers

// Largest k with thr[k] <= dt (thr[0] = 0, non-decreasing): the time bucket.
__device__ __forceinline__ int bucket_search(const int64_t* thr, int nb, int64_t dt) {
  if (dt <= 0) return 0;
  int lo = 0, hi = nb - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (thr[mid] <= dt) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Time bias and bucket of a 32-bit gap through the bin table (the table is
// exact for the divisor and the gap is below 2^31 - 1); a masked pair may hold
// any 32-bit pattern, and its index stays inside the table.
__device__ __forceinline__ float time_bias_lut(uint32_t dd, const int4* s_any, int& tb) {
  const uint32_t v = max(dd + 1u, 1u);
  const uint32_t fb = __float_as_uint(__uint2float_rz(v));
  const int4 e = s_any[int((fb >> 21) - 508u) & 127];
  const bool up = int(dd) >= e.x;
  tb = e.w + (up ? 1 : 0);
  return __int_as_float(up ? e.z : e.y);
}

// The padded rab_pos copy, written by the 256 row-group threads.
__device__ __forceinline__ void load_rp(const BwdParams& p, int t, float* s_rp) {
  const int n = p.pos_clamp + 1 + 2 * kPosPad;
  for (int k = t; k < n; k += 256) {
    const int q = k - kPosPad;
    s_rp[k] = __ldg(p.rab_pos + (q < 0 ? 0 : (q > p.pos_clamp ? p.pos_clamp : q)));
  }
}

// The per-CTA tables, written by the 256 row-group threads (t = 0..255).
__device__ __forceinline__ void load_tables(const BwdParams& p, int t, int64_t* s_thr, float* s_rt,
                                            int4* s_any) {
  const int nb = p.time_buckets;
  s_thr[t] = t < nb ? __ldg(p.thresholds + t) : (int64_t(1) << 62);
  s_rt[t] = t < nb ? __ldg(p.rab_time + t) : 0.0f;
  if (t < 128) {
    const int cand = __ldg(p.time_lut + t);
    const int nxt = cand + 1 < nb ? cand + 1 : cand;
    s_any[t] = make_int4(cand + 1 < nb ? __ldg(p.thr32 + cand + 1) : 0x7FFFFFFF,
                         __float_as_int(__ldg(p.rab_time + cand)),
                         __float_as_int(__ldg(p.rab_time + nxt)), cand);
  }
}

// sig(s) / n_norm (pre-scaled) and the two results of one pair.
struct Grad {
  float p;    // SiLU(s) / n_norm
  float ds;   // dA SiLU'(s) / n_norm
};
__device__ __forceinline__ Grad silu_grad(float s, float da, float inv_nn) {
  const float sig = fmaf(0.5f, tanh_approx(0.5f * s), 0.5f);
  const float sn = sig * inv_nn;
  const float w = fmaf(s, 1.0f - sig, 1.0f);
  Grad g;
  g.p = s * sn;
  g.ds = da * (sn * w);
  return g;
}

// Tensor-memory column of the bf16 operand (P or dS) for K-step kk of a TS MMA:
// group g writes its keys' packed pairs over the first half of its own 64
// score columns.
__device__ __forceinline__ uint32_t a_col(int kk) { return kk < 4 ? 8 * kk : 64 + 8 * (kk - 4); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Adds each lane's v (where pred holds and v != 0) to table[b], b per lane,
// with one shared add per distinct bucket: the lanes of a bucket are summed
// with shuffles first.  Shared-memory float adds from many lanes to one word
// are serialised by the hardware, and neighbouring rows mostly share a time
// bucket.  Every lane of the warp must call it.
__device__ __forceinline__ void warp_bucket_add(float* table, int b, float v, bool pred, int lane) {
  unsigned todo = __ballot_sync(0xffffffffu, pred && v != 0.0f);
  while (todo != 0u) {
    const int leader = __ffs(todo) - 1;
    const int bl = __shfl_sync(0xffffffffu, b, leader);
    const bool mine = ((todo >> lane) & 1u) != 0u && b == bl;
    const float s = warp_sum(mine ? v : 0.0f);
    if (lane == leader) red_add_shared(table + bl, s);
    todo &= ~__ballot_sync(0xffffffffu, mine);
  }
}

// Stages 32 rows x 32 fp32 columns of tensor memory (this warp's lanes) into a
// 128-byte-swizzled 4 KB box and writes it with a TMA store at (x, y).
__device__ __forceinline__ void store_box(uint32_t taddr, uint8_t* box, const CUtensorMap* m,
                                          int32_t x, int32_t y, int lane) {
  uint32_t r[32];
  tmem_ld32(taddr, r);
  tmem_ld_wait();
  const uint32_t row_addr = smem_u32(box + lane * 128);
#pragma unroll
  for (int e = 0; e < 8; ++e)
    st_shared_v4(row_addr + ((e ^ (lane & 7)) << 4), __uint_as_float(r[4 * e + 0]),
                 __uint_as_float(r[4 * e + 1]), __uint_as_float(r[4 * e + 2]),
                 __uint_as_float(r[4 * e + 3]));
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(m, box, x, y);
    bulk_commit_group();
    bulk_wait_group_read0();
  }
  __syncwarp();
}

// Adds v to the position-bucket gradient of relative position p (clamped); the
// clamped bucket's share goes to the row's register sum instead.
__device__ __forceinline__ void add_pos_grad(float* s_gpos, int p, int clamp, float v, float& acc_c) {
  const int b = p < 0 ? 0 : (p > clamp ? clamp : p);
  if (b == clamp) acc_c += v;
  else if (v != 0.0f) red_add_shared(s_gpos + b, v);
}

// Column sums of a warp's 32 x 16 chunk: after the butterfly, lane l (l even)
// holds the sum over all 32 lanes of column (l >> 1) & 15 (16 shuffles
// instead of one 5-step reduction per column).
__device__ __forceinline__ float column_sums16(const float (&v)[16], int lane) {
  float a[8], b[4], c[2];
  const bool h4 = lane & 16, h3 = lane & 8, h2 = lane & 4, h1 = lane & 2;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float send = h4 ? v[k] : v[k + 8];
    a[k] = (h4 ? v[k + 8] : v[k]) + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float send = h3 ? a[k] : a[k + 4];
    b[k] = (h3 ? a[k + 4] : a[k]) + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const float send = h2 ? b[k] : b[k + 2];
    c[k] = (h2 ? b[k + 2] : b[k]) + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  const float send = h1 ? c[0] : c[1];
  float s = (h1 ? c[1] : c[0]) + __shfl_xor_sync(0xffffffffu, send, 2);
  return s + __shfl_xor_sync(0xffffffffu, s, 1);
}

// ================================================================ dq kernel

// The time-bucket gradient is kept in kGCopies interleaved copies per CTA
// (entry b, copy c at b * kGCopies + c): the generic path's per-key flushes of
// lane l go to copy l mod kGCopies, so neighbouring rows that flush the same
// bucket at the same key add to different words (shared float adds to one
// word serialise); the copies are summed once at the end.
constexpr int kGCopies = 8;

template <int HD>
struct DqLayout {
  static constexpr int NS = HD == 128 ? 2 : 3;    // K / V ring stages
  static constexpr uint32_t kTile = 128 * HD * 2;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kDO = kTile;
  static constexpr uint32_t kK = 2 * kTile;
  static constexpr uint32_t kV = kK + NS * kTile;
  static constexpr uint32_t kKts = kV + NS * kTile;         // int64 [NS][128]
  static constexpr uint32_t kThr = kKts + NS * 1024;        // int64 [256]
  static constexpr uint32_t kRt = kThr + 2048;              // float [256]
  static constexpr uint32_t kGtime = kRt + 1024;            // float [256][kGCopies]
  static constexpr uint32_t kAny = kGtime + 1024 * kGCopies;   // int4 [128]
  static constexpr uint32_t kBars = kAny + 2048;
  static constexpr uint32_t kGpos = kBars + 256;            // float [clamp + 1], then the rab_pos copy
  static __host__ __device__ constexpr uint32_t rp_offset(int clamp) {
    return kGpos + ((uint32_t(clamp + 1) * 4 + 15) / 16) * 16;
  }
  static __host__ __device__ constexpr uint32_t smem_bytes(int clamp, bool rp) {
    return rp_offset(clamp) + (rp ? rp_bytes(clamp) : 0) + 1024;
  }
  static_assert(kK % 1024 == 0 && kV % 1024 == 0 && kTile % 1024 == 0, "tile alignment");
  static_assert(kKts % 128 == 0 && kBars % 8 == 0 && kAny % 16 == 0, "alignment");
  // dQ is staged in the Q and dO tiles: 8 warps x HD / 64 boxes of 4 KB
  static_assert(8 * (HD / 64) * 4096 == 2 * kTile, "dQ staging");
  static_assert(smem_bytes(kBwdMaxPos - 1, false) <= 227 * 1024, "shared memory budget");
};

template <int HD>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_ts,
                       const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  using L = DqLayout<HD>;
  constexpr int NS = L::NS;
  // ---- work item: one query tile of the pair order, one head
  const int per_head = 2 * p.num_pairs;
  const int h = blockIdx.x / per_head;
  const int rr = blockIdx.x % per_head;
  const int qt = 2 * p.order[rr >> 1] + (rr & 1);
  const int64_t r0 = int64_t(qt) * 128;
  if (r0 >= p.T) return;   // the missing second tile of the last pair (uniform over the CTA)
  int a0, e0;
  range_before(p.rows, r0, a0, e0);
  const int a_hi = e0 < qt ? (e0 > a0 ? e0 : a0) : qt;
  const int n_a = a_hi - a0;
  const int n_kt = n_a + 1;
  auto key_tile = [&](int j) -> int { return j < n_a ? a0 + j : qt; };

  extern __shared__ uint8_t smem_raw[];
  // aligned up to 1024 bytes by pointer arithmetic on the shared array, so that
  // the compiler keeps every access derived from it in the shared state space
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  int64_t* s_kts = reinterpret_cast<int64_t*>(smem + L::kKts);
  int64_t* s_thr = reinterpret_cast<int64_t*>(smem + L::kThr);
  float* s_rt = reinterpret_cast<float*>(smem + L::kRt);
  float* s_gtime = reinterpret_cast<float*>(smem + L::kGtime);
  int4* s_any = reinterpret_cast<int4*>(smem + L::kAny);
  float* s_gpos = reinterpret_cast<float*>(smem + L::kGpos);
  float* s_rp = reinterpret_cast<float*>(smem + L::rp_offset(p.pos_clamp));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* q_full = bars;
  uint64_t* kv_full = q_full + 1;      // [NS]
  uint64_t* kv_empty = kv_full + NS;   // [NS]
  uint64_t* s_full = kv_empty + NS;    // S and dA of the current key tile are in tensor memory
  uint64_t* ds_full = s_full + 1;      // dS written (256 arrivals)
  uint64_t* dq_done = ds_full + 1;     // every product is done
  uint64_t* drained = dq_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int d = p.d;
  const int clamp = p.pos_clamp;
  const int nb = p.time_buckets;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(ds_full, 256);
    mbar_init(dq_done, 1);
    mbar_init(drained, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp >= 4) {
    const int t = threadIdx.x - 128;
    load_tables(p, t, s_thr, s_rt, s_any);
    if (p.rp_smem) load_rp(p, t, s_rp);
    for (int k = t; k < 256 * kGCopies; k += 256) s_gtime[k] = 0.0f;
    for (int k = t; k <= clamp; k += 256) s_gpos[k] = 0.0f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tS = tmem_base;
  const uint32_t tdA = tmem_base + 128;
  const uint32_t tDQ = tmem_base + 256;

  if (warp == 0) {
    // ------------------------------------------------------------ loads
    if (lane == 0) {
      prefetch_tmap(&tm);
      prefetch_tmap(&tm_do);
      prefetch_tmap(&tm_ts);
      mbar_arrive_expect_tx(q_full, 2 * L::kTile);
#pragma unroll
      for (int b = 0; b < HD / 64; ++b) {
        tma_load_2d(smem + L::kQ + b * 16384, &tm, q_full, 2 * d + h * HD + b * 64, int32_t(r0));
        tma_load_2d(smem + L::kDO + b * 16384, &tm_do, q_full, h * HD + b * 64, int32_t(r0));
      }
      bool issued[NS];
      uint32_t issued_ph[NS];
      for (int s = 0; s < NS; ++s) issued[s] = false, issued_ph[s] = 0;
      for (int j = 0; j < n_kt && !*abort_flag; ++j) {
        const int s = j % NS;
        const uint32_t ph = (j / NS) & 1;
        if (!mbar_wait(&kv_empty[s], ph ^ 1, p.wait_limit)) { *abort_flag = 1; break; }
        const int32_t kb = key_tile(j) * 128;
        mbar_arrive_expect_tx(&kv_full[s], 2 * L::kTile + 1024);
#pragma unroll
        for (int b = 0; b < HD / 64; ++b) {
          tma_load_2d(smem + L::kK + s * L::kTile + b * 16384, &tm, &kv_full[s],
                      3 * d + h * HD + b * 64, kb);
          tma_load_2d(smem + L::kV + s * L::kTile + b * 16384, &tm, &kv_full[s],
                      d + h * HD + b * 64, kb);
        }
        tma_load_1d(s_kts + s * 128, &tm_ts, &kv_full[s], kb);
        issued[s] = true;
        issued_ph[s] = ph;
      }
      // no copy may still be in flight when the CTA ends
      mbar_wait(q_full, 0);
      for (int s = 0; s < NS; ++s)
        if (issued[s]) mbar_wait(&kv_full[s], issued_ph[s]);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_ss = idesc_bf16(128, 128, false, false);   // S, dA
      constexpr uint32_t idesc_dq = idesc_bf16(128, HD, false, true);     // dQ
      const uint32_t sQ = smem_u32(smem + L::kQ), sDO = smem_u32(smem + L::kDO);
      bool ok = mbar_wait(q_full, 0, p.wait_limit);
      for (int j = 0; ok && j < n_kt; ++j) {
        const int s = j % NS;
        if (!mbar_wait(&kv_full[s], (j / NS) & 1, p.wait_limit)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sK = smem_u32(smem + L::kK + s * L::kTile);
        const uint32_t sV = smem_u32(smem + L::kV + s * L::kTile);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tS, desc_sw128(sQ + off, 16, 1024), desc_sw128(sK + off, 16, 1024), idesc_ss,
                  kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tdA, desc_sw128(sDO + off, 16, 1024), desc_sw128(sV + off, 16, 1024), idesc_ss,
                  kk > 0);
        }
        umma_commit(s_full);
        if (!mbar_wait(ds_full, j & 1, p.wait_limit)) { ok = false; break; }
        tc_fence_after();
        // dQ += dS K_j: K = the 128 keys in 8 steps of 16, K_j consumed N-major
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tDQ, tS + a_col(kk), desc_sw128(sK + kk * 2048, 16384, 1024), idesc_dq,
                  (j > 0 || kk > 0));
        umma_commit(&kv_empty[s]);
      }
      if (!ok) *abort_flag = 1;
      umma_commit(dq_done);      // also releases the read-out after an abort
      umma_commit(drained);
      mbar_wait(drained, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ row groups
    const int g = (warp - 4) >> 2;           // key half of every tile
    const int wq = warp & 3;                 // tensor-memory lane quarter
    const int row = wq * 32 + lane;
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const int i = int(r0) + row;             // token indices fit in int32 (T <= 2^30)
    const bool valid = i < p.T;
    int lo = i, hi = i, pos = i;
    int64_t ti = 0, t_first = 0;
    if (valid) {
      const RowInfo ri = p.rows[i];
      lo = (ri.lo < 0 || ri.lo > i) ? i : ri.lo;
      hi = ri.hi;
      pos = ri.pos;
      ti = p.ts[i];
      t_first = p.ts[lo];
    }
    // every visible key of the row lies in its user at or after ts[lo]: below
    // 2^31 - 1 its gap fits the 32-bit bin-table path
    const bool narrow_row = !valid || ti - t_first < int64_t(0x7FFFFFFE);
    const uint32_t ti_lo = uint32_t(ti);
    const int nn = p.n_norm_fixed > 0 ? p.n_norm_fixed : p.counters[0];
    const float inv_nn = 1.0f / float(nn > 0 ? nn : 1);
    const bool narrow = p.lut_exact != 0 && __all_sync(0xffffffffu, narrow_row);
    const float rp_clamp = __ldg(p.rab_pos + clamp);
    const bool rp_smem = p.rp_smem != 0;
    // position buckets along the tile diagonals: every row of the warp valid and
    // positioned at its own index offset (history rows of one user)
    const int pos0 = __shfl_sync(0xffffffffu, pos, 0);
    const bool diag = __all_sync(0xffffffffu, valid && pos - lane == pos0);
    const bool col = !diag && __all_sync(0xffffffffu, valid && pos == pos0);
    named_bar_sync(1, 256);   // the tables
    bool aborted = false;
    float acc_c = 0.0f;       // the clamped position bucket's sum, added once at the end
    for (int j = 0; j < n_kt; ++j) {
      const int s = j % NS;
      const int kb = key_tile(j) * 128;
      bool ok = aborted ? false : mbar_wait(&kv_full[s], (j / NS) & 1, p.wait_limit);
      ok = ok && mbar_wait(s_full, j & 1, p.wait_limit);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        aborted = true;
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int64_t* kts = s_kts + s * 128;
      const int j0 = kb + 64 * g;   // first key of this group's half
      // ---- classify the row for this half tile
      const bool zero = __all_sync(0xffffffffu, !valid || i < j0);
      const bool full = valid && lo <= j0 && j0 + 63 < hi;
      int tb0 = 0, tb1 = 0;
      bool same = false;
      if (full) {
        tb0 = bucket_search(s_thr, nb, ti - kts[64 * g]);
        tb1 = bucket_search(s_thr, nb, ti - kts[64 * g + 63]);
        same = tb0 == tb1;
      }
      const bool fast = __all_sync(0xffffffffu, full && same && pos - (j0 + 63) >= clamp);
      // every pair visible and at most two time buckets per row: the position bias
      // per pair from the shared table, the time bias switching at one column
      const bool fastp = !fast && rp_smem && (diag || col) &&
                         __all_sync(0xffffffffu, full && tb0 - tb1 <= 1);
      const uint32_t tcol = lane_off + 64 * g;
      if (zero) {
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) pk[e] = 0u;
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_st8(tS + tcol + 8 * c, pk);
      } else if (fastp) {
        // the position bias per pair from the shared table, the time bias a row
        // constant; position gradients along the diagonals or the columns
        const int pos_rel = min(max(pos - kb, -1), clamp + 129);
        // keys from column jm on have a gap below thr[tb0] (bucket tb1): the count
        // of the half's keys with t_j <= t_i - thr[tb0] (sorted inside the user)
        int jm = 64;
        if (tb1 != tb0) {
          const int64_t cut = ti - s_thr[tb0];
          int pcount = 0;
#pragma unroll
          for (int step = 32; step > 0; step >>= 1)
            if (kts[64 * g + pcount + step - 1] <= cut) pcount += step;
          jm = pcount + (kts[64 * g + pcount] <= cut ? 1 : 0);
        }
        jm += 64 * g;
        const float ht0 = s_rt[tb0], ht1 = s_rt[tb1];
        float acc_t = 0.0f, acc_t1 = 0.0f;
        // diagonal sums over the half tile: slot w holds relative position
        // pos0 - (kb + 64 g) + lane - 32 w
        float dg0 = 0.0f, dg1 = 0.0f, dg2 = 0.0f;
        // the next chunk's tensor-memory loads run under this chunk's reductions
        uint32_t rs[16], ra[16];
        tmem_ld16(tS + tcol, rs);
        tmem_ld16(tdA + tcol, ra);
        tmem_ld_wait();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[8];
          const int jr0 = 64 * g + 16 * c;
          float dsv[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const bool lower = jr0 + e >= jm;
            const float rp = s_rp[kPosPad + pos_rel - (jr0 + e)];
            const Grad gr = silu_grad(__uint_as_float(rs[e]) + rp + (lower ? ht1 : ht0),
                                      __uint_as_float(ra[e]), inv_nn);
            dsv[e] = gr.ds;
            if (lower) acc_t1 += gr.ds; else acc_t += gr.ds;
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) pk[e] = pack_bf16x2(dsv[2 * e], dsv[2 * e + 1]);
          tmem_st8(tS + tcol + 8 * c, pk);
          if (c + 1 < 4) {
            tmem_ld16(tS + tcol + 16 * (c + 1), rs);
            tmem_ld16(tdA + tcol + 16 * (c + 1), ra);
          }
          if (diag) {
            // lane l takes pair (row (l + 16 c + e) mod 32, column e) of the chunk:
            // its relative position is pos0 - (kb + 64 g) + l - 32 w, w the wrap count
            // (chunks 0 and 1 wrap from slot 0 into slot 1, chunks 2 and 3 from 1 into 2)
            const int sh = lane + 16 * (c & 1);
            float acc_a = 0.0f, acc_b = 0.0f;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float v = __shfl_sync(0xffffffffu, dsv[e], (sh + e) & 31);
              if (sh + e < 32) acc_a += v; else acc_b += v;
            }
            if (c < 2) {
              dg0 += acc_a;
              dg1 += acc_b;
            } else {
              dg1 += acc_a;
              dg2 += acc_b;
            }
          } else {
            const float v = column_sums16(dsv, lane);
            if ((lane & 1) == 0)
              add_pos_grad(s_gpos, pos0 - (kb + jr0 + ((lane >> 1) & 15)), clamp, v, acc_c);
          }
          tmem_ld_wait();
        }
        if (diag) {
          const int p0 = pos0 - (kb + 64 * g) + lane;
          add_pos_grad(s_gpos, p0, clamp, dg0, acc_c);
          add_pos_grad(s_gpos, p0 - 32, clamp, dg1, acc_c);
          add_pos_grad(s_gpos, p0 - 64, clamp, dg2, acc_c);
        }
        warp_bucket_add(s_gtime, tb0 * kGCopies, acc_t, true, lane);
        warp_bucket_add(s_gtime, tb1 * kGCopies, acc_t1, true, lane);
      } else if (fast) {
        // every pair visible, clamped position, one time bucket per row; the
        // tensor-memory loads of chunk c + 1 overlap the arithmetic of chunk c
        const float hc = rp_clamp + s_rt[tb0];
        float acc = 0.0f;
        uint32_t xs[16], xa[16], ys[16], ya[16];
        tmem_ld16(tS + tcol, xs);
        tmem_ld16(tdA + tcol, xa);
        tmem_ld_wait();
#pragma unroll 1
        for (int c = 0; c < 4; c += 2) {
          tmem_ld16(tS + tcol + 16 * (c + 1), ys);
          tmem_ld16(tdA + tcol + 16 * (c + 1), ya);
          {
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              const Grad g0 = silu_grad(__uint_as_float(xs[e]) + hc, __uint_as_float(xa[e]), inv_nn);
              const Grad g1 = silu_grad(__uint_as_float(xs[e + 1]) + hc, __uint_as_float(xa[e + 1]), inv_nn);
              acc += g0.ds + g1.ds;
              pk[e >> 1] = pack_bf16x2(g0.ds, g1.ds);
            }
            tmem_st8(tS + tcol + 8 * c, pk);
          }
          tmem_ld_wait();
          if (c + 2 < 4) {
            tmem_ld16(tS + tcol + 16 * (c + 2), xs);
            tmem_ld16(tdA + tcol + 16 * (c + 2), xa);
          }
          {
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              const Grad g0 = silu_grad(__uint_as_float(ys[e]) + hc, __uint_as_float(ya[e]), inv_nn);
              const Grad g1 = silu_grad(__uint_as_float(ys[e + 1]) + hc, __uint_as_float(ya[e + 1]), inv_nn);
              acc += g0.ds + g1.ds;
              pk[e >> 1] = pack_bf16x2(g0.ds, g1.ds);
            }
            tmem_st8(tS + tcol + 8 * (c + 1), pk);
          }
          tmem_ld_wait();
        }
        acc_c += acc;   // the position bucket is the clamped one for every pair here
        warp_bucket_add(s_gtime, tb0 * kGCopies, acc, true, lane);
      } else {
        // any visibility: the mask, the position bucket and the exact time bucket
        // of every pair.  The time-bucket gradient is summed along runs of one
        // bucket; the position-bucket gradient along the tile diagonals (rows at
        // their own positions: lane l gathers the pairs of its diagonal from the
        // other lanes) or along the columns (rows at one position: M-FALCON
        // candidates), else per pair.
        const int pos_rel = min(max(pos - kb, -1), clamp + 129);
        int run_b = -1;
        float run_acc = 0.0f;
        float dg0 = 0.0f, dg1 = 0.0f, dg2 = 0.0f;   // diagonal sums, as on the two-bucket path
        uint32_t rs[16], ra[16];
        tmem_ld16(tS + tcol, rs);
        tmem_ld16(tdA + tcol, ra);
        tmem_ld_wait();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[8];
          const int jr0 = 64 * g + 16 * c;
          float dsv[16];
          int tbv[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int jr = jr0 + e;
            const int jj = kb + jr;
            const bool vis = valid && jj < p.T && ((lo <= jj && jj < hi) || jj == i);
            float rt;
            int tb;
            if (narrow) {
              rt = time_bias_lut(ti_lo - uint32_t(kts[jr]), s_any, tb);
            } else {
              int64_t gap = ti - kts[jr];
              tb = bucket_search(s_thr, nb, gap < 0 ? 0 : gap);
              rt = s_rt[tb];
            }
            float rp;
            if (rp_smem) {
              rp = s_rp[kPosPad + pos_rel - jr];
            } else {
              int dp = pos - jj;
              rp = __ldg(p.rab_pos + (dp < 0 ? 0 : (dp > clamp ? clamp : dp)));
            }
            const Grad gr = silu_grad(__uint_as_float(rs[e]) + rp + rt, __uint_as_float(ra[e]), inv_nn);
            dsv[e] = vis ? gr.ds : 0.0f;
            tbv[e] = vis ? tb : -1;
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) pk[e] = pack_bf16x2(dsv[2 * e], dsv[2 * e + 1]);
          tmem_st8(tS + tcol + 8 * c, pk);
          if (c + 1 < 4) {   // the next chunk's loads run under this chunk's reductions
            tmem_ld16(tS + tcol + 16 * (c + 1), rs);
            tmem_ld16(tdA + tcol + 16 * (c + 1), ra);
          }
          // time buckets: runs of one bucket along the row, without branches (a
          // run's sum is added when a visible pair of another bucket starts the next)
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const bool next = tbv[e] >= 0 && tbv[e] != run_b;
            red_add_shared_if(next && run_b >= 0,
                              s_gtime + (run_b < 0 ? 0 : run_b) * kGCopies + (lane & (kGCopies - 1)),
                              run_acc);
            run_acc = next ? dsv[e] : run_acc + dsv[e];
            run_b = next ? tbv[e] : run_b;
          }
          // position buckets
          if (diag) {
            // as on the two-bucket path: lane l takes pair (row (l + 16 c + e) mod 32,
            // column e) of the chunk, summed into slot w of its relative position
            // (chunks 0 and 1 wrap from slot 0 into slot 1, chunks 2 and 3 from 1 into 2)
            const int sh = lane + 16 * (c & 1);
            float acc_a = 0.0f, acc_b = 0.0f;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float v = __shfl_sync(0xffffffffu, dsv[e], (sh + e) & 31);
              if (sh + e < 32) acc_a += v; else acc_b += v;
            }
            if (c < 2) {
              dg0 += acc_a;
              dg1 += acc_b;
            } else {
              dg1 += acc_a;
              dg2 += acc_b;
            }
          } else if (col) {
            // one position per column (M-FALCON candidates): the column sums
            const float v = column_sums16(dsv, lane);
            if ((lane & 1) == 0)
              add_pos_grad(s_gpos, pos0 - (kb + jr0 + ((lane >> 1) & 15)), clamp, v, acc_c);
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              if (dsv[e] == 0.0f) continue;
              const int dp = pos - (kb + jr0 + e);
              const int b = dp < 0 ? 0 : (dp > clamp ? clamp : dp);
              if (b == clamp) acc_c += dsv[e]; else red_add_shared(s_gpos + b, dsv[e]);
            }
          }
          tmem_ld_wait();
        }
        warp_bucket_add(s_gtime, run_b * kGCopies, run_acc, run_b >= 0, lane);
        if (diag) {
          const int p0 = pos0 - (kb + 64 * g) + lane;
          add_pos_grad(s_gpos, p0, clamp, dg0, acc_c);
          add_pos_grad(s_gpos, p0 - 32, clamp, dg1, acc_c);
          add_pos_grad(s_gpos, p0 - 64, clamp, dg2, acc_c);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    {
      const float wsum = warp_sum(acc_c);
      if (lane == 0 && wsum != 0.0f) red_add_shared(s_gpos + clamp, wsum);
    }
    if (aborted) *abort_flag = 1;
    // ---- dQ -> the (now free) Q and dO tiles -> TMA stores; the rows past T are clipped
    bool w = aborted ? false : mbar_wait(dq_done, 0, p.wait_limit);
    w = __all_sync(0xffffffffu, w);
    if (w && !*abort_flag) {
      tc_fence_after();
      uint8_t* stage = smem + L::kQ + (g * 4 + wq) * (HD / 64) * 4096;
#pragma unroll 1
      for (int cb = 0; cb < HD / 64; ++cb) {
        const int col = g * (HD / 2) + cb * 32;
        store_box(tDQ + lane_off + col, stage + cb * 4096, &tm_dq, h * HD + col,
                  int32_t(r0) + wq * 32, lane);
      }
    } else {
      *abort_flag = 1;
    }
    // ---- the bias gradients of the CTA
    named_bar_sync(1, 256);
    const int t = threadIdx.x - 128;
    for (int k = t; k <= clamp; k += 256) {
      const float gv = s_gpos[k];
      if (gv != 0.0f) atomicAdd(p.d_rab_pos + k, gv);
    }
    if (t < nb) {
      float gv = 0.0f;
#pragma unroll
      for (int c = 0; c < kGCopies; ++c) gv += s_gtime[t * kGCopies + c];
      if (gv != 0.0f) atomicAdd(p.d_rab_time + t, gv);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.error, HSTU_DEVERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ================================================================ dkv kernel

template <int HD>
struct DkvLayout {
  static constexpr int NS = HD == 128 ? 2 : 3;    // Q / dO ring stages
  static constexpr uint32_t kTile = 128 * HD * 2;
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kTile;
  static constexpr uint32_t kQ = 2 * kTile;
  static constexpr uint32_t kDO = kQ + NS * kTile;
  static constexpr uint32_t kQf = kDO + NS * kTile;          // RowInfo [NS][128]
  static constexpr uint32_t kQts = kQf + NS * 2048;          // int64 [NS][128]
  static constexpr uint32_t kThr = kQts + NS * 1024;         // int64 [256]
  static constexpr uint32_t kRt = kThr + 2048;               // float [256]
  static constexpr uint32_t kAny = kRt + 1024;               // int4 [128]
  static constexpr uint32_t kBars = kAny + 2048;
  static constexpr uint32_t kRp = kBars + 256;               // the padded rab_pos copy
  static __host__ __device__ constexpr uint32_t smem_bytes(int clamp) {
    return kRp + rp_bytes(clamp) + 1024;
  }
  static_assert(kQ % 1024 == 0 && kDO % 1024 == 0 && kTile % 1024 == 0, "tile alignment");
  static_assert(kQf % 128 == 0 && kQts % 128 == 0 && kAny % 16 == 0, "alignment");
  // dK / dV are staged in the K and V tiles: 8 warps x HD / 64 boxes per pass, two passes
  static_assert(8 * (HD / 64) * 4096 == 2 * kTile, "dK / dV staging");
  static_assert(smem_bytes(kBwdMaxPos - 1) <= 227 * 1024, "shared memory budget");
};

template <int HD>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tm, const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ CUtensorMap tm_ts,
                        const __grid_constant__ CUtensorMap tm_rows,
                        const __grid_constant__ CUtensorMap tm_dk,
                        const __grid_constant__ CUtensorMap tm_dv, const BwdParams p) {
  using L = DkvLayout<HD>;
  constexpr int NS = L::NS;
  // ---- work item: one key tile (longest first), one head
  const int h = blockIdx.x / p.num_key_tiles;
  const int kt = p.key_order[blockIdx.x % p.num_key_tiles];
  const int64_t kb = int64_t(kt) * 128;
  // the query tiles that can see these keys: [kt, end of the user owning the last key)
  const int64_t r_last = kb + 127 < p.T ? kb + 127 : p.T - 1;
  int32_t u = p.rows[r_last].user;
  u = u < 0 ? 0 : (u >= p.B ? p.B - 1 : u);
  int64_t ue = p.offsets[u + 1];
  if (ue <= r_last) ue = r_last + 1;
  if (ue > p.T) ue = p.T;
  const int nq = int((ue + 127) / 128) - kt;   // >= 1

  extern __shared__ uint8_t smem_raw[];
  // aligned up to 1024 bytes by pointer arithmetic on the shared array, so that
  // the compiler keeps every access derived from it in the shared state space
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const RowInfo* s_qf = reinterpret_cast<const RowInfo*>(smem + L::kQf);
  const int64_t* s_qts = reinterpret_cast<const int64_t*>(smem + L::kQts);
  int64_t* s_thr = reinterpret_cast<int64_t*>(smem + L::kThr);
  float* s_rt = reinterpret_cast<float*>(smem + L::kRt);
  int4* s_any = reinterpret_cast<int4*>(smem + L::kAny);
  float* s_rp = reinterpret_cast<float*>(smem + L::kRp);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* kv_full = bars;
  uint64_t* q_full = kv_full + 1;      // [NS] Q, dO and the query facts of a tile landed
  uint64_t* q_empty = q_full + NS;     // [NS]
  uint64_t* s_full = q_empty + NS;     // S^T and dA^T are in tensor memory
  uint64_t* p_full = s_full + 1;       // P^T and dS^T written (256 arrivals)
  uint64_t* kv_done = p_full + 1;      // every product is done
  uint64_t* drained = kv_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int d = p.d;
  const int clamp = p.pos_clamp;
  const int nb = p.time_buckets;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 256);
    mbar_init(kv_done, 1);
    mbar_init(drained, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp >= 4) {
    load_tables(p, threadIdx.x - 128, s_thr, s_rt, s_any);
    load_rp(p, threadIdx.x - 128, s_rp);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tS = tmem_base;
  const uint32_t tdA = tmem_base + 128;
  const uint32_t tDK = tmem_base + 256;
  const uint32_t tDV = tmem_base + 256 + HD;

  if (warp == 0) {
    // ------------------------------------------------------------ loads
    if (lane == 0) {
      prefetch_tmap(&tm);
      prefetch_tmap(&tm_do);
      prefetch_tmap(&tm_ts);
      prefetch_tmap(&tm_rows);
      mbar_arrive_expect_tx(kv_full, 2 * L::kTile);
#pragma unroll
      for (int b = 0; b < HD / 64; ++b) {
        tma_load_2d(smem + L::kK + b * 16384, &tm, kv_full, 3 * d + h * HD + b * 64, int32_t(kb));
        tma_load_2d(smem + L::kV + b * 16384, &tm, kv_full, d + h * HD + b * 64, int32_t(kb));
      }
      bool issued[NS];
      uint32_t issued_ph[NS];
      for (int s = 0; s < NS; ++s) issued[s] = false, issued_ph[s] = 0;
      for (int it = 0; it < nq && !*abort_flag; ++it) {
        const int s = it % NS;
        const uint32_t ph = (it / NS) & 1;
        if (!mbar_wait(&q_empty[s], ph ^ 1, p.wait_limit)) { *abort_flag = 1; break; }
        const int32_t q0 = (kt + it) * 128;
        mbar_arrive_expect_tx(&q_full[s], 2 * L::kTile + 2048 + 1024);
#pragma unroll
        for (int b = 0; b < HD / 64; ++b) {
          tma_load_2d(smem + L::kQ + s * L::kTile + b * 16384, &tm, &q_full[s],
                      2 * d + h * HD + b * 64, q0);
          tma_load_2d(smem + L::kDO + s * L::kTile + b * 16384, &tm_do, &q_full[s],
                      h * HD + b * 64, q0);
        }
        // the query rows' facts (RowInfo as pairs of int64) and timestamps
        tma_load_1d(smem + L::kQf + s * 2048, &tm_rows, &q_full[s], 2 * q0);
        tma_load_1d(smem + L::kQts + s * 1024, &tm_ts, &q_full[s], q0);
        issued[s] = true;
        issued_ph[s] = ph;
      }
      mbar_wait(kv_full, 0);
      for (int s = 0; s < NS; ++s)
        if (issued[s]) mbar_wait(&q_full[s], issued_ph[s]);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_ss = idesc_bf16(128, 128, false, false);   // S^T, dA^T
      constexpr uint32_t idesc_kv = idesc_bf16(128, HD, false, true);     // dV, dK
      const uint32_t sK = smem_u32(smem + L::kK), sV = smem_u32(smem + L::kV);
      bool ok = mbar_wait(kv_full, 0, p.wait_limit);
      for (int it = 0; ok && it < nq; ++it) {
        const int s = it % NS;
        if (!mbar_wait(&q_full[s], (it / NS) & 1, p.wait_limit)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sQ = smem_u32(smem + L::kQ + s * L::kTile);
        const uint32_t sDO = smem_u32(smem + L::kDO + s * L::kTile);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tS, desc_sw128(sK + off, 16, 1024), desc_sw128(sQ + off, 16, 1024), idesc_ss,
                  kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tdA, desc_sw128(sV + off, 16, 1024), desc_sw128(sDO + off, 16, 1024), idesc_ss,
                  kk > 0);
        }
        umma_commit(s_full);
        if (!mbar_wait(p_full, it & 1, p.wait_limit)) { ok = false; break; }
        tc_fence_after();
        // K = the 128 queries in 8 steps of 16; dO_i and Q_i consumed N-major
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tDV, tS + a_col(kk), desc_sw128(sDO + kk * 2048, 16384, 1024), idesc_kv,
                  (it > 0 || kk > 0));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tDK, tdA + a_col(kk), desc_sw128(sQ + kk * 2048, 16384, 1024), idesc_kv,
                  (it > 0 || kk > 0));
        umma_commit(&q_empty[s]);
      }
      if (!ok) *abort_flag = 1;
      umma_commit(kv_done);
      umma_commit(drained);
      mbar_wait(drained, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ row groups (rows = keys)
    const int g = (warp - 4) >> 2;           // query half of every tile
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const int j = int(kb) + row;             // this thread's key (T <= 2^30)
    const bool valid = j < p.T;
    int64_t tj = 0, t_last = 0;
    if (valid) {
      tj = p.ts[j];
      // the queries that see key j lie in its user: their gaps are at most
      // ts[end of user - 1] - t_j
      int32_t u = p.rows[j].user;
      u = u < 0 ? 0 : (u >= p.B ? p.B - 1 : u);
      int64_t ue = p.offsets[u + 1];
      ue = ue <= j ? j + 1 : (ue > p.T ? p.T : ue);
      t_last = p.ts[ue - 1];
    }
    const bool narrow = p.lut_exact != 0 &&
                        __all_sync(0xffffffffu, !valid || t_last - tj < int64_t(0x7FFFFFFE));
    const uint32_t tj_lo = uint32_t(tj);
    const int nn = p.n_norm_fixed > 0 ? p.n_norm_fixed : p.counters[0];
    const float inv_nn = 1.0f / float(nn > 0 ? nn : 1);
    const float rp_clamp = __ldg(p.rab_pos + clamp);
    named_bar_sync(1, 256);   // the tables
    bool aborted = false;
    for (int it = 0; it < nq; ++it) {
      const int s = it % NS;
      const int q0 = (kt + it) * 128;
      bool ok = aborted ? false : mbar_wait(&q_full[s], (it / NS) & 1, p.wait_limit);
      ok = ok && mbar_wait(s_full, it & 1, p.wait_limit);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        aborted = true;
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const RowInfo* qf = s_qf + s * 128;
      const int64_t* qts = s_qts + s * 128;
      const int i0 = q0 + 64 * g;   // first query of this group's half
      // ---- classify the key row for this half tile: the half's queries' facts,
      // reduced over the warp (each lane reads two)
      int mx_lo, mn_hi, mn_pos, own;   // own: every query of the half at its own index
      {
        const RowInfo fa = qf[64 * g + lane], fb = qf[64 * g + 32 + lane];
        mx_lo = max(fa.lo, fb.lo);
        mn_hi = min(fa.hi, fb.hi);
        mn_pos = min(fa.pos, fb.pos);
        own = (fa.pos == i0 + lane && fb.pos == i0 + 32 + lane) ? 1 : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          mx_lo = max(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, o));
          mn_hi = min(mn_hi, __shfl_xor_sync(0xffffffffu, mn_hi, o));
          mn_pos = min(mn_pos, __shfl_xor_sync(0xffffffffu, mn_pos, o));
          own = min(own, __shfl_xor_sync(0xffffffffu, own, o));
        }
      }
      const bool all_rows = i0 + 63 < p.T;
      const bool zero = __all_sync(0xffffffffu, !valid || i0 + 63 < j);
      const bool full = valid && all_rows && mx_lo <= j && j < mn_hi;
      int tb0 = 0, tb1 = 0;
      bool same = false;
      if (full) {
        tb0 = bucket_search(s_thr, nb, qts[64 * g] - tj);
        tb1 = bucket_search(s_thr, nb, qts[64 * g + 63] - tj);
        same = tb0 == tb1;
      }
      const bool fast = __all_sync(0xffffffffu, full && same && mn_pos - j >= clamp);
      // every pair visible, one time bucket per key row, the queries at their
      // own positions: position iq - j, read from the padded table (every pair
      // visible keeps iq - j in [0, clamp + 95] when not all are clamped)
      const bool fastp = !fast && own && __all_sync(0xffffffffu, full && tb1 - tb0 <= 1);
      const uint32_t tcol = lane_off + 64 * g;
      if (zero) {
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) pk[e] = 0u;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_st8(tS + tcol + 8 * c, pk);
          tmem_st8(tdA + tcol + 8 * c, pk);
        }
      } else if (fastp) {
        // queries from column im on have a gap of at least thr[tb1] (bucket tb1):
        // the count of the half's queries with t_i < t_j + thr[tb1] (sorted)
        int im = 64;
        if (tb1 != tb0) {
          const int64_t cut = tj + s_thr[tb1];
          int pcount = 0;
#pragma unroll
          for (int step = 32; step > 0; step >>= 1)
            if (qts[64 * g + pcount + step - 1] < cut) pcount += step;
          im = pcount + (qts[64 * g + pcount] < cut ? 1 : 0);
        }
        const float ht0 = s_rt[tb0], ht1 = s_rt[tb1];
        const int base = kPosPad + i0 - j;   // + column offset inside the half
        auto chunk = [&](const uint32_t (&rs)[16], const uint32_t (&ra)[16], int c) {
          uint32_t pp[8], pd[8];
          float pv[16], dv[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float rp = s_rp[min(base + 16 * c + e, kPosPad + clamp + 129)];
            const float ht = 16 * c + e >= im ? ht1 : ht0;
            const Grad gr = silu_grad(__uint_as_float(rs[e]) + rp + ht, __uint_as_float(ra[e]), inv_nn);
            pv[e] = gr.p;
            dv[e] = gr.ds;
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            pp[e] = pack_bf16x2(pv[2 * e], pv[2 * e + 1]);
            pd[e] = pack_bf16x2(dv[2 * e], dv[2 * e + 1]);
          }
          tmem_st8(tS + tcol + 8 * c, pp);
          tmem_st8(tdA + tcol + 8 * c, pd);
        };
        // the tensor-memory loads of chunk c + 1 overlap the arithmetic of chunk c
        uint32_t xs[16], xa[16], ys[16], ya[16];
        tmem_ld16(tS + tcol, xs);
        tmem_ld16(tdA + tcol, xa);
        tmem_ld_wait();
#pragma unroll 1
        for (int c = 0; c < 4; c += 2) {
          tmem_ld16(tS + tcol + 16 * (c + 1), ys);
          tmem_ld16(tdA + tcol + 16 * (c + 1), ya);
          chunk(xs, xa, c);
          tmem_ld_wait();
          if (c + 2 < 4) {
            tmem_ld16(tS + tcol + 16 * (c + 2), xs);
            tmem_ld16(tdA + tcol + 16 * (c + 2), xa);
          }
          chunk(ys, ya, c + 1);
          tmem_ld_wait();
        }
      } else if (fast) {
        // the tensor-memory loads of chunk c + 1 overlap the arithmetic of chunk c
        const float hc = rp_clamp + s_rt[tb0];
        uint32_t xs[16], xa[16], ys[16], ya[16];
        tmem_ld16(tS + tcol, xs);
        tmem_ld16(tdA + tcol, xa);
        tmem_ld_wait();
#pragma unroll 1
        for (int c = 0; c < 4; c += 2) {
          tmem_ld16(tS + tcol + 16 * (c + 1), ys);
          tmem_ld16(tdA + tcol + 16 * (c + 1), ya);
          {
            uint32_t pp[8], pd[8];
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              const Grad g0 = silu_grad(__uint_as_float(xs[e]) + hc, __uint_as_float(xa[e]), inv_nn);
              const Grad g1 = silu_grad(__uint_as_float(xs[e + 1]) + hc, __uint_as_float(xa[e + 1]), inv_nn);
              pp[e >> 1] = pack_bf16x2(g0.p, g1.p);
              pd[e >> 1] = pack_bf16x2(g0.ds, g1.ds);
            }
            tmem_st8(tS + tcol + 8 * c, pp);
            tmem_st8(tdA + tcol + 8 * c, pd);
          }
          tmem_ld_wait();
          if (c + 2 < 4) {
            tmem_ld16(tS + tcol + 16 * (c + 2), xs);
            tmem_ld16(tdA + tcol + 16 * (c + 2), xa);
          }
          {
            uint32_t pp[8], pd[8];
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              const Grad g0 = silu_grad(__uint_as_float(ys[e]) + hc, __uint_as_float(ya[e]), inv_nn);
              const Grad g1 = silu_grad(__uint_as_float(ys[e + 1]) + hc, __uint_as_float(ya[e + 1]), inv_nn);
              pp[e >> 1] = pack_bf16x2(g0.p, g1.p);
              pd[e >> 1] = pack_bf16x2(g0.ds, g1.ds);
            }
            tmem_st8(tS + tcol + 8 * (c + 1), pp);
            tmem_st8(tdA + tcol + 8 * (c + 1), pd);
          }
          tmem_ld_wait();
        }
      } else {
        auto chunk = [&](const uint32_t (&rs)[16], const uint32_t (&ra)[16], int c) {
          uint32_t pp[8], pd[8];
          float pv[16], dv[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int ir = 64 * g + 16 * c + e;
            const int iq = q0 + ir;
            const RowInfo f = qf[ir];
            const bool vis = valid && iq < p.T && ((f.lo <= j && j < f.hi) || iq == j);
            float rt;
            if (narrow) {
              int tb;
              rt = time_bias_lut(uint32_t(qts[ir]) - tj_lo, s_any, tb);
            } else {
              const int64_t gap = qts[ir] - tj;
              rt = s_rt[bucket_search(s_thr, nb, gap < 0 ? 0 : gap)];
            }
            // the position of pair (iq, j) relative to this key tile, clamped into
            // the padded table
            const int pr = min(max(f.pos - int(kb), -1), clamp + 129);
            const float rp = s_rp[kPosPad + pr - row];
            const Grad gr = silu_grad(__uint_as_float(rs[e]) + rp + rt, __uint_as_float(ra[e]), inv_nn);
            pv[e] = vis ? gr.p : 0.0f;
            dv[e] = vis ? gr.ds : 0.0f;
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            pp[e] = pack_bf16x2(pv[2 * e], pv[2 * e + 1]);
            pd[e] = pack_bf16x2(dv[2 * e], dv[2 * e + 1]);
          }
          tmem_st8(tS + tcol + 8 * c, pp);
          tmem_st8(tdA + tcol + 8 * c, pd);
        };
        // the tensor-memory loads of chunk c + 1 overlap the arithmetic of chunk c
        uint32_t xs[16], xa[16], ys[16], ya[16];
        tmem_ld16(tS + tcol, xs);
        tmem_ld16(tdA + tcol, xa);
        tmem_ld_wait();
#pragma unroll 1
        for (int c = 0; c < 4; c += 2) {
          tmem_ld16(tS + tcol + 16 * (c + 1), ys);
          tmem_ld16(tdA + tcol + 16 * (c + 1), ya);
          chunk(xs, xa, c);
          tmem_ld_wait();
          if (c + 2 < 4) {
            tmem_ld16(tS + tcol + 16 * (c + 2), xs);
            tmem_ld16(tdA + tcol + 16 * (c + 2), xa);
          }
          chunk(ys, ya, c + 1);
          tmem_ld_wait();
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (aborted) *abort_flag = 1;
    // ---- dK (group 0) / dV (group 1) -> the free K and V tiles -> TMA stores
    bool w = aborted ? false : mbar_wait(kv_done, 0, p.wait_limit);
    w = __all_sync(0xffffffffu, w);
    if (w && !*abort_flag) {
      tc_fence_after();
      const uint32_t tacc = g == 0 ? tDK : tDV;
      const CUtensorMap* m = g == 0 ? &tm_dk : &tm_dv;
      uint8_t* stage = smem + L::kK + (g * 4 + wq) * (HD / 64) * 4096;
#pragma unroll 1
      for (int rd = 0; rd < 2; ++rd) {
#pragma unroll 1
        for (int cb = 0; cb < HD / 64; ++cb) {
          const int col = (rd * (HD / 64) + cb) * 32;
          store_box(tacc + lane_off + col, stage + cb * 4096, m, h * HD + col,
                    int32_t(kb) + wq * 32, lane);
        }
      }
    } else {
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.error, HSTU_DEVERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ================================================================ key-tile order

// One block: per key tile the number of query tiles that can see it (from the
// tile to the end of the user owning its last row), then a counting sort by
// descending count (longest processing time first).
__global__ void key_order_kernel(const RowInfo* __restrict__ rows,
                                 const int32_t* __restrict__ offsets, int32_t B, int64_t T,
                                 int32_t nkt, int32_t* __restrict__ cost,
                                 int32_t* __restrict__ order) {
  constexpr int NB = 4096;
  __shared__ int32_t hist[NB];
  __shared__ int32_t s_max;
  for (int c = threadIdx.x; c < NB; c += blockDim.x) hist[c] = 0;
  if (threadIdx.x == 0) s_max = 0;
  __syncthreads();
  int32_t local_max = 0;
  for (int32_t kt = threadIdx.x; kt < nkt; kt += blockDim.x) {
    const int64_t kb = int64_t(kt) * 128;
    const int64_t r_last = kb + 127 < T ? kb + 127 : T - 1;
    int32_t u = rows[r_last].user;
    u = u < 0 ? 0 : (u >= B ? B - 1 : u);
    int64_t ue = offsets[u + 1];
    if (ue <= r_last) ue = r_last + 1;
    if (ue > T) ue = T;
    const int32_t c = int32_t((ue + 127) / 128) - kt;
    cost[kt] = c;
    local_max = c > local_max ? c : local_max;
    atomicAdd(&hist[c < NB ? c : NB - 1], 1);
  }
  atomicMax(&s_max, local_max);
  __syncthreads();
  const int top = s_max < NB ? s_max : NB - 1;
  if (threadIdx.x == 0) {
    int32_t run = 0;
    for (int c = top; c >= 0; --c) {
      const int32_t n = hist[c];
      hist[c] = run;
      run += n;
    }
  }
  __syncthreads();
  for (int32_t kt = threadIdx.x; kt < nkt; kt += blockDim.x) {
    const int32_t c = cost[kt];
    const int32_t slot = atomicAdd(&hist[c < NB ? c : NB - 1], 1);
    order[slot] = kt;
  }
}

// ==== host side: launch configuration (no device code below this line) ====

template <int HD>
cudaError_t launch_bwd_hd(const AttnBwdArgs& a, const BwdParams& p, cudaStream_t st) {
  CUtensorMap tm, tm_do, tm_ts, tm_rows, tm_dq, tm_dk, tm_dv;
  if (!make_tmap_2d_bf16(&tm, a.uvqk, uint64_t(4 * a.d), uint64_t(a.T), uint64_t(4 * a.d) * 2,
                         64, 128))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d_bf16(&tm_do, a.dO, uint64_t(a.d), uint64_t(a.T), uint64_t(a.d) * 2, 64, 128))
    return cudaErrorInvalidValue;
  if (!make_tmap_1d_i64(&tm_ts, a.ts, uint64_t(a.T), 128)) return cudaErrorInvalidValue;
  if (!make_tmap_1d_i64(&tm_rows, a.rows, uint64_t(a.T) * 2, 256)) return cudaErrorInvalidValue;
  const uint64_t dd = uint64_t(a.d), tt = uint64_t(a.T);
  if (!make_tmap_2d_f32_sw128(&tm_dq, a.dq, dd, tt, dd * 4, 32, 32) ||
      !make_tmap_2d_f32_sw128(&tm_dk, a.dk, dd, tt, dd * 4, 32, 32) ||
      !make_tmap_2d_f32_sw128(&tm_dv, a.dv, dd, tt, dd * 4, 32, 32))
    return cudaErrorInvalidValue;
  static std::atomic<uint64_t> set_dq{0}, set_dkv{0};
  cudaError_t e = smem_opt_in(attn_bwd_dq_kernel<HD>, 227 * 1024, set_dq);
  if (e == cudaSuccess)
    e = smem_opt_in(attn_bwd_dkv_kernel<HD>, int(DkvLayout<HD>::smem_bytes(kBwdMaxPos - 1)),
                    set_dkv);
  if (e != cudaSuccess) return e;
  // the dq kernel keeps the padded rab_pos copy in shared memory when it fits
  BwdParams pq = p;
  pq.rp_smem = DqLayout<HD>::smem_bytes(a.pos_clamp, true) <= 227 * 1024 ? 1 : 0;
  const int64_t grid_q = int64_t(2) * p.num_pairs * a.H;
  attn_bwd_dq_kernel<HD><<<unsigned(grid_q), kBwdThreads,
                           DqLayout<HD>::smem_bytes(a.pos_clamp, pq.rp_smem != 0), st>>>(
      tm, tm_do, tm_ts, tm_dq, pq);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t grid_k = int64_t(p.num_key_tiles) * a.H;
  attn_bwd_dkv_kernel<HD><<<unsigned(grid_k), kBwdThreads, DkvLayout<HD>::smem_bytes(a.pos_clamp),
                            st>>>(
      tm, tm_do, tm_ts, tm_rows, tm_dk, tm_dv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_bwd_tc(const AttnBwdArgs& a, cudaStream_t st) {
  if (a.T <= 0 || a.B <= 0) return cudaSuccess;
  if (a.pos_clamp >= kBwdMaxPos || a.time_buckets > kBwdMaxBuckets) return cudaErrorInvalidValue;
  if (a.hd != 128 && a.hd != 64) return cudaErrorInvalidValue;
  BwdParams p;
  p.rows = a.rows;
  p.order = a.order;
  p.key_order = a.key_order;
  p.offsets = a.offsets;
  p.B = a.B;
  p.ts = a.ts;
  p.thresholds = a.thresholds;
  p.time_lut = a.time_lut;
  p.thr32 = a.thr32;
  p.rab_pos = a.rab_pos;
  p.rab_time = a.rab_time;
  p.counters = a.counters;
  p.error = a.error;
  p.d_rab_pos = a.d_rab_pos;
  p.d_rab_time = a.d_rab_time;
  p.T = a.T;
  p.d = a.d;
  p.H = a.H;
  p.num_pairs = int((a.T + 2 * kTile - 1) / (2 * kTile));
  p.num_key_tiles = int((a.T + kTile - 1) / kTile);
  p.pos_clamp = a.pos_clamp;
  p.time_buckets = a.time_buckets;
  p.n_norm_fixed = a.n_norm_fixed;
  p.lut_exact = a.lut_exact;
  p.rp_smem = 1;
  p.wait_limit = a.wait_limit > 0 ? a.wait_limit : kWaitLimit;
  key_order_kernel<<<1, 1024, 0, st>>>(a.rows, a.offsets, a.B, a.T, p.num_key_tiles, a.key_cost,
                                       a.key_order);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return a.hd == 128 ? launch_bwd_hd<128>(a, p, st) : launch_bwd_hd<64>(a, p, st);
}

}  // namespace hstu
