// Backward of the fused jagged pointwise attention on the tcgen05 tensor cores.
//
// For equation (2) of the HSTU layer (blog "Generative Recommendation 16:
// HSTU", section "HSTU Layer 到底改了什么"), with s = q.k + rab and
// a = vis * SiLU(s) / n_norm, O = a V, the gradients of sum(dO * O) are
//     dV = a^T dO,  dA = dO V^T,  dS = vis * dA * SiLU'(s) / n_norm,
//     dQ = dS K,    dK = dS^T Q,
// and every entry of rab_pos / rab_time collects dS of each visible
// (query, key, head) that reads it.  SiLU acts on each score alone (same blog,
// section "不对序列做 softmax"), so there are no row statistics to keep from
// the forward: S is recomputed tile by tile.
//
// One CTA per (128-key tile, head), 256 threads:
//   warp 0      TMA: the key tile's K, V and key timestamps once, then per
//               query tile its Q and dO (single buffers)
//   warp 1      tensor-memory allocation and MMA issue:
//                 S  = Q K^T, dA = dO V^T          (SS, both K-major)
//                 dV += P^T dO, dK += dS^T Q       (A = P or dS read M-major
//                                                   from shared memory, B N-major)
//                 dQ = dS K                        (A = dS K-major, B = K N-major)
//   warps 4-7   one query row per thread: P = a and dS from S and dA, written
//               as bf16 into 128-byte-swizzled shared tiles; the bias
//               gradients into shared accumulators; dQ added to global fp32
//               (reductions); at the end one key row per thread: dK and dV
//               of the key tile stored as fp32.
// Query tiles visited by key tile kt: [kt, end of the user owning the tile's
// last row) -- a query sees keys of its own user at or before its position
// (M-FALCON candidates: the history and themselves), so no earlier query tile
// and no later user's tile reads these keys.
//
// Tensor memory: S, then dQ, in columns [0, 128); dA in [128, 256); dK in
// [256, 256 + HD); dV in [256 + HD, 256 + 2 HD).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "sm100.cuh"

namespace hstu {
namespace {

using namespace sm100;

constexpr int kBwdThreads = 256;
constexpr int kBwdMaxPos = 4097;      // pos_clamp <= 4096
constexpr int kBwdMaxBuckets = 256;

struct AttnBwdParams {
  const RowInfo* rows;
  const int32_t* offsets;
  int32_t B;
  const int64_t* ts;
  const int64_t* thresholds;
  const float* rab_pos;
  const float* rab_time;
  const int32_t* counters;
  int32_t* error;
  float* dq;
  float* dk;
  float* dv;
  float* d_rab_pos;
  float* d_rab_time;
  int64_t T;
  int d, H, num_key_tiles;
  int pos_clamp, time_buckets, n_norm_fixed;
};

template <int HD>
struct BwdLayout {
  static constexpr uint32_t kTile = 128 * HD * 2;                   // bf16 [128][HD]
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kTile;
  static constexpr uint32_t kQ = kV + kTile;
  static constexpr uint32_t kDO = kQ + kTile;
  static constexpr uint32_t kP = kDO + kTile;                       // bf16 [128 q][128 k]
  static constexpr uint32_t kDS = kP + 32768;
  static constexpr uint32_t kKts = kDS + 32768;                     // int64 [128]
  static constexpr uint32_t kThr = kKts + 1024;                     // int64 [256]
  static constexpr uint32_t kGradTime = kThr + kBwdMaxBuckets * 8;  // float [256]
  static constexpr uint32_t kBars = kGradTime + kBwdMaxBuckets * 4;
  static constexpr uint32_t kGradPos = kBars + 256;                 // float [clamp + 1]
  static __host__ __device__ constexpr uint32_t smem_bytes(int clamp) {
    return kGradPos + ((uint32_t(clamp + 1) * 4 + 15) / 16) * 16 + 1024;
  }
  static_assert(kK % 1024 == 0 && kV % 1024 == 0 && kQ % 1024 == 0 && kDO % 1024 == 0 &&
                    kP % 1024 == 0 && kDS % 1024 == 0,
                "swizzled tiles start on 1024-byte boundaries");
  static_assert(kKts % 128 == 0 && kBars % 8 == 0, "alignment");
  static_assert(smem_bytes(kBwdMaxPos - 1) <= 227 * 1024, "shared memory budget");
};

// Largest k with thr[k] <= dt (thr[0] = 0, non-decreasing): the time bucket.
__device__ __forceinline__ int bwd_bucket(const int64_t* thr, int nb, int64_t dt) {
  if (dt <= 0) return 0;
  int lo = 0, hi = nb - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (thr[mid] <= dt) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Byte offset of column c (0..127) of row r in a [128][128] bf16 tile stored
// as two 64-column halves of 128-byte rows with the 128-byte swizzle (16-byte
// chunk index XOR row % 8): the layout of a TMA box of 64 x 128 bf16.
__device__ __forceinline__ uint32_t sw128_offset(int r, int c) {
  const int half = c >> 6;
  const int chunk = (c & 63) >> 3;
  return uint32_t(half * 16384 + r * 128 + ((chunk ^ (r & 7)) << 4) + (c & 7) * 2);
}

template <int HD>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_ts, const AttnBwdParams p) {
  using L = BwdLayout<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  int64_t* s_kts = reinterpret_cast<int64_t*>(smem + L::kKts);
  int64_t* s_thr = reinterpret_cast<int64_t*>(smem + L::kThr);
  float* s_gtime = reinterpret_cast<float*>(smem + L::kGradTime);
  float* s_gpos = reinterpret_cast<float*>(smem + L::kGradPos);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* kv_full = bars;         // K, V, key timestamps landed
  uint64_t* q_full = bars + 1;      // Q and dO of the current query tile landed
  uint64_t* q_empty = bars + 2;     // every MMA reading Q and dO is done
  uint64_t* s_full = bars + 3;      // S and dA are in tensor memory
  uint64_t* p_full = bars + 4;      // P and dS are in shared memory (128 arrivals)
  uint64_t* mma_done = bars + 5;    // dV, dK, dQ products of the tile are done
  uint64_t* tmem_free = bars + 6;   // dQ read out: S / dA columns free (128 arrivals)
  uint64_t* kv_done = bars + 7;     // every product of the CTA is done
  uint64_t* drained = bars + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 9);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int d = p.d;
  const int kt = blockIdx.x % p.num_key_tiles;
  const int h = blockIdx.x / p.num_key_tiles;
  const int64_t kb = int64_t(kt) * 128;

  // the query tiles that read this key tile: [kt, end of the last row's user)
  int64_t r_last = kb + 127 < p.T ? kb + 127 : p.T - 1;
  int32_t u = p.rows[r_last].user;
  u = u < 0 ? 0 : (u >= p.B ? p.B - 1 : u);
  int64_t ue = p.offsets[u + 1];
  if (ue <= r_last) ue = r_last + 1;
  if (ue > p.T) ue = p.T;
  const int q_begin = kt;
  const int nq = int((ue + 127) / 128) - q_begin;   // >= 1

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(mma_done, 1);
    mbar_init(tmem_free, 128);
    mbar_init(kv_done, 1);
    mbar_init(drained, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  // the tables and the gradient accumulators
  const int clamp = p.pos_clamp;
  const int nb = p.time_buckets;
  for (int k = threadIdx.x; k < kBwdMaxBuckets; k += blockDim.x) {
    s_thr[k] = k < nb ? p.thresholds[k] : (int64_t(1) << 62);
    s_gtime[k] = 0.0f;
  }
  for (int k = threadIdx.x; k <= clamp; k += blockDim.x) s_gpos[k] = 0.0f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tS = tmem_base;
  const uint32_t tdA = tmem_base + 128;
  const uint32_t tdK = tmem_base + 256;
  const uint32_t tdV = tmem_base + 256 + HD;

  if (warp == 0) {
    // ------------------------------------------------------------ loads
    if (lane == 0) {
      prefetch_tmap(&tm);
      prefetch_tmap(&tm_do);
      prefetch_tmap(&tm_ts);
      mbar_arrive_expect_tx(kv_full, 2 * L::kTile + 128 * 8);
#pragma unroll
      for (int b = 0; b < HD / 64; ++b) {
        tma_load_2d(smem + L::kK + b * 16384, &tm, kv_full, 3 * d + h * HD + b * 64, int32_t(kb));
        tma_load_2d(smem + L::kV + b * 16384, &tm, kv_full, d + h * HD + b * 64, int32_t(kb));
      }
      tma_load_1d(s_kts, &tm_ts, kv_full, int32_t(kb));
      int issued = 0;
      for (int it = 0; it < nq && !*abort_flag; ++it) {
        if (it > 0 && !mbar_wait(q_empty, (it - 1) & 1)) { *abort_flag = 1; break; }
        const int32_t row0 = (q_begin + it) * 128;
        mbar_arrive_expect_tx(q_full, 2 * L::kTile);
#pragma unroll
        for (int b = 0; b < HD / 64; ++b) {
          tma_load_2d(smem + L::kQ + b * 16384, &tm, q_full, 2 * d + h * HD + b * 64, row0);
          tma_load_2d(smem + L::kDO + b * 16384, &tm_do, q_full, h * HD + b * 64, row0);
        }
        issued = it + 1;
      }
      // no copy may still be in flight when the CTA ends
      mbar_wait(kv_full, 0);
      if (issued > 0) mbar_wait(q_full, (issued - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_kk = idesc_bf16(128, 128, false, false);   // S, dA
      constexpr uint32_t idesc_t = idesc_bf16(128, HD, true, true);       // dV, dK
      constexpr uint32_t idesc_q = idesc_bf16(128, HD, false, true);      // dQ
      const uint32_t sK = smem_u32(smem + L::kK), sV = smem_u32(smem + L::kV);
      const uint32_t sQ = smem_u32(smem + L::kQ), sDO = smem_u32(smem + L::kDO);
      const uint32_t sP = smem_u32(smem + L::kP), sDS = smem_u32(smem + L::kDS);
      bool ok = mbar_wait(kv_full, 0);
      for (int it = 0; ok && it < nq; ++it) {
        if (!mbar_wait(q_full, it & 1)) { ok = false; break; }
        if (it > 0 && !mbar_wait(tmem_free, (it - 1) & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tS, desc_sw128(sQ + off, 16, 1024), desc_sw128(sK + off, 16, 1024), idesc_kk,
                  kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tdA, desc_sw128(sDO + off, 16, 1024), desc_sw128(sV + off, 16, 1024), idesc_kk,
                  kk > 0);
        }
        umma_commit(s_full);
        if (!mbar_wait(p_full, it & 1)) { ok = false; break; }
        tc_fence_after();
        // K = the 128 query rows, in 8 steps of 16 (2048 bytes of 128-byte rows)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          umma_ss(tdV, desc_sw128(sP + kk * 2048, 16384, 1024),
                  desc_sw128(sDO + kk * 2048, 16384, 1024), idesc_t, (it > 0 || kk > 0));
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          umma_ss(tdK, desc_sw128(sDS + kk * 2048, 16384, 1024),
                  desc_sw128(sQ + kk * 2048, 16384, 1024), idesc_t, (it > 0 || kk > 0));
        }
        umma_commit(q_empty);
        // K = the 128 keys: dS K-major (two 64-key halves), K N-major
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tS, desc_sw128(sDS + off, 16, 1024), desc_sw128(sK + kk * 2048, 16384, 1024),
                  idesc_q, kk > 0);
        }
        umma_commit(mma_done);
      }
      if (!ok) *abort_flag = 1;
      umma_commit(kv_done);     // releases the final read-out (also on an abort)
      umma_commit(drained);
      mbar_wait(drained, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ rows
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const int nn = p.n_norm_fixed > 0 ? p.n_norm_fixed : p.counters[0];
    const float inv_nn = 1.0f / float(nn > 0 ? nn : 1);
    bool ok = mbar_wait(kv_full, 0);
    ok = __all_sync(0xffffffffu, ok);
    uint8_t* sP = smem + L::kP;
    uint8_t* sDS = smem + L::kDS;
    for (int it = 0; ok && it < nq; ++it) {
      const int64_t i = int64_t(q_begin + it) * 128 + row;
      const bool valid = i < p.T;
      int64_t lo = i, hi = i, pos = i, ti = 0;
      if (valid) {
        const RowInfo ri = p.rows[i];
        lo = (ri.lo < 0 || ri.lo > i) ? i : ri.lo;
        hi = ri.hi;
        pos = ri.pos;
        ti = p.ts[i];
      }
      bool w = mbar_wait(s_full, it & 1);
      w = __all_sync(0xffffffffu, w);
      if (!w) { ok = false; break; }
      tc_fence_after();
      bool any = false;
      // Along a row the keys advance in time inside the user, so the gap only
      // shrinks: the time bucket walks down from the previous visible key's (a
      // larger gap, i.e. input out of order, searches again).  The bias
      // gradients are summed in registers while the bucket stays the same
      // (time) or for the clamped entry (position), and added to shared
      // memory when the bucket changes and at the end of the tile.
      int tb = -1;
      float acc_t = 0.0f, acc_c = 0.0f;
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t rs[32], ra[32];
        tmem_ld32(tS + lane_off + c0, rs);
        tmem_ld32(tdA + lane_off + c0, ra);
        tmem_ld_wait();
        uint32_t pa[16], pd[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float av[2], dv[2];
#pragma unroll
          for (int f = 0; f < 2; ++f) {
            const int c = c0 + e + f;
            const int64_t j = kb + c;
            const bool vis = valid && j < p.T && ((lo <= j && j < hi) || j == i);
            av[f] = 0.0f;
            dv[f] = 0.0f;
            if (vis) {
              int64_t rel = pos - j;
              const int pidx = rel < 0 ? 0 : (rel > clamp ? clamp : int(rel));
              const int64_t gap = ti - s_kts[c];
              int tidx;
              if (tb < 0 || (tb + 1 < nb && gap >= s_thr[tb + 1])) {
                tidx = bwd_bucket(s_thr, nb, gap);
              } else {
                tidx = tb;
                while (tidx > 0 && gap < s_thr[tidx]) --tidx;
              }
              const float s = __uint_as_float(rs[e + f]) + __ldg(p.rab_pos + pidx) +
                              __ldg(p.rab_time + tidx);
              const float sig = 0.5f + 0.5f * tanh_approx(0.5f * s);
              av[f] = s * sig * inv_nn;
              const float ds = __uint_as_float(ra[e + f]) * (sig * (1.0f + s * (1.0f - sig))) * inv_nn;
              dv[f] = ds;
              if (pidx == clamp) acc_c += ds;
              else atomicAdd(s_gpos + pidx, ds);
              if (tidx != tb) {
                if (tb >= 0 && acc_t != 0.0f) atomicAdd(s_gtime + tb, acc_t);
                tb = tidx;
                acc_t = 0.0f;
              }
              acc_t += ds;
              any = true;
            }
          }
          pa[e / 2] = pack_bf16x2(av[0], av[1]);
          pd[e / 2] = pack_bf16x2(dv[0], dv[1]);
        }
        // 32 columns = four 16-byte chunks of P and of dS
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const uint32_t off = sw128_offset(row, c0 + g * 8);
          st_shared_v4_u32(smem_u32(sP + off), pa[4 * g], pa[4 * g + 1], pa[4 * g + 2], pa[4 * g + 3]);
          st_shared_v4_u32(smem_u32(sDS + off), pd[4 * g], pd[4 * g + 1], pd[4 * g + 2], pd[4 * g + 3]);
        }
      }
      if (tb >= 0 && acc_t != 0.0f) atomicAdd(s_gtime + tb, acc_t);
      if (acc_c != 0.0f) atomicAdd(s_gpos + clamp, acc_c);
      fence_proxy_async_smem();   // the tensor cores read P and dS through the async proxy
      tc_fence_before();
      mbar_arrive(p_full);
      w = mbar_wait(mma_done, it & 1);
      w = __all_sync(0xffffffffu, w);
      if (!w) { ok = false; break; }
      tc_fence_after();
      // dQ of this (query tile, key tile) into the global fp32 accumulator
      const bool add = __any_sync(0xffffffffu, any);
#pragma unroll 1
      for (int c0 = 0; add && c0 < HD; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tS + lane_off + c0, r);
        tmem_ld_wait();
        if (any) {
          float* dst = p.dq + i * d + h * HD + c0;
#pragma unroll
          for (int e = 0; e < 32; ++e) atomicAdd(dst + e, __uint_as_float(r[e]));
        }
      }
      tc_fence_before();
      mbar_arrive(tmem_free);
    }
    if (!ok) *abort_flag = 1;
    // dK and dV of the key tile: one key row per thread
    bool w = ok ? mbar_wait(kv_done, 0) : false;
    w = __all_sync(0xffffffffu, w);
    if (w) {
      tc_fence_after();
      const int64_t j = kb + row;
#pragma unroll 1
      for (int c0 = 0; c0 < HD; c0 += 32) {
        uint32_t rk[32], rv[32];
        tmem_ld32(tdK + lane_off + c0, rk);
        tmem_ld32(tdV + lane_off + c0, rv);
        tmem_ld_wait();
        if (j < p.T) {
          float4* gk = reinterpret_cast<float4*>(p.dk + j * d + h * HD + c0);
          float4* gv = reinterpret_cast<float4*>(p.dv + j * d + h * HD + c0);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            gk[e] = make_float4(__uint_as_float(rk[4 * e]), __uint_as_float(rk[4 * e + 1]),
                                __uint_as_float(rk[4 * e + 2]), __uint_as_float(rk[4 * e + 3]));
            gv[e] = make_float4(__uint_as_float(rv[4 * e]), __uint_as_float(rv[4 * e + 1]),
                                __uint_as_float(rv[4 * e + 2]), __uint_as_float(rv[4 * e + 3]));
          }
        }
      }
    } else {
      *abort_flag = 1;
    }
    // the bias gradients of the CTA
    named_bar_sync(1, 128);
    const int t = threadIdx.x - 128;
    for (int k = t; k <= clamp; k += 128) {
      const float g = s_gpos[k];
      if (g != 0.0f) atomicAdd(p.d_rab_pos + k, g);
    }
    for (int k = t; k < nb; k += 128) {
      const float g = s_gtime[k];
      if (g != 0.0f) atomicAdd(p.d_rab_time + k, g);
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

// ==== host side: launch configuration (no device code below this line) ====

template <int HD>
cudaError_t launch_bwd_hd(const AttnBwdArgs& a, cudaStream_t st) {
  using L = BwdLayout<HD>;
  CUtensorMap tm, tm_do, tm_ts;
  if (!make_tmap_2d_bf16(&tm, a.uvqk, uint64_t(4 * a.d), uint64_t(a.T), uint64_t(4 * a.d) * 2,
                         64, 128))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d_bf16(&tm_do, a.dO, uint64_t(a.d), uint64_t(a.T), uint64_t(a.d) * 2, 64, 128))
    return cudaErrorInvalidValue;
  if (!make_tmap_1d_i64(&tm_ts, a.ts, uint64_t(a.T), 128)) return cudaErrorInvalidValue;
  static std::atomic<uint64_t> smem_set{0};
  const cudaError_t e = smem_opt_in(attn_bwd_tc_kernel<HD>, int(L::smem_bytes(kBwdMaxPos - 1)),
                                    smem_set);
  if (e != cudaSuccess) return e;
  AttnBwdParams p;
  p.rows = a.rows;
  p.offsets = a.offsets;
  p.B = a.B;
  p.ts = a.ts;
  p.thresholds = a.thresholds;
  p.rab_pos = a.rab_pos;
  p.rab_time = a.rab_time;
  p.counters = a.counters;
  p.error = a.error;
  p.dq = a.dq;
  p.dk = a.dk;
  p.dv = a.dv;
  p.d_rab_pos = a.d_rab_pos;
  p.d_rab_time = a.d_rab_time;
  p.T = a.T;
  p.d = a.d;
  p.H = a.H;
  p.num_key_tiles = int((a.T + 127) / 128);
  p.pos_clamp = a.pos_clamp;
  p.time_buckets = a.time_buckets;
  p.n_norm_fixed = a.n_norm_fixed;
  const int64_t grid = int64_t(p.num_key_tiles) * a.H;
  attn_bwd_tc_kernel<HD><<<unsigned(grid), kBwdThreads, L::smem_bytes(a.pos_clamp), st>>>(
      tm, tm_do, tm_ts, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_bwd_tc(const AttnBwdArgs& a, cudaStream_t st) {
  if (a.T <= 0 || a.B <= 0) return cudaSuccess;
  if (a.pos_clamp >= kBwdMaxPos || a.time_buckets > kBwdMaxBuckets) return cudaErrorInvalidValue;
  if (a.hd == 128) return launch_bwd_hd<128>(a, st);
  if (a.hd == 64) return launch_bwd_hd<64>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace hstu
