// Fused jagged pointwise attention on the tcgen05 tensor cores.
//
// Equation (2) of the HSTU layer (blog "Generative Recommendation 16: HSTU",
// section "HSTU Layer 到底改了什么"):
//     O_i = sum_{j visible} SiLU(q_i . k_j + rab_pos[p(i,j)] + rab_time[t(i,j)]) v_j / n_norm
// The SiLU acts on each score alone: there is no softmax along the sequence
// (same blog, section "不对序列做 softmax"), hence no running maximum and no
// rescaling of the accumulator, and the n x n score matrix is never stored.
//
// One CTA computes one (128-query tile, head) work item:
//   warp 0      TMA: Q once, then K and V tiles into NS-stage rings
//   warp 1      MMA issue: S_j = Q K_j^T into one of two tensor-memory score
//               buffers (SS form, both operands K-major in shared memory), and
//               O += P_j V_j with P_j read back from tensor memory (TS form,
//               V consumed N-major straight from its row-major tile)
//   warps 2-5   one query row per thread: reads S_j from tensor memory, adds
//               the position and time biases, applies the mask and SiLU, and
//               writes P_j (bf16) over the first half of S_j's columns
// so the SiLU of tile j overlaps the MMAs of tiles j+1 (QK) and j-1 (PV).
//
// Key tiles: only tiles that hold a visible key for some row of the query
// tile are visited (see sched.cu); the last one is always the diagonal tile.
//
// Time buckets: timestamps are non-decreasing inside a user, so along a row
// the gap t_i - t_j only shrinks as j grows.  Each row keeps its current
// bucket b and the key-timestamp cut t_i - thr[b]; a key above the cut moves
// b down.  The threshold table thr holds, per bucket, the smallest integer
// gap of that bucket, so the integer compare reproduces
// floor(ln(1 + dt) / div) exactly.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "sm100.cuh"

namespace hstu {
namespace {

using namespace sm100;

constexpr int kMaxPosEntries = 4097;   // pos_clamp <= 4096
constexpr int kMaxTimeBuckets = 256;

struct AttnParams {
  const RowInfo* rows;
  const int32_t* order;
  const int64_t* ts;
  const int64_t* thresholds;
  const float* rab_pos;
  const float* rab_time;
  const int32_t* counters;
  int32_t* error;
  float* av;
  int64_t T;
  int d, H;
  int pos_clamp, time_buckets;
  int n_norm_fixed;
  int32_t* dump_pidx;
  int32_t* dump_tidx;
  uint8_t* dump_vis;
};

template <int HD>
struct AttnLayout {
  static constexpr int NS = HD == 128 ? 2 : 3;
  static constexpr uint32_t kTileBytes = 128 * HD * 2;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kTileBytes;
  static constexpr uint32_t kV = kK + NS * kTileBytes;
  static constexpr uint32_t kRabPos = kV + NS * kTileBytes;
  static constexpr uint32_t kRabTime = kRabPos + ((kMaxPosEntries * 4 + 15) / 16) * 16;
  static constexpr uint32_t kThr = kRabTime + kMaxTimeBuckets * 4;
  static constexpr uint32_t kKts = kThr + kMaxTimeBuckets * 8;
  static constexpr uint32_t kBars = kKts + 2 * 128 * 8;
  static constexpr uint32_t kSmemBytes = kBars + 256 + 1024;
};

__device__ __forceinline__ int bucket_search(const int64_t* thr, int nb, int64_t dt) {
  if (dt <= 0) return 0;
  int lo = 0, hi = nb - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (thr[mid] <= dt) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int HD, bool RECORD>
__global__ void __launch_bounds__(192, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm, const AttnParams p) {
  using L = AttnLayout<HD>;
  constexpr int NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* s_rab_pos = reinterpret_cast<float*>(smem + L::kRabPos);
  float* s_rab_time = reinterpret_cast<float*>(smem + L::kRabTime);
  int64_t* s_thr = reinterpret_cast<int64_t*>(smem + L::kThr);
  int64_t* s_kts = reinterpret_cast<int64_t*>(smem + L::kKts);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;
  uint64_t* k_empty = k_full + NS;
  uint64_t* v_full = k_empty + NS;
  uint64_t* v_empty = v_full + NS;
  uint64_t* s_full = v_empty + NS;   // [2]
  uint64_t* p_full = s_full + 2;     // [2]
  uint64_t* o_full = p_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int d = p.d;

  // ---- work item and its key-tile range
  const int w = blockIdx.x;
  const int qt = p.order[w / p.H];
  const int h = w % p.H;
  const int64_t r0 = int64_t(qt) * 128;
  const RowInfo ri0 = p.rows[r0];
  int64_t lo0 = ri0.lo;
  if (lo0 < 0 || lo0 > r0) lo0 = r0;
  int64_t vis_end = ri0.hi < r0 ? int64_t(ri0.hi) : r0;
  if (vis_end < lo0) vis_end = lo0;
  const int kt_begin = int(lo0 / 128);
  const int n_a = int((vis_end + 127) / 128) - kt_begin;   // tiles before the diagonal
  const int n_kt = n_a + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 128);
    }
    mbar_init(o_full, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tS = tmem_base;          // two 128-column score buffers
  const uint32_t tO = tmem_base + 256;    // HD-column output accumulator

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm);
      mbar_arrive_expect_tx(q_full, L::kTileBytes);
#pragma unroll
      for (int b = 0; b < HD / 64; ++b)
        tma_load_2d(smem + L::kQ + b * 16384, &tm, q_full, 2 * d + h * HD + b * 64, int32_t(r0));
      bool issued[NS];
      uint32_t issued_ph[NS];
      for (int s = 0; s < NS; ++s) issued[s] = false, issued_ph[s] = 0;
      for (int j = 0; j < n_kt; ++j) {
        const int s = j % NS;
        const uint32_t ph = (j / NS) & 1;
        const int32_t key_row = int32_t((j < n_a ? kt_begin + j : qt)) * 128;
        if (!mbar_wait(&k_empty[s], ph ^ 1)) { *abort_flag = 1; break; }
        mbar_arrive_expect_tx(&k_full[s], L::kTileBytes);
#pragma unroll
        for (int b = 0; b < HD / 64; ++b)
          tma_load_2d(smem + L::kK + s * L::kTileBytes + b * 16384, &tm, &k_full[s],
                      3 * d + h * HD + b * 64, key_row);
        if (!mbar_wait(&v_empty[s], ph ^ 1)) { *abort_flag = 1; break; }
        mbar_arrive_expect_tx(&v_full[s], L::kTileBytes);
#pragma unroll
        for (int b = 0; b < HD / 64; ++b)
          tma_load_2d(smem + L::kV + s * L::kTileBytes + b * 16384, &tm, &v_full[s],
                      d + h * HD + b * 64, key_row);
        issued[s] = true;
        issued_ph[s] = ph;
      }
      mbar_wait(q_full, 0);
      for (int s = 0; s < NS; ++s)
        if (issued[s]) {
          mbar_wait(&k_full[s], issued_ph[s]);
          mbar_wait(&v_full[s], issued_ph[s]);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, HD, false, true);
      const uint32_t sQ = smem_u32(smem + L::kQ);
      bool ok = mbar_wait(q_full, 0);
      tc_fence_after();
      auto issue_qk = [&](int j) -> bool {
        const int s = j % NS;
        if (!mbar_wait(&k_full[s], (j / NS) & 1)) return false;
        tc_fence_after();
        const uint32_t sK = smem_u32(smem + L::kK + s * L::kTileBytes);
        const uint32_t dS = tS + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(dS, desc_sw128(sQ + off, 16, 1024), desc_sw128(sK + off, 16, 1024), idesc_qk,
                  kk > 0);
        }
        umma_commit(&s_full[j & 1]);
        umma_commit(&k_empty[s]);
        return true;
      };
      if (ok) ok = issue_qk(0);
      for (int j = 0; ok && j < n_kt; ++j) {
        if (j + 1 < n_kt && !issue_qk(j + 1)) { ok = false; break; }
        if (!mbar_wait(&p_full[j & 1], (j >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const int s = j % NS;
        if (!mbar_wait(&v_full[s], (j / NS) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sV = smem_u32(smem + L::kV + s * L::kTileBytes);
        const uint32_t aP = tS + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          umma_ts(tO, aP + kk * 8, desc_sw128(sV + kk * 2048, 16384, 1024), idesc_pv,
                  (j > 0 || kk > 0));
        }
        umma_commit(&v_empty[s]);
      }
      if (!ok) *abort_flag = 1;
      umma_commit(o_full);   // also drains: fires once every MMA above is done
      mbar_wait(o_full, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int t = threadIdx.x - 64;           // 0..127 for cooperative loads
    const int q = warp & 3;                   // tensor-memory lane quarter
    const int row = q * 32 + lane;            // query row inside the tile
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    const int clamp = p.pos_clamp;
    const int nb = p.time_buckets;
    for (int k = t; k <= clamp; k += 128) s_rab_pos[k] = p.rab_pos[k];
    for (int k = t; k < nb; k += 128) {
      s_rab_time[k] = p.rab_time[k];
      s_thr[k] = p.thresholds[k];
    }
    {
      const int64_t kb0 = int64_t(n_a > 0 ? kt_begin : qt) * 128;
      s_kts[t] = (kb0 + t < p.T) ? p.ts[kb0 + t] : int64_t(0);
    }
    named_bar_sync(1, 128);

    const int64_t i = r0 + row;
    const bool valid = i < p.T;
    int64_t lo = i + 1, hi = 0, pos = 0, ti = 0;
    if (valid) {
      const RowInfo ri = p.rows[i];
      lo = (ri.lo < 0 || ri.lo > i) ? i : int64_t(ri.lo);
      hi = ri.hi;
      pos = ri.pos;
      ti = p.ts[i];
    }
    int b = 0;
    int64_t cut = ti;
    if (valid) {
      b = bucket_search(s_thr, nb, ti - p.ts[lo]);
      cut = ti - s_thr[b];
    }
    const int nn = p.n_norm_fixed > 0 ? p.n_norm_fixed : p.counters[0];
    const float inv_nn = 1.0f / float(nn > 0 ? nn : 1);
    bool aborted = false;

    for (int j = 0; j < n_kt; ++j) {
      const int64_t kb = int64_t(j < n_a ? kt_begin + j : qt) * 128;
      int64_t nxt = 0;
      if (j + 1 < n_kt) {
        const int64_t kbn = int64_t(j + 1 < n_a ? kt_begin + j + 1 : qt) * 128;
        nxt = (kbn + t < p.T) ? p.ts[kbn + t] : int64_t(0);
      }
      bool ok = aborted ? false : mbar_wait(&s_full[j & 1], (j >> 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        aborted = true;
        *abort_flag = 1;
      }
      if (!aborted) {
        tc_fence_after();
        const int64_t* kts = s_kts + (j & 1) * 128;
        const uint32_t taddr = tS + (j & 1) * 128 + lane_off;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float pv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int col = c * 32 + e + u;
              const int64_t jj = kb + col;
              const int64_t tk = kts[col];
              if (jj >= lo && jj <= i) {
                while (b > 0 && tk > cut) {
                  --b;
                  cut = ti - s_thr[b];
                }
              }
              int64_t dp = pos - jj;
              const int pidx = dp < 0 ? 0 : (dp > clamp ? clamp : int(dp));
              const float sc = __uint_as_float(r[e + u]) + s_rab_pos[pidx] + s_rab_time[b];
              const bool vis = (jj >= lo && jj < hi) || jj == i;
              const float hh = 0.5f * sc;
              const float sl = fmaf(hh, tanh_approx(hh), hh);
              pv[u] = vis ? sl : 0.0f;
              if constexpr (RECORD) {
                if (h == 0 && valid && jj < p.T) {
                  const int64_t at = i * p.T + jj;
                  p.dump_pidx[at] = pidx;
                  p.dump_tidx[at] = b;
                  p.dump_vis[at] = vis ? 1 : 0;
                }
              }
            }
            pk[e >> 1] = pack_bf16x2(pv[0], pv[1]);
          }
          tmem_st16(taddr + c * 16, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[j & 1]);
      }
      s_kts[((j + 1) & 1) * 128 + t] = nxt;
      named_bar_sync(1, 128);
    }

    bool ok = aborted ? false : mbar_wait(o_full, 0);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + lane_off + c * 32, r);
        tmem_ld_wait();
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(p.av + i * d + h * HD + c * 32);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(r[4 * e + 0]) * inv_nn,
                                 __uint_as_float(r[4 * e + 1]) * inv_nn,
                                 __uint_as_float(r[4 * e + 2]) * inv_nn,
                                 __uint_as_float(r[4 * e + 3]) * inv_nn);
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

template <int HD, bool RECORD>
cudaError_t launch_hd(const AttnArgs& a, cudaStream_t st) {
  using L = AttnLayout<HD>;
  CUtensorMap tm;
  if (!make_tmap_2d_bf16(&tm, a.uvqk, uint64_t(4 * a.d), uint64_t(a.T), uint64_t(4 * a.d) * 2,
                         64, 128))
    return cudaErrorInvalidValue;
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<HD, RECORD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(L::kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  AttnParams p;
  p.rows = a.rows;
  p.order = a.order;
  p.ts = a.ts;
  p.thresholds = a.thresholds;
  p.rab_pos = a.rab_pos;
  p.rab_time = a.rab_time;
  p.counters = a.counters;
  p.error = a.error;
  p.av = a.av;
  p.T = a.T;
  p.d = a.d;
  p.H = a.H;
  p.pos_clamp = a.pos_clamp;
  p.time_buckets = a.time_buckets;
  p.n_norm_fixed = a.n_norm_fixed;
  p.dump_pidx = a.dump_pidx;
  p.dump_tidx = a.dump_tidx;
  p.dump_vis = a.dump_vis;
  const int64_t grid = int64_t(a.num_qtiles) * a.H;
  attn_tc_kernel<HD, RECORD><<<unsigned(grid), 192, L::kSmemBytes, st>>>(tm, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_tc(const AttnArgs& a, cudaStream_t st, bool record) {
  if (a.T <= 0) return cudaSuccess;
  if (a.pos_clamp >= kMaxPosEntries || a.time_buckets > kMaxTimeBuckets) return cudaErrorInvalidValue;
  if (a.hd == 128) return record ? launch_hd<128, true>(a, st) : launch_hd<128, false>(a, st);
  if (a.hd == 64) return record ? launch_hd<64, true>(a, st) : launch_hd<64, false>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace hstu
