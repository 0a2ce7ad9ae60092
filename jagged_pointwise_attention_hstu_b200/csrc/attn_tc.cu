// Fused jagged pointwise attention on the tcgen05 tensor cores.
//
// Equation (2) of the HSTU layer (blog "Generative Recommendation 16: HSTU",
// section "HSTU Layer 到底改了什么"):
//     O_i = sum_{j visible} SiLU(q_i . k_j + rab_pos[p(i,j)] + rab_time[t(i,j)]) v_j / n_norm
// The SiLU acts on each score alone: there is no softmax along the sequence
// (same blog, section "不对序列做 softmax"), hence no running maximum and no
// rescaling of the accumulator, and the n x n score matrix is never stored.
//
// One CTA computes one (128-query tile, head) work item with 10 warps:
//   warp 0      TMA: Q once, then K and V tiles into NS-stage rings
//   warp 1      MMA issue: S_j = Q K_j^T into tensor-memory score buffer j % 2
//               (SS form, both operands K-major in shared memory), and
//               O += P_j V_j with P_j read back from tensor memory (TS form,
//               V consumed N-major straight from its row-major tile)
//   warps 2-5   row group 0, one query row per thread, key tiles j = 0, 2, 4..
//   warps 6-9   row group 1, same rows, key tiles j = 1, 3, 5..
// A row group reads S_j from tensor memory, adds the position and time
// biases, applies the mask and SiLU and writes P_j (bf16) over the first half
// of S_j's columns, while the tensor cores run S_{j+1} and P_{j-1} V_{j-1}.
//
// Key tiles: only tiles that hold a visible key for some row of the query
// tile are visited (see sched.cu); the last one is always the diagonal tile.
// Work items are ordered head-major, so the CTAs resident at one time share
// one head's K and V in L2.
//
// Bias buckets without a per-score logarithm.  Timestamps are non-decreasing
// inside a user, so along a row the gap t_i - t_j only shrinks as j grows.
// Each row keeps its current time bucket b and the key-timestamp cut
// t_i - thr[b] (thr[k] = the smallest integer gap of bucket >= k, built on the
// host from the fp64 rule), so an integer compare reproduces
// floor(ln(1 + dt) / div) exactly.  Per (warp, key tile) the rows are
// classified once:
//   kFast  every key visible to every row of the warp and one time bucket per
//          row: the whole bias is a per-row constant (plus the position
//          gather when the position bucket is not clamped);
//   kMed   every key visible, at most two time buckets per row: one 32-bit
//          compare of the key's timestamp (relative to the tile's first key)
//          against the row's cut picks the bias;
//   kGen   anything else (diagonal tiles, user and history boundaries): the
//          mask, the position clamp and the bucket walk per score.
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
constexpr int kThreads = 320;
constexpr int kFast = 0, kMed = 1, kGen = 2;

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
  int d, H, num_qtiles;
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
  static constexpr uint32_t kKts = kThr + kMaxTimeBuckets * 8;       // int64 [group][buf][128]
  static constexpr uint32_t kKrel = kKts + 2 * 2 * 128 * 8;          // int32 [group][buf][128]
  static constexpr uint32_t kBars = kKrel + 2 * 2 * 128 * 4;
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

// Moves the row's bucket down to the bucket of a key with timestamp tk.
__device__ __forceinline__ void walk_to(int& b, int64_t& cut, int64_t tk, int64_t ti,
                                        const int64_t* thr) {
  while (b > 0 && tk > cut) {
    --b;
    cut = ti - thr[b];
  }
}

__device__ __forceinline__ int clamp_i32(int64_t v, int lo, int hi) {
  return v < lo ? lo : (v > hi ? hi : int(v));
}

__device__ __forceinline__ float silu_half(float hh) {
  // SiLU(s) with hh = s / 2:  s * sigmoid(s) = hh * (1 + tanh(hh))
  return fmaf(hh, tanh_approx(hh), hh);
}

// Per-row state of one row group for the current key tile.
struct Row {
  int lo_rel, hi_rel, i_rel, pos_rel;  // relative to the tile's first key, clamped
  int b, b_last;                        // time bucket at the walk position / tile end
  int64_t ti, cut, cut_last;
  float hc, hc_hi, hc_lo;               // half-bias constants of the fast paths
  int cutr;                             // 32-bit cut relative to the tile's first key
};

struct Record {
  int32_t* pidx;
  int32_t* tidx;
  uint8_t* vis;
  int64_t T, i, kb;
  bool on;
};

template <int MODE, bool PC, bool RECORD>
__device__ __forceinline__ void score_tile(uint32_t taddr, Row& R, const float* s_rp,
                                           const float* s_rt, const int64_t* s_thr,
                                           const int64_t* kts, const int32_t* krel, int clamp,
                                           const Record& rec) {
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    uint32_t r[32];
    tmem_ld32(taddr + c * 32, r);
    tmem_ld_wait();
    int kr[32];
    if constexpr (MODE == kMed) {
      const int4* k4 = reinterpret_cast<const int4*>(krel + c * 32);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int4 v = k4[q];
        kr[4 * q + 0] = v.x; kr[4 * q + 1] = v.y; kr[4 * q + 2] = v.z; kr[4 * q + 3] = v.w;
      }
    }
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      float pv[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int jr = c * 32 + e + u;
        const float acc = __uint_as_float(r[e + u]);
        if constexpr (MODE == kFast || MODE == kMed) {
          float add;
          int tb = R.b;
          if constexpr (MODE == kFast) {
            add = R.hc;
          } else {
            const bool hi = kr[e + u] <= R.cutr;
            add = hi ? R.hc_hi : R.hc_lo;
            tb = hi ? R.b : R.b_last;
          }
          int pidx = clamp;
          if constexpr (!PC) {
            pidx = min(R.pos_rel - jr, clamp);
            add = fmaf(0.5f, s_rp[pidx], add);
          }
          pv[u] = silu_half(fmaf(acc, 0.5f, add));
          if constexpr (RECORD) {
            if (rec.on) {
              const int64_t at = rec.i * rec.T + rec.kb + jr;
              rec.pidx[at] = pidx;
              rec.tidx[at] = tb;
              rec.vis[at] = 1;
            }
          }
        } else {
          const int64_t tk = kts[jr];
          if (jr >= R.lo_rel && jr <= R.i_rel) walk_to(R.b, R.cut, tk, R.ti, s_thr);
          const int dp = R.pos_rel - jr;
          const int pidx = dp < 0 ? 0 : (dp > clamp ? clamp : dp);
          const bool vis = (unsigned(jr - R.lo_rel) < unsigned(R.hi_rel - R.lo_rel)) ||
                           jr == R.i_rel;
          const float sc = acc + s_rp[pidx] + s_rt[R.b];
          pv[u] = vis ? silu_half(0.5f * sc) : 0.0f;
          if constexpr (RECORD) {
            if (rec.on && rec.kb + jr < rec.T) {
              const int64_t at = rec.i * rec.T + rec.kb + jr;
              rec.pidx[at] = pidx;
              rec.tidx[at] = R.b;
              rec.vis[at] = vis ? 1 : 0;
            }
          }
        }
      }
      pk[e >> 1] = pack_bf16x2(pv[0], pv[1]);
    }
    tmem_st16(taddr + c * 16, pk);
  }
}

template <int HD, bool RECORD>
__global__ void __launch_bounds__(kThreads, 1)
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
  int32_t* s_krel = reinterpret_cast<int32_t*>(smem + L::kKrel);
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

  // ---- work item (head-major) and its key-tile range
  const int w = blockIdx.x;
  const int h = w / p.num_qtiles;
  const int qt = p.order[w % p.num_qtiles];
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
    // ------------------------------------------------------------ row groups
    const int g = (warp - 2) >> 2;             // row group 0 or 1
    const int t = threadIdx.x - 64 - 128 * g;  // 0..127 inside the group
    const int q = warp & 3;                    // tensor-memory lane quarter
    const int row = q * 32 + lane;             // query row inside the tile
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    const int clamp = p.pos_clamp;
    const int nb = p.time_buckets;
    const int bar_id = 1 + g;
    // tables: each group loads half, then both groups meet once
    for (int k = threadIdx.x - 64; k <= clamp; k += 256) s_rab_pos[k] = p.rab_pos[k];
    for (int k = threadIdx.x - 64; k < nb; k += 256) {
      s_rab_time[k] = p.rab_time[k];
      s_thr[k] = p.thresholds[k];
    }
    int64_t* kts_g = s_kts + g * 256;
    int32_t* krel_g = s_krel + g * 256;
    auto key_base = [&](int j) -> int64_t { return int64_t(j < n_a ? kt_begin + j : qt) * 128; };
    auto load_key = [&](int j, int64_t& tsv, int32_t& rel) {
      const int64_t kb = key_base(j);
      const int64_t t0 = p.ts[kb];
      tsv = (kb + t < p.T) ? p.ts[kb + t] : t0;
      const int64_t dr = tsv - t0;
      rel = dr < 0 ? 0 : (dr > 0x7FFFFFFF ? 0x7FFFFFFF : int32_t(dr));
    };
    if (g < n_kt) {
      int64_t tsv;
      int32_t rel;
      load_key(g, tsv, rel);
      kts_g[t] = tsv;
      krel_g[t] = rel;
    }
    named_bar_sync(3, 256);

    const int64_t i = r0 + row;
    const bool valid = i < p.T;
    int64_t lo = 0, hi = 0, pos = 0;   // rows past T see nothing
    Row R;
    R.ti = 0;
    if (valid) {
      const RowInfo ri = p.rows[i];
      lo = (ri.lo < 0 || ri.lo > i) ? i : int64_t(ri.lo);
      hi = ri.hi;
      pos = ri.pos;
      R.ti = p.ts[i];
    }
    R.b = 0;
    R.cut = R.ti;
    if (valid) {
      R.b = bucket_search(s_thr, nb, R.ti - p.ts[lo]);
      R.cut = R.ti - s_thr[R.b];
    }
    const int nn = p.n_norm_fixed > 0 ? p.n_norm_fixed : p.counters[0];
    const float inv_nn = 1.0f / float(nn > 0 ? nn : 1);
    bool aborted = false;

    int n = 0;
    for (int j = g; j < n_kt; j += 2, ++n) {
      const int buf = n & 1;
      const int64_t kb = key_base(j);
      int64_t nxt_ts = 0;
      int32_t nxt_rel = 0;
      if (j + 2 < n_kt) load_key(j + 2, nxt_ts, nxt_rel);
      const int64_t* kts = kts_g + buf * 128;
      const int32_t* krel = krel_g + buf * 128;

      // ---- classify this row for the tile
      R.lo_rel = clamp_i32(lo - kb, -1, 129);
      R.hi_rel = clamp_i32(hi - kb, -1, 129);
      R.i_rel = valid ? clamp_i32(i - kb, -1, 129) : -1;
      R.pos_rel = clamp_i32(pos - kb, -1, clamp + 129);
      const bool full = valid && lo <= kb && hi >= kb + 128;
      const bool posc = (pos - (kb + 127)) >= clamp;
      int lev = 99;
      if (full) {
        walk_to(R.b, R.cut, kts[0], R.ti, s_thr);
        R.b_last = R.b;
        R.cut_last = R.cut;
        walk_to(R.b_last, R.cut_last, kts[127], R.ti, s_thr);
        lev = R.b - R.b_last;
      }
      const bool wide = (kts[127] - kts[0]) >= int64_t(0x7FFFFFFE);
      const int mode = __all_sync(0xffffffffu, full && lev == 0)
                           ? kFast
                           : (__all_sync(0xffffffffu, full && lev <= 1 && !wide) ? kMed : kGen);
      const bool pc = __all_sync(0xffffffffu, posc);
      if (mode != kGen) {
        const float rp_c = pc ? s_rab_pos[clamp] : 0.0f;
        R.hc_hi = 0.5f * (rp_c + s_rab_time[R.b]);
        R.hc_lo = 0.5f * (rp_c + s_rab_time[R.b_last]);
        R.hc = R.hc_hi;
        const int64_t cr = R.cut - kts[0];
        R.cutr = cr < -1 ? -1 : (cr > 0x7FFFFFFE ? 0x7FFFFFFE : int32_t(cr));
      }
      Record rec;
      rec.pidx = p.dump_pidx;
      rec.tidx = p.dump_tidx;
      rec.vis = p.dump_vis;
      rec.T = p.T;
      rec.i = i;
      rec.kb = kb;
      rec.on = RECORD && h == 0 && valid;

      bool ok = aborted ? false : mbar_wait(&s_full[j & 1], (j >> 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        aborted = true;
        *abort_flag = 1;
      }
      if (!aborted) {
        tc_fence_after();
        const uint32_t taddr = tS + (j & 1) * 128 + lane_off;
        if (mode == kFast) {
          if (pc) score_tile<kFast, true, RECORD>(taddr, R, s_rab_pos, s_rab_time, s_thr, kts, krel, clamp, rec);
          else score_tile<kFast, false, RECORD>(taddr, R, s_rab_pos, s_rab_time, s_thr, kts, krel, clamp, rec);
        } else if (mode == kMed) {
          if (pc) score_tile<kMed, true, RECORD>(taddr, R, s_rab_pos, s_rab_time, s_thr, kts, krel, clamp, rec);
          else score_tile<kMed, false, RECORD>(taddr, R, s_rab_pos, s_rab_time, s_thr, kts, krel, clamp, rec);
        } else {
          score_tile<kGen, false, RECORD>(taddr, R, s_rab_pos, s_rab_time, s_thr, kts, krel, clamp, rec);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[j & 1]);
      }
      if (mode != kGen) {
        R.b = R.b_last;
        R.cut = R.cut_last;
      }
      kts_g[(buf ^ 1) * 128 + t] = nxt_ts;
      krel_g[(buf ^ 1) * 128 + t] = nxt_rel;
      named_bar_sync(bar_id, 128);
    }

    bool ok = aborted ? false : mbar_wait(o_full, 0);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      // group g writes the columns [g * HD / 2, (g + 1) * HD / 2) of its rows
#pragma unroll 1
      for (int c = g * (HD / 64); c < (g + 1) * (HD / 64); ++c) {
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
  p.num_qtiles = a.num_qtiles;
  p.pos_clamp = a.pos_clamp;
  p.time_buckets = a.time_buckets;
  p.n_norm_fixed = a.n_norm_fixed;
  p.dump_pidx = a.dump_pidx;
  p.dump_tidx = a.dump_tidx;
  p.dump_vis = a.dump_vis;
  const int64_t grid = int64_t(a.num_qtiles) * a.H;
  attn_tc_kernel<HD, RECORD><<<unsigned(grid), kThreads, L::kSmemBytes, st>>>(tm, p);
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
