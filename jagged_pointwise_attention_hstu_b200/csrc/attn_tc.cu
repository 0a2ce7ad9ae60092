// Fused jagged pointwise attention on the tcgen05 tensor cores.
//
// Equation (2) of the HSTU layer (blog "Generative Recommendation 16: HSTU",
// section "HSTU Layer 到底改了什么"):
//     O_i = sum_{j visible} SiLU(q_i . k_j + rab_pos[p(i,j)] + rab_time[t(i,j)]) v_j / n_norm
// The SiLU acts on each score alone: there is no softmax along the sequence
// (same blog, section "不对序列做 softmax"), hence no running maximum and no
// rescaling of the accumulator, and the n x n score matrix is never stored.
//
// Two kernels compute it.  Head dim 128 runs on the CTA-pair kernel at the end
// of this file (clusters of two SMs, cta_group::2 products, persistent over the
// work items, three row groups); head dim 64 and the bucket-recording variant
// run on this one.
//
// One CTA computes one work item -- a pair of adjacent 128-query tiles and
// one head -- with 12 warps:
//   warp 0      TMA: both Q tiles once, then K tiles into an NSK-stage ring and
//               the tiles' key timestamps into a 4-stage ring
//   warp 1      MMA issue for query tile 0, warp 3 for query tile 1:
//               S_q = Q_q K_j^T into tensor-memory score buffer q (SS form, both
//               operands K-major in shared memory) and O_q += P_q V_j with P_q
//               read back from tensor memory (TS form, V consumed N-major
//               straight from its row-major tile).  Two issuing threads keep the
//               tensor pipe fed while either one waits for its row group.
//   warp 2      TMA: V tiles into an NSV-stage ring
//   warps 4-7   row group 0: one row of query tile 0 per thread
//   warps 8-11  row group 1: one row of query tile 1 per thread
// A row group reads S_q from tensor memory, adds the position and time
// biases, applies the mask and SiLU and writes P_q (bf16) over the first half
// of S_q's columns.  While one group scores key tile j, the tensor cores run
// the other group's products, and every K and V tile loaded feeds both query
// tiles, which halves the K/V traffic per flop.  At the end each group scales
// its O_q by 1/n_norm, stages it in Q_q's (now free) shared buffer and writes
// it with TMA stores.
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
// floor(ln(1 + dt) / div) exactly.  The keys' timestamps arrive by TMA with
// each V tile.  Per (warp, key tile) the rows are classified once:
//   kFast  every key visible to every row of the warp and one time bucket per
//          row: the whole bias is a per-row constant (plus the position
//          gather when the position bucket is not clamped);
//   kMed   every key visible, at most two time buckets per row: the column
//          where the row's bucket drops is found once per tile (a binary
//          search over the tile's sorted key timestamps) and each score
//          compares its column with it;
//   kCut   every key visible, at most four time buckets per row: three such
//          split columns and a select chain;
//   kAny   any visibility (the causal diagonal, user and history boundaries,
//          M-FALCON candidates) with every visible gap of the warp's rows
//          below 2^31: the full mask per score and the exact bucket of each
//          gap without a walk -- v = dt + 1 falls in a bin (floor(log2 v) and
//          the next two bits) spanning less than one bucket; a per-CTA table
//          gives, per bin, the next bucket's integer threshold and both
//          candidate biases, so one 16-byte shared load and one compare give
//          the time bias;
//   kGen   anything else (the table is not exact for the divisor, or a gap of
//          2^31 or more): the full mask, position clamp and bucket walk per
//          score;
//   kSelf  no row of the warp sees a key of the tile other than itself (the
//          M-FALCON candidates on their own tiles: a candidate sees the history
//          and itself only): one SiLU per row, the rest of P is 0.
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
constexpr int kThreads = 384;
constexpr int kPairThreads = 512;   // CTA-pair kernel: one load/MMA warpgroup, three row groups
// The shared copy of rab_pos is padded on both sides with its end values, so
// that any relative position pos_rel - column in [-kPosPad, clamp + kPosPad]
// reads the clamped entry without a min/max.
constexpr int kPosPad = 130;
constexpr int kFast = 0, kMed = 1, kCut = 2, kAny = 3, kGen = 4, kZero = 5, kSelf = 6;

struct AttnParams {
  const RowInfo* rows;
  const int32_t* order;
  const int64_t* ts;
  const int64_t* thresholds;
  const uint8_t* time_lut;
  const int32_t* thr32;
  const float* rab_pos;
  const float* rab_time;
  const int32_t* counters;
  int32_t* error;
  float* av;
  int64_t T;
  int d, H, num_pairs;
  int pos_clamp, time_buckets;
  int n_norm_fixed;
  int lut_exact;
  int num_splits;     // 2: each pair's key range is split over two CTAs
  long long wait_limit;
  int32_t* dump_pidx;
  int32_t* dump_tidx;
  uint8_t* dump_vis;
};

template <int HD>
struct AttnLayout {
  static constexpr int NSK = HD == 128 ? 2 : 3;   // K ring stages
  static constexpr int NSV = HD == 128 ? 2 : 3;   // V ring stages
  static constexpr uint32_t kTileBytes = 128 * HD * 2;
  static constexpr uint32_t kQ = 0;                                  // two Q tiles
  static constexpr uint32_t kK = kQ + 2 * kTileBytes;
  static constexpr uint32_t kV = kK + NSK * kTileBytes;
  static constexpr int NST = 4;                   // key-timestamp ring stages
  static constexpr uint32_t kKts = kV + NSV * kTileBytes;            // int64 [stage][128], TMA
  static constexpr uint32_t kThr = kKts + NST * 128 * 8;
  static constexpr uint32_t kThr32 = kThr + kMaxTimeBuckets * 8;     // int32 [257] (+pad)
  static constexpr uint32_t kLut = kThr32 + 260 * 4;                 // uint8 [128]
  static constexpr uint32_t kAnyTab = kLut + 128;                    // int4 [128]
  static constexpr uint32_t kRabTime = kAnyTab + 128 * 16;
  static constexpr uint32_t kBars = kRabTime + kMaxTimeBuckets * 4;
  // float [clamp + 1 + 2 kPosPad]: rab_pos[clamp(k, 0, clamp)] at k + kPosPad
  static constexpr uint32_t kRabPos = kBars + 256;
  static __host__ __device__ constexpr uint32_t smem_bytes(int clamp) {
    return kRabPos + ((uint32_t(clamp + 1 + 2 * kPosPad) * 4 + 15) / 16) * 16 + 1024;
  }
  // every TMA destination starts on a 1024-byte (swizzled tiles) or 128-byte boundary
  static_assert(kQ % 1024 == 0 && kK % 1024 == 0 && kV % 1024 == 0, "tile alignment");
  static_assert(kTileBytes % 1024 == 0, "tile stride alignment");
  static_assert(kKts % 128 == 0, "timestamp stage alignment");
  static_assert(kBars % 8 == 0, "mbarrier alignment");
  // O of query tile q is staged for its TMA stores in Q_q's tile, in two passes:
  // per warp a quarter of the tile holds HD / 64 boxes of 32 rows x 32 fp32 columns
  static_assert((kTileBytes / 4) % 4096 == 0 && (kTileBytes / 4) / 4096 == HD / 64, "O staging");
  static_assert(smem_bytes(kMaxPosEntries - 1) <= 227 * 1024, "shared memory budget");
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
  float hc2, hc3;                       // kCut: half-bias of buckets b - 2, b - 3
  int j1, j2, j3;                       // kMed/kCut: keys from column j_m on drop one more bucket
  uint32_t ti_lo;                       // low 32 bits of t_i (kMed, kCut, kAny)
};

struct Record {
  int32_t* pidx;
  int32_t* tidx;
  uint8_t* vis;
  int64_t T, i, kb;
  bool on;
};

// One score element: returns P (bf16-ready float) for key column jr of the tile.
template <int MODE, bool PC, bool RECORD>
__device__ __forceinline__ float score_one(float acc, int jr, int64_t tk, Row& R,
                                           const float* s_rp, const float* s_rt,
                                           const int64_t* s_thr, const uint8_t* s_lut,
                                           const int32_t* s_thr32, int clamp, const Record& rec) {
  if constexpr (MODE == kFast || MODE == kMed || MODE == kCut) {
    float add = R.hc;
    int tb = R.b;
    if constexpr (MODE != kFast) {
      // timestamps are sorted inside the user: the gap shrinks as the column grows
      const bool d1 = jr >= R.j1;
      add = d1 ? R.hc_lo : R.hc;
      if constexpr (RECORD) tb = R.b - (d1 ? 1 : 0);
      if constexpr (MODE == kCut) {
        const bool d2 = jr >= R.j2;
        const bool d3 = jr >= R.j3;
        add = d2 ? (d3 ? R.hc3 : R.hc2) : add;
        if constexpr (RECORD) tb -= (d2 ? 1 : 0) + (d3 ? 1 : 0);
      }
    }
    if constexpr (!PC) add = fmaf(0.5f, s_rp[-jr], add);
    if constexpr (RECORD) {
      const int pidx = PC ? clamp : min(R.pos_rel - jr, clamp);
      if (rec.on) {
        const int64_t at = rec.i * rec.T + rec.kb + jr;
        rec.pidx[at] = pidx;
        rec.tidx[at] = tb;
        rec.vis[at] = 1;
      }
    }
    return silu_half(fmaf(acc, 0.5f, add));
  } else if constexpr (MODE == kAny) {
    const bool vis = (unsigned(jr - R.lo_rel) < unsigned(R.hi_rel - R.lo_rel)) || jr == R.i_rel;
    const uint32_t dd = R.ti_lo - uint32_t(tk);     // the gap; < 2^31 - 1 for visible keys
    // masked keys may hold any gap (even -1, i.e. v = 0): keep v >= 1 so the
    // table index stays in [0, 127] for every input
    const uint32_t v = max(dd + 1u, 1u);
    // the bin index floor(log2 v) * 4 + the next two bits of v, read off the
    // exponent and top mantissa bits of v converted with truncation (exact:
    // truncation never carries into the exponent); the conversion runs beside
    // the tanh instead of competing with it on the multi-function unit, as a
    // leading-zero count would
    const uint32_t fb = __float_as_uint(__uint2float_rz(v));
    const int idx = int((fb >> 21) - 508u) & 127;
    const int4 ent = reinterpret_cast<const int4*>(s_lut)[idx];   // {thr, rt_lo, rt_hi, cand}
    const bool up = int(dd) >= ent.x;
    const float rt = __int_as_float(up ? ent.z : ent.y);
    if constexpr (RECORD) {
      const int pidx = min(max(R.pos_rel - jr, 0), clamp);
      if (rec.on && rec.kb + jr < rec.T) {
        const int64_t at = rec.i * rec.T + rec.kb + jr;
        rec.pidx[at] = pidx;
        rec.tidx[at] = ent.w + (up ? 1 : 0);
        rec.vis[at] = vis ? 1 : 0;
      }
    }
    const float hh = 0.5f * (acc + s_rp[-jr] + rt);
    return vis ? silu_half(hh) : 0.0f;
  } else {
    if (jr >= R.lo_rel && jr <= R.i_rel) walk_to(R.b, R.cut, tk, R.ti, s_thr);
    const bool vis = (unsigned(jr - R.lo_rel) < unsigned(R.hi_rel - R.lo_rel)) || jr == R.i_rel;
    if constexpr (RECORD) {
      const int dp = R.pos_rel - jr;
      const int pidx = dp < 0 ? 0 : (dp > clamp ? clamp : dp);
      if (rec.on && rec.kb + jr < rec.T) {
        const int64_t at = rec.i * rec.T + rec.kb + jr;
        rec.pidx[at] = pidx;
        rec.tidx[at] = R.b;
        rec.vis[at] = vis ? 1 : 0;
      }
    }
    const float sc = acc + s_rp[-jr] + s_rt[R.b];
    return vis ? silu_half(0.5f * sc) : 0.0f;
  }
}

template <int MODE, bool PC, bool RECORD>
__device__ __forceinline__ void score_chunk(const uint32_t (&r)[16], int c, uint32_t taddr,
                                            Row& R, const float* s_rp, const float* s_rt,
                                            const int64_t* s_thr, const uint8_t* s_lut,
                                            const int32_t* s_thr32, const int64_t* kts, int clamp,
                                            const Record& rec) {
  uint32_t pk[8];
  const longlong2* k2 = reinterpret_cast<const longlong2*>(kts + c * 16);
#pragma unroll
  for (int e = 0; e < 16; e += 2) {
    int64_t t0 = 0, t1 = 0;
    if constexpr (MODE == kAny || MODE == kGen) {
      const longlong2 kk = k2[e >> 1];
      t0 = kk.x;
      t1 = kk.y;
    }
    const float p0 = score_one<MODE, PC, RECORD>(__uint_as_float(r[e]), c * 16 + e, t0, R, s_rp,
                                                 s_rt, s_thr, s_lut, s_thr32, clamp, rec);
    const float p1 = score_one<MODE, PC, RECORD>(__uint_as_float(r[e + 1]), c * 16 + e + 1, t1,
                                                 R, s_rp, s_rt, s_thr, s_lut, s_thr32, clamp, rec);
    pk[e >> 1] = pack_bf16x2(p0, p1);
  }
  tmem_st8(taddr + c * 8, pk);
}

// Writes P = 0 for a tile whose keys are all later than every row of the warp.
template <bool RECORD>
__device__ __forceinline__ void zero_tile(uint32_t taddr, const Record& rec) {
  uint32_t pk[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) pk[e] = 0u;
#pragma unroll
  for (int c = 0; c < 8; ++c) tmem_st8(taddr + c * 8, pk);
  if constexpr (RECORD) {
    if (rec.on)
      for (int jr = 0; jr < 128 && rec.kb + jr < rec.T; ++jr) {
        const int64_t at = rec.i * rec.T + rec.kb + jr;
        rec.pidx[at] = 0;
        rec.tidx[at] = 0;
        rec.vis[at] = 0;
      }
  }
}

// Writes P for a tile in which the only key a row may see is the row itself
// (column i_rel; its gap is 0, so its time bucket is 0): one SiLU per row.
// The warp's rows are consecutive, so their own columns fall in at most two
// 16-key chunks, which are the only ones read.
template <bool RECORD>
__device__ __forceinline__ void self_tile(uint32_t taddr, const Row& R, const float* rp_row,
                                          const float* s_rt, int clamp, const Record& rec) {
  const int cs = (R.i_rel >= 0 && R.i_rel < 128) ? R.i_rel : -1;   // own column, or none
  float p_self = 0.0f;
#pragma unroll 1
  for (int c = 0; c < 8; ++c) {
    if (!__any_sync(0xffffffffu, cs >= 0 && (cs >> 4) == c)) continue;
    uint32_t r[16];
    tmem_ld16(taddr + c * 16, r);
    tmem_ld_wait();
    if (cs >= 0 && (cs >> 4) == c) {
      float sv = 0.0f;
#pragma unroll
      for (int e = 0; e < 16; ++e) sv = e == (cs & 15) ? __uint_as_float(r[e]) : sv;
      p_self = silu_half(0.5f * (sv + rp_row[-cs] + s_rt[0]));
    }
  }
  const uint32_t val = (cs & 1) ? pack_bf16x2(0.0f, p_self) : pack_bf16x2(p_self, 0.0f);
#pragma unroll 1
  for (int c = 0; c < 8; ++c) {
    uint32_t pk[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) pk[e] = (cs >= 0 && (cs >> 4) == c && ((cs & 15) >> 1) == e) ? val : 0u;
    tmem_st8(taddr + c * 8, pk);
  }
  if constexpr (RECORD) {
    if (rec.on && cs >= 0 && rec.kb + cs < rec.T) {
      const int64_t at = rec.i * rec.T + rec.kb + cs;
      const int dp = R.pos_rel - cs;
      rec.pidx[at] = dp < 0 ? 0 : (dp > clamp ? clamp : dp);
      rec.tidx[at] = 0;
      rec.vis[at] = 1;
    }
  }
}

// Scores one 128-key tile of S for this thread's row and writes P over its
// first 64 columns, 16 keys at a time; the tensor-memory load of the next 16
// scores overlaps the SiLU of the current ones.  P chunk c lands on columns
// [8c, 8c + 8), which hold scores already consumed.  On the masked paths a
// chunk whose keys are all later than every row of the warp is written as 0
// without being scored.
template <int MODE, bool PC, bool RECORD>
__device__ __forceinline__ void score_tile(uint32_t taddr, Row& R, const float* s_rp,
                                           const float* s_rt, const int64_t* s_thr,
                                           const uint8_t* s_lut, const int32_t* s_thr32,
                                           const int64_t* kts, int clamp, const Record& rec,
                                           uint64_t* half_bar) {
  int live = 8;   // chunks holding a key visible to some row of the warp
  if constexpr (MODE == kAny || MODE == kGen) {
    int last = R.i_rel;   // every visible key of the row is <= its own column
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
    live = min(8, last / 16 + 1);
  }
  uint32_t ra[16], rb[16];
  tmem_ld16(taddr, ra);
  tmem_ld_wait();
#pragma unroll 1
  for (int c = 0; c < 8; c += 2) {
    if (c >= live) {
      uint32_t pk[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) pk[e] = 0u;
      tmem_st8(taddr + c * 8, pk);
      tmem_st8(taddr + (c + 1) * 8, pk);
      if (c == 2) {
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(half_bar);
      }
      if constexpr (RECORD) {
        if (rec.on)
          for (int jr = c * 16; jr < 128 && rec.kb + jr < rec.T; ++jr) {
            const int64_t at = rec.i * rec.T + rec.kb + jr;
            rec.pidx[at] = 0;
            rec.tidx[at] = 0;
            rec.vis[at] = 0;
          }
      }
      continue;
    }
    tmem_ld16(taddr + (c + 1) * 16, rb);
    score_chunk<MODE, PC, RECORD>(ra, c, taddr, R, s_rp, s_rt, s_thr, s_lut, s_thr32, kts, clamp, rec);
    tmem_ld_wait();
    if (c + 2 < 8) tmem_ld16(taddr + (c + 2) * 16, ra);
    score_chunk<MODE, PC, RECORD>(rb, c + 1, taddr, R, s_rp, s_rt, s_thr, s_lut, s_thr32, kts, clamp, rec);
    tmem_ld_wait();
    if (c == 2) {   // P of the first 64 keys is written: their products may start
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(half_bar);
    }
  }
}

template <int HD, bool RECORD>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm, const __grid_constant__ CUtensorMap tm_ts,
                   const __grid_constant__ CUtensorMap tm_o,
                   const AttnParams p) {
  using L = AttnLayout<HD>;
  constexpr int NSK = L::NSK;
  constexpr int NSV = L::NSV;
  constexpr int NST = L::NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* s_rab_pos = reinterpret_cast<float*>(smem + L::kRabPos);
  float* s_rab_time = reinterpret_cast<float*>(smem + L::kRabTime);
  int64_t* s_thr = reinterpret_cast<int64_t*>(smem + L::kThr);
  int32_t* s_thr32 = reinterpret_cast<int32_t*>(smem + L::kThr32);
  uint8_t* s_lut = reinterpret_cast<uint8_t*>(smem + L::kLut);
  int4* s_any = reinterpret_cast<int4*>(smem + L::kAnyTab);
  int64_t* s_kts = reinterpret_cast<int64_t*>(smem + L::kKts);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;
  uint64_t* k_empty = k_full + NSK;
  uint64_t* v_full = k_empty + NSK;
  uint64_t* v_empty = v_full + NSV;
  uint64_t* s_full = v_empty + NSV;  // [2] one per query tile
  uint64_t* p_full = s_full + 2;     // [2]
  uint64_t* o_full = p_full + 2;     // [2] every product of a query tile is done
  uint64_t* drained = o_full + 2;    // [2] every MMA of one issuer is done
  uint64_t* t_full = drained + 2;    // [NST] key timestamps of a tile landed
  uint64_t* t_empty = t_full + NST;  // [NST] every row-group warp is done with them
  uint64_t* p_half = t_empty + NST;  // [2] P of the first 64 keys written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(p_half + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int d = p.d;

  // ---- work item (head-major, then the pairs longest first, then the key-range
  // splits of a pair) and its key tiles
  const int w = blockIdx.x;
  const int per_head = p.num_pairs * p.num_splits;
  const int h = w / per_head;
  const int pr = p.order[(w % per_head) / p.num_splits];
  const int split = (w % per_head) % p.num_splits;
  const int qt0 = 2 * pr;
  const PairTiles pt = pair_tiles(p.rows, p.T, pr);
  const int nq = pt.n_diag;              // query tiles in this pair (1 or 2)
  const int n_a = pt.n_a;
  const int n_all = n_a + nq;            // the pair's key tiles, of which this item takes
  const int jb = split * n_all / p.num_splits;
  const int n_kt = (split + 1) * n_all / p.num_splits - jb;   // [jb, jb + n_kt)
  if (n_kt <= 0) return;   // more splits than key tiles (uniform over the CTA)
  auto key_tile = [&](int j) -> int {
    j += jb;
    return j < n_a ? pt.a_lo + j : qt0 + (j - n_a);
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], nq);   // one commit per MMA issuer
    }
    for (int s = 0; s < NSV; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], nq);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 128);
    }
    mbar_init(&p_half[0], 128);
    mbar_init(&p_half[1], 128);
    mbar_init(&o_full[0], 1);
    mbar_init(&o_full[1], 1);
    mbar_init(&drained[0], 1);
    mbar_init(&drained[1], 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&t_full[s], 1);
      mbar_init(&t_empty[s], 4 * nq);   // the warps of every row group that has rows
    }
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
  // columns: S_0 [0,128), S_1 [128,256), O_0 [256, 256+HD), O_1 [256+HD, 256+2HD)
  auto tS = [&](int q) -> uint32_t { return tmem_base + q * 128; };
  auto tO = [&](int q) -> uint32_t { return tmem_base + 256 + q * HD; };

  if (warp == 0) {
    // ------------------------------------------------------------ Q, K and key timestamp loads
    if (lane == 0) {
      prefetch_tmap(&tm);
      prefetch_tmap(&tm_ts);
      mbar_arrive_expect_tx(q_full, nq * L::kTileBytes);
      for (int q = 0; q < nq; ++q)
#pragma unroll
        for (int b = 0; b < HD / 64; ++b)
          tma_load_2d(smem + L::kQ + q * L::kTileBytes + b * 16384, &tm, q_full,
                      2 * d + h * HD + b * 64, (qt0 + q) * 128);
      bool issued[NSK], t_issued[NST];
      uint32_t issued_ph[NSK], t_issued_ph[NST];
      for (int s = 0; s < NSK; ++s) issued[s] = false, issued_ph[s] = 0;
      for (int s = 0; s < NST; ++s) t_issued[s] = false, t_issued_ph[s] = 0;
      for (int j = 0; j < n_kt && !*abort_flag; ++j) {
        const int s = j % NSK;
        const uint32_t ph = (j / NSK) & 1;
        if (!mbar_wait(&k_empty[s], ph ^ 1, p.wait_limit)) { *abort_flag = 1; break; }
        mbar_arrive_expect_tx(&k_full[s], L::kTileBytes);
#pragma unroll
        for (int b = 0; b < HD / 64; ++b)
          tma_load_2d(smem + L::kK + s * L::kTileBytes + b * 16384, &tm, &k_full[s],
                      3 * d + h * HD + b * 64, key_tile(j) * 128);
        issued[s] = true;
        issued_ph[s] = ph;
        // the tile's key timestamps (a deeper ring: the row groups classify ahead)
        const int st = j % NST;
        const uint32_t tph = (j / NST) & 1;
        if (!mbar_wait(&t_empty[st], tph ^ 1, p.wait_limit)) { *abort_flag = 1; break; }
        mbar_arrive_expect_tx(&t_full[st], 128 * 8);
        tma_load_1d(s_kts + st * 128, &tm_ts, &t_full[st], key_tile(j) * 128);
        t_issued[st] = true;
        t_issued_ph[st] = tph;
      }
      mbar_wait(q_full, 0);
      for (int s = 0; s < NSK; ++s)
        if (issued[s]) mbar_wait(&k_full[s], issued_ph[s]);
      for (int s = 0; s < NST; ++s)
        if (t_issued[s]) mbar_wait(&t_full[s], t_issued_ph[s]);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ V loads
    if (lane == 0) {
      bool issued[NSV];
      uint32_t issued_ph[NSV];
      for (int s = 0; s < NSV; ++s) issued[s] = false, issued_ph[s] = 0;
      for (int j = 0; j < n_kt && !*abort_flag; ++j) {
        const int s = j % NSV;
        const uint32_t ph = (j / NSV) & 1;
        if (!mbar_wait(&v_empty[s], ph ^ 1, p.wait_limit)) { *abort_flag = 1; break; }
        mbar_arrive_expect_tx(&v_full[s], L::kTileBytes);
#pragma unroll
        for (int b = 0; b < HD / 64; ++b)
          tma_load_2d(smem + L::kV + s * L::kTileBytes + b * 16384, &tm, &v_full[s],
                      d + h * HD + b * 64, key_tile(j) * 128);
        issued[s] = true;
        issued_ph[s] = ph;
      }
      for (int s = 0; s < NSV; ++s)
        if (issued[s]) mbar_wait(&v_full[s], issued_ph[s]);
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------ MMA issue, one thread per
    // query tile (warp 1: tile 0, warp 3: tile 1).  Two issuers keep the tensor pipe fed while
    // either one waits for its row group: an issuing thread that stops for a wait lets the
    // pipe drain.
    const int q = warp == 1 ? 0 : 1;
    if (lane == 0 && q < nq) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, HD, false, true);
      bool ok = mbar_wait(q_full, 0, p.wait_limit);
      tc_fence_after();
      const uint32_t sQ = smem_u32(smem + L::kQ + q * L::kTileBytes);
      // S_q = Q_q K_j^T; the K stage is released once every issuer's product has read it
      auto issue_qk = [&](int j) -> bool {
        const int s = j % NSK;
        if (!mbar_wait(&k_full[s], (j / NSK) & 1, p.wait_limit)) return false;
        tc_fence_after();
        const uint32_t sK = smem_u32(smem + L::kK + s * L::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tS(q), desc_sw128(sQ + off, 16, 1024), desc_sw128(sK + off, 16, 1024),
                  idesc_qk, kk > 0);
        }
        umma_commit(&s_full[q]);
        umma_commit(&k_empty[s]);
        return true;
      };
      if (ok) ok = issue_qk(0);
      bool o_done = false;
      for (int j = 0; ok && j < n_kt; ++j) {
        const int s = j % NSV;
        if (!mbar_wait(&v_full[s], (j / NSV) & 1, p.wait_limit)) { ok = false; break; }
        if (!mbar_wait(&p_half[q], j & 1, p.wait_limit)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sV = smem_u32(smem + L::kV + s * L::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          umma_ts(tO(q), tS(q) + kk * 8, desc_sw128(sV + kk * 2048, 16384, 1024), idesc_pv,
                  (j > 0 || kk > 0));
        }
        if (!mbar_wait(&p_full[q], j & 1, p.wait_limit)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 4; kk < 8; ++kk) {
          umma_ts(tO(q), tS(q) + kk * 8, desc_sw128(sV + kk * 2048, 16384, 1024), idesc_pv, 1);
        }
        umma_commit(&v_empty[s]);
        if (j + 1 == n_kt) {
          umma_commit(&o_full[q]);
          o_done = true;
        }
        // S_q is rewritten only after P_q V_j (issued just above, executed in order)
        if (j + 1 < n_kt && !issue_qk(j + 1)) ok = false;
      }
      if (!ok) *abort_flag = 1;
      if (!o_done) umma_commit(&o_full[q]);   // release the row group on an abort
      umma_commit(&drained[q]);              // fires once every MMA of this issuer is done
      mbar_wait(&drained[q], 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ row groups
    const int q = (warp - 4) >> 2;             // query tile of this row group
    const int wq = warp & 3;                   // tensor-memory lane quarter
    const int row = wq * 32 + lane;            // query row inside the tile
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const int clamp = p.pos_clamp;
    const int nb = p.time_buckets;
    {
      // the tables, eight global loads in flight per thread before the stores
      const int t = threadIdx.x - 128;
      const int n_rp = clamp + 1 + 2 * kPosPad;
#pragma unroll 1
      for (int k0 = t; k0 < n_rp; k0 += 8 * 256) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int k = k0 + u * 256;
          v[u] = k < n_rp ? __ldg(p.rab_pos + min(max(k - kPosPad, 0), clamp)) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (k0 + u * 256 < n_rp) s_rab_pos[k0 + u * 256] = v[u];
      }
      const float rt = t < nb ? __ldg(p.rab_time + t) : 0.0f;
      const int64_t th = t < nb ? __ldg(p.thresholds + t) : 0;
      const int32_t t32a = __ldg(p.thr32 + t);
      const int32_t t32b = t + 256 < 257 ? __ldg(p.thr32 + t + 256) : 0;
      const uint8_t lu = t < 128 ? __ldg(p.time_lut + t) : 0;
      if (t < nb) {
        s_rab_time[t] = rt;
        s_thr[t] = th;
      }
      s_thr32[t] = t32a;
      if (t + 256 < 257) s_thr32[t + 256] = t32b;
      if (t < 128) s_lut[t] = lu;
    }
    named_bar_sync(1, 256);
    if (threadIdx.x - 128 < 128) {
      // per bin: {threshold of the next bucket, bias of the bin's bucket, bias of the next, bucket}
      const int idx = threadIdx.x - 128;
      const int cand = s_lut[idx];
      const int nxt = cand + 1 < nb ? cand + 1 : cand;
      s_any[idx] = make_int4(cand + 1 < nb ? s_thr32[cand + 1] : 0x7FFFFFFF,
                             __float_as_int(s_rab_time[cand]), __float_as_int(s_rab_time[nxt]),
                             cand);
    }
    named_bar_sync(1, 256);
    const uint8_t* s_anyb = reinterpret_cast<const uint8_t*>(s_any);

    // token indices fit in int32 (T <= 2^30, checked at create)
    const int i = (qt0 + q) * 128 + row;
    const bool valid = q < nq && i < p.T;
    int lo = 0, hi = 0, pos = 0;   // rows past T see nothing
    Row R;
    R.ti = 0;
    if (valid) {
      const RowInfo ri = p.rows[i];
      lo = (ri.lo < 0 || ri.lo > i) ? i : ri.lo;
      hi = ri.hi;
      pos = ri.pos;
      R.ti = p.ts[i];
    }
    R.ti_lo = uint32_t(R.ti);
    // every visible key of the row lies in its user, at or after ts[lo]: its gap is
    // at most t_i - ts[lo], so this bound decides whether 32-bit gaps are exact
    const bool row_narrow = !valid || R.ti - p.ts[lo] < int64_t(0x7FFFFFFE);
    R.b = 0;
    R.cut = R.ti;
    if (valid) {
      R.b = bucket_search(s_thr, nb, R.ti - p.ts[lo]);
      R.cut = R.ti - s_thr[R.b];
    }
    const int nn = p.n_norm_fixed > 0 ? p.n_norm_fixed : p.counters[0];
    const float inv_nn = 1.0f / float(nn > 0 ? nn : 1);
    bool aborted = false;

    for (int j = 0; q < nq && j < n_kt; ++j) {
      const int kb = key_tile(j) * 128;
      const int st = j % NST;
      const int64_t* kts = s_kts + st * 128;
      // The key timestamps of tile j come through their own ring, loaded well
      // ahead of the scores: classify the rows first, off the critical path.
      bool ok = aborted ? false : mbar_wait(&t_full[st], (j / NST) & 1, p.wait_limit);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        aborted = true;
        *abort_flag = 1;
        continue;
      }
      // ---- classify this row for the tile
      R.lo_rel = min(max(lo - kb, -1), 129);
      R.hi_rel = min(max(hi - kb, -1), 129);
      R.i_rel = valid ? min(max(i - kb, -1), 129) : -1;
      R.pos_rel = min(max(pos - kb, -1), clamp + 129);
      const bool full = valid && lo <= kb && hi - kb >= 128;
      const bool posc = pos - kb - 127 >= clamp;
      int lev = 99;
      if (full) {
        walk_to(R.b, R.cut, kts[0], R.ti, s_thr);
        R.b_last = R.b;
        R.cut_last = R.cut;
        walk_to(R.b_last, R.cut_last, kts[127], R.ti, s_thr);
        lev = R.b - R.b_last;
      }
      int mode;
      if (__all_sync(0xffffffffu, R.i_rel < 0)) mode = kZero;   // every key is later than every row
      else if (__all_sync(0xffffffffu, full && lev == 0)) mode = kFast;
      else if (__all_sync(0xffffffffu, full && lev <= 1)) mode = kMed;
      else if (__all_sync(0xffffffffu, full && lev <= 3)) mode = kCut;
      else if (__all_sync(0xffffffffu, !valid || hi <= kb))
        mode = kSelf;  // candidates on their own tiles: only the row itself is visible
      else if (p.lut_exact && __all_sync(0xffffffffu, row_narrow))
        mode = kAny;   // the causal diagonal, user and history boundaries, candidates
      else mode = kGen;
      const bool pc = __all_sync(0xffffffffu, posc);
      if (mode == kFast || mode == kMed || mode == kCut) {
        // R.b = bucket of the tile's first key (the largest gap); a gap below
        // thr[R.b - m + 1] drops the bucket below R.b - m + 1
        const float rp_c = pc ? s_rab_pos[kPosPad + clamp] : 0.0f;
        const int b0 = R.b;
        R.hc = 0.5f * (rp_c + s_rab_time[b0]);
        R.hc_lo = 0.5f * (rp_c + s_rab_time[max(b0 - 1, 0)]);
        R.hc2 = 0.5f * (rp_c + s_rab_time[max(b0 - 2, 0)]);
        R.hc3 = 0.5f * (rp_c + s_rab_time[max(b0 - 3, 0)]);
        if (mode != kFast) {
          // first column whose gap is below thr[b0 - m + 1]: the count of keys with
          // t_j <= t_i - thr[b0 - m + 1] (the tile's timestamps are sorted)
          const int64_t c1 = R.ti - s_thr[b0];
          const int64_t c2 = R.ti - s_thr[max(b0 - 1, 0)];
          const int64_t c3 = R.ti - s_thr[max(b0 - 2, 0)];
          int p1 = 0, p2 = 0, p3 = 0;
#pragma unroll
          for (int step = 64; step > 0; step >>= 1) {
            if (kts[p1 + step - 1] <= c1) p1 += step;
            if (mode == kCut) {
              if (kts[p2 + step - 1] <= c2) p2 += step;
              if (kts[p3 + step - 1] <= c3) p3 += step;
            }
          }
          // seven halvings leave p in [0, 127]; one more compare completes the count
          R.j1 = p1 + (kts[p1] <= c1 ? 1 : 0);
          R.j2 = p2 + (kts[p2] <= c2 ? 1 : 0);
          R.j3 = p3 + (kts[p3] <= c3 ? 1 : 0);
        }
      }
      Record rec;
      rec.pidx = p.dump_pidx;
      rec.tidx = p.dump_tidx;
      rec.vis = p.dump_vis;
      rec.T = p.T;
      rec.i = i;
      rec.kb = kb;
      rec.on = RECORD && h == 0 && valid;

      ok = mbar_wait(&s_full[q], j & 1, p.wait_limit);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        aborted = true;
        *abort_flag = 1;
        continue;
      }
      tc_fence_after();
      const uint32_t taddr = tS(q) + lane_off;
      // rp_row[-column] = rab_pos[clamp(pos_rel - column, 0, clamp)]
      const float* rp_row = s_rab_pos + kPosPad + R.pos_rel;
      if (mode == kZero) {
        zero_tile<RECORD>(taddr, rec);
      } else if (mode == kSelf) {
        self_tile<RECORD>(taddr, R, rp_row, s_rab_time, clamp, rec);
      } else if (mode == kFast) {
        if (pc) score_tile<kFast, true, RECORD>(taddr, R, rp_row, s_rab_time, s_thr, s_anyb, s_thr32, kts, clamp, rec, &p_half[q]);
        else score_tile<kFast, false, RECORD>(taddr, R, rp_row, s_rab_time, s_thr, s_anyb, s_thr32, kts, clamp, rec, &p_half[q]);
      } else if (mode == kMed) {
        if (pc) score_tile<kMed, true, RECORD>(taddr, R, rp_row, s_rab_time, s_thr, s_anyb, s_thr32, kts, clamp, rec, &p_half[q]);
        else score_tile<kMed, false, RECORD>(taddr, R, rp_row, s_rab_time, s_thr, s_anyb, s_thr32, kts, clamp, rec, &p_half[q]);
      } else if (mode == kCut) {
        if (pc) score_tile<kCut, true, RECORD>(taddr, R, rp_row, s_rab_time, s_thr, s_anyb, s_thr32, kts, clamp, rec, &p_half[q]);
        else score_tile<kCut, false, RECORD>(taddr, R, rp_row, s_rab_time, s_thr, s_anyb, s_thr32, kts, clamp, rec, &p_half[q]);
      } else if (mode == kAny) {
        score_tile<kAny, false, RECORD>(taddr, R, rp_row, s_rab_time, s_thr, s_anyb, s_thr32, kts, clamp, rec, &p_half[q]);
      } else {
        score_tile<kGen, false, RECORD>(taddr, R, rp_row, s_rab_time, s_thr, s_anyb, s_thr32, kts, clamp, rec, &p_half[q]);
      }
      if (mode == kZero || mode == kSelf) {
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_half[q]);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[q]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&t_empty[st]);
      if (mode == kFast || mode == kMed || mode == kCut) {
        R.b = R.b_last;
        R.cut = R.cut_last;
      }
    }

    // ---- O_q / n_norm -> shared memory (128-byte swizzled boxes of 32 rows x 32
    // columns, per warp) -> TMA stores, which clip the rows past T.  Once o_full[q]
    // fired, every MMA of this query tile is done, so Q_q's tile is free to stage in.
    if (q < nq) {
      bool ok = aborted ? false : mbar_wait(&o_full[q], 0, p.wait_limit);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        uint8_t* stage = smem + L::kQ + q * L::kTileBytes + wq * (L::kTileBytes / 4);
        constexpr int kBoxes = HD / 64;   // boxes per pass; two passes cover HD columns
#pragma unroll 1
        for (int rd = 0; rd < 2; ++rd) {
#pragma unroll 1
          for (int cb = 0; cb < kBoxes; ++cb) {
            uint32_t r[32];
            tmem_ld32(tO(q) + lane_off + (rd * kBoxes + cb) * 32, r);
            tmem_ld_wait();
            const uint32_t row_addr = smem_u32(stage + cb * 4096 + lane * 128);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              st_shared_v4(row_addr + ((e ^ (lane & 7)) << 4),
                           __uint_as_float(r[4 * e + 0]) * inv_nn,
                           __uint_as_float(r[4 * e + 1]) * inv_nn,
                           __uint_as_float(r[4 * e + 2]) * inv_nn,
                           __uint_as_float(r[4 * e + 3]) * inv_nn);
          }
          fence_proxy_async_smem();   // make the stores visible to the TMA unit
          __syncwarp();
          if (lane == 0) {
            for (int cb = 0; cb < kBoxes; ++cb) {
              const int32_t x = h * HD + (rd * kBoxes + cb) * 32;
              const int32_t y = (qt0 + q) * 128 + wq * 32;
              // a split's partial sum is added to the others' (O starts at zero)
              if (p.num_splits > 1) tma_reduce_add_2d(&tm_o, stage + cb * 4096, x, y);
              else tma_store_2d(&tm_o, stage + cb * 4096, x, y);
            }
            bulk_commit_group();
            bulk_wait_group_read0();   // the boxes are reused by the next pass
          }
          __syncwarp();
        }
      } else {
        *abort_flag = 1;
      }
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

// ================================================================ CTA-pair kernel (head dim 128)
//
// The same work items -- a pair of adjacent 128-query tiles and one head --
// computed by clusters of two CTAs on two SMs, one query tile each, each
// cluster looping over the items c, c + clusters, ... (persistent: the tables
// load once per SM, and an item's first products run while the previous
// item's O is read out).  The leader CTA's MMA thread issues every product
// with cta_group::2 (M = 256: rows 0-127 from the leader's Q and tensor
// memory, 128-255 from the peer's); K and V are split between the CTAs along
// the products' N (each CTA loads 64 keys of K and 64 columns of V per key
// tile), so each SM reads half of every K and V tile.  With one query tile per
// CTA, tensor memory holds three S buffers beside O, and three row groups
// (warps 4-7, 8-11, 12-15) score the key tiles in turn: group g takes the tiles
// whose running count over the CTA's items is g mod 3, so it always reads the
// same S buffer, and three tiles are scored at once (three scoring warps per SM
// sub-partition keep the multi-function unit busier than two: 2-3% faster on
// one 8 x 8192-token layer than two groups on alternate tiles).  The K, V,
// timestamp and S rings run on one tile count across the items.
struct PairLayout {
  static constexpr int NSK = 4, NSV = 4, NST = 6;
  static constexpr uint32_t kQ = 0;                            // 128 x 128: two 64-column boxes
  static constexpr uint32_t kK = 32768;                        // [NSK] 64 keys x 128: two 8 KB boxes
  static constexpr uint32_t kV = kK + NSK * 16384;             // [NSV] 128 keys x 64 columns
  static constexpr uint32_t kStage = kV + NSV * 16384;         // O staging: 8 warps x 4 KB
  static constexpr uint32_t kKts = kStage + 8 * 4096;          // int64 [NST][128]
  static constexpr uint32_t kThr = kKts + NST * 1024;
  static constexpr uint32_t kThr32 = kThr + kMaxTimeBuckets * 8;
  static constexpr uint32_t kLut = kThr32 + 260 * 4;
  static constexpr uint32_t kAnyTab = kLut + 128;
  static constexpr uint32_t kRabTime = kAnyTab + 128 * 16;
  static constexpr uint32_t kBars = kRabTime + kMaxTimeBuckets * 4;
  static constexpr uint32_t kRabPos = kBars + 512;
  static __host__ __device__ constexpr uint32_t smem_bytes(int clamp) {
    return kRabPos + ((uint32_t(clamp + 1 + 2 * kPosPad) * 4 + 15) / 16) * 16 + 1024;
  }
  static_assert(kK % 1024 == 0 && kV % 1024 == 0 && kStage % 1024 == 0 && kKts % 128 == 0,
                "alignment");
  static_assert(kAnyTab % 16 == 0 && kBars % 8 == 0, "alignment");
  // mbarriers (q_full, q_empty, the K, V and timestamp rings, s_full and p_full
  // [3] each, o_full, o_empty, drained, p_half) and two words
  static_assert((2 + 2 * NSK + 2 * NSV + 2 * NST + 10) * 8 + 8 <= 512, "barrier block");
};
static_assert(PairLayout::smem_bytes(kMaxPosEntries - 1) <= 227 * 1024, "shared memory budget");

// One work item of the pair kernel: head, pair, and its key tiles.
struct PairItem {
  int h, qt0, nq, n_a, a_lo, jb, n_kt;
  __device__ __forceinline__ int key_tile(int j) const {
    j += jb;
    return j < n_a ? a_lo + j : qt0 + (j - n_a);
  }
};

__device__ __forceinline__ PairItem pair_item(const AttnParams& p, int w) {
  const int per_head = p.num_pairs * p.num_splits;
  PairItem it;
  it.h = w / per_head;
  const int pr = p.order[(w % per_head) / p.num_splits];
  const int split = (w % per_head) % p.num_splits;
  it.qt0 = 2 * pr;
  const PairTiles pt = pair_tiles(p.rows, p.T, pr);
  it.nq = pt.n_diag;
  it.n_a = pt.n_a;
  it.a_lo = pt.a_lo;
  const int n_all = pt.n_a + pt.n_diag;
  it.jb = split * n_all / p.num_splits;
  it.n_kt = (split + 1) * n_all / p.num_splits - it.jb;   // <= 0: nothing to do
  return it;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    attn_tc_pair_kernel(const __grid_constant__ CUtensorMap tm,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_ts,
                        const __grid_constant__ CUtensorMap tm_o, const AttnParams p) {
  using L = PairLayout;
  constexpr int HD = 128;
  constexpr bool RECORD = false;
  constexpr int NSK = L::NSK;
  constexpr int NSV = L::NSV;
  constexpr int NST = L::NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* s_rab_pos = reinterpret_cast<float*>(smem + L::kRabPos);
  float* s_rab_time = reinterpret_cast<float*>(smem + L::kRabTime);
  int64_t* s_thr = reinterpret_cast<int64_t*>(smem + L::kThr);
  int32_t* s_thr32 = reinterpret_cast<int32_t*>(smem + L::kThr32);
  uint8_t* s_lut = reinterpret_cast<uint8_t*>(smem + L::kLut);
  int4* s_any = reinterpret_cast<int4*>(smem + L::kAnyTab);
  int64_t* s_kts = reinterpret_cast<int64_t*>(smem + L::kKts);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* q_full = bars;             // (leader) both Q tiles of an item landed
  uint64_t* q_empty = q_full + 1;      // the item's last QK^T read Q
  uint64_t* k_full = q_empty + 1;      // [NSK] (leader) both K halves landed
  uint64_t* k_empty = k_full + NSK;    // [NSK] the products reading the stage are done
  uint64_t* v_full = k_empty + NSK;    // [NSV] (leader)
  uint64_t* v_empty = v_full + NSV;    // [NSV]
  uint64_t* s_full = v_empty + NSV;    // [3] S buffer b holds the scores of its key tile
  uint64_t* p_full = s_full + 3;       // [3] (leader) P written by the scoring warps of both CTAs
  uint64_t* o_full = p_full + 3;       // every product of an item is done
  uint64_t* o_empty = o_full + 1;      // (leader) both CTAs read O out
  uint64_t* drained = o_empty + 1;
  uint64_t* t_full = drained + 1;      // [NST] key timestamps of a tile landed (local)
  uint64_t* t_empty = t_full + NST;    // [NST]
  uint64_t* p_half = t_empty + NST;    // arrivals of the half-tile hand-over (unused here)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(p_half + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t rank = cluster_rank();
  const int q = int(rank);             // this CTA's query tile within each pair
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int d = p.d;
  const int num_items = p.num_pairs * p.num_splits * p.H;
  const int cid = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < NSV; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 3; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 8);   // one arrival per warp of the scoring group of each CTA
    }
    mbar_init(o_full, 1);
    mbar_init(o_empty, 16);       // every warp of row groups 0 and 1 of both CTAs
    mbar_init(drained, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&t_full[s], 1);
      mbar_init(&t_empty[s], 4);  // the warps of the row group scoring the tile
    }
    mbar_init(p_half, 128);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // columns: S buffers [0, 128), [128, 256), [256, 384); O [384, 512)
  auto tS = [&](int b) -> uint32_t { return tmem_base + b * 128; };
  const uint32_t tO = tmem_base + 384;
  auto leader = [&](uint64_t* bar) -> uint32_t { return map_to_rank(smem_u32(bar), 0); };

  if (warp == 0) {
    // ------------------------------------------------------------ loads (both CTAs)
    if (lane == 0) {
      prefetch_tmap(&tm);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_ts);
      int last_k[NSK], last_v[NSV];
      bool t_issued[NST];
      uint32_t t_ph[NST];
      for (int s = 0; s < NSK; ++s) last_k[s] = -1;
      for (int s = 0; s < NSV; ++s) last_v[s] = -1;
      for (int s = 0; s < NST; ++s) t_issued[s] = false, t_ph[s] = 0;
      int G = 0, n_done = 0;
      for (int w = cid; w < num_items && !*abort_flag; w += n_clusters) {
        const PairItem I = pair_item(p, w);
        if (I.n_kt <= 0) continue;   // uniform over the cluster
        // Q of this item once the previous item's last QK^T has read Q
        if (n_done > 0 && !mbar_wait(q_empty, (n_done - 1) & 1, p.wait_limit)) {
          *abort_flag = 1;
          break;
        }
        if (rank == 0) mbar_arrive_expect_tx(q_full, 2 * 32768);
#pragma unroll
        for (int b = 0; b < 2; ++b)
          tma_load_2d_pair(smem + L::kQ + b * 16384, &tm, leader(q_full),
                           2 * d + I.h * HD + b * 64, (I.qt0 + q) * 128);
        bool ok = true;
        for (int j = 0; j < I.n_kt && ok; ++j) {
          const int g = G + j;
          const int kb = I.key_tile(j) * 128;
          const int s = g % NSK;
          if (!mbar_wait(&k_empty[s], ((g / NSK) & 1) ^ 1, p.wait_limit)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&k_full[s], 2 * 16384);
#pragma unroll
          for (int b = 0; b < 2; ++b)
            tma_load_2d_pair(smem + L::kK + s * 16384 + b * 8192, &tm_k, leader(&k_full[s]),
                             3 * d + I.h * HD + b * 64, kb + 64 * q);
          last_k[s] = g;
          const int sv = g % NSV;
          if (!mbar_wait(&v_empty[sv], ((g / NSV) & 1) ^ 1, p.wait_limit)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&v_full[sv], 2 * 16384);
          tma_load_2d_pair(smem + L::kV + sv * 16384, &tm, leader(&v_full[sv]),
                           d + I.h * HD + 64 * q, kb);
          last_v[sv] = g;
          const int st = g % NST;
          const uint32_t tph = (g / NST) & 1;
          if (!mbar_wait(&t_empty[st], tph ^ 1, p.wait_limit)) { ok = false; break; }
          mbar_arrive_expect_tx(&t_full[st], 128 * 8);
          tma_load_1d(s_kts + st * 128, &tm_ts, &t_full[st], kb);
          t_issued[st] = true;
          t_ph[st] = tph;
        }
        if (!ok) {
          *abort_flag = 1;
          break;
        }
        G += I.n_kt;
        ++n_done;
      }
      // no copy may still be in flight when the CTA ends: a stage's copies have
      // landed once the products that read it are done (the leader counts the
      // bytes of both CTAs), and the last Q once the last QK^T is
      for (int s = 0; s < NSK; ++s)
        if (last_k[s] >= 0) mbar_wait(&k_empty[s], (last_k[s] / NSK) & 1);
      for (int s = 0; s < NSV; ++s)
        if (last_v[s] >= 0) mbar_wait(&v_empty[s], (last_v[s] / NSV) & 1);
      for (int s = 0; s < NST; ++s)
        if (t_issued[s]) mbar_wait(&t_full[s], t_ph[s]);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue (leader)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(256, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(256, HD, false, true);
      const uint32_t sQ = smem_u32(smem + L::kQ);
      bool ok = true;
      int G = 0, n_done = 0;
      for (int w = cid; ok && w < num_items && !*abort_flag; w += n_clusters) {
        const PairItem I = pair_item(p, w);
        if (I.n_kt <= 0) continue;
        if (!mbar_wait(q_full, n_done & 1, p.wait_limit)) { ok = false; break; }
        tc_fence_after();
        // S of the item's tile j = Q K^T into buffer (G + j) % 3, after the products
        // issued before it (in order): the K stage is released when it is done, Q
        // after the item's last one
        auto issue_s = [&](int j) -> bool {
          const int g = G + j;
          const int s = g % NSK;
          if (!mbar_wait(&k_full[s], (g / NSK) & 1, p.wait_limit)) return false;
          tc_fence_after();
          const uint32_t sK = smem_u32(smem + L::kK + s * 16384);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t oq = (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t ok2 = (kk >> 2) * 8192 + (kk & 3) * 32;
            umma_ss_pair(tS(g % 3), desc_sw128(sQ + oq, 16, 1024), desc_sw128(sK + ok2, 16, 1024),
                         idesc_qk, kk > 0);
          }
          umma_commit_pair(&s_full[g % 3]);
          umma_commit_pair(&k_empty[s]);
          if (j + 1 == I.n_kt) umma_commit_pair(q_empty);
          return true;
        };
        for (int j = 0; ok && j < 3 && j < I.n_kt; ++j) ok = issue_s(j);
        // O is rewritten from zero only after both CTAs read the previous item's O
        if (ok && n_done > 0 && !mbar_wait(o_empty, (n_done - 1) & 1, p.wait_limit)) ok = false;
        tc_fence_after();
        for (int j = 0; ok && j < I.n_kt; ++j) {
          const int g = G + j;
          const int b = g % 3;
          const int sv = g % NSV;
          if (!mbar_wait(&p_full[b], (g / 3) & 1, p.wait_limit)) { ok = false; break; }
          if (!mbar_wait(&v_full[sv], (g / NSV) & 1, p.wait_limit)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sV = smem_u32(smem + L::kV + sv * 16384);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ts_pair(tO, tS(b) + kk * 8, desc_sw128(sV + kk * 2048, 16384, 1024), idesc_pv,
                         (j > 0 || kk > 0));
          umma_commit_pair(&v_empty[sv]);
          if (j + 1 == I.n_kt) umma_commit_pair(o_full);
          // buffer b is rewritten only after P_j V_j (issued just above, executed in order)
          if (j + 3 < I.n_kt && !issue_s(j + 3)) ok = false;
        }
        G += I.n_kt;
        ++n_done;
      }
      if (!ok) *abort_flag = 1;
      umma_commit_pair(drained);   // fires once every product issued here is done
      mbar_wait(drained, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ row groups
    const int g = (warp - 4) >> 2;             // this group scores the tiles counted g mod 3
    const int wq = warp & 3;                   // tensor-memory lane quarter
    const int row = wq * 32 + lane;
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const int clamp = p.pos_clamp;
    const int nb = p.time_buckets;
    {
      // the tables, eight global loads in flight per thread before the stores,
      // written by the first 256 row-group threads
      const int t = threadIdx.x - 128;
      const int n_rp = clamp + 1 + 2 * kPosPad;
      if (t < 256) {
#pragma unroll 1
      for (int k0 = t; k0 < n_rp; k0 += 8 * 256) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int k = k0 + u * 256;
          v[u] = k < n_rp ? __ldg(p.rab_pos + min(max(k - kPosPad, 0), clamp)) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (k0 + u * 256 < n_rp) s_rab_pos[k0 + u * 256] = v[u];
      }
      const float rt = t < nb ? __ldg(p.rab_time + t) : 0.0f;
      const int64_t th = t < nb ? __ldg(p.thresholds + t) : 0;
      const int32_t t32a = __ldg(p.thr32 + t);
      const int32_t t32b = t + 256 < 257 ? __ldg(p.thr32 + t + 256) : 0;
      const uint8_t lu = t < 128 ? __ldg(p.time_lut + t) : 0;
      if (t < nb) {
        s_rab_time[t] = rt;
        s_thr[t] = th;
      }
      s_thr32[t] = t32a;
      if (t + 256 < 257) s_thr32[t + 256] = t32b;
      if (t < 128) s_lut[t] = lu;
      }
    }
    named_bar_sync(1, 384);
    if (threadIdx.x - 128 < 128) {
      // per bin: {threshold of the next bucket, bias of the bin's bucket, bias of the next, bucket}
      const int idx = threadIdx.x - 128;
      const int cand = s_lut[idx];
      const int nxt = cand + 1 < nb ? cand + 1 : cand;
      s_any[idx] = make_int4(cand + 1 < nb ? s_thr32[cand + 1] : 0x7FFFFFFF,
                             __float_as_int(s_rab_time[cand]), __float_as_int(s_rab_time[nxt]),
                             cand);
    }
    named_bar_sync(1, 384);
    const uint8_t* s_anyb = reinterpret_cast<const uint8_t*>(s_any);
    const int nn = p.n_norm_fixed > 0 ? p.n_norm_fixed : p.counters[0];
    const float inv_nn = 1.0f / float(nn > 0 ? nn : 1);
    Record rec;
    rec.pidx = nullptr;
    rec.tidx = nullptr;
    rec.vis = nullptr;
    rec.T = p.T;
    rec.kb = 0;
    rec.on = false;
    bool aborted = false;
    int G = 0, n_done = 0;

    for (int w = cid; w < num_items && !aborted && !*abort_flag; w += n_clusters) {
      const PairItem I = pair_item(p, w);
      if (I.n_kt <= 0) continue;
      // the row's facts (token indices fit in int32: T <= 2^30, checked at create)
      const int i = (I.qt0 + q) * 128 + row;
      const bool valid = q < I.nq && i < p.T;
      int lo = 0, hi = 0, pos = 0;   // rows past T see nothing
      Row R;
      R.ti = 0;
      int64_t t_lo = 0;
      if (valid) {
        const RowInfo ri = p.rows[i];
        lo = (ri.lo < 0 || ri.lo > i) ? i : ri.lo;
        hi = ri.hi;
        pos = ri.pos;
        R.ti = p.ts[i];
        t_lo = p.ts[lo];
      }
      R.ti_lo = uint32_t(R.ti);
      const bool row_narrow = !valid || R.ti - t_lo < int64_t(0x7FFFFFFE);
      R.b = 0;
      R.cut = R.ti;
      if (valid) {
        R.b = bucket_search(s_thr, nb, R.ti - t_lo);
        R.cut = R.ti - s_thr[R.b];
      }
      rec.i = i;

      for (int j = ((g - G) % 3 + 3) % 3; j < I.n_kt; j += 3) {
        const int gt = G + j;
        const int kb = I.key_tile(j) * 128;
        const int st = gt % NST;
        const int64_t* kts = s_kts + st * 128;
        bool ok = mbar_wait(&t_full[st], (gt / NST) & 1, p.wait_limit);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
          aborted = true;
          *abort_flag = 1;
          break;
        }
        // ---- classify this row for the tile
        R.lo_rel = min(max(lo - kb, -1), 129);
        R.hi_rel = min(max(hi - kb, -1), 129);
        R.i_rel = valid ? min(max(i - kb, -1), 129) : -1;
        R.pos_rel = min(max(pos - kb, -1), clamp + 129);
        const bool full = valid && lo <= kb && hi - kb >= 128;
        const bool posc = pos - kb - 127 >= clamp;
        int lev = 99;
        if (full) {
          walk_to(R.b, R.cut, kts[0], R.ti, s_thr);
          R.b_last = R.b;
          R.cut_last = R.cut;
          walk_to(R.b_last, R.cut_last, kts[127], R.ti, s_thr);
          lev = R.b - R.b_last;
        }
        int mode;
        if (__all_sync(0xffffffffu, R.i_rel < 0)) mode = kZero;   // every key is later than every row
        else if (__all_sync(0xffffffffu, full && lev == 0)) mode = kFast;
        else if (__all_sync(0xffffffffu, full && lev <= 1)) mode = kMed;
        else if (__all_sync(0xffffffffu, full && lev <= 3)) mode = kCut;
        else if (__all_sync(0xffffffffu, !valid || hi <= kb))
          mode = kSelf;  // candidates on their own tiles: only the row itself is visible
        else if (p.lut_exact && __all_sync(0xffffffffu, row_narrow))
          mode = kAny;   // the causal diagonal, user and history boundaries, candidates
        else mode = kGen;
        const bool pc = __all_sync(0xffffffffu, posc);
        if (mode == kFast || mode == kMed || mode == kCut) {
          // R.b = bucket of the tile's first key (the largest gap); a gap below
          // thr[R.b - m + 1] drops the bucket below R.b - m + 1
          const float rp_c = pc ? s_rab_pos[kPosPad + clamp] : 0.0f;
          const int b0 = R.b;
          R.hc = 0.5f * (rp_c + s_rab_time[b0]);
          R.hc_lo = 0.5f * (rp_c + s_rab_time[max(b0 - 1, 0)]);
          R.hc2 = 0.5f * (rp_c + s_rab_time[max(b0 - 2, 0)]);
          R.hc3 = 0.5f * (rp_c + s_rab_time[max(b0 - 3, 0)]);
          if (mode != kFast) {
            // first column whose gap is below thr[b0 - m + 1]: the count of keys with
            // t_j <= t_i - thr[b0 - m + 1] (the tile's timestamps are sorted)
            const int64_t c1 = R.ti - s_thr[b0];
            const int64_t c2 = R.ti - s_thr[max(b0 - 1, 0)];
            const int64_t c3 = R.ti - s_thr[max(b0 - 2, 0)];
            int p1 = 0, p2 = 0, p3 = 0;
#pragma unroll
            for (int step = 64; step > 0; step >>= 1) {
              if (kts[p1 + step - 1] <= c1) p1 += step;
              if (mode == kCut) {
                if (kts[p2 + step - 1] <= c2) p2 += step;
                if (kts[p3 + step - 1] <= c3) p3 += step;
              }
            }
            // seven halvings leave p in [0, 127]; one more compare completes the count
            R.j1 = p1 + (kts[p1] <= c1 ? 1 : 0);
            R.j2 = p2 + (kts[p2] <= c2 ? 1 : 0);
            R.j3 = p3 + (kts[p3] <= c3 ? 1 : 0);
          }
        }
        ok = mbar_wait(&s_full[gt % 3], (gt / 3) & 1, p.wait_limit);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
          aborted = true;
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tS(gt % 3) + lane_off;
        // rp_row[-column] = rab_pos[clamp(pos_rel - column, 0, clamp)]
        const float* rp_row = s_rab_pos + kPosPad + R.pos_rel;
        if (mode == kZero) {
          zero_tile<RECORD>(taddr, rec);
        } else if (mode == kSelf) {
          self_tile<RECORD>(taddr, R, rp_row, s_rab_time, clamp, rec);
        } else if (mode == kFast) {
          if (pc) score_tile<kFast, true, RECORD>(taddr, R, rp_row, s_rab_time, s_thr, s_anyb, s_thr32, kts, clamp, rec, p_half);
          else score_tile<kFast, false, RECORD>(taddr, R, rp_row, s_rab_time, s_thr, s_anyb, s_thr32, kts, clamp, rec, p_half);
        } else if (mode == kMed) {
          if (pc) score_tile<kMed, true, RECORD>(taddr, R, rp_row, s_rab_time, s_thr, s_anyb, s_thr32, kts, clamp, rec, p_half);
          else score_tile<kMed, false, RECORD>(taddr, R, rp_row, s_rab_time, s_thr, s_anyb, s_thr32, kts, clamp, rec, p_half);
        } else if (mode == kCut) {
          if (pc) score_tile<kCut, true, RECORD>(taddr, R, rp_row, s_rab_time, s_thr, s_anyb, s_thr32, kts, clamp, rec, p_half);
          else score_tile<kCut, false, RECORD>(taddr, R, rp_row, s_rab_time, s_thr, s_anyb, s_thr32, kts, clamp, rec, p_half);
        } else if (mode == kAny) {
          score_tile<kAny, false, RECORD>(taddr, R, rp_row, s_rab_time, s_thr, s_anyb, s_thr32, kts, clamp, rec, p_half);
        } else {
          score_tile<kGen, false, RECORD>(taddr, R, rp_row, s_rab_time, s_thr, s_anyb, s_thr32, kts, clamp, rec, p_half);
        }
        // each warp hands its 32 rows of P over on its own: no warp waits for the
        // others of its group
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          arrive_leader(leader(&p_full[gt % 3]));
          mbar_arrive(&t_empty[st]);
        }
        if (mode == kFast || mode == kMed || mode == kCut) {
          R.b = R.b_last;
          R.cut = R.cut_last;
        }
      }
      if (aborted) break;

      // ---- O / n_norm -> staging (32 columns per warp and pass, group g columns
      // [64 g, 64 g + 64)) -> TMA stores, or reductions into a zeroed O when the
      // pair's key range is split; then O's columns are released to the next item.
      // Groups 0 and 1 read O out; group 2 goes on to the next item's tiles.
      if (g == 2) {
        G += I.n_kt;
        ++n_done;
        continue;
      }
      bool ok = mbar_wait(o_full, n_done & 1, p.wait_limit);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        aborted = true;
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      if (q < I.nq) {
        uint8_t* stage = smem + L::kStage + (g * 4 + wq) * 4096;
#pragma unroll 1
        for (int rd = 0; rd < 2; ++rd) {
          const int col = 64 * g + 32 * rd;
          uint32_t r[32];
          tmem_ld32(tO + lane_off + col, r);
          tmem_ld_wait();
          const uint32_t row_addr = smem_u32(stage + lane * 128);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            st_shared_v4(row_addr + ((e ^ (lane & 7)) << 4), __uint_as_float(r[4 * e + 0]) * inv_nn,
                         __uint_as_float(r[4 * e + 1]) * inv_nn, __uint_as_float(r[4 * e + 2]) * inv_nn,
                         __uint_as_float(r[4 * e + 3]) * inv_nn);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int32_t x = I.h * HD + col;
            const int32_t y = (I.qt0 + q) * 128 + wq * 32;
            if (p.num_splits > 1) tma_reduce_add_2d(&tm_o, stage, x, y);
            else tma_store_2d(&tm_o, stage, x, y);
            bulk_commit_group();
            bulk_wait_group_read0();   // the box is reused by the next pass or item
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_leader(leader(o_empty));
      G += I.n_kt;
      ++n_done;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();   // the peer's tensor memory, barriers and shared memory stay valid until both are done
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.error, HSTU_DEVERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

// ==== host side: launch configuration (no device code below this line) ====

// Key-range splits per pair: with fewer than one and a half work items per
// SM, a pair's key tiles are shared by two CTAs, so that no single CTA carries
// a long user's whole key range while most SMs idle (measured: 9% faster at
// 124 items, 2% slower at 368, where the extra zeroing and reductions cost
// more than the shorter critical path saves).  Two partial sums added into a
// zeroed O give the same result in either order (0 + a + b = 0 + b + a in
// floating point), so the output stays deterministic; more splits would not.
int attention_splits(int num_pairs, int H) {
  const int64_t items = int64_t(num_pairs) * H;
  return 2 * items < 3 * 148 ? 2 : 1;
}

template <int HD, bool RECORD>
cudaError_t launch_hd(const AttnArgs& a, cudaStream_t st) {
  using L = AttnLayout<HD>;
  CUtensorMap tm, tm_ts, tm_o, tm_k;
  if (!make_tmap_2d_bf16(&tm, a.uvqk, uint64_t(4 * a.d), uint64_t(a.T), uint64_t(4 * a.d) * 2,
                         64, 128))
    return cudaErrorInvalidValue;
  if (!make_tmap_1d_i64(&tm_ts, a.ts, uint64_t(a.T), 128)) return cudaErrorInvalidValue;
  if (!make_tmap_2d_f32_sw128(&tm_o, a.av, uint64_t(a.d), uint64_t(a.T), uint64_t(a.d) * 4, 32, 32))
    return cudaErrorInvalidValue;
  static std::atomic<uint64_t> smem_set{0};
  const cudaError_t e = smem_opt_in(attn_tc_kernel<HD, RECORD>,
                                    int(L::smem_bytes(kMaxPosEntries - 1)), smem_set);
  if (e != cudaSuccess) return e;
  AttnParams p;
  p.rows = a.rows;
  p.order = a.order;
  p.ts = a.ts;
  p.thresholds = a.thresholds;
  p.time_lut = a.time_lut;
  p.thr32 = a.thr32;
  p.lut_exact = a.lut_exact;
  p.num_splits = RECORD ? 1 : attention_splits(a.num_pairs, a.H);
  p.wait_limit = a.wait_limit > 0 ? a.wait_limit : kWaitLimit;
  p.rab_pos = a.rab_pos;
  p.rab_time = a.rab_time;
  p.counters = a.counters;
  p.error = a.error;
  p.av = a.av;
  p.T = a.T;
  p.d = a.d;
  p.H = a.H;
  p.num_pairs = a.num_pairs;
  p.pos_clamp = a.pos_clamp;
  p.time_buckets = a.time_buckets;
  p.n_norm_fixed = a.n_norm_fixed;
  p.dump_pidx = a.dump_pidx;
  p.dump_tidx = a.dump_tidx;
  p.dump_vis = a.dump_vis;
  if (p.num_splits > 1) {
    // the splits add their partial sums into O: zero the rows the pairs cover
    const cudaError_t ez = cudaMemsetAsync(a.av + size_t(a.q_row0) * size_t(a.d), 0,
                                           size_t(a.T - a.q_row0) * size_t(a.d) * 4, st);
    if (ez != cudaSuccess) return ez;
  }
  const int64_t grid = int64_t(a.num_pairs) * a.H * p.num_splits;
  if (HD == 128 && !RECORD) {
    // CTA pairs: K halves come through their own tensor map
    if (!make_tmap_2d_bf16(&tm_k, a.uvqk, uint64_t(4 * a.d), uint64_t(a.T), uint64_t(4 * a.d) * 2,
                           64, 64))
      return cudaErrorInvalidValue;
    static std::atomic<uint64_t> pair_set{0};
    const cudaError_t ep = smem_opt_in(attn_tc_pair_kernel,
                                       int(PairLayout::smem_bytes(kMaxPosEntries - 1)), pair_set);
    if (ep != cudaSuccess) return ep;
    // persistent: one cluster per two SMs (or per item, when there are fewer)
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t clusters = grid < sms / 2 ? grid : int64_t(sms / 2 > 0 ? sms / 2 : 1);
    attn_tc_pair_kernel<<<unsigned(2 * clusters), kPairThreads, PairLayout::smem_bytes(a.pos_clamp),
                          st>>>(tm, tm_k, tm_ts, tm_o, p);
    return cudaGetLastError();
  }
  attn_tc_kernel<HD, RECORD><<<unsigned(grid), kThreads, L::smem_bytes(a.pos_clamp), st>>>(tm, tm_ts, tm_o, p);
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
