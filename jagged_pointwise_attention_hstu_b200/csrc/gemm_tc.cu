// f1 and f2 of the HSTU layer as tcgen05 GEMMs over the jagged token axis.
//
//   f1:  UVQK = SiLU(X W1^T + b1)      (blog "Generative Recommendation 16:
//        HSTU", section "HSTU Layer 到底改了什么", equation (1); the split into
//        U, V, Q, K is the column order of the output, so it costs nothing)
//   f2:  Y = G W2^T + b2 + X           (equation (3) plus the residual)
//
// The token axis is never padded: M = T rows ("fully ragged GEMM", item 1 of
// the same blog's list of extra pieces); TMA zero-fills rows past T and the
// epilogue masks them.
//
// Persistent, warp-specialised: warp 0 streams A/B k-blocks with TMA into a
// 4-stage ring, warp 1 issues 128 x BN x 16 MMAs into one of two tensor-memory
// accumulators, warps 2-9 drain the other accumulator through the fused
// epilogue (two warps per tensor-memory lane quarter, each taking half of the
// columns), so the epilogue of tile t overlaps the MMAs of tile t+1.  Each
// epilogue warp stages 32 rows x 128 bytes of output at a time in its own
// 128-byte-swizzled shared box and writes it with a TMA store, which clips the
// rows past M.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "sm100.cuh"

namespace hstu {
namespace {

using namespace sm100;

constexpr int kBK = 64;   // one 128-byte swizzle row of bf16

struct GemmParams {
  int64_t M;
  int N, K;
  int epi;              // Epi
  const float* bias;
  void* out;
  const void* residual;
  int io_fp32;
  int out_bf16;         // fp32 out: also store bf16(out) through tma_out2
  long long wait_limit; // bound of the pipeline waits (the drains keep the default)
  int32_t* error;
};

// PAIR: a cluster of two CTAs computes a 256 x BN tile with cta_group::2
// products (each CTA holds 128 rows of A and BN / 2 rows of the B tile).
// RES (with PAIR, fp32 output + fp32 residual): the residual comes in by TMA
// through a ring of kResSlots boxes per epilogue warp, two 32-column chunks
// ahead of use; the output is formed in place in the residual's box and
// stored from there, so the plain output boxes are not needed.  The epilogue
// is the bound there, so the operand ring is shorter.
constexpr int kResSlots = 3;
template <int BN, bool PAIR, bool RES = false>
struct GemmLayout {
  static_assert(!RES || PAIR, "the residual ring is laid out for CTA pairs");
  static constexpr int kStages = RES ? 3 : (PAIR ? 5 : 4);
  static constexpr uint32_t kABytes = 128 * kBK * 2;
  static constexpr uint32_t kBBytes = (PAIR ? BN / 2 : BN) * kBK * 2;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kOutOffset = kStages * kStageBytes;   // 8 boxes of 4 KB (not RES)
  // PAIR: 8 boxes of 2 KB of their own for the bf16 copy of an fp32 output
  static constexpr uint32_t kOut2Offset = kOutOffset + (RES ? 0 : 8 * 4096);
  static constexpr uint32_t kResOffset = kOut2Offset + (PAIR ? 8 * 2048 : 0);
  static constexpr uint32_t kBarOffset = kResOffset + (RES ? 8 * kResSlots * 4096 : 0);
  static constexpr uint32_t kSmemBytes = kBarOffset + 512 + 1024;   // + alignment slack
  static_assert(kABytes % 1024 == 0 && kStageBytes % 1024 == 0, "TMA destinations 1024-aligned");
  static_assert(kOut2Offset % 1024 == 0 && kResOffset % 1024 == 0, "box alignment");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  // mbarriers: the ring (2 kStages), 4 accumulator, drain, 8 x kResSlots residual; two words
  static_assert((2 * kStages + 5 + 8 * kResSlots) * 8 + 8 <= 512, "barrier block");
};

// SiLU(v) = v / (1 + e^-v) with the hardware exp2 and reciprocal (relative
// error ~1e-7, far below the bf16 rounding that follows).  For v < -88 the
// exponential overflows to +inf and the quotient is -0, the correct limit.
__device__ __forceinline__ float silu_f(float v) { return __fdividef(v, 1.0f + __expf(-v)); }

constexpr int kGemmThreads = 320;

template <int BN, bool PAIR, bool RES>
__device__ __forceinline__ void gemm_body(const CUtensorMap* tma_a, const CUtensorMap* tma_b,
                                          const CUtensorMap* tma_out, const CUtensorMap* tma_out2,
                                          const CUtensorMap* tma_res, const GemmParams& p) {
  using L = GemmLayout<BN, PAIR, RES>;
  constexpr int kStages = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOffset);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;   // [2]
  uint64_t* acc_empty = acc_full + 2;     // [2]
  uint64_t* drain = acc_empty + 2;
  uint64_t* res_full = drain + 1;         // [8 warps][kResSlots] (RES)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(res_full + 8 * kResSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // PAIR: this CTA's half of the cluster's 256-row tile; the leader (rank 0)
  // counts both CTAs' loads and epilogue releases and issues every product
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  auto leader = [&](uint64_t* bar) -> uint32_t { return map_to_rank(smem_u32(bar), 0); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], PAIR ? 16 : 256);   // PAIR: each epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    for (int r = 0; r < 8 * kResSlots; ++r) mbar_init(&res_full[r], 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, 2 * BN);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, 2 * BN);
      tmem_relinquish();
    }
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(tma_a);
    prefetch_tmap(tma_b);
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();   // the leader's barriers exist before the peer's loads signal them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  constexpr int kTileM = PAIR ? 256 : 128;
  const int64_t m_tiles = (p.M + kTileM - 1) / kTileM;
  const int n_tiles = p.N / BN;
  const int64_t total = m_tiles * n_tiles;
  const int kblocks = p.K / kBK;
  const int64_t t0 = PAIR ? int64_t(blockIdx.x >> 1) : int64_t(blockIdx.x);
  const int64_t t_step = PAIR ? int64_t(gridDim.x >> 1) : int64_t(gridDim.x);

  if (warp == 0) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t issued_phase[kStages];
      bool issued[kStages];
      for (int s = 0; s < kStages; ++s) issued[s] = false, issued_phase[s] = 0;
      for (int64_t t = t0; t < total && !*abort_flag; t += t_step) {
        const int64_t mt = t / n_tiles;
        const int nt = int(t % n_tiles);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, p.wait_limit)) { *abort_flag = 1; break; }
          uint8_t* sa = smem + stage * L::kStageBytes;
          if constexpr (PAIR) {
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * L::kStageBytes);
            tma_load_2d_pair(sa, tma_a, leader(&full[stage]), kb * kBK,
                             int32_t(mt * 256 + rank * 128));
            tma_load_2d_pair(sa + L::kABytes, tma_b, leader(&full[stage]), kb * kBK,
                             nt * BN + int(rank) * (BN / 2));
          } else {
            mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
            tma_load_2d(sa, tma_a, &full[stage], kb * kBK, int32_t(mt * 128));
            tma_load_2d(sa + L::kABytes, tma_b, &full[stage], kb * kBK, nt * BN);
          }
          issued[stage] = true;
          issued_phase[stage] = phase;
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
      // every load this thread issued has landed before the CTA may exit (PAIR:
      // the leader counts them, so wait for the products that read the stage)
      for (int s = 0; s < kStages; ++s)
        if (issued[s]) {
          if constexpr (PAIR) mbar_wait(&empty[s], issued_phase[s]);
          else mbar_wait(&full[s], issued_phase[s]);
        }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16(PAIR ? 256 : 128, BN, false, false);
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool any = false;
      for (int64_t t = t0; t < total && !*abort_flag; t += t_step) {
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, p.wait_limit)) { *abort_flag = 1; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.wait_limit)) { *abort_flag = 1; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * L::kStageBytes);
          const uint32_t b_addr = a_addr + L::kABytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            if constexpr (PAIR)
              umma_ss_pair(d_tmem, desc_sw128(a_addr + k * 32, 16, 1024),
                           desc_sw128(b_addr + k * 32, 16, 1024), idesc, (kb | k) != 0);
            else
              umma_ss(d_tmem, desc_sw128(a_addr + k * 32, 16, 1024),
                      desc_sw128(b_addr + k * 32, 16, 1024), idesc, (kb | k) != 0);
          }
          if constexpr (PAIR) umma_commit_pair(&empty[stage]);
          else umma_commit(&empty[stage]);
          any = true;
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if constexpr (PAIR) umma_commit_pair(&acc_full[acc]);
        else umma_commit(&acc_full[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      if (any) {
        if constexpr (PAIR) umma_commit_pair(drain);
        else umma_commit(drain);
        mbar_wait(drain, 0);
      }
    }
  } else {
    // epilogue: warps 2..9; warp w reads the 32 tensor-memory lanes of quarter
    // w % 4 and the column half (w - 2) / 4 of the tile
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int c_begin = ((warp - 2) >> 2) * (BN / 2);
    uint8_t* box = smem + L::kOutOffset + (warp - 2) * 4096;
    uint8_t* box2 = smem + L::kOut2Offset + (warp - 2) * 2048;   // PAIR only
    const uint32_t row_addr = smem_u32(box + lane * 128);
    // 16-byte chunk e of this thread's 128-byte box row (128-byte swizzle)
    auto chunk = [&](int e) -> uint32_t { return row_addr + ((e ^ (lane & 7)) << 4); };
    const bool out_bf16 = p.epi == int(Epi::kSiluSplit) || !p.io_fp32;
    const int step = out_bf16 ? 64 : 32;   // columns per 128-byte box row
    uint32_t acc = 0, acc_phase = 0;
    if constexpr (RES) {
      // fp32 output = acc + bias + the fp32 residual, 32 columns per chunk; the
      // warp's chunk k is tile t0 + (k / kChunks) t_step, columns c_begin + 32 (k % kChunks)
      constexpr int kChunks = (BN / 2) / 32;
      const int wi = warp - 2;
      uint8_t* rbox = smem + L::kResOffset + wi * kResSlots * 4096;
      uint64_t* rbar = res_full + wi * kResSlots;
      int64_t issued = -1;   // the last chunk whose residual load was issued (lane 0)
      auto issue_res = [&](int64_t k) {
        const int64_t tt = t0 + (k / kChunks) * t_step;
        if (tt >= total) return;
        const int cc = c_begin + 32 * int(k % kChunks);
        const int slot = int(k % kResSlots);
        mbar_arrive_expect_tx(&rbar[slot], 4096);
        tma_load_2d(rbox + slot * 4096, tma_res, &rbar[slot], int(tt % n_tiles) * BN + cc,
                    int32_t((tt / n_tiles) * kTileM + int64_t(rank) * 128 + q * 32));
        issued = k;
      };
      if (lane == 0) {
        issue_res(0);
        issue_res(1);
      }
      int64_t k = 0;
      bool ok = true;
      for (int64_t t = t0; ok && t < total; t += t_step) {
        if (*abort_flag) break;
        const int64_t mt = t / n_tiles;
        const int nt = int(t % n_tiles);
        const int64_t row0 = mt * kTileM + int64_t(rank) * 128;   // this CTA's first row
        if (!mbar_wait(&acc_full[acc], acc_phase, p.wait_limit)) { *abort_flag = 1; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c = c_begin; c < c_begin + BN / 2; c += 32, ++k) {
          const int col0 = nt * BN + c;
          const int slot = int(k % kResSlots);
          uint32_t r[32];
          tmem_ld32(tmem_base + acc * BN + c + (uint32_t(q * 32) << 16), r);
          ok = __all_sync(0xffffffffu,
                          mbar_wait(&rbar[slot], uint32_t(k / kResSlots) & 1, p.wait_limit));
          tmem_ld_wait();
          if (!ok) {
            *abort_flag = 1;
            break;
          }
          // the residual's box row of this thread (128-byte swizzle), overwritten by the output
          const uint32_t xrow = smem_u32(rbox + slot * 4096 + lane * 128);
          const float4* b4 = reinterpret_cast<const float4*>(p.bias + col0);
          float v[32];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t at = xrow + ((e ^ (lane & 7)) << 4);
            const float4 x = ld_shared_v4(at);
            const float4 bb = __ldg(b4 + e);
            v[4 * e + 0] = __uint_as_float(r[4 * e + 0]) + bb.x + x.x;
            v[4 * e + 1] = __uint_as_float(r[4 * e + 1]) + bb.y + x.y;
            v[4 * e + 2] = __uint_as_float(r[4 * e + 2]) + bb.z + x.z;
            v[4 * e + 3] = __uint_as_float(r[4 * e + 3]) + bb.w + x.w;
            st_shared_v4(at, v[4 * e + 0], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
          }
          // the previous chunk's stores have read their boxes: its residual slot
          // takes chunk k + 2, and the bf16 box is refilled
          if (lane == 0) {
            bulk_wait_group_read0();
            issue_res(k + 2);
          }
          __syncwarp();
          if (p.out_bf16) {
            // 64-byte box rows, 64-byte swizzle (16-byte chunk e of row r sits at
            // chunk e ^ ((r / 2) mod 4))
            const uint32_t row64 = smem_u32(box2 + lane * 64);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              st_shared_v4_u32(row64 + ((e ^ ((lane >> 1) & 3)) << 4),
                               pack_bf16x2(v[8 * e + 0], v[8 * e + 1]),
                               pack_bf16x2(v[8 * e + 2], v[8 * e + 3]),
                               pack_bf16x2(v[8 * e + 4], v[8 * e + 5]),
                               pack_bf16x2(v[8 * e + 6], v[8 * e + 7]));
          }
          fence_proxy_async_smem();   // make the stores visible to the TMA unit
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(tma_out, rbox + slot * 4096, col0, int32_t(row0 + q * 32));
            if (p.out_bf16) tma_store_2d(tma_out2, box2, col0, int32_t(row0 + q * 32));
            bulk_commit_group();
          }
          __syncwarp();
        }
        if (!ok) break;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_leader(leader(&acc_empty[acc]));
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      // no residual load lands and no store reads shared memory after the exit
      if (lane == 0) {
        for (int64_t kk = k; kk <= issued; ++kk)
          mbar_wait(&rbar[kk % kResSlots], uint32_t(kk / kResSlots) & 1, p.wait_limit);
        bulk_wait_group_read0();
      }
      __syncwarp();
    } else {
    for (int64_t t = t0; t < total; t += t_step) {
      if (*abort_flag) break;
      const int64_t mt = t / n_tiles;
      const int nt = int(t % n_tiles);
      const int64_t row0 = mt * kTileM + int64_t(rank) * 128;   // this CTA's first row
      const int64_t grow = row0 + row;
      const bool valid = grow < p.M;   // rows past M are computed on zeros and clipped by the store
      // fp32 residual: the loads of a chunk are issued one chunk ahead (the
      // first chunk's before the wait for the accumulator), so that their
      // latency overlaps the products and the previous chunk's epilogue
      const float4* res_row = reinterpret_cast<const float4*>(
          static_cast<const float*>(p.residual) + grow * int64_t(p.N) + nt * BN);
      float4 xnext[8];
      if (!out_bf16) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          xnext[e] = valid ? res_row[c_begin / 4 + e] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      if (!mbar_wait(&acc_full[acc], acc_phase, p.wait_limit)) { *abort_flag = 1; break; }
      tc_fence_after();
#pragma unroll 1
      for (int c = c_begin; c < c_begin + BN / 2; c += step) {
        const int col0 = nt * BN + c;
        if (!out_bf16) {
          // fp32 output: acc + bias + the fp32 residual (32 columns)
          float4 xres[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) xres[e] = xnext[e];
          if (c + step < c_begin + BN / 2) {
#pragma unroll
            for (int e = 0; e < 8; ++e)
              xnext[e] = valid ? res_row[(c + step) / 4 + e] : make_float4(0.f, 0.f, 0.f, 0.f);
          }
          uint32_t r[32];
          tmem_ld32(tmem_base + acc * BN + c + (uint32_t(q * 32) << 16), r);
          tmem_ld_wait();
          const float4* b4 = reinterpret_cast<const float4*>(p.bias + col0);
          float v[32];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float4 bb = __ldg(b4 + e);
            const float4 x = xres[e];
            v[4 * e + 0] = __uint_as_float(r[4 * e + 0]) + bb.x + x.x;
            v[4 * e + 1] = __uint_as_float(r[4 * e + 1]) + bb.y + x.y;
            v[4 * e + 2] = __uint_as_float(r[4 * e + 2]) + bb.z + x.z;
            v[4 * e + 3] = __uint_as_float(r[4 * e + 3]) + bb.w + x.w;
          }
          // the boxes went to the TMA unit in the previous step: refill them once
          // it has read them (the wait overlaps this step's loads and arithmetic)
          if (lane == 0) bulk_wait_group_read0();
          __syncwarp();
#pragma unroll
          for (int e = 0; e < 8; ++e)
            st_shared_v4(chunk(e), v[4 * e + 0], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
          // bf16 copy of the 32 fp32 columns: 64-byte box rows, 64-byte swizzle
          // (16-byte chunk e of row r sits at chunk e ^ ((r / 2) mod 4)); PAIR
          // stages it in a box of its own, else in the fp32 box once that is read
          auto stage_bf16 = [&](uint8_t* b) {
            const uint32_t row64 = smem_u32(b + lane * 64);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              st_shared_v4_u32(row64 + ((e ^ ((lane >> 1) & 3)) << 4),
                               pack_bf16x2(v[8 * e + 0], v[8 * e + 1]),
                               pack_bf16x2(v[8 * e + 2], v[8 * e + 3]),
                               pack_bf16x2(v[8 * e + 4], v[8 * e + 5]),
                               pack_bf16x2(v[8 * e + 6], v[8 * e + 7]));
          };
          if (PAIR && p.out_bf16) stage_bf16(box2);
          fence_proxy_async_smem();   // make the stores visible to the TMA unit
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(tma_out, box, col0, int32_t(row0 + q * 32));
            if (PAIR && p.out_bf16) tma_store_2d(tma_out2, box2, col0, int32_t(row0 + q * 32));
            bulk_commit_group();
          }
          __syncwarp();
          if (!PAIR && p.out_bf16) {
            if (lane == 0) bulk_wait_group_read0();
            __syncwarp();
            stage_bf16(box);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(tma_out2, box, col0, int32_t(row0 + q * 32));
              bulk_commit_group();
            }
            __syncwarp();
          }
          continue;
        }
        // bf16 output (64 columns): SiLU-split, or + bias + the bf16 residual
        float v[64];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t r[32];
          tmem_ld32(tmem_base + acc * BN + c + 32 * h + (uint32_t(q * 32) << 16), r);
          tmem_ld_wait();
          const float4* b4 = reinterpret_cast<const float4*>(p.bias + col0 + 32 * h);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float4 bb = __ldg(b4 + e);
            v[32 * h + 4 * e + 0] = __uint_as_float(r[4 * e + 0]) + bb.x;
            v[32 * h + 4 * e + 1] = __uint_as_float(r[4 * e + 1]) + bb.y;
            v[32 * h + 4 * e + 2] = __uint_as_float(r[4 * e + 2]) + bb.z;
            v[32 * h + 4 * e + 3] = __uint_as_float(r[4 * e + 3]) + bb.w;
          }
        }
        // the box went to the TMA unit in the previous step: refill it once read
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
        if (p.epi == int(Epi::kSiluSplit)) {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            st_shared_v4_u32(chunk(e), pack_bf16x2(silu_f(v[8 * e + 0]), silu_f(v[8 * e + 1])),
                             pack_bf16x2(silu_f(v[8 * e + 2]), silu_f(v[8 * e + 3])),
                             pack_bf16x2(silu_f(v[8 * e + 4]), silu_f(v[8 * e + 5])),
                             pack_bf16x2(silu_f(v[8 * e + 6]), silu_f(v[8 * e + 7])));
        } else {
          const uint4* res = reinterpret_cast<const uint4*>(
              static_cast<const uint16_t*>(p.residual) + grow * int64_t(p.N) + col0);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint4 x = valid ? res[e] : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
            uint32_t os[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const float lo = __uint_as_float(xs[w] << 16);
              const float hi = __uint_as_float(xs[w] & 0xFFFF0000u);
              os[w] = pack_bf16x2(v[8 * e + 2 * w] + lo, v[8 * e + 2 * w + 1] + hi);
            }
            st_shared_v4_u32(chunk(e), os[0], os[1], os[2], os[3]);
          }
        }
        fence_proxy_async_smem();   // make the stores visible to the TMA unit
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(tma_out, box, col0, int32_t(row0 + q * 32));
          bulk_commit_group();
        }
        __syncwarp();
      }
      tc_fence_before();
      if constexpr (PAIR) {
        __syncwarp();
        if (lane == 0) arrive_leader(leader(&acc_empty[acc]));
      } else {
        mbar_arrive(&acc_empty[acc]);
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    if (lane == 0) bulk_wait_group_read0();   // no store still reads shared memory at exit
    __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();   // the leader's products read the peer's memory until done
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.error, HSTU_DEVERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, 2 * BN);
    else tmem_dealloc(tmem_base, 2 * BN);
  }
}

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tma_a,
                   const __grid_constant__ CUtensorMap tma_b,
                   const __grid_constant__ CUtensorMap tma_out,
                   const __grid_constant__ CUtensorMap tma_out2,
                   const __grid_constant__ CUtensorMap tma_res, const GemmParams p) {
  gemm_body<BN, false, false>(&tma_a, &tma_b, &tma_out, &tma_out2, &tma_res, p);
}

// 256 x 256 output tiles on a cluster of two CTAs (M = 256 cta_group::2
// products): each SM brings in half of every B tile, so the L2 -> shared
// memory operand stream per output element is a third smaller than with
// 128 x 256 tiles.  The loads are plain (no multicast).
// RES: the fp32-residual epilogue with the residual brought in by TMA.
template <bool RES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_tc_pair_kernel(const __grid_constant__ CUtensorMap tma_a,
                        const __grid_constant__ CUtensorMap tma_b,
                        const __grid_constant__ CUtensorMap tma_out,
                        const __grid_constant__ CUtensorMap tma_out2,
                        const __grid_constant__ CUtensorMap tma_res, const GemmParams p) {
  gemm_body<256, true, RES>(&tma_a, &tma_b, &tma_out, &tma_out2, &tma_res, p);
}

template <int BN, bool PAIR, bool RES = false>
cudaError_t launch_bn(const GemmArgs& a, int num_sms, cudaStream_t st, int32_t* error) {
  using L = GemmLayout<BN, PAIR, RES>;
  CUtensorMap ta, tb, to, to2, tr;
  if (!make_tmap_2d_bf16(&ta, a.a, uint64_t(a.K), uint64_t(a.M), uint64_t(a.K) * 2, kBK, 128))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d_bf16(&tb, a.b, uint64_t(a.K), uint64_t(a.N), uint64_t(a.K) * 2, kBK,
                         PAIR ? BN / 2 : BN))
    return cudaErrorInvalidValue;
  // output boxes: 32 rows x 128 bytes (64 bf16 or 32 fp32 columns)
  const bool out_f32 = a.epi == Epi::kBiasResidual && a.io_fp32;
  const bool ok_o = out_f32 ? make_tmap_2d_f32_sw128(&to, a.out, uint64_t(a.N), uint64_t(a.M),
                                                     uint64_t(a.N) * 4, 32, 32)
                            : make_tmap_2d_bf16(&to, a.out, uint64_t(a.N), uint64_t(a.M),
                                                uint64_t(a.N) * 2, 64, 32);
  if (!ok_o) return cudaErrorInvalidValue;
  const bool copy = out_f32 && a.out_bf16 != nullptr;
  to2 = to;   // unused unless copy
  if (copy && !make_tmap_2d_bf16_sw64(&to2, a.out_bf16, uint64_t(a.N), uint64_t(a.M),
                                      uint64_t(a.N) * 2, 32, 32))
    return cudaErrorInvalidValue;
  tr = to;   // unused unless RES: the fp32 residual in the output's box format
  if (RES && !make_tmap_2d_f32_sw128(&tr, a.residual, uint64_t(a.N),
                                     uint64_t(a.M), uint64_t(a.N) * 4, 32, 32))
    return cudaErrorInvalidValue;
  static std::atomic<uint64_t> smem_set{0};
  const cudaError_t e =
      PAIR ? smem_opt_in(gemm_tc_pair_kernel<RES>, int(L::kSmemBytes), smem_set)
           : smem_opt_in(gemm_tc_kernel<BN>, int(L::kSmemBytes), smem_set);
  if (e != cudaSuccess) return e;
  GemmParams p;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.epi = int(a.epi);
  p.bias = a.bias;
  p.out = a.out;
  p.residual = a.residual;
  p.io_fp32 = a.io_fp32;
  p.out_bf16 = copy ? 1 : 0;
  p.wait_limit = a.wait_limit > 0 ? a.wait_limit : kWaitLimit;
  p.error = error;
  if constexpr (PAIR) {
    const int64_t tiles = ((a.M + 255) / 256) * (a.N / BN);
    const int64_t clusters = tiles < num_sms / 2 ? tiles : int64_t(num_sms / 2);
    gemm_tc_pair_kernel<RES><<<unsigned(2 * clusters), kGemmThreads, L::kSmemBytes, st>>>(
        ta, tb, to, to2, tr, p);
  } else {
    const int64_t tiles = ((a.M + 127) / 128) * (a.N / BN);
    const int grid = int(tiles < num_sms ? tiles : num_sms);
    gemm_tc_kernel<BN><<<grid, kGemmThreads, L::kSmemBytes, st>>>(ta, tb, to, to2, tr, p);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_tc(const GemmArgs& a, int num_sms, cudaStream_t st, int32_t* error) {
  if (a.M <= 0) return cudaSuccess;
  if (a.K % kBK != 0 || a.N % 128 != 0) return cudaErrorInvalidValue;
  // CTA pairs when there are 256 x 256 tiles for every pair of SMs (measured
  // on one c3 layer: f1 7.5% and f2 4% faster than 128 x 256 tiles)
  if (a.N % 256 == 0 && num_sms >= 2 &&
      ((a.M + 255) / 256) * (a.N / 256) >= num_sms / 2) {
    if (a.epi == Epi::kBiasResidual && a.io_fp32) return launch_bn<256, true, true>(a, num_sms, st, error);
    return launch_bn<256, true>(a, num_sms, st, error);
  }
  // 128 x 256 tiles when they fill a wave, else 128 x 128 (twice the tiles)
  if (a.N % 256 == 0 && ((a.M + 127) / 128) * (a.N / 256) >= num_sms)
    return launch_bn<256, false>(a, num_sms, st, error);
  return launch_bn<128, false>(a, num_sms, st, error);
}

}  // namespace hstu
