// Candidate blocks of the M-FALCON history cache.
//
// M-FALCON scores a user's candidates against the user's history; the history
// computation does not depend on the candidates, so it is done once and kept
// (ltzyclt blog, section 5.2, M-FALCON: candidates see the history and
// themselves, and micro-batches of candidates share the history work; blog
// "Generative Recommendation 16", item 3 "M-FALCON": the candidate-independent
// history computation is cached).  The cache keeps, per layer, the history
// rows of SiLU(f1(X)) in a buffer laid out as
//   rows [0, T_h)          the histories, packed by user (as a causal batch)
//   rows [q0, q0 + P)      q0 = T_h rounded up to 2 * 128: this call's candidates,
//                          user b's block at [q0 + blk[b], q0 + blk[b + 1])
// Each user's block is padded to whole pairs of query tiles so that every pair
// of the attention belongs to one user and visits only that user's history
// tiles.  A candidate row's facts point at its user's history: lo = history
// start, hi = history end (keys [lo, hi) plus itself), pos = history end, so
// that a history key j sits at position n_h - j(local) and the candidate
// itself at position 0.  Padding rows take the same facts (they are scored and
// dropped) and zero inputs, so every value they feed the tensor cores is finite.
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace hstu {
namespace {

// Largest b in [0, B - 1] with blk[b] <= r, for 0 <= r < blk[B]: the block
// that holds row r (blocks of zero rows share their start with the next one).
__device__ __forceinline__ int32_t block_of(const int32_t* __restrict__ blk, int32_t B, int32_t r) {
  int32_t lo = 0, hi = B - 1;
  while (lo < hi) {
    const int32_t mid = (lo + hi + 1) >> 1;
    if (blk[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void candidate_rows_kernel(const int32_t* __restrict__ table,
                                      const int32_t* __restrict__ hoff, int32_t B, int64_t T_h,
                                      int64_t q0, int32_t P, const int64_t* __restrict__ cand_ts,
                                      int64_t* __restrict__ ts, RowInfo* __restrict__ rows) {
  const int32_t r = int32_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= P) return;
  const int32_t* blk = table;
  const int32_t* coff = table + B + 1;
  const int32_t b = block_of(blk, B, r);
  const int32_t c = r - blk[b];
  const int32_t n_c = coff[b + 1] - coff[b];
  // history offsets as the prefill received them, clamped into [0, T_h]
  int64_t h_lo = hoff[b], h_hi = hoff[b + 1];
  h_lo = h_lo < 0 ? 0 : (h_lo > T_h ? T_h : h_lo);
  h_hi = h_hi < h_lo ? h_lo : (h_hi > T_h ? T_h : h_hi);
  const int32_t i = int32_t(q0 + r);
  RowInfo ri;
  if (h_hi > h_lo) {
    ri.lo = int32_t(h_lo);
    ri.hi = int32_t(h_hi);
  } else {   // no history: the row sees itself only
    ri.lo = i;
    ri.hi = i;
  }
  ri.pos = int32_t(h_hi);
  ri.user = b;
  rows[i] = ri;
  int64_t t;
  if (c < n_c) t = cand_ts[coff[b] + c];
  else if (h_hi > h_lo) t = ts[h_hi - 1];                  // padding: the history's last time
  else t = n_c > 0 ? cand_ts[coff[b] + n_c - 1] : 0;
  ts[i] = t;
}

// Pairs of the block ordered by descending cost (history length of their
// user), ties by index: the longest-first order of the attention's work items.
__global__ void candidate_order_kernel(const int32_t* __restrict__ table,
                                       const int32_t* __restrict__ hoff, int32_t B, int64_t T_h,
                                       int32_t n_pairs, int32_t pair0, int32_t* __restrict__ order) {
  extern __shared__ int32_t cost[];
  const int32_t* blk = table;
  for (int32_t k = threadIdx.x; k < n_pairs; k += blockDim.x) {
    const int32_t b = block_of(blk, B, k * 2 * kTile);
    int64_t h_lo = hoff[b], h_hi = hoff[b + 1];
    h_lo = h_lo < 0 ? 0 : (h_lo > T_h ? T_h : h_lo);
    h_hi = h_hi < h_lo ? h_lo : (h_hi > T_h ? T_h : h_hi);
    cost[k] = int32_t(h_hi - h_lo);
  }
  __syncthreads();
  for (int32_t k = threadIdx.x; k < n_pairs; k += blockDim.x) {
    const int32_t ck = cost[k];
    int32_t rank = 0;
    for (int32_t q = 0; q < n_pairs; ++q) {
      const int32_t cq = cost[q];
      rank += (cq > ck || (cq == ck && q < k)) ? 1 : 0;
    }
    order[rank] = pair0 + k;
  }
}

// One block per block row; 16-byte chunks.
__global__ void candidate_copy_kernel(const int32_t* __restrict__ table, int32_t B,
                                      int32_t chunks, const uint4* __restrict__ src,
                                      uint4* __restrict__ dst, int to_block) {
  const int32_t r = blockIdx.x;
  const int32_t* blk = table;
  const int32_t* coff = table + B + 1;
  const int32_t b = block_of(blk, B, r);
  const int32_t c = r - blk[b];
  const bool real = c < coff[b + 1] - coff[b];
  const int64_t packed = int64_t(coff[b]) + c;
  if (to_block) {
    uint4* d = dst + int64_t(r) * chunks;
    if (real) {
      const uint4* s = src + packed * chunks;
      for (int32_t k = threadIdx.x; k < chunks; k += blockDim.x) d[k] = s[k];
    } else {
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
      for (int32_t k = threadIdx.x; k < chunks; k += blockDim.x) d[k] = z;
    }
  } else if (real) {
    const uint4* s = src + int64_t(r) * chunks;
    uint4* d = dst + packed * chunks;
    for (int32_t k = threadIdx.x; k < chunks; k += blockDim.x) d[k] = s[k];
  }
}

}  // namespace

cudaError_t launch_candidate_rows(const int32_t* table, const int32_t* hoff, int32_t B,
                                  int64_t T_h, int64_t q0, int32_t P, const int64_t* cand_ts,
                                  int64_t* ts, RowInfo* rows, int32_t* order, cudaStream_t st) {
  if (P <= 0 || B <= 0) return cudaSuccess;
  const int32_t n_pairs = P / (2 * kTile);
  if (n_pairs * 2 * kTile != P || n_pairs > kMaxCandidatePairs) return cudaErrorInvalidValue;
  candidate_rows_kernel<<<(P + 255) / 256, 256, 0, st>>>(table, hoff, B, T_h, q0, P, cand_ts, ts,
                                                        rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  candidate_order_kernel<<<1, 1024, size_t(n_pairs) * 4, st>>>(table, hoff, B, T_h, n_pairs,
                                                               int32_t(q0 / (2 * kTile)), order);
  return cudaGetLastError();
}

cudaError_t launch_candidate_copy(const int32_t* table, int32_t B, int32_t P, int64_t row_bytes,
                                  const void* src, void* dst, bool to_block, cudaStream_t st) {
  if (P <= 0 || B <= 0) return cudaSuccess;
  if (row_bytes % 16 != 0) return cudaErrorInvalidValue;
  const int32_t chunks = int32_t(row_bytes / 16);
  const int threads = chunks < 256 ? ((chunks + 31) / 32) * 32 : 256;
  candidate_copy_kernel<<<P, threads, 0, st>>>(table, B, chunks, static_cast<const uint4*>(src),
                                               static_cast<uint4*>(dst), to_block ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace hstu
