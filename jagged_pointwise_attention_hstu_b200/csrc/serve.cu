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

// One block per row of the candidate block: thread 0 writes the row's facts
// and timestamp, and the block moves its input row from the packed candidates
// (padding rows: zeros), in 16-byte chunks.
__global__ void candidate_block_kernel(const int32_t* __restrict__ table,
                                       const int32_t* __restrict__ hoff, int32_t B, int64_t T_h,
                                       int64_t q0, const int64_t* __restrict__ cand_ts,
                                       int64_t* __restrict__ ts, RowInfo* __restrict__ rows,
                                       int32_t chunks, const uint4* __restrict__ src,
                                       uint4* __restrict__ dst) {
  const int32_t r = blockIdx.x;
  const int32_t* blk = table;
  const int32_t* coff = table + B + 1;
  const int32_t b = block_of(blk, B, r);
  const int32_t c = r - blk[b];
  const int32_t n_c = coff[b + 1] - coff[b];
  const bool real = c < n_c;
  if (threadIdx.x == 0) {
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
    if (real) t = cand_ts[coff[b] + c];
    else if (h_hi > h_lo) t = ts[h_hi - 1];                  // padding: the history's last time
    else t = n_c > 0 ? cand_ts[coff[b] + n_c - 1] : 0;
    ts[i] = t;
  }
  uint4* d = dst + int64_t(r) * chunks;
  if (real) {
    const uint4* s = src + (int64_t(coff[b]) + c) * chunks;
    for (int32_t k = threadIdx.x; k < chunks; k += blockDim.x) d[k] = s[k];
  } else {
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int32_t k = threadIdx.x; k < chunks; k += blockDim.x) d[k] = z;
  }
}

// Block rows back to the packed order (padding rows dropped), 16-byte chunks.
__global__ void candidate_out_kernel(const int32_t* __restrict__ table, int32_t B, int32_t chunks,
                                     const uint4* __restrict__ src, uint4* __restrict__ dst) {
  const int32_t r = blockIdx.x;
  const int32_t* blk = table;
  const int32_t* coff = table + B + 1;
  const int32_t b = block_of(blk, B, r);
  const int32_t c = r - blk[b];
  if (c >= coff[b + 1] - coff[b]) return;
  const uint4* s = src + int64_t(r) * chunks;
  uint4* d = dst + (int64_t(coff[b]) + c) * chunks;
  for (int32_t k = threadIdx.x; k < chunks; k += blockDim.x) d[k] = s[k];
}

}  // namespace

cudaError_t launch_candidate_block(const int32_t* table, const int32_t* hoff, int32_t B,
                                   int64_t T_h, int64_t q0, int32_t P, const int64_t* cand_ts,
                                   int64_t* ts, RowInfo* rows, int64_t row_bytes, const void* src,
                                   void* dst, cudaStream_t st) {
  if (P <= 0 || B <= 0) return cudaSuccess;
  if (row_bytes % 16 != 0) return cudaErrorInvalidValue;
  const int32_t chunks = int32_t(row_bytes / 16);
  const int threads = chunks < 256 ? ((chunks + 31) / 32) * 32 : 256;
  candidate_block_kernel<<<P, threads, 0, st>>>(table, hoff, B, T_h, q0, cand_ts, ts, rows, chunks,
                                                static_cast<const uint4*>(src),
                                                static_cast<uint4*>(dst));
  return cudaGetLastError();
}

cudaError_t launch_candidate_copy(const int32_t* table, int32_t B, int32_t P, int64_t row_bytes,
                                  const void* src, void* dst, bool to_block, cudaStream_t st) {
  if (P <= 0 || B <= 0) return cudaSuccess;
  if (row_bytes % 16 != 0 || to_block) return cudaErrorInvalidValue;
  const int32_t chunks = int32_t(row_bytes / 16);
  const int threads = chunks < 256 ? ((chunks + 31) / 32) * 32 : 256;
  candidate_out_kernel<<<P, threads, 0, st>>>(table, B, chunks, static_cast<const uint4*>(src),
                                              static_cast<uint4*>(dst));
  return cudaGetLastError();
}

}  // namespace hstu
