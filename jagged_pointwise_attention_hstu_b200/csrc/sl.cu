// Stochastic Length on the device: builds the sampled training batch.
//
// A user's sequence of n actions is kept whole with probability N_c^alpha /
// n^2, otherwise a sub-sequence of N_c actions is sampled (ltzyclt blog on
// HSTU, section 5.1; blog "Generative Recommendation 16", item 2 "Stochastic
// Length": alpha = 1.6 keeps length 4096 mostly at 776).  The draws are
// inputs: u_b per user (whole iff u_b * n^2 < N_c^alpha, fp64, or n <= N_c)
// and a 32-bit key per action; the sub-sequence is the N_c actions with the
// smallest (key, position) pairs, kept in time order.
//
// Four launches, all bound by memory traffic:
//   select  one block per user: the decision, and for a sampled user a
//           bitonic sort of its (key, position) pairs in shared memory; flags
//           the kept actions and counts them
//   scan    one block: the new offsets (running sums of the counts)
//   index   one block per user: a block-wide scan of the flags gives every kept
//           action its output slot: global index and timestamp
//   rows    gathers the kept rows of the values (16-byte chunks)
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace hstu {
namespace {

constexpr int kSlThreads = 1024;

// The user's range, clamped so that a bad offset table stays in bounds
// (such a user counts as empty and sets the offsets error bit).
__device__ __forceinline__ bool user_range(const int32_t* offs, int32_t B, int64_t T, int32_t b,
                                           int64_t& lo, int64_t& hi) {
  lo = offs[b];
  hi = offs[b + 1];
  const bool bad = lo < 0 || hi < lo || hi > T || (b == 0 && lo != 0) || (b == B - 1 && hi != T);
  if (bad) {
    lo = 0;
    hi = 0;
  }
  return !bad;
}

__global__ void __launch_bounds__(kSlThreads)
sl_select_kernel(const int32_t* __restrict__ offs, int32_t B, int64_t T,
                 const double* __restrict__ u, const uint32_t* __restrict__ keys, int32_t n_c,
                 double numerator, uint8_t* __restrict__ flags, int32_t* __restrict__ kept,
                 int32_t* __restrict__ err) {
  extern __shared__ unsigned long long s_pairs[];   // kSlMaxLen
  const int32_t b = blockIdx.x;
  const int tid = threadIdx.x;
  int64_t lo, hi;
  const bool ok = user_range(offs, B, T, b, lo, hi);
  if (!ok && tid == 0) atomicOr(err, HSTU_DEVERR_OFFSETS);
  const int64_t n = hi - lo;
  const bool whole = n <= n_c || u[b] * double(n * n) < numerator;
  if (whole || n > kSlMaxLen) {
    const uint8_t f = whole ? 1 : 0;
    for (int64_t i = tid; i < n; i += blockDim.x) flags[lo + i] = f;
    if (tid == 0) {
      kept[b] = whole ? int32_t(n) : 0;
      if (!whole) atomicOr(err, HSTU_DEVERR_SL_TOO_LONG);
    }
    return;
  }
  int32_t m = 1;   // the sort's size: a power of two >= n (n <= kSlMaxLen)
  while (m < n) m <<= 1;
  for (int32_t i = tid; i < m; i += blockDim.x)
    s_pairs[i] = i < n ? (static_cast<unsigned long long>(keys[lo + i]) << 32) | uint32_t(i)
                       : ~0ull;
  __syncthreads();
  for (int32_t k = 2; k <= m; k <<= 1) {
    for (int32_t j = k >> 1; j > 0; j >>= 1) {
      for (int32_t i = tid; i < m; i += blockDim.x) {
        const int32_t p = i ^ j;
        if (p > i) {
          const unsigned long long a = s_pairs[i], c = s_pairs[p];
          const bool ascending = (i & k) == 0;
          if ((a > c) == ascending) {
            s_pairs[i] = c;
            s_pairs[p] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  const unsigned long long last = s_pairs[n_c - 1];   // the n_c-th smallest pair
  for (int32_t i = tid; i < n; i += blockDim.x) {
    const unsigned long long key = (static_cast<unsigned long long>(keys[lo + i]) << 32) | uint32_t(i);
    flags[lo + i] = key <= last ? 1 : 0;
  }
  if (tid == 0) kept[b] = n_c;
}

// Inclusive sum over the block of v (blockDim.x a multiple of 32, <= 1024);
// *total receives the block's sum.  Every thread must call it.
__device__ __forceinline__ int64_t block_inclusive_sum(int64_t v, int64_t* s_warp, int64_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  if (lane == 31) s_warp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int64_t w = lane < nwarps ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t t = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += t;
    }
    if (lane < nwarps) s_warp[lane] = w;   // inclusive over warps
  }
  __syncthreads();
  if (warp > 0) v += s_warp[warp - 1];
  *total = s_warp[nwarps - 1];
  __syncthreads();   // s_warp is reused by the next call
  return v;
}

// New offsets: running sums of the kept counts, capped at T so that a bad
// offset table (overlapping users) cannot push any write past the outputs.
__global__ void __launch_bounds__(kSlThreads)
sl_scan_kernel(const int32_t* __restrict__ kept, int32_t B, int64_t T,
               int32_t* __restrict__ out_offs) {
  __shared__ int64_t s_warp[32];
  int64_t carry = 0;
  for (int32_t base = 0; base < B; base += blockDim.x) {
    const int32_t i = base + threadIdx.x;
    const int64_t v = i < B ? kept[i] : 0;
    int64_t total;
    const int64_t inc = block_inclusive_sum(v, s_warp, &total);
    if (i < B) {
      const int64_t ex = carry + inc - v;
      out_offs[i] = int32_t(ex < T ? ex : T);
    }
    carry += total;
  }
  if (threadIdx.x == 0) out_offs[B] = int32_t(carry < T ? carry : T);
}

__global__ void __launch_bounds__(kSlThreads)
sl_index_kernel(const int32_t* __restrict__ offs, int32_t B, int64_t T,
                const uint8_t* __restrict__ flags, const int32_t* __restrict__ out_offs,
                const int64_t* __restrict__ ts, int64_t* __restrict__ out_index,
                int64_t* __restrict__ out_ts) {
  __shared__ int64_t s_warp[32];
  const int32_t b = blockIdx.x;
  int64_t lo, hi;
  user_range(offs, B, T, b, lo, hi);
  const int64_t n = hi - lo;
  const int64_t base = out_offs[b];
  const int64_t cap = int64_t(out_offs[b + 1]) - base;
  int64_t run = 0;
  for (int64_t c = 0; c < n; c += blockDim.x) {
    const int64_t i = c + threadIdx.x;
    const int64_t f = i < n ? flags[lo + i] : 0;
    int64_t total;
    const int64_t slot = run + block_inclusive_sum(f, s_warp, &total) - f;
    if (f && slot < cap) {
      out_index[base + slot] = lo + i;
      if (out_ts != nullptr) out_ts[base + slot] = ts[lo + i];
    }
    run += total;
  }
}

__global__ void sl_rows_kernel(const int32_t* __restrict__ out_offs, int32_t B, int64_t T,
                               const int64_t* __restrict__ out_index, int32_t chunks,
                               const uint4* __restrict__ src, uint4* __restrict__ dst) {
  const int64_t total = out_offs[B];
  for (int64_t r = blockIdx.x; r < total; r += gridDim.x) {
    const int64_t s = out_index[r];
    uint4* d = dst + r * chunks;
    if (s < 0 || s >= T) {   // a slot left unwritten by a bad offset table
      for (int32_t k = threadIdx.x; k < chunks; k += blockDim.x) d[k] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const uint4* p = src + s * chunks;
    for (int32_t k = threadIdx.x; k < chunks; k += blockDim.x) d[k] = p[k];
  }
}

}  // namespace

cudaError_t launch_stochastic_length(const SlArgs& a, int num_sms, cudaStream_t st) {
  static std::atomic<uint64_t> smem_set{0};
  const int smem = kSlMaxLen * int(sizeof(unsigned long long));
  cudaError_t e = smem_opt_in(sl_select_kernel, smem, smem_set);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(a.err, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return e;
  if (a.B > 0) {
    sl_select_kernel<<<a.B, kSlThreads, smem, st>>>(a.offs, a.B, a.T, a.u, a.keys, a.n_c,
                                                    a.numerator, a.flags, a.kept, a.err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  sl_scan_kernel<<<1, kSlThreads, 0, st>>>(a.kept, a.B, a.T, a.out_offs);
  e = cudaGetLastError();
  if (e != cudaSuccess || a.B == 0) return e;
  sl_index_kernel<<<a.B, kSlThreads, 0, st>>>(a.offs, a.B, a.T, a.flags, a.out_offs, a.ts,
                                              a.out_index, a.out_ts);
  e = cudaGetLastError();
  if (e != cudaSuccess || a.values == nullptr || a.T == 0) return e;
  const int32_t chunks = int32_t(a.row_bytes / 16);
  const int threads = chunks < 256 ? ((chunks + 31) / 32) * 32 : 256;
  const int64_t want = a.T < int64_t(num_sms) * 16 ? a.T : int64_t(num_sms) * 16;
  sl_rows_kernel<<<int(want), threads, 0, st>>>(a.out_offs, a.B, a.T, a.out_index, chunks,
                                                static_cast<const uint4*>(a.values),
                                                static_cast<uint4*>(a.out_values));
  return cudaGetLastError();
}

}  // namespace hstu
