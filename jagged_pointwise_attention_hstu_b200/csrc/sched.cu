// Jagged scheduler: per-token row facts, input validation and the work order
// of the attention kernels (pairs of adjacent query tiles).
//
// The batch is jagged (per-user sequences packed without padding; blog
// "Generative Recommendation 16: HSTU", item 1 "Ragged/Jagged kernel").  Query
// tiles are 128 consecutive rows of the packed token axis, so short users
// share a tile.  For the tile starting at row r0 every visible key lies in
//   [lo(r0), min(r0, hi(r0)))  (keys of the tile's first user before the tile)
//   [r0, r0 + 128)             (the diagonal tile)
// because later users in the tile start inside it and a candidate of the first
// user sees only that user's history and itself (ltzyclt blog, section 5.2,
// M-FALCON).  Every other key tile is fully masked and never visited.  A work
// item is a pair of adjacent query tiles (2p, 2p+1), which visits the union of
// both tiles' key ranges; the pairs are ordered by descending cost (key tiles
// visited), a longest-processing-time-first order that keeps the power-law
// lengths balanced.
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace hstu {
namespace {

__global__ void rows_kernel(const int32_t* __restrict__ offs, int32_t B, int64_t T,
                            const int32_t* __restrict__ ncand, int mfalcon,
                            const int64_t* __restrict__ ts, RowInfo* __restrict__ rows,
                            int32_t* __restrict__ counters, int32_t* __restrict__ err) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  // user-level checks, one thread per user
  if (i <= B) {
    const int32_t o = offs[i];
    int bits = 0;
    if (i == 0 && o != 0) bits |= HSTU_DEVERR_OFFSETS;
    if (i == B && int64_t(o) != T) bits |= HSTU_DEVERR_OFFSETS;
    if (i < B) {
      const int32_t o1 = offs[i + 1];
      const int32_t len = o1 - o;
      if (len < 0) bits |= HSTU_DEVERR_OFFSETS;
      if (mfalcon) {
        const int32_t c = ncand[i];
        if (c < 0 || c > len) bits |= HSTU_DEVERR_CANDIDATES;
      }
      if (len > 0) atomicMax(&counters[0], len);
    }
    if (bits) atomicOr(err, bits);
  }
  if (i >= T) return;
  // largest b with offs[b] <= i  (b in [0, B-1])
  int32_t lo_b = 0, hi_b = B - 1;
  while (lo_b < hi_b) {
    const int32_t mid = (lo_b + hi_b + 1) >> 1;
    if (int64_t(offs[mid]) <= i) lo_b = mid; else hi_b = mid - 1;
  }
  const int32_t b = lo_b;
  int32_t lo = offs[b];
  int32_t end = offs[b + 1];
  // invalid offsets: clamp so that downstream kernels stay in bounds
  if (lo < 0 || int64_t(lo) > i) lo = int32_t(i);
  if (int64_t(end) <= i || int64_t(end) > T) end = int32_t(i) + 1;
  int32_t nc = mfalcon ? ncand[b] : 0;
  if (nc < 0) nc = 0;
  if (nc > end - lo) nc = end - lo;
  const int32_t he = end - nc;
  RowInfo r;
  r.lo = lo;
  r.user = b;
  if (i < he) {
    r.hi = int32_t(i) + 1;
    r.pos = int32_t(i);
  } else {
    r.hi = he;
    r.pos = he;
  }
  rows[i] = r;
  const int64_t t = ts[i];
  bool bad = (t < 0) || (t >= kMaxTimestamp);
  if (i > lo && ts[i - 1] > t) bad = true;
  if (bad) atomicOr(err, HSTU_DEVERR_TIMESTAMPS);
}

// One block: cost of every pair of query tiles (key tiles it visits), then a
// counting sort by descending cost (longest processing time first).
__global__ void order_kernel(const RowInfo* __restrict__ rows, int64_t T, int32_t npairs,
                             int32_t* __restrict__ cost, int32_t* __restrict__ order,
                             int32_t* __restrict__ counters) {
  constexpr int NB = 4096;   // cost bins; costs above NB-1 share the top bin
  __shared__ int32_t hist[NB];
  __shared__ int32_t s_max;
  for (int c = threadIdx.x; c < NB; c += blockDim.x) hist[c] = 0;
  if (threadIdx.x == 0) s_max = 0;
  __syncthreads();
  int32_t local_max = 0;
  for (int32_t pr = threadIdx.x; pr < npairs; pr += blockDim.x) {
    const PairTiles t = pair_tiles(rows, T, pr);
    const int32_t c = t.n_a + t.n_diag;
    cost[pr] = c;
    local_max = c > local_max ? c : local_max;
    atomicAdd(&hist[c < NB ? c : NB - 1], 1);
  }
  atomicMax(&s_max, local_max);
  __syncthreads();
  const int top = s_max < NB ? s_max : NB - 1;
  if (threadIdx.x == 0) {
    int32_t run = 0;   // exclusive prefix over descending cost
    for (int c = top; c >= 0; --c) {
      const int32_t n = hist[c];
      hist[c] = run;
      run += n;
    }
    counters[1] = s_max;
  }
  __syncthreads();
  for (int32_t pr = threadIdx.x; pr < npairs; pr += blockDim.x) {
    const int32_t c = cost[pr];
    const int32_t slot = atomicAdd(&hist[c < NB ? c : NB - 1], 1);
    order[slot] = pr;
  }
}

__global__ void cast_bf16_kernel(const float4* __restrict__ x, uint2* __restrict__ y, int64_t n4) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += int64_t(gridDim.x) * blockDim.x) {
    const float4 v = x[i];
    uint2 o;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o.x) : "f"(v.y), "f"(v.x));
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o.y) : "f"(v.w), "f"(v.z));
    y[i] = o;
  }
}

}  // namespace

cudaError_t launch_schedule(const hstu_handle_s* h, int64_t T, const int32_t* offsets, int32_t B,
                            const int64_t* ts, int mask_mode, const int32_t* ncand,
                            cudaStream_t st) {
  const Workspace& ws = h->ws;
  cudaError_t e = cudaMemsetAsync(ws.counters, 0, 4 * sizeof(int32_t), st);
  if (e != cudaSuccess) return e;
  const int64_t n = (T > int64_t(B) + 1) ? T : int64_t(B) + 1;
  const int threads = 256;
  const unsigned blocks = unsigned((n + threads - 1) / threads);
  rows_kernel<<<blocks, threads, 0, st>>>(offsets, B, T, ncand, mask_mode == HSTU_MASK_MFALCON,
                                          ts, ws.rows, ws.counters, ws.error);
  e = cudaGetLastError();
  if (e != cudaSuccess || T == 0) return e;
  const int32_t npairs = int32_t((T + 2 * kTile - 1) / (2 * kTile));
  order_kernel<<<1, 1024, 0, st>>>(ws.rows, T, npairs, ws.qtile_cost, ws.qtile_order, ws.counters);
  return cudaGetLastError();
}

cudaError_t launch_schedule_raw(int64_t T, const int32_t* offsets, int32_t B, const int64_t* ts,
                                int mask_mode, const int32_t* ncand, RowInfo* rows, int32_t* cost,
                                int32_t* order, int32_t* counters, int32_t* err, cudaStream_t st) {
  const int64_t n = (T > int64_t(B) + 1) ? T : int64_t(B) + 1;
  const int threads = 256;
  const unsigned blocks = unsigned((n + threads - 1) / threads);
  rows_kernel<<<blocks, threads, 0, st>>>(offsets, B, T, ncand, mask_mode == HSTU_MASK_MFALCON,
                                          ts, rows, counters, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || T == 0) return e;
  const int32_t npairs = int32_t((T + 2 * kTile - 1) / (2 * kTile));
  order_kernel<<<1, 1024, 0, st>>>(rows, T, npairs, cost, order, counters);
  return cudaGetLastError();
}

cudaError_t launch_cast_bf16(const float* x, void* xb, int64_t n, cudaStream_t st) {
  // n is a multiple of 4 (d is a multiple of 16)
  const int64_t n4 = n / 4;
  if (n4 == 0) return cudaSuccess;
  int64_t blocks = (n4 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  cast_bf16_kernel<<<unsigned(blocks), 256, 0, st>>>(reinterpret_cast<const float4*>(x),
                                                     reinterpret_cast<uint2*>(xb), n4);
  return cudaGetLastError();
}

}  // namespace hstu
