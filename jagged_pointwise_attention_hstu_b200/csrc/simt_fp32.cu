// fp32 path of the HSTU layer (compute_dtype = FP32): every product and sum
// in fp32 on the CUDA cores.  Used for fp32 layer configurations, where the
// result must track an fp64 reference to ~1e-4; the tensor-core path serves
// the bf16 configurations.
//
//   gemm_f32_kernel       f1 (SiLU, split order U|V|Q|K) and f2 (+ b2 + X)
//   attention_f32_kernel  equation (2), one warp per (query row, head); keys
//                         visible to the row are walked in order and the bias
//                         buckets are computed per pair from the threshold
//                         table (no reliance on sorted timestamps)
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace hstu {
namespace {

constexpr int kBM = 64, kBN = 64, kBK = 16;

template <int EPI>
__global__ void __launch_bounds__(256)
    gemm_f32_kernel(const float* __restrict__ A, const float* __restrict__ B, int64_t M, int N,
                    int K, const float* __restrict__ bias, float* out,
                    const float* residual) {
  __shared__ float As[kBK][kBM + 4];
  __shared__ float Bs[kBK][kBN + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t m0 = int64_t(blockIdx.y) * kBM;
  const int n0 = blockIdx.x * kBN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kBK) {
    for (int e = threadIdx.x; e < kBM * kBK; e += 256) {
      const int r = e / kBK, c = e % kBK;
      const int64_t gm = m0 + r;
      const int gk = k0 + c;
      As[c][r] = (gm < M && gk < K) ? A[gm * K + gk] : 0.f;
      const int gn = n0 + r;
      Bs[c][r] = (gn < N && gk < K) ? B[int64_t(gn) * K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kBK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = As[kk][ty * 4 + u];
        b[u] = Bs[kk][tx * 4 + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t gm = m0 + ty * 4 + u;
    if (gm >= M) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int gn = n0 + tx * 4 + v;
      if (gn >= N) continue;
      const float x = acc[u][v] + bias[gn];
      if (EPI == int(Epi::kSiluSplit)) {
        out[gm * N + gn] = x / (1.0f + expf(-x));
      } else {
        out[gm * N + gn] = x + residual[gm * N + gn];
      }
    }
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int bucket_of(const int64_t* thr, int nb, int64_t dt) {
  if (dt <= 0) return 0;
  int lo = 0, hi = nb - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (thr[mid] <= dt) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int E>   // head_dim = 32 * E
__global__ void __launch_bounds__(256)
    attention_f32_kernel(const float* __restrict__ uvqk, float* __restrict__ av,
                         const RowInfo* __restrict__ rows, const int64_t* __restrict__ ts,
                         const int64_t* __restrict__ thresholds,
                         const float* __restrict__ rab_pos, const float* __restrict__ rab_time,
                         const int32_t* __restrict__ counters, int n_norm_fixed, int64_t T,
                         int d, int H, int pos_clamp, int nb) {
  __shared__ int64_t s_thr[256];
  for (int k = threadIdx.x; k < nb; k += blockDim.x) s_thr[k] = thresholds[k];
  __syncthreads();
  constexpr int HD = 32 * E;
  const int lane = threadIdx.x & 31;
  const int64_t wid = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (wid >= T * H) return;
  const int64_t i = wid / H;
  const int h = int(wid % H);
  const int64_t ld = 4 * int64_t(d);
  const RowInfo ri = rows[i];
  int64_t lo = ri.lo;
  if (lo < 0 || lo > i) lo = i;
  int64_t hi = ri.hi;
  if (hi > i + 1) hi = i + 1;
  const int64_t pos = ri.pos;
  const int64_t ti = ts[i];
  float q[E], o[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    q[e] = uvqk[i * ld + 2 * d + h * HD + lane + 32 * e];
    o[e] = 0.f;
  }
  const int nn = n_norm_fixed > 0 ? n_norm_fixed : counters[0];
  for (int64_t j = lo;; ++j) {
    if (j >= hi) {
      if (j > i || hi == i + 1) break;   // history rows: done at hi = i + 1
      j = i;                               // candidates: jump to the self key
    }
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) s = fmaf(q[e], uvqk[j * ld + 3 * d + h * HD + lane + 32 * e], s);
    s = warp_sum(s);
    const int64_t dp = pos - j;
    const int pidx = dp < 0 ? 0 : (dp > pos_clamp ? pos_clamp : int(dp));
    s += rab_pos[pidx] + rab_time[bucket_of(s_thr, nb, ti - ts[j])];
    const float p = s / (1.0f + expf(-s));
#pragma unroll
    for (int e = 0; e < E; ++e)
      o[e] = fmaf(p, uvqk[j * ld + d + h * HD + lane + 32 * e], o[e]);
    if (j == i) break;
  }
  const float inv = 1.0f / float(nn > 0 ? nn : 1);
#pragma unroll
  for (int e = 0; e < E; ++e) av[i * d + h * HD + lane + 32 * e] = o[e] * inv;
}

}  // namespace

cudaError_t launch_gemm_f32(const float* a, const float* b, int64_t M, int N, int K, Epi epi,
                            const float* bias, float* out, const float* residual,
                            cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  const dim3 grid(unsigned((N + kBN - 1) / kBN), unsigned((M + kBM - 1) / kBM));
  if (epi == Epi::kSiluSplit)
    gemm_f32_kernel<0><<<grid, 256, 0, st>>>(a, b, M, N, K, bias, out, residual);
  else
    gemm_f32_kernel<1><<<grid, 256, 0, st>>>(a, b, M, N, K, bias, out, residual);
  return cudaGetLastError();
}

cudaError_t launch_attention_f32(const AttnArgs& a, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  const int64_t warps = a.T * a.H;
  const unsigned blocks = unsigned((warps + 7) / 8);
  const float* u = static_cast<const float*>(a.uvqk);
#define HSTU_F32_ATTN(E)                                                                     \
  attention_f32_kernel<E><<<blocks, 256, 0, st>>>(u, a.av, a.rows, a.ts, a.thresholds,      \
                                                  a.rab_pos, a.rab_time, a.counters,         \
                                                  a.n_norm_fixed, a.T, a.d, a.H, a.pos_clamp, \
                                                  a.time_buckets)
  switch (a.hd) {
    case 32: HSTU_F32_ATTN(1); break;
    case 64: HSTU_F32_ATTN(2); break;
    case 96: HSTU_F32_ATTN(3); break;
    case 128: HSTU_F32_ATTN(4); break;
    default: return cudaErrorInvalidValue;
  }
#undef HSTU_F32_ATTN
  return cudaGetLastError();
}

}  // namespace hstu
