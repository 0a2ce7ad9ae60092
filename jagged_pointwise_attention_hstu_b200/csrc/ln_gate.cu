// G = LayerNorm(O) (.) U  -- the gate that replaces the feed-forward block
// (blog "Generative Recommendation 16: HSTU", section "用门控代替独立 FFN";
// equation (3) of section "HSTU Layer 到底改了什么").
//
// One warp per token row: the row of O (fp32) is read once with coalesced
// vector loads into registers, the mean and the biased variance are two
// register passes closed by warp-shuffle reductions, and U is read from the
// first d columns of the f1 output.  HBM-bound: per token 4d bytes of O,
// d * sizeof(U) bytes of U and d * sizeof(G) bytes of G.
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace hstu {
namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
  const float4 x = *reinterpret_cast<const float4*>(p);
  v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}

__device__ __forceinline__ void load4(const uint16_t* p, float (&v)[4]) {
  const uint2 x = *reinterpret_cast<const uint2*>(p);
  v[0] = __uint_as_float(x.x << 16);
  v[1] = __uint_as_float(x.x & 0xFFFF0000u);
  v[2] = __uint_as_float(x.y << 16);
  v[3] = __uint_as_float(x.y & 0xFFFF0000u);
}

__device__ __forceinline__ void store4(float* p, const float (&v)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void store4(uint16_t* p, const float (&v)[4]) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack2(v[0], v[1]), pack2(v[2], v[3]));
}

// CH = d / 128 chunks of 4 consecutive columns per lane.
template <int CH, typename TU>
__global__ void __launch_bounds__(256)
    ln_gate_kernel(const float* __restrict__ av, const TU* __restrict__ uvqk, TU* __restrict__ g,
                   const float* __restrict__ gamma, const float* __restrict__ beta, int64_t T,
                   float eps) {
  constexpr int D = CH * 128;
  const int lane = threadIdx.x & 31;
  const int64_t row = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= T) return;
  const float* a = av + row * D;
  float x[CH][4];
#pragma unroll
  for (int c = 0; c < CH; ++c) load4(a + c * 128 + lane * 4, x[c]);
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < CH; ++c) s += (x[c][0] + x[c][1]) + (x[c][2] + x[c][3]);
  const float mu = warp_sum(s) * (1.0f / D);
  float v = 0.f;
#pragma unroll
  for (int c = 0; c < CH; ++c)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float dx = x[c][e] - mu;
      v = fmaf(dx, dx, v);
    }
  const float var = warp_sum(v) * (1.0f / D);
  const float rstd = rsqrtf(var + eps);
  const TU* u = uvqk + row * (4 * D);
  TU* out = g + row * D;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int col = c * 128 + lane * 4;
    float uu[4], gg[4], bb[4], o[4];
    load4(u + col, uu);
    load4(gamma + col, gg);
    load4(beta + col, bb);
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] = fmaf((x[c][e] - mu) * rstd, gg[e], bb[e]) * uu[e];
    store4(out + col, o);
  }
}

// d = 64: one 2-column chunk per lane.
template <typename TU>
__global__ void __launch_bounds__(256)
    ln_gate_d64_kernel(const float* __restrict__ av, const TU* __restrict__ uvqk,
                       TU* __restrict__ g, const float* __restrict__ gamma,
                       const float* __restrict__ beta, int64_t T, float eps) {
  const int lane = threadIdx.x & 31;
  const int64_t row = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= T) return;
  const int col = lane * 2;
  const float x0 = av[row * 64 + col], x1 = av[row * 64 + col + 1];
  const float mu = warp_sum(x0 + x1) * (1.0f / 64);
  const float var = warp_sum((x0 - mu) * (x0 - mu) + (x1 - mu) * (x1 - mu)) * (1.0f / 64);
  const float rstd = rsqrtf(var + eps);
  const TU* u = uvqk + row * 256;
  float u0, u1;
  if constexpr (sizeof(TU) == 4) {
    u0 = float(u[col]);
    u1 = float(u[col + 1]);
  } else {
    u0 = __uint_as_float(uint32_t(u[col]) << 16);
    u1 = __uint_as_float(uint32_t(u[col + 1]) << 16);
  }
  const float o0 = fmaf((x0 - mu) * rstd, gamma[col], beta[col]) * u0;
  const float o1 = fmaf((x1 - mu) * rstd, gamma[col + 1], beta[col + 1]) * u1;
  if constexpr (sizeof(TU) == 4) {
    g[row * 64 + col] = TU(o0);
    g[row * 64 + col + 1] = TU(o1);
  } else {
    *reinterpret_cast<uint32_t*>(&g[row * 64 + col]) = pack2(o0, o1);
  }
}

template <typename TU>
cudaError_t launch_typed(const float* av, const void* uvqk, void* g, const float* gamma,
                         const float* beta, int64_t T, int d, float eps, cudaStream_t st) {
  const unsigned blocks = unsigned((T + 7) / 8);
  const TU* u = static_cast<const TU*>(uvqk);
  TU* gg = static_cast<TU*>(g);
  switch (d) {
    case 64: ln_gate_d64_kernel<TU><<<blocks, 256, 0, st>>>(av, u, gg, gamma, beta, T, eps); break;
    case 128: ln_gate_kernel<1, TU><<<blocks, 256, 0, st>>>(av, u, gg, gamma, beta, T, eps); break;
    case 256: ln_gate_kernel<2, TU><<<blocks, 256, 0, st>>>(av, u, gg, gamma, beta, T, eps); break;
    case 384: ln_gate_kernel<3, TU><<<blocks, 256, 0, st>>>(av, u, gg, gamma, beta, T, eps); break;
    case 512: ln_gate_kernel<4, TU><<<blocks, 256, 0, st>>>(av, u, gg, gamma, beta, T, eps); break;
    case 768: ln_gate_kernel<6, TU><<<blocks, 256, 0, st>>>(av, u, gg, gamma, beta, T, eps); break;
    case 1024: ln_gate_kernel<8, TU><<<blocks, 256, 0, st>>>(av, u, gg, gamma, beta, T, eps); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ln_gate(const float* av, const void* uvqk, void* g, const float* gamma,
                           const float* beta, int64_t T, int d, float eps, int compute_fp32,
                           cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  if (compute_fp32) return launch_typed<float>(av, uvqk, g, gamma, beta, T, d, eps, st);
  return launch_typed<uint16_t>(av, uvqk, g, gamma, beta, T, d, eps, st);
}

}  // namespace hstu
