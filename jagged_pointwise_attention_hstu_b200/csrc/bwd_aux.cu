// Memory-bound steps of the HSTU layer backward (the gradients of equations
// (1) and (3) of blog "Generative Recommendation 16: HSTU", section "HSTU Layer
// 到底改了什么"; the attention step is attn_bwd_tc.cu, the products run on the
// tensor-core GEMM of gemm_tc.cu):
//   ln_gate_bwd   from dG = dY W2: dU = dG (.) N, dO through the LayerNorm
//                 (N and its statistics recomputed from O), G = N (.) U for the
//                 W2 gradient, and the gamma / beta gradients;
//   silu_bwd      dH1 = [dU | dV | dQ | dK] (.) SiLU'(H1) and the b1 gradient;
//   colsum        the b2 gradient (column sums of dY);
//   transpose     [R, C] -> [C, ldd] bf16 with zero padding, so that every
//                 weight gradient is a plain K-major GEMM over the tokens.
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

__device__ __forceinline__ float bf16_to_f(uint16_t x) { return __uint_as_float(uint32_t(x) << 16); }

__device__ __forceinline__ uint16_t f_to_bf16(float f) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(0.0f), "f"(f));
  return uint16_t(r & 0xFFFFu);
}

__device__ __forceinline__ float load_f(const float* p) { return *p; }
__device__ __forceinline__ float load_f(const uint16_t* p) { return bf16_to_f(*p); }

// One warp per token row at a time (grid-stride); lane owns CH chunks of 4
// consecutive columns, the same columns for every row, so the gamma / beta
// gradients stay in registers until one shared and one global add per column.
template <int CH>
__global__ void __launch_bounds__(256)
    ln_gate_bwd_kernel(const float* __restrict__ dG, const uint16_t* __restrict__ uvqk,
                       const float* __restrict__ av, const float* __restrict__ gamma,
                       const float* __restrict__ beta, int64_t T, float eps,
                       float* __restrict__ dU, uint16_t* __restrict__ dO,
                       uint16_t* __restrict__ G, float* __restrict__ dgamma,
                       float* __restrict__ dbeta) {
  constexpr int D = CH * 128;
  __shared__ float s_g[D];
  __shared__ float s_b[D];
  for (int c = threadIdx.x; c < D; c += blockDim.x) s_g[c] = s_b[c] = 0.0f;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  float pg[CH][4], pb[CH][4];
#pragma unroll
  for (int k = 0; k < CH; ++k)
#pragma unroll
    for (int e = 0; e < 4; ++e) pg[k][e] = pb[k][e] = 0.0f;
  for (int64_t row = int64_t(blockIdx.x) * 8 + warp; row < T; row += int64_t(gridDim.x) * 8) {
    float o[CH][4], u[CH][4], g[CH][4];
    float s = 0.0f;
#pragma unroll
    for (int k = 0; k < CH; ++k)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = k * 128 + lane * 4 + e;
        o[k][e] = av[row * D + c];
        u[k][e] = bf16_to_f(uvqk[row * 4 * D + c]);
        g[k][e] = dG[row * D + c];
        s += o[k][e];
      }
    const float mu = warp_sum(s) * (1.0f / D);
    float v = 0.0f;
#pragma unroll
    for (int k = 0; k < CH; ++k)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float t = o[k][e] - mu;
        v += t * t;
      }
    const float rstd = rsqrtf(warp_sum(v) * (1.0f / D) + eps);
    float m1 = 0.0f, m2 = 0.0f;
#pragma unroll
    for (int k = 0; k < CH; ++k)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = k * 128 + lane * 4 + e;
        const float gmc = __ldg(gamma + c);
        const float oh = (o[k][e] - mu) * rstd;
        const float n = oh * gmc + __ldg(beta + c);
        const float dn = g[k][e] * u[k][e];
        dU[row * D + c] = g[k][e] * n;
        G[row * D + c] = f_to_bf16(n * u[k][e]);
        pg[k][e] += dn * oh;
        pb[k][e] += dn;
        const float doh = dn * gmc;
        m1 += doh;
        m2 += doh * oh;
        o[k][e] = oh;        // keep Ohat
        g[k][e] = doh;       // keep dOhat
      }
    m1 = warp_sum(m1) * (1.0f / D);
    m2 = warp_sum(m2) * (1.0f / D);
#pragma unroll
    for (int k = 0; k < CH; ++k)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = k * 128 + lane * 4 + e;
        dO[row * D + c] = f_to_bf16(rstd * (g[k][e] - m1 - o[k][e] * m2));
      }
  }
#pragma unroll
  for (int k = 0; k < CH; ++k)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = k * 128 + lane * 4 + e;
      atomicAdd(s_g + c, pg[k][e]);
      atomicAdd(s_b + c, pb[k][e]);
    }
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    if (s_g[c] != 0.0f) atomicAdd(dgamma + c, s_g[c]);
    if (s_b[c] != 0.0f) atomicAdd(dbeta + c, s_b[c]);
  }
}

// Thread = one column of [T, 4d]; blocks split the rows.  dZ's column c comes
// from dU, dV, dQ or dK ([T, d] each) by c / d.
__global__ void __launch_bounds__(256)
    silu_bwd_kernel(const float* __restrict__ dUp, const float* __restrict__ dVp,
                    const float* __restrict__ dQp, const float* __restrict__ dKp,
                    const float* __restrict__ H1, int64_t T, int d, int64_t rows_per_block,
                    uint16_t* __restrict__ dH1, float* __restrict__ db1) {
  const int c = blockIdx.y * blockDim.x + threadIdx.x;
  if (c >= 4 * d) return;
  const int seg = c / d;
  const int lc = c - seg * d;
  const float* src = seg == 0 ? dUp : (seg == 1 ? dVp : (seg == 2 ? dQp : dKp));
  const int64_t r0 = int64_t(blockIdx.x) * rows_per_block;
  const int64_t r1 = r0 + rows_per_block < T ? r0 + rows_per_block : T;
  float acc = 0.0f;
  for (int64_t r = r0; r < r1; ++r) {
    const float h = H1[r * 4 * d + c];
    const float sg = 1.0f / (1.0f + __expf(-h));
    const float g = src[r * d + lc] * (sg * (1.0f + h * (1.0f - sg)));
    dH1[r * 4 * d + c] = f_to_bf16(g);
    acc += g;
  }
  if (acc != 0.0f) atomicAdd(db1 + c, acc);
}

template <typename TS>
__global__ void __launch_bounds__(256)
    colsum_kernel(const TS* __restrict__ src, int64_t T, int n, int64_t rows_per_block,
                  float* __restrict__ out) {
  const int c = blockIdx.y * blockDim.x + threadIdx.x;
  if (c >= n) return;
  const int64_t r0 = int64_t(blockIdx.x) * rows_per_block;
  const int64_t r1 = r0 + rows_per_block < T ? r0 + rows_per_block : T;
  float acc = 0.0f;
  for (int64_t r = r0; r < r1; ++r) acc += load_f(src + r * n + c);
  if (acc != 0.0f) atomicAdd(out + c, acc);
}

// dst[c * ldd + r] = bf16(src[r * lds + c]) for r < R, c < C; rows R..ldd-1 of
// every dst row are written as zeros.  32 x 32 tiles through shared memory.
template <typename TS>
__global__ void transpose_bf16_kernel(const TS* __restrict__ src, int64_t R, int C, int64_t lds,
                                      uint16_t* __restrict__ dst, int64_t ldd) {
  __shared__ float tile[32][33];
  const int64_t r0 = int64_t(blockIdx.x) * 32;
  const int c0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;   // 32 x 8
#pragma unroll
  for (int y = 0; y < 32; y += 8) {
    const int64_t r = r0 + ty + y;
    const int c = c0 + tx;
    tile[ty + y][tx] = (r < R && c < C) ? load_f(src + r * lds + c) : 0.0f;
  }
  __syncthreads();
#pragma unroll
  for (int y = 0; y < 32; y += 8) {
    const int c = c0 + ty + y;
    const int64_t r = r0 + tx;
    if (c < C && r < ldd) dst[int64_t(c) * ldd + r] = f_to_bf16(tile[tx][ty + y]);
  }
}

int blocks_for_rows(int64_t T, int num_sms, int64_t& rows_per_block) {
  const int64_t want = int64_t(num_sms) * 4;
  const int64_t nb = T < want ? T : want;
  rows_per_block = (T + nb - 1) / nb;
  return int((T + rows_per_block - 1) / rows_per_block);
}

}  // namespace

cudaError_t launch_ln_gate_bwd(const float* dG, const void* uvqk, const float* av,
                               const float* gamma, const float* beta, int64_t T, int d, float eps,
                               float* dU, void* dO, void* G, float* dgamma, float* dbeta,
                               int num_sms, cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  const int64_t want = int64_t(num_sms) * 4;
  const int64_t need = (T + 7) / 8;
  const unsigned grid = unsigned(need < want ? need : want);
  const uint16_t* u = static_cast<const uint16_t*>(uvqk);
  uint16_t* o = static_cast<uint16_t*>(dO);
  uint16_t* g = static_cast<uint16_t*>(G);
  switch (d / 128) {
    case 1: ln_gate_bwd_kernel<1><<<grid, 256, 0, st>>>(dG, u, av, gamma, beta, T, eps, dU, o, g, dgamma, dbeta); break;
    case 2: ln_gate_bwd_kernel<2><<<grid, 256, 0, st>>>(dG, u, av, gamma, beta, T, eps, dU, o, g, dgamma, dbeta); break;
    case 3: ln_gate_bwd_kernel<3><<<grid, 256, 0, st>>>(dG, u, av, gamma, beta, T, eps, dU, o, g, dgamma, dbeta); break;
    case 4: ln_gate_bwd_kernel<4><<<grid, 256, 0, st>>>(dG, u, av, gamma, beta, T, eps, dU, o, g, dgamma, dbeta); break;
    case 6: ln_gate_bwd_kernel<6><<<grid, 256, 0, st>>>(dG, u, av, gamma, beta, T, eps, dU, o, g, dgamma, dbeta); break;
    case 8: ln_gate_bwd_kernel<8><<<grid, 256, 0, st>>>(dG, u, av, gamma, beta, T, eps, dU, o, g, dgamma, dbeta); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_silu_bwd(const float* dU, const float* dV, const float* dQ, const float* dK,
                            const float* H1, int64_t T, int d, void* dH1, float* db1, int num_sms,
                            cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  int64_t rpb = 1;
  const int gx = blocks_for_rows(T, num_sms, rpb);
  const dim3 grid(unsigned(gx), unsigned((4 * d + 255) / 256));
  silu_bwd_kernel<<<grid, 256, 0, st>>>(dU, dV, dQ, dK, H1, T, d, rpb,
                                        static_cast<uint16_t*>(dH1), db1);
  return cudaGetLastError();
}

cudaError_t launch_colsum(const void* src, bool fp32, int64_t T, int n, float* out, int num_sms,
                          cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  int64_t rpb = 1;
  const int gx = blocks_for_rows(T, num_sms, rpb);
  const dim3 grid(unsigned(gx), unsigned((n + 255) / 256));
  if (fp32)
    colsum_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(src), T, n, rpb, out);
  else
    colsum_kernel<uint16_t><<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(src), T, n, rpb, out);
  return cudaGetLastError();
}

cudaError_t launch_transpose_bf16(const void* src, bool fp32, int64_t R, int C, int64_t lds,
                                  void* dst, int64_t ldd, cudaStream_t st) {
  if (ldd <= 0 || C <= 0) return cudaSuccess;
  const dim3 grid(unsigned((ldd + 31) / 32), unsigned((C + 31) / 32));
  const dim3 block(32, 8);
  if (fp32)
    transpose_bf16_kernel<float><<<grid, block, 0, st>>>(static_cast<const float*>(src), R, C, lds,
                                                         static_cast<uint16_t*>(dst), ldd);
  else
    transpose_bf16_kernel<uint16_t><<<grid, block, 0, st>>>(
        static_cast<const uint16_t*>(src), R, C, lds, static_cast<uint16_t*>(dst), ldd);
  return cudaGetLastError();
}

}  // namespace hstu
