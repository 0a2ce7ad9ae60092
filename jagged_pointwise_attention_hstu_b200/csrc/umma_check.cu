// One-tile tensor-core product used by the tests to check, in isolation, the
// three operand layouts the GEMM and attention kernels rely on:
//   mode 0  A [128, k] and B [n, k], both K-major in shared memory (f1, f2, Q K^T)
//   mode 1  A K-major in shared memory, B given [k, n] (N-major; the V tile of P V)
//   mode 2  A staged in tensor memory (bf16 pairs per 32-bit column), B N-major
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "sm100.cuh"

namespace hstu {
namespace {

using namespace sm100;

constexpr uint32_t kSmem = 128 * 128 * 2 + 256 * 128 * 2 + 1024 + 256;

__global__ void __launch_bounds__(128, 1)
    umma_tile_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
                     int mode, int n, int k, const uint16_t* __restrict__ a_glob,
                     float* __restrict__ c, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + 128 * 128 * 2;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sB + 256 * 128 * 2);
  uint64_t* done = bar + 1;
  uint32_t* slot = reinterpret_cast<uint32_t*>(done + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    mbar_init(done, 1);
    fence_mbarrier_init();
  }
  if (warp == 0) {
    tmem_alloc(slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const uint32_t tD = tmem, tA = tmem + 256;
  bool ok = true;
  if (threadIdx.x == 0) {
    const uint32_t a_bytes = 128 * k * 2, b_bytes = n * k * 2;
    mbar_arrive_expect_tx(bar, (mode == 2 ? 0u : a_bytes) + b_bytes);
    if (mode != 2)
      for (int b = 0; b < k / 64; ++b) tma_load_2d(sA + b * 16384, &ta, bar, b * 64, 0);
    if (mode == 0) {
      for (int b = 0; b < k / 64; ++b) tma_load_2d(sB + b * (n * 128), &tb, bar, b * 64, 0);
    } else {
      for (int b = 0; b < n / 64; ++b) tma_load_2d(sB + b * (k * 128), &tb, bar, b * 64, 0);
    }
    ok = mbar_wait(bar, 0);
  }
  if (mode == 2) {
    // thread row r = 32 * warp + lane stages A[r, :] into tensor-memory lane r
    const int r = warp * 32 + lane;
    for (int cch = 0; cch < k / 32; ++cch) {
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const uint32_t lo = a_glob[r * k + cch * 32 + 2 * e];
        const uint32_t hi = a_glob[r * k + cch * 32 + 2 * e + 1];
        pk[e] = lo | (hi << 16);
      }
      tmem_st16(tA + (uint32_t(warp * 32) << 16) + cch * 16, pk);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && ok) {
    tc_fence_after();
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    for (int kk = 0; kk < k / 16; ++kk) {
      if (mode == 0) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        const uint32_t boff = (kk >> 2) * (n * 128) + (kk & 3) * 32;
        umma_ss(tD, desc_sw128(a0 + off, 16, 1024), desc_sw128(b0 + boff, 16, 1024),
                idesc_bf16(128, n, false, false), kk > 0);
      } else if (mode == 1) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        umma_ss(tD, desc_sw128(a0 + off, 16, 1024), desc_sw128(b0 + kk * 2048, k * 128, 1024),
                idesc_bf16(128, n, false, true), kk > 0);
      } else {
        umma_ts(tD, tA + kk * 8, desc_sw128(b0 + kk * 2048, k * 128, 1024),
                idesc_bf16(128, n, false, true), kk > 0);
      }
    }
    umma_commit(done);
    ok = mbar_wait(done, 0);
    if (!ok) *status = 1;
  }
  if (threadIdx.x == 0 && !ok) *status = 1;
  __syncthreads();
  tc_fence_after();
  const int r = warp * 32 + lane;
  for (int cc = 0; cc < n; cc += 32) {
    uint32_t v[32];
    tmem_ld32(tD + (uint32_t(warp * 32) << 16) + cc, v);
    tmem_ld_wait();
    for (int e = 0; e < 32; ++e) c[r * n + cc + e] = __uint_as_float(v[e]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t run_umma_tile(int mode, const void* a, const void* b, float* c, int n, int k) {
  CUtensorMap ta, tb;
  if (!make_tmap_2d_bf16(&ta, a, uint64_t(k), 128, uint64_t(k) * 2, 64, 128))
    return cudaErrorInvalidValue;
  if (mode == 0) {
    if (!make_tmap_2d_bf16(&tb, b, uint64_t(k), uint64_t(n), uint64_t(k) * 2, 64, uint32_t(n)))
      return cudaErrorInvalidValue;
  } else {
    if (!make_tmap_2d_bf16(&tb, b, uint64_t(n), uint64_t(k), uint64_t(n) * 2, 64, uint32_t(k)))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(umma_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(kSmem));
  if (e != cudaSuccess) return e;
  int* status = nullptr;
  e = cudaMalloc(&status, sizeof(int));
  if (e != cudaSuccess) return e;
  cudaMemset(status, 0, sizeof(int));
  umma_tile_kernel<<<1, 128, kSmem>>>(ta, tb, mode, n, k, static_cast<const uint16_t*>(a), c,
                                      status);
  e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  int hs = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&hs, status, sizeof(int), cudaMemcpyDeviceToHost);
  cudaFree(status);
  if (e == cudaSuccess && hs != 0) e = cudaErrorLaunchTimeout;
  return e;
}

}  // namespace hstu
