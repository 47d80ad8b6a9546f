// Microbenchmark (diagnostics): tcgen05.mma throughput of one CTA per SM on
// operands already in shared memory (no TMA).  For N in {64,128,256}: issue R
// K blocks of 4 MMAs (M = 128, K = 16 each), with a commit to an mbarrier
// after every K block (as the GEMMs do) or only at the end, zero or random
// bf16 operands, on 1 or 148 CTAs; time with the global timer.  Build:
// python -m block_text_diffusion_b200.build --mma-bench.
#include <cstdio>
#include <cuda.h>
#include <cuda_runtime.h>
#include "../csrc/dg_device.cuh"

__global__ void __launch_bounds__(128, 1) k_mma_bench(int N, int R, int commit_each, int random, long long* out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t bar, bar_final;
  __shared__ uint32_t tmem_base;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < (16384 + 32768) / 4; i += blockDim.x) {
    // random: pairs of bf16 values of magnitude ~1 with varying signs and mantissas
    uint32_t h = (uint32_t)i * 2654435761u + 12345u;
    h ^= h >> 13; h *= 0x5bd1e995u; h ^= h >> 15;
    const uint32_t lo = 0x3F00u | (h & 0x807Fu), hi = 0x3F00u | ((h >> 16) & 0x807Fu);
    reinterpret_cast<uint32_t*>(smem)[i] = random ? (lo | (hi << 16)) : 0u;
  }
  if (threadIdx.x == 0) { mbar_init(&bar, 1); mbar_init(&bar_final, 1); fence_mbar_init(); }
  if (warp == 0) tmem_alloc(&tmem_base, 256);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  long long t0 = 0, t1 = 0;
  int ok = 1;
  if (warp == 1 && lane == 0) {
    const uint32_t idesc = idesc_bf16(128, N);
    const uint32_t a_addr = smem_u32(smem), b_addr = a_addr + 16384;
    const uint64_t ad = sdesc_sw128(a_addr), bd = sdesc_sw128(b_addr);
    t0 = (long long)global_ns();
    for (int i = 0; i < R; ++i) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) tc_mma_bf16(tmem, ad + 2 * kk, bd + 2 * kk, idesc, (i | kk) != 0);
      if (commit_each) tc_commit(&bar);
    }
    tc_commit(&bar_final);
    ok = mbar_wait(&bar_final, 0, nullptr, 0) ? 1 : 0;
    t1 = (long long)global_ns();
    if (blockIdx.x == 0) {
      out[0] = t1 - t0;
      out[1] = ok;
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

int main() {
  long long* d;
  cudaMalloc(&d, 64);
  const int smem = 16384 + 32768 + 1024;
  cudaFuncSetAttribute(k_mma_bench, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  for (int grid : {1, 148})
  for (int random = 0; random < 2; ++random)
  for (int commit_each = 0; commit_each < 2; ++commit_each)
    for (int N : {64, 128, 256}) {
      const int R = 200;
      long long h[2] = {0, 0};
      for (int rep = 0; rep < 3; ++rep) {
        k_mma_bench<<<grid, 128, smem>>>(N, R, commit_each, random, d);
        cudaError_t e = cudaDeviceSynchronize();
        if (e != cudaSuccess) { printf("error %s\n", cudaGetErrorString(e)); return 1; }
      }
      cudaMemcpy(h, d, 16, cudaMemcpyDeviceToHost);
      const double us = h[0] / 1000.0;
      const double flop = 2.0 * 128 * N * 64 * R;
      printf("grid %3d random %d N %3d commit_each %d: %.2f us for %d k-blocks = %.3f us/k-block, %.2f TFLOP/s per SM (ok %lld)\n", grid, random, N,
             commit_each, us, R, us / R, flop / (us * 1e-6) / 1e12, h[1]);
    }
  // many CTAs: one per SM
  return 0;
}
