// Split-K GEMM whose scratch lives in a fixed-size file-scope device array,
// for callers that must not allocate device memory (see include/dg.h,
// dg_gemm_splitk_noalloc).  This file has its own tensor-map helper and its
// own copy of the GEMM kernel instantiation; it shares nothing at run time
// with the other entry points except the kernel code in dg_gemm.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/dg.h"
#include "dg_gemm.cuh"

namespace {

// Partial-sum slabs of every call: k_splits x N x M floats (64 MiB).  Every
// GPU that loads the library holds this array until the process exits.
constexpr long long kNoAllocScratchFloats = 16ll << 20;
__device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];
__device__ __align__(256) int g_noalloc_err[8];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_ptr[kMaxDevices] = {};
int* g_err_ptr[kMaxDevices] = {};

typedef CUresult (*PFN_encode)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                               const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                               CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                               CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point, looked up
// once (a function-local static is initialised once even when several host
// threads make their first call at the same time).
PFN_encode lookup_encode() {
  cudaDriverEntryPointQueryResult q;
  void* p = nullptr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return (PFN_encode)p;
}

bool tensor_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  static const PFN_encode fn = lookup_encode();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// out[i] = sum over the split slabs of the scratch, in split order.
__global__ void k_noalloc_reduce(const float* __restrict__ scratch, float* __restrict__ out, long long n,
                                 int splits) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    float v = scratch[i];
    for (int s = 1; s < splits; ++s) v += scratch[s * n + i];
    out[i] = v;
  }
}

// Device addresses of the two arrays on the current device, looked up once
// per device (host code cannot use the array names as device addresses).
dg_status device_arrays(float** scratch, int** err) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DG_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* s = nullptr;
    void* e = nullptr;
    if (cudaGetSymbolAddress(&s, g_noalloc_scratch) != cudaSuccess) return DG_ERR_CUDA;
    if (cudaGetSymbolAddress(&e, g_noalloc_err) != cudaSuccess) return DG_ERR_CUDA;
    g_scratch_ptr[dev] = (float*)s;
    g_err_ptr[dev] = (int*)e;
  }
  *scratch = g_scratch_ptr[dev];
  *err = g_err_ptr[dev];
  return DG_OK;
}

constexpr int kBN = 256, kStages = 4;

}  // namespace

extern "C" dg_status dg_gemm_splitk_noalloc(const void* A, const void* B, float* out, int32_t M, int32_t N,
                                            int32_t K, int32_t k_splits, void* stream) {
  if (!A || !B || !out || M < 1 || N < 1 || K < 1 || K % 8 || k_splits < 1) return DG_ERR_INVALID_ARG;
  const int kb_total = (K + 63) / 64;
  const int splits = k_splits < kb_total ? k_splits : kb_total;
  if ((long long)splits * N * M > kNoAllocScratchFloats) return DG_ERR_INVALID_ARG;   // beyond the fixed scratch
  float* scratch = nullptr;
  int* err = nullptr;
  dg_status st = device_arrays(&scratch, &err);
  if (st != DG_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  CUtensorMap ta;
  BMaps tb;
  bool maps_ok = tensor_map(&ta, A, (uint64_t)M, (uint64_t)K, 128);
  for (int i = 0; i < 4; ++i) maps_ok = maps_ok && tensor_map(&tb.m[i], B, (uint64_t)N, (uint64_t)K, 32u << i);
  if (!maps_ok) return DG_ERR_CUDA;
  using C = GemmTcCfg<kBN, kStages>;
  if (cudaFuncSetAttribute(k_gemm_tc<kBN, kStages>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem) !=
      cudaSuccess)
    return DG_ERR_CUDA;
  // the error word starts at zero on every call; the partial slabs are
  // overwritten in full by the GEMM, so they need no clearing
  if (cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess) return DG_ERR_CUDA;
  GemmArgs a{};
  a.M = M;
  a.m_tiles = (M + 127) / 128;
  a.kb_total = kb_total;
  a.k_splits = splits;
  a.N = N;
  a.n_tile = kBN;
  a.alpha = 1.0f;
  a.out = scratch;
  a.ldo = M;
  a.split_stride = (long long)N * M;
  a.err = err;
  const long long grid = (long long)a.m_tiles * splits * ((N + kBN - 1) / kBN);
  k_gemm_tc<kBN, kStages><<<(unsigned)grid, 128, C::kSmem, s>>>(ta, tb, a);
  if (cudaGetLastError() != cudaSuccess) return DG_ERR_CUDA;
  const long long n = (long long)N * M;
  const int blocks = (int)((n + 255) / 256 < 148 * 16 ? (n + 255) / 256 : 148 * 16);
  k_noalloc_reduce<<<blocks, 256, 0, s>>>(scratch, out, n, splits);
  if (cudaGetLastError() != cudaSuccess) return DG_ERR_CUDA;
  int e = 0;
  if (cudaMemcpyAsync(&e, err, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return DG_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DG_ERR_CUDA;
  return e ? DG_ERR_TIMEOUT : DG_OK;
}
