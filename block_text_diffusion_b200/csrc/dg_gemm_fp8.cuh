// FP8 expert weights: quantisation and the grouped GEMM that streams them.
//
// Format (a reading of the FP8 deployment the DiffusionGemma release news,
// section "速度数据", reports): expert weights are OCP E4M3 codes (4 exponent
// bits, bias 7, 3 mantissa bits, largest finite 448) with one power-of-two
// scale per 128 consecutive inputs of each output row,
//   s = 2^ceil(log2(amax / 448)),  q = round-to-nearest-even(w / s),
// so q s is exactly a bfloat16 value and a GEMM over the dequantised weights
// is the bf16 GEMM of the model with those weights.  Activations stay bf16.
//
// The GEMM halves the weight bytes the expert GEMMs stream: TMA brings
// 128-row x 128-input E4M3 tiles (16 KB) into a raw buffer, eight converter
// warps expand them into the 128-byte-swizzled bf16 layout tcgen05.mma reads
// (two 64-input K blocks), applying the row's scale, and the MMA warp runs the
// same instructions as the bf16 kernel.  So on identical dequantised weights
// the result equals the bf16 GEMM's bit for bit.
#pragma once
#include <cuda_fp8.h>
#include "dg_gemm.cuh"

constexpr int kF8Chunk = 128;                 // inputs per scale block and per ring slot
constexpr int kF8ConvWarps = 8;
constexpr int kF8Threads = 192 + 32 * kF8ConvWarps;
constexpr int kF8WorkSmem = 256;

// Scale exponent of a block from its largest magnitude (a normal binary32
// value or 0): the least e with amax <= 448 * 2^e.  With amax = f 2^ea,
// f in [1, 2): e = ea - 8, plus 1 when f > 1.75 (448 = 1.75 * 2^8).
__device__ __forceinline__ int f8_scale_exp(float amax) {
  const uint32_t b = __float_as_uint(amax);
  if ((b & 0x7FFFFFFFu) == 0u) return 0;
  const int ea = (int)((b >> 23) & 0xFF) - 127;
  return ea - 8 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
}

// One warp per (row, 128-input block) of w [rows][K] (bf16): codes [rows][K]
// (E4M3 bytes) and scales [rows][ceil(K / 128)] (fp32 powers of two).
__global__ void k_quant_f8(const bf16* __restrict__ w, long long rows, int K, uint8_t* __restrict__ codes,
                           float* __restrict__ scales) {
  const int n_chunks = (K + kF8Chunk - 1) / kF8Chunk;
  const long long unit = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (unit >= rows * n_chunks) return;
  const int lane = threadIdx.x & 31;
  const long long r = unit / n_chunks;
  const int c = (int)(unit % n_chunks);
  const int k0 = c * kF8Chunk + lane * 4;            // this lane's 4 inputs
  float v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) v[j] = (k0 + j < K) ? __bfloat162float(w[r * K + k0 + j]) : 0.0f;
  float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const int e = f8_scale_exp(amax);
  const float inv_s = __int_as_float((127 - e) << 23);   // 2^-e, exact
  const __nv_fp8x2_storage_t lo =
      __nv_cvt_float2_to_fp8x2(make_float2(v[0] * inv_s, v[1] * inv_s), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi =
      __nv_cvt_float2_to_fp8x2(make_float2(v[2] * inv_s, v[3] * inv_s), __NV_SATFINITE, __NV_E4M3);
  const uint8_t q[4] = {(uint8_t)(lo & 0xFF), (uint8_t)(lo >> 8), (uint8_t)(hi & 0xFF), (uint8_t)(hi >> 8)};
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if (k0 + j < K) codes[r * K + k0 + j] = q[j];
  if (lane == 0) scales[r * n_chunks + c] = __int_as_float((127 + e) << 23);
}

// Dequantised weights back to bf16 (read-back for the tests): w = q s.
__global__ void k_dequant_f8(const uint8_t* __restrict__ codes, const float* __restrict__ scales, long long rows,
                             int K, bf16* __restrict__ w) {
  const int n_chunks = (K + kF8Chunk - 1) / kF8Chunk;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < rows * K;
       i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / K;
    const int k = (int)(i % K);
    const __half_raw h = __nv_cvt_fp8_to_halfraw(codes[i], __NV_E4M3);
    const float s = scales[r * n_chunks + k / kF8Chunk];
    w[i] = __float2bfloat16_rn(__half2float(__half(h)) * s);
  }
}

// Expands 16 E4M3 codes (one 16-byte raw chunk) into 16 bf16 values q s
// (two 16-byte chunks).  Every step is exact: E4M3 -> f16 (each E4M3 value
// is a normal f16 or zero), f16 -> f32, times a power of two, f32 -> bf16 of
// a bf16-representable value.
__device__ __forceinline__ void f8_expand16(uint4 raw, float s, uint4& o0, uint4& o1) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t out[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)((w[i] >> (16 * h)) & 0xFFFF),
                                                       __NV_E4M3);
      const float2 f = __half22float2(__half2(hr));
      const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * s, f.y * s);
      out[i * 2 + h] = *reinterpret_cast<const uint32_t*>(&b);
    }
  }
  o0 = make_uint4(out[0], out[1], out[2], out[3]);
  o1 = make_uint4(out[4], out[5], out[6], out[7]);
}

struct F8Args {
  const float* scales;   // [A rows][n_chunks]
  int n_chunks;          // ceil(K / 128); GemmArgs::kb_total counts 128-input chunks here
  long long a_rows;      // rows of the weight tensor (scale reads stay inside it)
};

// Persistent grouped GEMM over FP8 weights, MT = 1 (128-row tiles), BN <= 256.
// Warps: 0 = TMA producer, 1 = MMA issuer, 2..5 = epilogue (TMEM lanes
// 32 (w % 4) ..), 6..13 = converters (thread 2 r + j expands input half j of
// tile row r).  Ring slot: converted A (2 x 16 KB) | raw A (16 KB) | B
// (2 x b_half).  Barriers per slot: full (TMA bytes landed), conv (256
// converter arrivals, after a proxy fence), empty (MMA commit).  Waits are
// bounded; a timeout sets the error word and the roles stop.
template <int BN>
__global__ void __launch_bounds__(kF8Threads, 1)
k_gemm_f8w_persistent(const __grid_constant__ CUtensorMap tmA8, const __grid_constant__ BMaps tmB, GemmArgs p_in,
                      F8Args f8, int items_dense, int smem_budget) {
  constexpr int kAccCols = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));
  constexpr int kMaxStages = 8;
  constexpr int kConvBytes = 2 * 16384, kRawBytes = 16384;
  pdl_launch();
  GemmArgs p = p_in;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full_bar[kMaxStages], conv_bar[kMaxStages], empty_bar[kMaxStages];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2];
  __shared__ uint32_t tmem_base;
  __shared__ int4 s_work[kF8WorkSmem];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&conv_bar[s], 32 * kF8ConvWarps);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 128); }
    fence_mbar_init();
    prefetch_tmap(&tmA8);
    for (int i = 0; i < 4; ++i) prefetch_tmap(&tmB.m[i]);
  }
  if (warp == 0) tmem_alloc(&tmem_base, 2 * kAccCols);
  pdl_wait();
  if (p.k_splits_dev) p.k_splits = max(1, min(*p.k_splits_dev, p.kb_total));
  const int n_items = p.work ? *p.work_count : items_dense;
  int rows_max = BN;
  if (p.max_rows_dev) rows_max = min(BN, max(kBoxRowsB, *p.max_rows_dev));
  const int b_half = ((rows_max + kBoxRowsB - 1) / kBoxRowsB) * kBoxRowsB * 128;
  const int stage_bytes = kConvBytes + kRawBytes + 2 * b_half;
  const int n_stages = max(1, min(kMaxStages, smem_budget / stage_bytes));
  const int total = p.m_tiles * p.k_splits * n_items;
  const bool work_smem = p.work != nullptr && n_items <= kF8WorkSmem;
  if (work_smem)
    for (int i = threadIdx.x; i < n_items; i += blockDim.x) s_work[i] = p.work[i];
  const int4* work = work_smem ? s_work : p.work;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  // tile -> (m tile, split, a_row0, b_row0, n_valid, out_row0)
  auto decode = [&](int tile, GemmTile& t) {
    t.m_tile = tile % p.m_tiles;
    const int r = tile / p.m_tiles;
    t.split = r % p.k_splits;
    const int item = r / p.k_splits;
    if (p.work) {
      const int4 w = work[item];
      t.a_row0 = w.x * p.a_group_rows; t.b_row0 = w.y; t.n_valid = w.z; t.out_row0 = w.w;
    } else {
      t.a_row0 = 0; t.b_row0 = item * p.n_tile; t.out_row0 = t.b_row0;
      t.n_valid = min(p.n_tile, p.N - t.b_row0);
    }
  };

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        GemmTile t;
        decode(tile, t);
        int c0, c1;
        split_range(p, t.split, c0, c1);
        const int n_boxes = (min(BN, (t.n_valid + 15) & ~15) + kBoxRowsB - 1) / kBoxRowsB;
        const uint32_t tx = kRawBytes + 2 * n_boxes * kBoxRowsB * 128;
        for (int c = c0; c < c1; ++c, ++it) {
          const int s = it % n_stages;
          const uint32_t ph = (it / n_stages) & 1;
          if (it >= n_stages && !mbar_wait(&empty_bar[s], ph ^ 1, p.err, DGDEV_TIMEOUT_TMA)) { ok = false; break; }
          uint8_t* st = smem + s * stage_bytes;
          mbar_expect_tx(&full_bar[s], tx);
          tma_load_2d(st + kConvBytes, &tmA8, c * kF8Chunk, t.a_row0 + t.m_tile * 128, &full_bar[s]);
          for (int j = 0; j < 2; ++j)
            tma_load_b_rows(st + kConvBytes + kRawBytes + j * b_half, &tmB, c * kF8Chunk + j * 64, t.b_row0,
                            n_boxes * kBoxRowsB, &full_bar[s]);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      int it = 0, local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++local) {
        GemmTile t;
        decode(tile, t);
        int c0, c1;
        split_range(p, t.split, c0, c1);
        const int n_mma = min(BN, (t.n_valid + 15) & ~15);
        const uint32_t idesc = idesc_bf16(128, n_mma);
        const int buf = local & 1;
        if (local >= 2 && !mbar_wait(&acc_empty[buf], ((local >> 1) & 1) ^ 1, p.err, DGDEV_TIMEOUT_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + buf * kAccCols;
        for (int c = c0; c < c1; ++c, ++it) {
          const int s = it % n_stages;
          const uint32_t ph = (it / n_stages) & 1;
          if (!mbar_wait(&conv_bar[s], ph, p.err, DGDEV_TIMEOUT_MMA)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * stage_bytes);
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const uint64_t ad = sdesc_sw128(st + j * 16384);
            const uint64_t bd = sdesc_sw128(st + kConvBytes + kRawBytes + j * b_half);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc_mma_bf16(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (c > c0 || j > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&empty_bar[s]);
        }
        tc_commit(&acc_full[buf]);
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // epilogue warps 2..5
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    int local = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
      GemmTile t;
      decode(tile, t);
      int c0, c1;
      split_range(p, t.split, c0, c1);
      const int n_mma = min(BN, (t.n_valid + 15) & ~15);
      const int buf = local & 1;
      const bool ok =
          __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (local >> 1) & 1, p.err, DGDEV_TIMEOUT_EPI));
      tc_fence_after();
      const int m0 = t.m_tile * 128;
      const bool m_ok = (m0 + row) < p.M;
      float* outp = p.out + (long long)t.split * p.split_stride + (long long)t.out_row0 * p.ldo + m0 + row;
      if (ok && c1 > c0) {
        epilogue_store(tmem + buf * kAccCols + ((uint32_t)(quad * 32) << 16), n_mma, t.n_valid, m_ok, outp,
                       p.ldo, p.alpha);
      } else if (ok && m_ok) {
        for (int n = 0; n < t.n_valid; ++n) outp[(long long)n * p.ldo] = 0.0f;
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
      if (!ok) break;
    }
  } else {
    // converter warps 6..13: thread 2 r + j expands inputs 64 j .. 64 j + 63 of tile row r
    const int tc = threadIdx.x - 192;
    const int r = tc >> 1, j = tc & 1;
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      GemmTile t;
      decode(tile, t);
      int c0, c1;
      split_range(p, t.split, c0, c1);
      const long long a_row = (long long)t.a_row0 + t.m_tile * 128 + r;
      const bool row_ok = (t.m_tile * 128 + r) < p.M && a_row < f8.a_rows;
      for (int c = c0; c < c1; ++c, ++it) {
        const int s = it % n_stages;
        const uint32_t ph = (it / n_stages) & 1;
        if (!mbar_wait(&full_bar[s], ph, p.err, DGDEV_TIMEOUT_MMA)) { ok = false; break; }
        const float sc = row_ok ? f8.scales[a_row * f8.n_chunks + c] : 0.0f;
        uint8_t* st = smem + s * stage_bytes;
        const uint8_t* raw_row = st + kConvBytes + r * 128;
        uint8_t* conv_row = st + j * 16384 + r * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int rc = 4 * j + i;                                   // raw 16-byte chunk of the row
          const uint4 raw = *reinterpret_cast<const uint4*>(raw_row + ((rc ^ (r & 7)) << 4));
          uint4 o0, o1;
          f8_expand16(raw, sc, o0, o1);
          *reinterpret_cast<uint4*>(conv_row + (((2 * i) ^ (r & 7)) << 4)) = o0;
          *reinterpret_cast<uint4*>(conv_row + (((2 * i + 1) ^ (r & 7)) << 4)) = o1;
        }
        fence_async_smem();   // generic-proxy writes -> visible to the tensor core
        mbar_arrive(&conv_bar[s]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 2 * kAccCols);
}
