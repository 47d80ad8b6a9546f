// GEMMs of the denoising step.
//
// Every projection is computed "swap-AB": out[n][m] = alpha * sum_k A[m][k] B[n][k]
// with A a weight matrix stored [out_features][in_features] (K-major) and B the
// activations [tokens][in_features] (K-major).  Weights fill the 128-row M side
// of tcgen05.mma, tokens the N side (16..256), so a 256-token canvas streams
// every weight byte exactly once and a small expert group (16 rows) still uses
// full-height MMA tiles.
//
// Work items.  Dense launches tile N by blockIdx; grouped (MoE) launches read
// work items (group, b_row0, n_valid, out_row0) built on the device by the
// permute kernel, one per (expert, token tile).  Split-K writes fp32 partials
// to out + split * split_stride; consumers sum the splits in index order.
#pragma once
#include "dg_device.cuh"


// Fused QKV post-process for the dense bf16 GEMM (head_dim 128, one split):
// each 128-row tile of the fused QKV weight is one head; q and k heads get
// rotate-half RoPE at their positions, q goes to Q [t][Hq][128], k into the
// K cache [lbh][pos][128], v transposed into the V^T cache [lbh][128][pos].
struct QkvEpi {
  bf16* q;
  bf16* kc;
  bf16* vt;
  const float2* rope;   // [pos][64] (cos, sin)
  int Hq, Hkv;
  int n_per;            // tokens per canvas in the launch
  int pos0;             // position of a canvas's first token
  int b0, B, layer, S;  // first canvas, canvases in the cache, layer, key slot stride
};

struct GemmArgs {
  int M;                   // valid A rows per work item
  int m_tiles;             // ceil(M / tile M)
  int kb_total;            // number of 64-wide K blocks
  int k_splits;            // split-K factor (k blocks divided evenly, last takes the rest)
  int N;                   // dense: total B rows
  int n_tile;              // dense: B rows per CTA
  float alpha;
  float* out;
  long long ldo;           // out row stride (elements)
  long long split_stride;  // elements between split-K partial outputs
  const int4* work;        // grouped: (group, b_row0, n_valid, out_row0); nullptr = dense
  int a_group_rows;        // grouped: A rows per group (a_row0 = group * a_group_rows)
  const int* work_count;
  const int* k_splits_dev; // persistent kernel: split-K factor chosen on the device (overrides k_splits)
  const int* max_rows_dev; // persistent kernel: rows of the largest work item (sizes the ring stages)
  int qkv_on;              // dense, one split, MT 1: fused QKV post-process (see QkvEpi)
  QkvEpi qkv;
  void* act;               // persistent gate|up: when non-null and the split factor is 1, the
                           // epilogue writes round(silu(g) u) (bf16, row stride act_ld) instead
                           // of the fp32 output; A rows interleave gate / up in blocks of 64
  int act_ld;
  int* err;
};

struct GemmTile {
  int m_tile, split, a_row0, b_row0, n_valid, out_row0;
};

__device__ __forceinline__ bool gemm_decode(const GemmArgs& p, GemmTile& t) {
  const int bid = blockIdx.x;
  t.m_tile = bid % p.m_tiles;
  const int r = bid / p.m_tiles;
  t.split = r % p.k_splits;
  const int item = r / p.k_splits;
  if (p.work) {
    if (item >= *p.work_count) return false;
    const int4 w = p.work[item];
    t.a_row0 = w.x * p.a_group_rows; t.b_row0 = w.y; t.n_valid = w.z; t.out_row0 = w.w;
  } else {
    const int n0 = item * p.n_tile;
    t.a_row0 = 0; t.b_row0 = n0; t.out_row0 = n0;
    t.n_valid = min(p.n_tile, p.N - n0);
  }
  return t.n_valid > 0;
}

__device__ __forceinline__ void split_range(const GemmArgs& p, int split, int& kb0, int& kb1) {
  const int per = p.kb_total / p.k_splits;
  kb0 = split * per;
  kb1 = (split == p.k_splits - 1) ? p.kb_total : kb0 + per;
}

// ---------------------------------------------------------------------------
// tcgen05 GEMM, bf16 in / fp32 out.  128 threads: warp 0 lane 0 issues TMA,
// warp 1 lane 0 issues MMAs, then all four warps drain TMEM (warp w owns
// accumulator rows 32w..32w+31).  A tiles 128 x 64, B tiles BN x 64 loaded
// 32 rows per TMA box; STAGES-deep mbarrier ring.  MT = 2 gives a CTA two
// 128-row accumulators that share every B tile (M tile 256): for the big
// vocabulary GEMMs this halves how often the activations stream from L2.
// ---------------------------------------------------------------------------
constexpr int kBoxRowsB = 32;   // B rows are loaded in multiples of 32

// Epilogue of one accumulator row (this thread's TMEM lane) of n_mma columns:
// out[c * ldo] = alpha * acc[c] for c < n_valid.  TMEM loads are issued four
// at a time (64 columns) before one wait.  Warp-collective: n_mma uniform.
__device__ __forceinline__ void epilogue_store(uint32_t taddr, int n_mma, int n_valid, bool m_ok, float* outp,
                                               long long ldo, float alpha) {
  for (int c0 = 0; c0 < n_mma; c0 += 64) {
    uint32_t v[4][16];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (c0 + q * 16 < n_mma) tmem_ld16_nw(taddr + c0 + q * 16, v[q]);
    tmem_wait_ld();
    if (m_ok) {
      float* o = outp + (long long)c0 * ldo;
      if (c0 + 64 <= n_valid) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int j = 0; j < 16; ++j) o[(long long)(q * 16 + j) * ldo] = __uint_as_float(v[q][j]) * alpha;
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + q * 16 + j < n_valid) o[(long long)(q * 16 + j) * ldo] = __uint_as_float(v[q][j]) * alpha;
      }
    }
  }
}

// Fused QKV epilogue of one 128-row tile (head `head`) of the dense GEMM,
// 128 threads (thread = channel c = TMEM lane), up to 64 tokens per pass.
// q / k heads: RoPE pairs channels c and c + 64; the upper-half threads pass
// their values to the lower half through shared memory, the lower half
// rotates and writes the bf16 head rows of the pass into a [token][channel]
// staging tile, and all threads then copy whole 256-byte rows (16-byte
// stores) to Q or the K cache.  v heads: each thread owns one V^T row and
// writes its run of positions with 16-byte stores when the tokens are
// consecutive positions of one canvas (scalar stores otherwise).
// `xch` is the pipeline ring (free after the mainloop).
__device__ __forceinline__ void qkv_epilogue(const QkvEpi& e, uint32_t taddr, int head, int tok0, int n_valid,
                                             int n_mma, bool have, uint8_t* xch_raw) {
  float* xch = reinterpret_cast<float*>(xch_raw);                      // [64][65] fp32
  bf16* st = reinterpret_cast<bf16*>(xch_raw + 64 * 65 * 4 + 256);     // [64][136] bf16
  constexpr int kStPitch = 136;
  const int c = threadIdx.x;   // 0..127
  for (int c0 = 0; c0 < n_mma; c0 += 64) {
    uint32_t v[4][16];
    if (have) {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (c0 + q * 16 < n_mma) tmem_ld16_nw(taddr + c0 + q * 16, v[q]);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int j = 0; j < 16; ++j) v[q][j] = 0u;
    }
    const int nt = min(64, n_valid - c0);   // tokens of this pass
    if (head < e.Hq + e.Hkv) {
      if (c >= 64) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int j = 0; j < 16; ++j) xch[(c - 64) * 65 + q * 16 + j] = __uint_as_float(v[q][j]);
      }
      __syncthreads();
      if (c < 64) {
        const int t = tok0 + c0;
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = q * 16 + j;
            if (n < nt) {
              const int pn = e.pos0 + (t + n) % e.n_per;
              const float2 cs = e.rope[(long long)pn * 64 + c];
              const float x0 = __uint_as_float(v[q][j]), x1 = xch[c * 65 + n];
              st[n * kStPitch + c] = __float2bfloat16_rn(x0 * cs.x - x1 * cs.y);
              st[n * kStPitch + c + 64] = __float2bfloat16_rn(x0 * cs.y + x1 * cs.x);
            }
          }
      }
      __syncthreads();
      // copy: 16 threads per token row (16 x 16 B = 256 B)
      for (int id = threadIdx.x; id < nt * 16; id += 128) {
        const int n = id >> 4, part = id & 15;
        const int t = tok0 + c0 + n;
        const int b = e.b0 + t / e.n_per, pn = e.pos0 + t % e.n_per;
        bf16* dst;
        if (head < e.Hq) {
          dst = e.q + ((long long)t * e.Hq + head) * 128;
        } else {
          const long long lbh = ((long long)e.layer * e.B + b) * e.Hkv + (head - e.Hq);
          dst = e.kc + (lbh * e.S + pn) * 128;
        }
        *reinterpret_cast<uint4*>(dst + part * 8) = *reinterpret_cast<const uint4*>(st + n * kStPitch + part * 8);
      }
      __syncthreads();
    } else {
      const int g = head - e.Hq - e.Hkv;
      const int t0 = tok0 + c0;
      const int b = e.b0 + t0 / e.n_per, p0 = e.pos0 + t0 % e.n_per;
      const long long lbh = ((long long)e.layer * e.B + b) * e.Hkv + g;
      bf16* row = e.vt + (lbh * 128 + c) * e.S + p0;
      const bool vec = nt == 64 && (t0 % e.n_per) + 64 <= e.n_per && (p0 % 8) == 0 && (e.S % 8) == 0;
      if (vec) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t pk[8];
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const __nv_bfloat162 pr = __floats2bfloat162_rn(__uint_as_float(v[q][j]), __uint_as_float(v[q][j + 1]));
            pk[j / 2] = *reinterpret_cast<const uint32_t*>(&pr);
          }
          *reinterpret_cast<uint4*>(row + q * 16) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(row + q * 16 + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = q * 16 + j;
            if (n < nt) {
              const int t = t0 + n;
              const int bb = e.b0 + t / e.n_per, pn = e.pos0 + t % e.n_per;
              const long long lb = ((long long)e.layer * e.B + bb) * e.Hkv + g;
              e.vt[(lb * 128 + c) * e.S + pn] = __float2bfloat16_rn(__uint_as_float(v[q][j]));
            }
          }
      }
    }
  }
}

// Tensor maps of one B operand with boxes of 32, 64, 128 and 256 rows: a tile
// of n rows is fetched with the fewest boxes (greedy, largest first), since
// every TMA box costs a fixed issue overhead (measured: 8 boxes of 32 rows per
// k-block made a 256-row tile 50% slower than one box of 256).
struct BMaps {
  CUtensorMap m[4];   // box rows 32 << i
};

// Loads rows [row0, row0 + n_load) (n_load a multiple of 32, <= 256) of K
// block x into dst (rows contiguous, 128 B each) on barrier bar.
__device__ __forceinline__ void tma_load_b_rows(uint8_t* dst, const BMaps* bm, int x, int row0, int n_load,
                                                uint64_t* bar) {
  int r = 0;
#pragma unroll 1
  for (int i = 3; i >= 0; --i) {
    const int box = 32 << i;
    while (n_load - r >= box) {
      tma_load_2d(dst + r * 128, &bm->m[i], x, row0 + r, bar);
      r += box;
    }
  }
}

template <int BN, int STAGES, int MT = 1>
struct GemmTcCfg {
  static constexpr int kABytes = MT * 128 * 128;     // MT x (128 rows x 64 bf16)
  static constexpr int kBBytes = BN * 128;           // BN rows x 64 bf16
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kTmemCols = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));
  static constexpr int kSmem = STAGES * kStage + 1024;
};

template <int BN, int STAGES, int MT = 1>
__global__ void __launch_bounds__(128, 1)
k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ BMaps tmB,
          GemmArgs p) {
  using C = GemmTcCfg<BN, STAGES, MT>;
  static_assert(MT * C::kTmemCols <= 512, "tensor memory holds 512 columns");
  pdl_launch();
  // grouped work items come from the permute kernel: decode after the wait;
  // dense tiles are pure index arithmetic and prefetch weight tiles first
  const bool grouped = p.work != nullptr;
  if (grouped) pdl_wait();
  GemmTile t;
  if (!gemm_decode(p, t)) {
    if (!grouped) pdl_wait();
    return;
  }
  int kb0, kb1;
  split_range(p, t.split, kb0, kb1);
  const int nkb = kb1 - kb0;
  const int n_mma = min(BN, (t.n_valid + 15) & ~15);
  const int n_boxes = (n_mma + kBoxRowsB - 1) / kBoxRowsB;   // B rows loaded >= n_mma (extra rows unused)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full_bar[STAGES], empty_bar[STAGES], done_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
    mbar_init(&done_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    for (int i = 0; i < 4; ++i) prefetch_tmap(&tmB.m[i]);
  }
  if (warp == 0) tmem_alloc(&tmem_base, MT * C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const int m0 = t.m_tile * 128 * MT;

  const uint32_t tx = C::kABytes + n_boxes * kBoxRowsB * 128;
  // dense: the first ring slots' weight tiles are fetched before the wait
  const int n_pre = grouped ? 0 : min(STAGES, nkb);
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < n_pre; ++i) {
      mbar_expect_tx(&full_bar[i], tx);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
        tma_load_2d(smem + i * C::kStage + mt * 16384, &tmA, (kb0 + i) * 64, t.a_row0 + m0 + mt * 128,
                    &full_bar[i]);
    }
  }
  if (!grouped) pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < nkb; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (i >= STAGES && !mbar_wait(&empty_bar[s], ph ^ 1, p.err, DGDEV_TIMEOUT_TMA)) {
          abort_flag = 1;
          break;
        }
        uint8_t* a_s = smem + s * C::kStage;
        uint8_t* b_s = a_s + C::kABytes;
        const int kx = (kb0 + i) * 64;
        if (i >= n_pre) {
          mbar_expect_tx(&full_bar[s], tx);
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
            tma_load_2d(a_s + mt * 16384, &tmA, kx, t.a_row0 + m0 + mt * 128, &full_bar[s]);
        }
        tma_load_b_rows(b_s, &tmB, kx, t.b_row0, n_boxes * kBoxRowsB, &full_bar[s]);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, n_mma);
      bool ok = true;
      for (int i = 0; i < nkb && ok; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&full_bar[s], ph, p.err, DGDEV_TIMEOUT_MMA)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * C::kStage);
        const uint32_t b_addr = a_addr + C::kABytes;
        const uint64_t bd = sdesc_sw128(b_addr);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
            tc_mma_bf16(tmem + mt * C::kTmemCols, sdesc_sw128(a_addr + mt * 16384) + 2 * kk, bd + 2 * kk, idesc,
                        (i | kk) != 0);
        tc_commit(&empty_bar[s]);
      }
      // Completes when every MMA above has finished (also on the abort path).
      tc_commit(&done_bar);
    }
    __syncwarp();
  }

  // Epilogue: TMEM -> registers -> out[(out_row0 + n) * ldo + m0 + row].
  // tcgen05.ld is warp-collective: agree on the wait outcome across the warp.
  const bool ok = __all_sync(0xffffffffu, mbar_wait(&done_bar, 0, p.err, DGDEV_TIMEOUT_EPI));
  tc_fence_after();
  if (MT == 1 && p.qkv_on) {
    qkv_epilogue(p.qkv, tmem + ((uint32_t)(warp * 32) << 16), t.m_tile, t.out_row0, t.n_valid, n_mma,
                 ok && nkb > 0, smem);
  } else
  for (int mt = 0; mt < MT; ++mt) {
    const int row = mt * 128 + warp * 32 + lane;
    const bool m_ok = (m0 + row) < p.M;
    float* outp = p.out + (long long)t.split * p.split_stride + (long long)t.out_row0 * p.ldo + m0 + row;
    if (ok && nkb > 0) {
      epilogue_store(tmem + mt * C::kTmemCols + ((uint32_t)(warp * 32) << 16), n_mma, t.n_valid, m_ok, outp,
                     p.ldo, p.alpha);
    } else if (nkb == 0 && ok && m_ok) {
      for (int n = 0; n < t.n_valid; ++n) outp[(long long)n * p.ldo] = 0.0f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, MT * C::kTmemCols);
}

// ---------------------------------------------------------------------------
// Persistent variant for long tile lists (expert GEMMs, LM head): one CTA per
// SM slot walks tiles blockIdx.x, +gridDim.x, ...  The TMA ring runs across
// tile boundaries, and the accumulator is double-buffered in TMEM so the
// epilogue of tile i overlaps the mainloop of tile i+1.
// Warps: 0 = TMA producer, 1 = MMA issuer, 2..5 = epilogue (warp w drains
// TMEM lanes 32*(w%4)..+31).  192 threads.
// ---------------------------------------------------------------------------
constexpr int kWorkSmem = 512;   // work items staged in shared memory (more are read from global)


// Barrier among the four epilogue warps (threads 64..191) of the persistent kernel.
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int BN, int STAGES, int MT = 1>
__global__ void __launch_bounds__(192, 1)
k_gemm_tc_persistent(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ BMaps tmB,
                     GemmArgs p_in, int items_dense) {
  using C = GemmTcCfg<BN, STAGES, MT>;
  constexpr int kAccCols = C::kTmemCols;               // one 128-row accumulator
  // MT = 1: two accumulator buffers (the epilogue of one tile overlaps the
  // next tile's mainloop).  MT = 2: one buffer of two accumulators (a 256-row
  // tile: every B tile feeds twice the MMA work).
  constexpr int kNBuf = MT == 1 ? 2 : 1;
  constexpr int kAllocCols = kNBuf * MT * kAccCols;
  static_assert(kAllocCols <= 512, "tensor memory holds 512 columns");
  constexpr int kTileRows = 128 * MT;
  // The ring holds STAGES full-size stages; when every work item has fewer
  // rows than BN, stages shrink to A + the rows actually loaded and the ring
  // holds more of them (more weight bytes in flight per SM).
  constexpr int kMaxStages = 3 * STAGES;
  pdl_launch();
  GemmArgs p = p_in;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full_bar[kMaxStages], empty_bar[kMaxStages], acc_full[2], acc_empty[2];
  __shared__ uint32_t tmem_base;
  __shared__ int4 s_work[kWorkSmem];
  __shared__ float s_xfer[64 * 17];   // fused SwiGLU: up values of one 16-column chunk
  __shared__ int s_epi_fail;          // fused SwiGLU: an epilogue wait ran out
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxStages; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 128); }
    fence_mbar_init();
    prefetch_tmap(&tmA);
    for (int i = 0; i < 4; ++i) prefetch_tmap(&tmB.m[i]);
    s_epi_fail = 0;
  }
  if (warp == 0) tmem_alloc(&tmem_base, kAllocCols);
  // the split factor and the work list are written by the permute kernel
  pdl_wait();
  if (p.k_splits_dev) p.k_splits = max(1, min(*p.k_splits_dev, p.kb_total));
  constexpr int tile_rows = kTileRows, nbuf = kNBuf, acc_stride = MT, a_bytes = C::kABytes;
  const int n_items = p.work ? *p.work_count : items_dense;
  // ring geometry from the largest B tile any work item loads
  int rows_max = BN;
  if (p.max_rows_dev) rows_max = min(BN, max(kBoxRowsB, *p.max_rows_dev));
  const int stage_bytes = a_bytes + ((rows_max + kBoxRowsB - 1) / kBoxRowsB) * kBoxRowsB * 128;
  const int n_stages = min(kMaxStages, (STAGES * C::kStage) / stage_bytes);
  const int total = p.m_tiles * p.k_splits * n_items;
  // work items are read by all three roles once per tile: stage them on chip
  const bool work_smem = p.work != nullptr && n_items <= kWorkSmem;
  if (work_smem)
    for (int i = threadIdx.x; i < n_items; i += blockDim.x) s_work[i] = p.work[i];
  const int4* work = work_smem ? s_work : p.work;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  // 128-row halves of tile m_t that hold rows below M (the last tile of an
  // odd number of halves loads and multiplies only its first half)
  auto halves = [&](int m_t) { return MT == 1 ? 1 : min(MT, (p.M - m_t * kTileRows + 127) / 128); };

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;   // global k-block counter across tiles (ring position)
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        GemmTile t;
        // decode with blockIdx replaced by `tile`
        t.m_tile = tile % p.m_tiles;
        const int r = tile / p.m_tiles;
        t.split = r % p.k_splits;
        const int item = r / p.k_splits;
        if (p.work) {
          const int4 w = work[item];
          t.a_row0 = w.x * p.a_group_rows; t.b_row0 = w.y; t.n_valid = w.z;
        } else {
          t.a_row0 = 0; t.b_row0 = item * p.n_tile; t.n_valid = min(p.n_tile, p.N - t.b_row0);
        }
        int kb0, kb1;
        split_range(p, t.split, kb0, kb1);
        const int nh = halves(t.m_tile);
        const int n_boxes = (min(BN, (t.n_valid + 15) & ~15) + kBoxRowsB - 1) / kBoxRowsB;
        const uint32_t tx = nh * 16384 + n_boxes * kBoxRowsB * 128;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % n_stages;
          const uint32_t ph = (it / n_stages) & 1;
          if (it >= n_stages && !mbar_wait(&empty_bar[s], ph ^ 1, p.err, DGDEV_TIMEOUT_TMA)) { ok = false; break; }
          uint8_t* a_s = smem + s * stage_bytes;
          uint8_t* b_s = a_s + a_bytes;
          mbar_expect_tx(&full_bar[s], tx);
          for (int h = 0; h < nh; ++h)
            tma_load_2d(a_s + h * 16384, &tmA, kb * 64, t.a_row0 + t.m_tile * tile_rows + h * 128, &full_bar[s]);
          tma_load_b_rows(b_s, &tmB, kb * 64, t.b_row0, n_boxes * kBoxRowsB, &full_bar[s]);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      int it = 0, local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++local) {
        const int m_t = tile % p.m_tiles;
        const int r = tile / p.m_tiles;
        const int split = r % p.k_splits;
        const int item = r / p.k_splits;
        const int n_valid = p.work ? work[item].z : min(p.n_tile, p.N - item * p.n_tile);
        const int nh = halves(m_t);
        int kb0, kb1;
        split_range(p, split, kb0, kb1);
        const int n_mma = min(BN, (n_valid + 15) & ~15);
        const uint32_t idesc = idesc_bf16(128, n_mma);
        const int buf = local % nbuf;
        // wait until the epilogue drained this buffer (nbuf tiles ago)
        if (local >= nbuf &&
            !mbar_wait(&acc_empty[buf], ((local / nbuf) & 1) ^ 1, p.err, DGDEV_TIMEOUT_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + buf * acc_stride * kAccCols;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % n_stages;
          const uint32_t ph = (it / n_stages) & 1;
          if (!mbar_wait(&full_bar[s], ph, p.err, DGDEV_TIMEOUT_MMA)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * stage_bytes);
          const uint64_t bd = sdesc_sw128(a_addr + a_bytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
#pragma unroll
            for (int h = 0; h < MT; ++h)
              if (h < nh)
                tc_mma_bf16(d_tmem + h * kAccCols, sdesc_sw128(a_addr + h * 16384) + 2 * kk, bd + 2 * kk, idesc,
                            (kb > kb0 || kk > 0) ? 1u : 0u);
          tc_commit(&empty_bar[s]);
        }
        tc_commit(&acc_full[buf]);
      }
    }
    __syncwarp();
  } else {
    // epilogue warps 2..5
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    int local = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
      const int m_t = tile % p.m_tiles;
      const int r = tile / p.m_tiles;
      const int split = r % p.k_splits;
      const int item = r / p.k_splits;
      int n_valid, out_row0;
      if (p.work) { const int4 w = work[item]; n_valid = w.z; out_row0 = w.w; }
      else { out_row0 = item * p.n_tile; n_valid = min(p.n_tile, p.N - out_row0); }
      int kb0, kb1;
      split_range(p, split, kb0, kb1);
      const int n_mma = min(BN, (n_valid + 15) & ~15);
      const int nh = halves(m_t);
      const int buf = local % nbuf;
      const bool ok =
          __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (local / nbuf) & 1, p.err, DGDEV_TIMEOUT_EPI));
      tc_fence_after();
      if (p.act && p.k_splits == 1) {
        // fused SwiGLU: in each 128-row half, rows 0..63 are gate rows of SwiGLU
        // outputs f = 64 (half index) .. + 63 and rows 64..127 the matching up
        // rows.  The up quads hand their values to the gate quads through shared
        // memory.  The four warps first agree on the wait outcome (they share
        // barriers).
        if (lane == 0 && !ok) s_epi_fail = 1;
        epi_sync();
        const bool ok_all = s_epi_fail == 0;
        bf16* act = reinterpret_cast<bf16*>(p.act);
        for (int h = 0; h < nh; ++h) {
          const int f = (m_t * (tile_rows / 128) + h) * 64 + (quad & 1) * 32 + lane;
          const uint32_t tbase = tmem + (buf * acc_stride + h) * kAccCols + ((uint32_t)(quad * 32) << 16);
          for (int c0 = 0; c0 < n_mma; c0 += 16) {
            uint32_t v[16];
            if (ok_all && kb1 > kb0) {
              tmem_ld16_nw(tbase + c0, v);
              tmem_wait_ld();
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) v[j] = 0u;
            }
            if (quad >= 2) {
#pragma unroll
              for (int j = 0; j < 16; ++j) s_xfer[((quad - 2) * 32 + lane) * 17 + j] = __uint_as_float(v[j]);
            }
            epi_sync();
            if (quad < 2) {
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                if (c0 + j < n_valid) {
                  const float g = __uint_as_float(v[j]);
                  const float u = s_xfer[(quad * 32 + lane) * 17 + j];
                  act[(long long)(out_row0 + c0 + j) * p.act_ld + f] =
                      __float2bfloat16_rn(g / (1.0f + expf(-g)) * u);
                }
              }
            }
            epi_sync();
          }
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[buf]);
        if (!ok_all) break;
        continue;
      }
      for (int h = 0; h < nh; ++h) {
        const int m0 = m_t * tile_rows + h * 128;
        const bool m_ok = (m0 + row) < p.M;
        float* outp = p.out + (long long)split * p.split_stride + (long long)out_row0 * p.ldo + m0 + row;
        if (ok && kb1 > kb0) {
          epilogue_store(tmem + (buf * acc_stride + h) * kAccCols + ((uint32_t)(quad * 32) << 16), n_mma, n_valid, m_ok,
                         outp, p.ldo, p.alpha);
        } else if (ok && m_ok) {
          for (int n = 0; n < n_valid; ++n) outp[(long long)n * p.ldo] = 0.0f;
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
      if (!ok) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kAllocCols);
}

// ---------------------------------------------------------------------------
// fp32 SIMT GEMM with the same contract (the fp32 workload's projections):
// 64 x 64 output tile per CTA, 256 threads, 4 x 4 outputs per thread.
// ---------------------------------------------------------------------------
static __global__ void __launch_bounds__(256)
k_gemm_f32(const float* __restrict__ A, long long lda, const float* __restrict__ B, long long ldb,
           int K, GemmArgs p) {
  pdl_enter();
  GemmTile t;
  if (!gemm_decode(p, t)) return;
  int kb0, kb1;
  split_range(p, t.split, kb0, kb1);
  const int k_begin = kb0 * 64, k_end = min(K, kb1 * 64);
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = t.m_tile * 64;
  float acc[4][4] = {};
  for (int k0 = k_begin; k0 < k_end; k0 += 16) {
    for (int i = threadIdx.x; i < 16 * 64; i += 256) {
      const int kk = i % 16, r = i / 16;
      const int k = k0 + kk;
      const int am = m0 + r;
      As[kk][r] = (k < k_end && am < p.M) ? A[(long long)(t.a_row0 + am) * lda + k] : 0.0f;
      Bs[kk][r] = (k < k_end && r < t.n_valid) ? B[(long long)(t.b_row0 + r) * ldb + k] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty * 4 + i]; b[i] = Bs[kk][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* outp = p.out + (long long)t.split * p.split_stride;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= p.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = tx * 4 + j;
      if (n < t.n_valid) outp[(long long)(t.out_row0 + n) * p.ldo + m] = acc[i][j] * p.alpha;
    }
  }
}
