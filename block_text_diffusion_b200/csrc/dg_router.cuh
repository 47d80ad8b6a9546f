// MoE router as one kernel: router logits on the tensor cores, split-K
// partials reduced through distributed shared memory, top-k and gate softmax.
//
// r[t][e] = sum_k x[t][k] Wr[e][k] (+ b_e) (+ c[t][e], an optional per-token
// bias given as input), fp32 accumulation; the k largest
// (ties to the lower expert id) in descending order; gates = softmax over the
// k selected logits.  (Mixture-of-Experts FFN of the DiffusionGemma
// technical-report explainer, section 二: each token goes to top_k experts.)
//
// Grid: (token tiles of 32) x kRouterSplits CTAs; the kRouterSplits CTAs of a
// token tile form one thread-block cluster and each accumulates one K range
// of the [E <= 128 experts] x [32 tokens] logit tile in TMEM.  After a cluster
// barrier, CTA r sums the partials of tokens 4r..4r+3 over the cluster in rank
// order (the same order as the split-K consumers elsewhere) and runs the
// top-k, one warp per token.
#pragma once
#include "dg_device.cuh"

constexpr int kRouterSplits = 8;
constexpr int kRouterBN = 32;
constexpr int kRouterStages = 4;
constexpr int kRouterStage = 16384 + kRouterBN * 128;      // A (128 x 64 bf16) + B (32 x 64 bf16)
constexpr int kRouterSmem = kRouterStages * kRouterStage + kRouterBN * 128 * 4 + 1024;

struct RouterArgs {
  int E, k, n_tok, kb_total;
  const float* bias;   // [E] or null
  const float* tok_bias;   // [n_tok][E] or null
  int* ids;            // [n_tok][k]
  float* gate;         // [n_tok][k]
  int* err;
};

__global__ void __cluster_dims__(kRouterSplits, 1, 1) __launch_bounds__(128, 1)
k_router_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, RouterArgs p) {
  pdl_launch();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  float* part = reinterpret_cast<float*>(smem + kRouterStages * kRouterStage);   // [32 tokens][128 experts]
  __shared__ __align__(8) uint64_t full_bar[kRouterStages], empty_bar[kRouterStages], done_bar;
  __shared__ uint32_t tmem_base;
  uint32_t rank;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
  const int tile = blockIdx.x / kRouterSplits;
  const int n0 = tile * kRouterBN;
  const int n_valid = min(kRouterBN, p.n_tok - n0);
  const int per = p.kb_total / kRouterSplits;
  const int kb0 = (int)rank * per;
  const int kb1 = rank == kRouterSplits - 1 ? p.kb_total : kb0 + per;
  const int nkb = kb1 - kb0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t tx = 16384 + kRouterBN * 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRouterStages; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
    mbar_init(&done_bar, 1);
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 0) tmem_alloc(&tmem_base, 32);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  // router weights are never written by the step: first ring slots before the wait
  const int n_pre = min(kRouterStages, nkb);
  if (warp == 0 && lane == 0)
    for (int i = 0; i < n_pre; ++i) {
      mbar_expect_tx(&full_bar[i], tx);
      tma_load_2d(smem + i * kRouterStage, &tmA, (kb0 + i) * 64, 0, &full_bar[i]);
    }
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < nkb; ++i) {
        const int s = i % kRouterStages;
        const uint32_t ph = (i / kRouterStages) & 1;
        if (i >= kRouterStages && !mbar_wait(&empty_bar[s], ph ^ 1, p.err, DGDEV_TIMEOUT_TMA)) break;
        uint8_t* a_s = smem + s * kRouterStage;
        if (i >= n_pre) {
          mbar_expect_tx(&full_bar[s], tx);
          tma_load_2d(a_s, &tmA, (kb0 + i) * 64, 0, &full_bar[s]);
        }
        tma_load_2d(a_s + 16384, &tmB, (kb0 + i) * 64, n0, &full_bar[s]);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, kRouterBN);
      for (int i = 0; i < nkb; ++i) {
        const int s = i % kRouterStages;
        if (!mbar_wait(&full_bar[s], (i / kRouterStages) & 1, p.err, DGDEV_TIMEOUT_MMA)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * kRouterStage);
        const uint64_t ad = sdesc_sw128(a_addr), bd = sdesc_sw128(a_addr + 16384);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) tc_mma_bf16(tmem, ad + 2 * kk, bd + 2 * kk, idesc, (i | kk) != 0);
        tc_commit(&empty_bar[s]);
      }
      tc_commit(&done_bar);
    }
    __syncwarp();
  }

  // partial logits of this K range -> shared memory [token][expert]
  const bool ok = __all_sync(0xffffffffu, mbar_wait(&done_bar, 0, p.err, DGDEV_TIMEOUT_EPI));
  tc_fence_after();
  {
    const int e = warp * 32 + lane;
    uint32_t v[2][16];
    if (ok && nkb > 0) {
      tmem_ld16_nw(tmem + ((uint32_t)(warp * 32) << 16), v[0]);
      tmem_ld16_nw(tmem + ((uint32_t)(warp * 32) << 16) + 16, v[1]);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c) v[c >> 4][c & 15] = 0u;
    }
#pragma unroll
    for (int c = 0; c < 32; ++c) part[c * 128 + e] = __uint_as_float(v[c >> 4][c & 15]);
  }
  tc_fence_before();
  cluster_sync_all();

  // tokens 4 rank .. 4 rank + 3: one warp each
  const int tl = (int)rank * 4 + warp;
  if (tl < n_valid) {
    const long long t = n0 + tl;
    float lg[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = lane + 32 * q;
      float acc = 0.0f;
      for (int r = 0; r < kRouterSplits; ++r) acc += cluster_peer(part, r)[tl * 128 + e];
      lg[q] = (e < p.E) ? acc + (p.bias ? p.bias[e] : 0.0f) + (p.tok_bias ? p.tok_bias[t * p.E + e] : 0.0f)
                        : -INFINITY;
    }
    float sel = 0.0f, top = 0.0f;
    int sid = 0;
    for (int j = 0; j < p.k; ++j) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int e = lane + 32 * q;
        if (e < p.E && (lg[q] > bv || (lg[q] == bv && e < bi))) { bv = lg[q]; bi = e; }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      if (j == 0) top = bv;
      if (lane == j) { sel = bv; sid = bi; }
#pragma unroll
      for (int q = 0; q < 4; ++q)   // the owner lane removes the winner
        if (bi == lane + 32 * q) lg[q] = -INFINITY;
    }
    const float ex = lane < p.k ? expf(sel - top) : 0.0f;
    float den = ex;
#pragma unroll
    for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (lane < p.k) {
      p.ids[t * p.k + lane] = sid;
      p.gate[t * p.k + lane] = ex / den;
    }
  }
  // no CTA may leave while another still reads its partials
  cluster_sync_all();
  if (warp == 0) tmem_dealloc(tmem, 32);
}
