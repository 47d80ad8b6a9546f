// Attention of canvas queries over [prompt KV ; canvas KV] (bidirectional,
// no mask) and of prompt queries over the prompt (causal, for the encode).
//
// KV cache layout (owned by the library, inside the caller's buffer):
//   K  [L][B][Hkv][S][hd]   keys, one row per position
//   Vt [L][B][Hkv][hd][S]   values transposed, so both tensor-core operands
//                           (K for S = Q K^T, V^T for O = P V) are K-major
// S = slot stride >= P + 256, positions 0..P-1 prompt, P..P+255 canvas.
//
// tcgen05 kernel: one CTA = 128 query rows (128/G tokens x the G query heads
// sharing one KV head) x one split of the key range.  Warp 4 issues TMA
// (Q once, K/V blocks of 128 keys double-buffered), warp 5 issues the MMAs,
// warps 0-3 run the online softmax: thread = query row = TMEM lane.
// S = Q K^T lives in TMEM columns [0,128), O in [128,256).  P is written as
// bf16 into shared memory in the 128B-swizzled K-major layout the MMA reads.
// Each split writes its normalised partial O and log2-sum-exp; a combine
// kernel merges the splits in index order.
#pragma once
#include "dg_device.cuh"

struct AttnArgs {
  int n_q;              // query tokens per canvas in this launch
  int q_pos0;           // absolute position of query token 0
  int n_keys;           // keys per canvas visible to this launch
  int causal;           // 1: key j visible to query at position p iff j <= p
  int G;                // query heads per KV head
  int Hq, Hkv;
  int q_tiles;          // ceil(n_q * G / 128)
  int n_splits;
  int blocks_per_split; // KV blocks of 128 keys per split
  int lbh0;             // (layer * B + b0) * Hkv: outer index of canvas b0's head 0
  int n_canvas;         // canvases in this launch
  float scale_log2;     // log2(e) / sqrt(hd)
  float* o_part;        // [n_splits][n_canvas * n_q * Hq][hd] fp32
  float* lse_part;      // [n_splits][n_canvas * n_q * Hq]
  int* err;
};

constexpr int kAttnThreads = 192;
constexpr int kAttnSmem = 32768 /*Q*/ + 2 * 65536 /*K,V x2*/ + 32768 /*P*/ + 1024;

__global__ void __launch_bounds__(kAttnThreads, 1)
k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
          const __grid_constant__ CUtensorMap tmV, AttnArgs a) {
  pdl_enter();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;                 // 2 x [128 rows][128 B]
  uint8_t* sKV = smem + 32768;        // stage s: K (2 x 16 KB) then V (2 x 16 KB)
  uint8_t* sP = smem + 32768 + 2 * 65536;
  __shared__ __align__(8) uint64_t q_full, kv_full[2], kv_empty[2], s_full, p_full, o_done;
  __shared__ uint32_t tmem_base;

  int bid = blockIdx.x;
  const int split = bid % a.n_splits; bid /= a.n_splits;
  const int qt = bid % a.q_tiles; bid /= a.q_tiles;
  const int g = bid % a.Hkv;
  const int bc = bid / a.Hkv;                   // canvas within the launch
  const int tok_per_tile = 128 / a.G;
  const int tok0 = qt * tok_per_tile;
  const int lbh = a.lbh0 + bc * a.Hkv + g;

  // key blocks of this split (causal: only blocks reaching the tile's last query)
  const int n_blocks_all = (a.n_keys + 127) / 128;
  int kb_begin = split * a.blocks_per_split;
  int kb_end = min(n_blocks_all, kb_begin + a.blocks_per_split);
  if (a.causal) {
    const int last_pos = a.q_pos0 + min(a.n_q, tok0 + tok_per_tile) - 1;
    kb_end = min(kb_end, last_pos / 128 + 1);
  }
  const int nblk = max(0, kb_end - kb_begin);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < 2; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
    mbar_init(&s_full, 1);
    mbar_init(&p_full, 128);
    mbar_init(&o_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&tmem_base, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const uint32_t tS = tmem, tO = tmem + 128;
  const uint32_t idesc = idesc_bf16(128, 128);

  if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && nblk > 0) {
      mbar_expect_tx(&q_full, 32768);
      const int zq = bc * a.n_q + tok0;
      tma_load_3d(sQ, &tmQ, 0, g * a.G, zq, &q_full);
      tma_load_3d(sQ + 16384, &tmQ, 64, g * a.G, zq, &q_full);
      for (int j = 0; j < nblk; ++j) {
        const int s = j & 1;
        if (j >= 2 && !mbar_wait(&kv_empty[s], ((j >> 1) & 1) ^ 1, a.err, DGDEV_TIMEOUT_TMA)) break;
        uint8_t* kv = sKV + s * 65536;
        const int key0 = (kb_begin + j) * 128;
        mbar_expect_tx(&kv_full[s], 65536);
        tma_load_3d(kv, &tmK, 0, key0, lbh, &kv_full[s]);
        tma_load_3d(kv + 16384, &tmK, 64, key0, lbh, &kv_full[s]);
        tma_load_3d(kv + 32768, &tmV, key0, 0, lbh, &kv_full[s]);
        tma_load_3d(kv + 49152, &tmV, key0 + 64, 0, lbh, &kv_full[s]);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && nblk > 0) {
      bool ok = mbar_wait(&q_full, 0, a.err, DGDEV_TIMEOUT_MMA);
      const uint32_t q_addr = smem_u32(sQ), p_addr = smem_u32(sP);
      for (int j = 0; j <= nblk && ok; ++j) {
        if (j > 0) {
          // O += P_{j-1} V_{j-1}
          if (!mbar_wait(&p_full, (j - 1) & 1, a.err, DGDEV_TIMEOUT_MMA)) { ok = false; break; }
          tc_fence_after();
          const uint32_t v_addr = smem_u32(sKV + ((j - 1) & 1) * 65536 + 32768);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ad = sdesc_sw128(p_addr + (kk >> 2) * 16384) + 2 * (kk & 3);
            const uint64_t bd = sdesc_sw128(v_addr + (kk >> 2) * 16384) + 2 * (kk & 3);
            tc_mma_bf16(tO, ad, bd, idesc, (j > 1 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&o_done);
          tc_commit(&kv_empty[(j - 1) & 1]);
        }
        if (j < nblk) {
          // S = Q K_j^T
          if (!mbar_wait(&kv_full[j & 1], (j >> 1) & 1, a.err, DGDEV_TIMEOUT_MMA)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sKV + (j & 1) * 65536);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ad = sdesc_sw128(q_addr + (kk >> 2) * 16384) + 2 * (kk & 3);
            const uint64_t bd = sdesc_sw128(k_addr + (kk >> 2) * 16384) + 2 * (kk & 3);
            tc_mma_bf16(tS, ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
          tc_commit(&s_full);
        }
      }
    }
    __syncwarp();
  } else {
    // ---------------- softmax warps 0-3: thread = query row ----------------
    const int r = threadIdx.x;                      // TMEM lane / Q row
    const int tok = tok0 + r / a.G;
    const int head = g * a.G + r % a.G;
    const int qpos = a.q_pos0 + tok;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    // tcgen05.ld/st are warp-collective: every branch around them is kept
    // uniform across the warp (wait outcomes are agreed with __all_sync).
    for (int j = 0; j < nblk && ok; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full, j & 1, a.err, DGDEV_TIMEOUT_EPI))) { ok = false; break; }
      tc_fence_after();
      const int key0 = (kb_begin + j) * 128;
      // pass 1: block max (scaled to log2 units)
      float mx = -INFINITY;
      for (int c0 = 0; c0 < 128; c0 += 16) {
        float v[16];
        tmem_ld16(tS + lane_off + c0, v);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int key = key0 + c0 + q;
          const bool vis = key < a.n_keys && (!a.causal || key <= qpos);
          if (vis) mx = fmaxf(mx, v[q] * a.scale_log2);
        }
      }
      const float m_new = fmaxf(m_run, mx);
      // PV of the previous block must be done before P and O are touched
      if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(&o_done, (j - 1) & 1, a.err, DGDEV_TIMEOUT_EPI))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float alpha = (m_run == -INFINITY) ? 0.0f : exp2f(m_run - m_new);
      // pass 2: P = exp2(s - m_new) as bf16 into the swizzled tile
      float lsum = 0.0f;
      for (int c0 = 0; c0 < 128; c0 += 16) {
        float v[16];
        tmem_ld16(tS + lane_off + c0, v);
        uint32_t pk[8];
#pragma unroll
        for (int q = 0; q < 16; q += 2) {
          float p2[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int key = key0 + c0 + q + u;
            const bool vis = key < a.n_keys && (!a.causal || key <= qpos);
            const float pv = (vis && m_new != -INFINITY) ? exp2f(v[q + u] * a.scale_log2 - m_new) : 0.0f;
            const bf16 pb = __float2bfloat16_rn(pv);
            lsum += __bfloat162float(pb);
            p2[u] = __bfloat162float(pb);
          }
          const __nv_bfloat162 pr = __floats2bfloat162_rn(p2[0], p2[1]);
          pk[q / 2] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        // 16 keys = two 16-byte chunks of row r in column block c0/64
        const int cb = c0 >> 6;
        const int ch0 = (c0 & 63) >> 3;
        uint8_t* rowp = sP + cb * 16384 + r * 128;
        *reinterpret_cast<uint4*>(rowp + (((ch0) ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(rowp + (((ch0 + 1) ^ (r & 7)) << 4)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
      // rescale the running output (skipped only when no row of the warp needs it)
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
        for (int c0 = 0; c0 < 128; c0 += 16) {
          float v[16];
          tmem_ld16(tO + lane_off + c0, v);
#pragma unroll
          for (int q = 0; q < 16; ++q) v[q] *= alpha;
          tmem_st16(tO + lane_off + c0, v);
        }
      }
      l_run = l_run * alpha + lsum;
      m_run = m_new;
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full);
    }
    // epilogue: normalised partial O and log2-sum-exp of this split
    if (ok && nblk > 0) ok = __all_sync(0xffffffffu, mbar_wait(&o_done, (nblk - 1) & 1, a.err, DGDEV_TIMEOUT_EPI));
    tc_fence_after();
    // TMEM loads are warp-collective: every lane loads, only valid rows store.
    const bool row_valid = tok < a.n_q;
    const long long row = ((long long)(bc * a.n_q + min(tok, a.n_q - 1))) * a.Hq + head;
    const long long rows_total = (long long)a.n_canvas * a.n_q * a.Hq;
    float* op = a.o_part + ((long long)split * rows_total + row) * 128;
    const bool loaded = ok && nblk > 0;
    const bool have = loaded && l_run > 0.0f;
    const float inv_l = have ? 1.0f / l_run : 0.0f;
    for (int c0 = 0; c0 < 128; c0 += 16) {
      float v[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) v[q] = 0.0f;
      if (loaded) tmem_ld16(tO + lane_off + c0, v);
      if (row_valid) {
#pragma unroll
        for (int q = 0; q < 16; q += 4) {
          const float4 o4 = have ? make_float4(v[q] * inv_l, v[q + 1] * inv_l, v[q + 2] * inv_l,
                                               v[q + 3] * inv_l)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
          *reinterpret_cast<float4*>(op + c0 + q) = o4;
        }
      }
    }
    if (row_valid) a.lse_part[(long long)split * rows_total + row] = have ? m_run + log2f(l_run) : -INFINITY;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------------------
// fp32 SIMT attention (the fp32 workload): one warp per (query, head),
// online softmax over the visible keys; same partial-output contract.
// ---------------------------------------------------------------------------
__global__ void k_attn_f32(const float* __restrict__ Q, const float* __restrict__ Kc,
                           const float* __restrict__ Vt, int S, int hd, AttnArgs a) {
  pdl_enter();
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int rows = a.n_canvas * a.n_q * a.Hq;
  if (gw >= rows) return;
  const int head = gw % a.Hq, tq = gw / a.Hq;
  const int bc = tq / a.n_q, tok = tq % a.n_q;
  const int g = head / a.G;
  const int lbh = a.lbh0 + bc * a.Hkv + g;
  const int qpos = a.q_pos0 + tok;
  const int per = hd / 32;   // hd <= 128
  float q[4], acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int u = 0; u < per; ++u) q[u] = Q[(long long)gw * hd + lane + 32 * u];
  float m = -INFINITY, l = 0.0f;
  const float scale = a.scale_log2;
  const int nk = a.causal ? min(a.n_keys, qpos + 1) : a.n_keys;
  for (int j = 0; j < nk; ++j) {
    const float* kr = Kc + ((long long)lbh * S + j) * hd;
    float s = 0.0f;
    for (int u = 0; u < per; ++u) s = fmaf(q[u], kr[lane + 32 * u], s);
    s = warp_sum(s) * scale;
    const float mn = fmaxf(m, s);
    const float al = exp2f(m - mn), p = exp2f(s - mn);
    l = l * al + p;
    for (int u = 0; u < per; ++u)
      acc[u] = acc[u] * al + p * Vt[((long long)lbh * hd + lane + 32 * u) * S + j];
    m = mn;
  }
  float* op = a.o_part + (long long)gw * hd;
  for (int u = 0; u < per; ++u) op[lane + 32 * u] = acc[u] / l;
  if (lane == 0) a.lse_part[gw] = m + log2f(l);
}

// Merge split partials: o = sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M),
// splits in index order.  One warp per (token, head) row; hd % 32 == 0.
template <typename T>
__global__ void k_attn_combine(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                               int n_splits, long long rows, int hd, T* __restrict__ out) {
  pdl_enter();
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float M = -INFINITY;
  for (int s = 0; s < n_splits; ++s) M = fmaxf(M, lse_part[s * rows + row]);
  float den = 0.0f;
  for (int s = 0; s < n_splits; ++s) {
    const float l = lse_part[s * rows + row];
    den += (l == -INFINITY) ? 0.0f : exp2f(l - M);
  }
  const float inv = den > 0.0f ? 1.0f / den : 0.0f;
  for (int c0 = lane * 4; c0 < hd; c0 += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < n_splits; ++s) {
      const float l = lse_part[s * rows + row];
      if (l == -INFINITY) continue;
      const float wgt = exp2f(l - M);
      const float4 o = *reinterpret_cast<const float4*>(o_part + (s * rows + row) * hd + c0);
      acc.x += wgt * o.x; acc.y += wgt * o.y; acc.z += wgt * o.z; acc.w += wgt * o.w;
    }
    T* dst = out + row * hd + c0;
    dst[0] = from_f<T>(acc.x * inv);
    dst[1] = from_f<T>(acc.y * inv);
    dst[2] = from_f<T>(acc.z * inv);
    dst[3] = from_f<T>(acc.w * inv);
  }
}
