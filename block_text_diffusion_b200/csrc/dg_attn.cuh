// Attention of canvas queries over [prompt KV ; canvas KV] (bidirectional,
// no mask) and of prompt queries over the prompt (causal, for the encode).
//
// KV cache layout (owned by the library, inside the caller's buffer):
//   K  [L][B][Hkv][S][hd]   keys, one row per position
//   Vt [L][B][Hkv][hd][S]   values transposed, so both tensor-core operands
//                           (K for S = Q K^T, V^T for O = P V) are K-major
// S = slot stride >= P + 256, positions 0..P-1 prompt, P..P+255 canvas.
//
// tcgen05 kernel: S = Q K^T and O live in TMEM, P is written as bf16 into
// shared memory in the 128B-swizzled K-major layout the MMA reads.  The key
// range is split over CTAs.  With at most kAttnMaxCluster splits the split
// CTAs of a query-tile pair form one thread-block cluster and merge their
// results through distributed shared memory, writing the bf16 attention
// output directly; with more, each split writes its normalised partial O and
// log2-sum-exp and a combine kernel merges the splits.  Either way the merge
// runs in split order.
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
  int blocks_per_split; // KV blocks of 64 keys per split
  int lbh0;             // (layer * B + b0) * Hkv: outer index of canvas b0's head 0
  int n_canvas;         // canvases in this launch
  float scale_log2;     // log2(e) / sqrt(hd)
  int cluster;          // 1: the n_splits CTAs of a pair are one cluster and merge in the kernel
  bf16* o_out;          // cluster merge: attention output [n_canvas * n_q][Hq][hd] (bf16)
  float* o_part;        // otherwise: [n_splits][n_canvas * n_q * Hq][hd] fp32
  float* lse_part;      // otherwise: [n_splits][n_canvas * n_q * Hq]
  int* err;
};

// One CTA = two query tiles (A and B, 128 rows each: 128/G tokens x the G
// query heads of one KV head) x one split of the key range, so every K/V
// block fetched serves 256 query rows.  320 threads:
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B (thread = query
//              row = TMEM lane; warp w reaches lanes 32 (w % 4) ..);
//   warp 8     TMA: Q of both tiles once, then K / V^T blocks of 64 keys
//              through a 3-stage ring;
//   warp 9     MMA issuer.
// TMEM (512 columns): S_A0 [0,64), S_A1 [64,128), S_B0 [128,192), S_B1
// [192,256), O_A [256,384), O_B [384,512).  S is double-buffered: the issuer
// computes S_t(j+2) as soon as tile t's softmax has read S_t(j) and handed
// P_t(j), so a softmax group never waits for a QK^T after handing its P --
// only the short PV of the previous block stands between two blocks.
constexpr int kAttnThreads = 320;
constexpr int kAttnBK = 64;                                   // keys per block
constexpr int kAttnStages = 3;
constexpr int kAttnQBytes = 32768;                            // one Q tile
constexpr int kAttnKVBytes = 2 * 8192 + 16384;                // K (2 chunks) + V^T of one block
constexpr int kAttnPBytes = 16384;                            // one P tile
constexpr int kAttnSmem = 2 * kAttnQBytes + kAttnStages * kAttnKVBytes + 2 * kAttnPBytes + 1024;
constexpr int kAttnMaxCluster = 8;                            // portable cluster size
static_assert(256 * 128 * 4 <= kAttnSmem - 1024, "the merge staging reuses the pipeline buffers");

// Grid of the tensor-core attention: q_tiles tiles of 128 query rows, paired
// per CTA; the key range is split so that pairs x splits fill the SMs about
// once (one CTA per SM), capped by the partial-output rows available.  The
// in-kernel cluster merge (at most kAttnMaxCluster splits, no partial
// outputs in global memory, no combine launch) is taken when its clusters
// all fit on the GPU at once (max_clusters[c] = clusters of c CTAs that can
// be resident together; null: SMs / c) and its estimated time -- key blocks
// per split plus the merge -- beats the wider split with the global partials
// and the combine kernel.
struct AttnPlan {
  int q_tiles, n_splits, blocks_per_split, ctas, cluster;
};
inline AttnPlan attn_plan(long long n_q, int G, int Hkv, int n_canvas, int n_keys, long long rows,
                          long long part_rows_cap, const int* max_clusters = nullptr) {
  AttnPlan p;
  p.q_tiles = (int)((n_q * G + 127) / 128);
  const int nblocks = (n_keys + kAttnBK - 1) / kAttnBK;
  const int base = (p.q_tiles + 1) / 2 * Hkv * n_canvas;
  const int wide = std::max(1, std::min(nblocks, kSMs / std::max(1, base)));
  // microseconds: ~0.8 per key block, ~1.5 for the cluster merge, ~7.5 for
  // the partial outputs plus the combine kernel
  auto blocks_of = [&](int splits) { return (nblocks + splits - 1) / splits; };
  double best = 0.8 * blocks_of(wide) + 7.5;
  int splits = wide;
  p.cluster = 0;
  for (int c = std::min(wide, kAttnMaxCluster); c >= 1; --c) {
    const int n = (nblocks + blocks_of(c) - 1) / blocks_of(c);   // splits actually used
    const int fit = max_clusters ? max_clusters[n] : kSMs / n;
    if (base > fit) continue;
    const double t = 0.8 * blocks_of(c) + 1.5;
    if (t < best) { best = t; splits = c; p.cluster = 1; }
  }
  if (!p.cluster)
    while (splits > 1 && (long long)splits * rows > part_rows_cap) --splits;
  p.blocks_per_split = (nblocks + splits - 1) / splits;
  p.n_splits = (nblocks + p.blocks_per_split - 1) / p.blocks_per_split;
  p.ctas = base * p.n_splits;
  return p;
}

__global__ void __launch_bounds__(kAttnThreads, 1)
k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
          const __grid_constant__ CUtensorMap tmV, AttnArgs a) {
  pdl_launch();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;                                   // tile t at t * 32 KB
  uint8_t* sKV = smem + 2 * kAttnQBytes;                // stage s: K chunk 0, K chunk 1, V^T
  uint8_t* sP = sKV + kAttnStages * kAttnKVBytes;       // tile t at t * 16 KB
  __shared__ __align__(8) uint64_t q_full, kv_full[kAttnStages], kv_empty[kAttnStages];
  __shared__ __align__(8) uint64_t s_full[2][2], p_full[2], o_done[2];
  __shared__ uint32_t tmem_base;
  __shared__ float s_lse[256];                          // cluster merge: log2-sum-exp per row

  int bid = blockIdx.x;
  const int split = bid % a.n_splits; bid /= a.n_splits;
  const int n_pairs = (a.q_tiles + 1) / 2;
  const int qp = bid % n_pairs; bid /= n_pairs;
  const int g = bid % a.Hkv;
  const int bc = bid / a.Hkv;                   // canvas within the launch
  const int tok_per_tile = 128 / a.G;
  const int tok0 = 2 * qp * tok_per_tile;       // first token of tile A (tile B follows)
  const int lbh = a.lbh0 + bc * a.Hkv + g;

  // key blocks of this split (causal: only blocks reaching the pair's last query)
  const int n_blocks_all = (a.n_keys + kAttnBK - 1) / kAttnBK;
  const int kb_begin = split * a.blocks_per_split;
  int kb_end = min(n_blocks_all, kb_begin + a.blocks_per_split);
  if (a.causal) {
    const int last_pos = a.q_pos0 + min(a.n_q, tok0 + 2 * tok_per_tile) - 1;
    kb_end = min(kb_end, last_pos / kAttnBK + 1);
  }
  const int nblk = max(0, kb_end - kb_begin);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < kAttnStages; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t][0], 1); mbar_init(&s_full[t][1], 1);
      mbar_init(&p_full[t], 128); mbar_init(&o_done[t], 1);
    }
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&tmem_base, 512);
  pdl_wait();   // q and the cache are written by the previous kernels
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp == 8) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && nblk > 0) {
      mbar_expect_tx(&q_full, 2 * kAttnQBytes);
      for (int t = 0; t < 2; ++t) {
        const int zq = bc * a.n_q + tok0 + t * tok_per_tile;
        tma_load_3d(sQ + t * kAttnQBytes, &tmQ, 0, g * a.G, zq, &q_full);
        tma_load_3d(sQ + t * kAttnQBytes + 16384, &tmQ, 64, g * a.G, zq, &q_full);
      }
      for (int j = 0; j < nblk; ++j) {
        const int s = j % kAttnStages;
        if (j >= kAttnStages &&
            !mbar_wait(&kv_empty[s], ((j / kAttnStages) & 1) ^ 1, a.err, DGDEV_TIMEOUT_TMA))
          break;
        uint8_t* kv = sKV + s * kAttnKVBytes;
        const int key0 = (kb_begin + j) * kAttnBK;
        mbar_expect_tx(&kv_full[s], kAttnKVBytes);
        tma_load_3d(kv, &tmK, 0, key0, lbh, &kv_full[s]);
        tma_load_3d(kv + 8192, &tmK, 64, key0, lbh, &kv_full[s]);
        tma_load_3d(kv + 16384, &tmV, key0, 0, lbh, &kv_full[s]);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && nblk > 0) {
      bool ok = mbar_wait(&q_full, 0, a.err, DGDEV_TIMEOUT_MMA);
      const uint32_t idesc_s = idesc_bf16(128, kAttnBK), idesc_o = idesc_bf16(128, 128);
      // S_t(j) = Q_t K(j)^T into buffer j & 1 of tile t
      auto issue_s = [&](int j) {
        const uint32_t k_addr = smem_u32(sKV + (j % kAttnStages) * kAttnKVBytes);
        for (int t = 0; t < 2; ++t) {
          const uint32_t q_addr = smem_u32(sQ + t * kAttnQBytes);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc_mma_bf16(tmem + (2 * t + (j & 1)) * kAttnBK, sdesc_sw128(q_addr + (kk >> 2) * 16384) + 2 * (kk & 3),
                        sdesc_sw128(k_addr + (kk >> 2) * 8192) + 2 * (kk & 3), idesc_s, kk > 0 ? 1u : 0u);
          tc_commit(&s_full[t][j & 1]);
        }
      };
      for (int j = 0; j < 2 && j < nblk && ok; ++j) {
        if (!mbar_wait(&kv_full[j % kAttnStages], (j / kAttnStages) & 1, a.err, DGDEV_TIMEOUT_MMA)) { ok = false; break; }
        tc_fence_after();
        issue_s(j);
      }
      for (int j = 0; j < nblk && ok; ++j) {
        // O_t += P_t(j) V(j), each tile as soon as its softmax handed P_t(j)
        const uint32_t v_addr = smem_u32(sKV + (j % kAttnStages) * kAttnKVBytes + 16384);
        for (int t = 0; t < 2; ++t) {
          if (!mbar_wait(&p_full[t], j & 1, a.err, DGDEV_TIMEOUT_MMA)) { ok = false; break; }
          tc_fence_after();
          const uint32_t p_addr = smem_u32(sP + t * kAttnPBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_bf16(tmem + 256 + t * 128, sdesc_sw128(p_addr) + 2 * kk, sdesc_sw128(v_addr) + 2 * kk, idesc_o,
                        (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&o_done[t]);
        }
        if (!ok) break;
        tc_commit(&kv_empty[j % kAttnStages]);
        // both tiles have read S(j): its buffers take S(j + 2)
        if (j + 2 < nblk) {
          if (!mbar_wait(&kv_full[(j + 2) % kAttnStages], ((j + 2) / kAttnStages) & 1, a.err, DGDEV_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s(j + 2);
        }
      }
    }
    __syncwarp();
  } else {
    // ---------------- softmax: warps 0-3 tile A, 4-7 tile B ----------------
    const int t = warp >> 2;
    const int r = threadIdx.x & 127;                // TMEM lane / Q row of the tile
    const int tok = tok0 + t * tok_per_tile + r / a.G;
    const int head = g * a.G + r % a.G;
    const int qpos = a.q_pos0 + tok;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + 256 + t * 128 + lane_off;
    uint8_t* rowp = sP + t * kAttnPBytes + r * 128;
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    // tcgen05.ld/st are warp-collective: every branch around them is kept
    // uniform across the warp (wait outcomes are agreed with __all_sync).
    for (int j = 0; j < nblk && ok; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[t][j & 1], (j >> 1) & 1, a.err, DGDEV_TIMEOUT_EPI))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tmem + (2 * t + (j & 1)) * kAttnBK + lane_off;
      const int key0 = (kb_begin + j) * kAttnBK;
      float v[kAttnBK];
      {
        uint32_t w[kAttnBK / 16][16];
#pragma unroll
        for (int q = 0; q < kAttnBK / 16; ++q) tmem_ld16_nw(tS + q * 16, w[q]);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < kAttnBK / 16; ++q)
#pragma unroll
          for (int u = 0; u < 16; ++u) v[q * 16 + u] = __uint_as_float(w[q][u]);
      }
      // keys past the end (or after the query, causal) get -inf; the max is
      // taken on raw scores (scale_log2 > 0) and scaled once
      if (a.causal || key0 + kAttnBK > a.n_keys) {
#pragma unroll
        for (int c = 0; c < kAttnBK; ++c) {
          const int key = key0 + c;
          const bool vis = key < a.n_keys && (!a.causal || key <= qpos);
          if (!vis) v[c] = -INFINITY;
        }
      }
      float mt[kAttnBK / 2];
#pragma unroll
      for (int c = 0; c < kAttnBK / 2; ++c) mt[c] = fmaxf(v[2 * c], v[2 * c + 1]);
#pragma unroll
      for (int w2 = kAttnBK / 4; w2 >= 1; w2 >>= 1)
#pragma unroll
        for (int c = 0; c < w2; ++c) mt[c] = fmaxf(mt[c], mt[c + w2]);
      const float mx = mt[0] * a.scale_log2;
      // The running reference max moves only when the block max exceeds it by
      // more than 8 (a factor 256 in P), so O is rarely rescaled; the final
      // normalisation uses the same reference, so the result is unchanged.
      const float m_new = (m_run == -INFINITY || mx > m_run + 8.0f) ? mx : m_run;
      const float alpha = (m_run == -INFINITY) ? 0.0f : ex2_approx(m_run - m_new);
      // p = 2^(s * scale - m) with one FFMA and one MUFU.EX2 (exp2(-inf) = 0);
      // the row sum adds the fp32 values.  The exponentials are computed
      // before waiting for the previous block's PV (which reads P_t).
      const float nm = m_new == -INFINITY ? 0.0f : -m_new;
      uint32_t pk[kAttnBK / 2];
      float ls[kAttnBK / 8];
#pragma unroll
      for (int ch = 0; ch < kAttnBK / 8; ++ch) {
        float acc = 0.0f;
#pragma unroll
        for (int q = 0; q < 8; q += 2) {
          const float p0 = ex2_approx(fmaf(v[ch * 8 + q], a.scale_log2, nm));
          const float p1 = ex2_approx(fmaf(v[ch * 8 + q + 1], a.scale_log2, nm));
          acc += p0 + p1;
          const __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
          pk[ch * 4 + q / 2] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        ls[ch] = acc;
      }
#pragma unroll
      for (int w2 = kAttnBK / 16; w2 >= 1; w2 >>= 1)
#pragma unroll
        for (int c = 0; c < w2; ++c) ls[c] += ls[c + w2];
      const float lsum = ls[0];
      // PV of the previous block must be done before P_t and O_t are touched
      if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(&o_done[t], (j - 1) & 1, a.err, DGDEV_TIMEOUT_EPI))) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < kAttnBK / 8; ++ch)
        *reinterpret_cast<uint4*>(rowp + ((ch ^ (r & 7)) << 4)) =
            make_uint4(pk[ch * 4], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
      // rescale the running output (skipped only when no row of the warp needs it)
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t o[4][16];
#pragma unroll
          for (int q = 0; q < 4; ++q) tmem_ld16_nw(tO + half * 64 + q * 16, o[q]);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int u = 0; u < 16; ++u) o[q][u] = __float_as_uint(__uint_as_float(o[q][u]) * alpha);
#pragma unroll
          for (int q = 0; q < 4; ++q) tmem_st16_nw(tO + half * 64 + q * 16, o[q]);
          tmem_wait_st();
        }
      }
      l_run = l_run * alpha + lsum;
      m_run = m_new;
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }
    // epilogue: normalised O and log2-sum-exp of this split
    if (ok && nblk > 0) ok = __all_sync(0xffffffffu, mbar_wait(&o_done[t], (nblk - 1) & 1, a.err, DGDEV_TIMEOUT_EPI));
    tc_fence_after();
    // TMEM loads are warp-collective: every lane loads, only valid rows store.
    const bool row_valid = tok < a.n_q;
    const long long row = ((long long)(bc * a.n_q + min(tok, a.n_q - 1))) * a.Hq + head;
    const long long rows_total = (long long)a.n_canvas * a.n_q * a.Hq;
    const bool loaded = ok && nblk > 0;
    const bool have = loaded && l_run > 0.0f;
    const float inv_l = have ? 1.0f / l_run : 0.0f;
    const float lse = have ? m_run + log2f(l_run) : -INFINITY;
    const int wt = warp & 3;   // warp within the tile's group
    if (a.cluster) {
      // both tiles' MMAs are complete: every pipeline buffer is free.  Row
      // R = 128 t + r of the pair goes to the staging area [256][32 float4],
      // float4 c at position c ^ (R & 31) (conflict-free both ways).
      asm volatile("bar.sync 1, 256;" ::: "memory");
      float4* stage = reinterpret_cast<float4*>(smem);
      const int R = t * 128 + r;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t o[4][16];
        if (loaded) {
#pragma unroll
          for (int q = 0; q < 4; ++q) tmem_ld16_nw(tO + half * 64 + q * 16, o[q]);
          tmem_wait_ld();
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int u = 0; u < 16; u += 4) {
            const int c = (half * 64 + q * 16 + u) >> 2;
            stage[R * 32 + (c ^ (R & 31))] =
                have ? make_float4(__uint_as_float(o[q][u]) * inv_l, __uint_as_float(o[q][u + 1]) * inv_l,
                                   __uint_as_float(o[q][u + 2]) * inv_l, __uint_as_float(o[q][u + 3]) * inv_l)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
          }
      }
      s_lse[R] = lse;
    } else {
      // Staged through this tile's Q buffer (free after its last QK^T): each
      // thread writes its row's 64 columns of a half into shared memory, then
      // the tile's four warps copy whole 256-byte row segments with coalesced
      // 16-byte stores (two rows per warp instruction).
      // [128 rows][16 float4], float4 index XOR (row & 15): conflict-free both ways
      float4* stage = reinterpret_cast<float4*>(sQ + t * kAttnQBytes);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t o[4][16];
        if (loaded) {
#pragma unroll
          for (int q = 0; q < 4; ++q) tmem_ld16_nw(tO + half * 64 + q * 16, o[q]);
          tmem_wait_ld();
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int u = 0; u < 16; u += 4) {
            const float4 o4 = have ? make_float4(__uint_as_float(o[q][u]) * inv_l, __uint_as_float(o[q][u + 1]) * inv_l,
                                                 __uint_as_float(o[q][u + 2]) * inv_l,
                                                 __uint_as_float(o[q][u + 3]) * inv_l)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
            stage[r * 16 + (((q * 16 + u) >> 2) ^ (r & 15))] = o4;
          }
        asm volatile("bar.sync %0, 128;" ::"r"(2 + t) : "memory");
        // rows 2i, 2i+1 of the tile per warp instruction; lane l copies float4 l % 16
        for (int rr = wt * 2; rr < 128; rr += 8) {
          const int rl = rr + (lane >> 4);
          const int tok_r = tok0 + t * tok_per_tile + rl / a.G;
          if (tok_r < a.n_q) {
            const long long grow = ((long long)(bc * a.n_q + tok_r)) * a.Hq + g * a.G + rl % a.G;
            float* dst = a.o_part + ((long long)split * rows_total + grow) * 128 + half * 64;
            *reinterpret_cast<float4*>(dst + (lane & 15) * 4) = stage[rl * 16 + ((lane & 15) ^ (rl & 15))];
          }
        }
        asm volatile("bar.sync %0, 128;" ::"r"(2 + t) : "memory");
      }
      if (row_valid) a.lse_part[(long long)split * rows_total + row] = lse;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (a.cluster) {
    // every split of the pair has staged its rows: CTA `split` merges rows
    // [r0, r1) of the pair over all splits, in split order, and writes them
    // as bf16.  Remote reads are batched: first every split's log2-sum-exp of
    // those rows (one load per thread), then per row all splits' float4 of a
    // lane at once.
    if (a.n_splits > 1) cluster_sync_all();
    const int ns = a.n_splits;
    const int per = (256 + ns - 1) / ns;
    const int r0 = split * per, r1 = min(256, r0 + per);
    const int nrows = max(0, r1 - r0);
    float* s_w = reinterpret_cast<float*>(sP);          // [nrows][ns] merge weights (P buffers are free)
    float* s_inv = s_w + 256 + kAttnMaxCluster;         // [nrows] 1 / sum of weights
    for (int i = threadIdx.x; i < nrows * ns; i += kAttnThreads) {
      const int q = i % ns;
      const float* src = &s_lse[r0 + i / ns];
      s_w[i] = ns > 1 ? *cluster_peer(src, q) : *src;
    }
    __syncthreads();
    for (int rr = threadIdx.x; rr < nrows; rr += kAttnThreads) {
      float M = -INFINITY;
      for (int q = 0; q < ns; ++q) M = fmaxf(M, s_w[rr * ns + q]);
      float den = 0.0f;
      for (int q = 0; q < ns; ++q) {
        const float l = s_w[rr * ns + q];
        const float w = (l == -INFINITY) ? 0.0f : exp2f(l - M);
        s_w[rr * ns + q] = w;
        den += w;
      }
      s_inv[rr] = den > 0.0f ? 1.0f / den : 0.0f;
    }
    __syncthreads();
    const float4* stage = reinterpret_cast<const float4*>(smem);
    for (int rr = warp; rr < nrows; rr += kAttnThreads / 32) {
      const int R = r0 + rr;
      const int tt = R >> 7, rl = R & 127;
      const int tok_r = tok0 + tt * tok_per_tile + rl / a.G;
      if (tok_r >= a.n_q) continue;
      const float4* src = &stage[R * 32 + (lane ^ (R & 31))];
      float4 o[kAttnMaxCluster];
#pragma unroll
      for (int q = 0; q < kAttnMaxCluster; ++q)
        if (q < ns) o[q] = ns > 1 ? *cluster_peer(src, q) : *src;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < kAttnMaxCluster; ++q)
        if (q < ns) {
          const float w = s_w[rr * ns + q];
          acc.x += w * o[q].x; acc.y += w * o[q].y; acc.z += w * o[q].z; acc.w += w * o[q].w;
        }
      const float inv = s_inv[rr];
      const long long grow = ((long long)(bc * a.n_q + tok_r)) * a.Hq + g * a.G + rl % a.G;
      store4<bf16>(a.o_out + grow * 128 + lane * 4, acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
    // peers read this CTA's staging: keep it until every CTA is done
    if (a.n_splits > 1) cluster_sync_all();
  }
  if (warp == 0) tmem_dealloc(tmem, 512);
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
    store4<T>(out + row * hd + c0, acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  }
}
