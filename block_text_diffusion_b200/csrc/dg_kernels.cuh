// Memory-bound and integer kernels of the denoising step.
#pragma once
#include "dg_device.cuh"

// Device-resident loop state, read by every kernel that depends on the round.
struct DevState {
  int step;           // current round s
  float t;            // diffusion time of the round (1 -> 0)
  int n_steps;        // round budget N
  int use_selfcond;   // 0 at round 0 (self-conditioning input is zero)
  int active;         // number of canvases not yet stopped
  int cond;           // 1 while the block loop should continue
  int err;            // first device error code
  int pad;
};

// ---------------------------------------------------------------------------
// Weight initialisation: w = round(0.02 * sqrt(-2 ln u1) * cos(2 pi u2)),
// u1/u2 from words 0/1 of Philox(key = seed, ctr = (j lo, j hi, tensor, 3)),
// j the element's row-major index in its logical tensor.  `outer`/`inner`
// place logical element j at physical index (j / inner) * outer + j % inner
// + offset, which packs gate/up experts and the fused QKV matrix.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float init_value(uint64_t j, uint64_t seed, uint32_t tensor_id) {
  const uint4 w = philox4x32_10(make_uint4((uint32_t)j, (uint32_t)(j >> 32), tensor_id, STREAM_WEIGHTS),
                                (uint32_t)seed, (uint32_t)(seed >> 32));
  const float u1 = uniform_open(w.x), u2 = uniform_open(w.y);
  const float r = __fsqrt_rn(__fmul_rn(dg_logf(u1), -2.0f));
  const float z = __fmul_rn(r, dg_cos2pif(u2));
  return __fmul_rn(DG_F(0x3CA3D70Au), z);   // 0.02f
}

template <typename T>
__global__ void k_init_weights(T* __restrict__ out, uint64_t n, uint64_t inner, uint64_t outer,
                               uint64_t offset, uint64_t seed, uint32_t tensor_id) {
  for (uint64_t j = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; j < n;
       j += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t phys = (j / inner) * outer + (j % inner) + offset;
    out[phys] = from_f<T>(init_value(j, seed, tensor_id));
  }
}

// Transposed copy of a logical [rows][cols] tensor: out[c][r] = w(r * cols + c).
template <typename T>
__global__ void k_init_weights_t(T* __restrict__ out, uint64_t rows, uint64_t cols, uint64_t seed,
                                 uint32_t tensor_id) {
  const uint64_t n = rows * cols;
  for (uint64_t p = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; p < n;
       p += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t c = p / rows, r = p % rows;
    out[p] = from_f<T>(init_value(r * cols + c, seed, tensor_id));
  }
}

// RoPE table: (cos, sin) of pos * theta^(-2i/hd) in fp64, stored fp32.
__global__ void k_rope_table(float2* __restrict__ tab, int n_pos, int half, int hd, double theta) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_pos * half) return;
  const int pos = i / half, c = i % half;
  const double ang = (double)pos * pow(theta, -2.0 * c / hd);
  double s, co;
  sincos(ang, &s, &co);
  tab[i] = make_float2((float)co, (float)s);
}


// Block-wide sum of one float per thread (blockDim.x a multiple of 32, <= 1024).
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x < 32) {
    float w = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
    w = warp_sum(w);
    if (threadIdx.x == 0) red[0] = w;
  }
  __syncthreads();
  const float s = red[0];
  __syncthreads();
  return s;
}

// Normalise the (already stored) row hr into xr: x = h / sqrt(mean(h^2) + eps).
// Each thread reads back only the elements it wrote itself.
template <typename T>
__device__ __forceinline__ void rownorm_store(const T* hr, T* xr, int d, float eps, float ss, float* red) {
  const float tot = block_sum(ss, red);
  const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(tot, (float)d), eps)));
  for (int i = threadIdx.x; i < d; i += blockDim.x) xr[i] = from_f<T>(to_f(hr[i]) * r);
}

// Same, for rows written in groups of 4 consecutive elements per thread.
template <typename T>
__device__ __forceinline__ void rownorm_store4(const T* hr, T* xr, int d, float eps, float ss, float* red) {
  const float tot = block_sum(ss, red);
  const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(tot, (float)d), eps)));
  for (int i = threadIdx.x * 4; i < d; i += blockDim.x * 4)
#pragma unroll
    for (int q = 0; q < 4; ++q) xr[i + q] = from_f<T>(to_f(hr[i + q]) * r);
}

// Embedding (+ self-conditioning add) fused with the first RMSNorm:
// h[t] = E[ids[t]] (+ s[t]);  x[t] = RMSNorm(h[t]).
template <typename T>
__global__ void k_embed_norm(const int* __restrict__ ids, const T* __restrict__ E, const T* __restrict__ sc,
                             const int* __restrict__ use_sc, T* __restrict__ h, T* __restrict__ x, int d,
                             int vocab, float eps, int* err) {
  pdl_enter();
  __shared__ float red[32];
  const long long t = blockIdx.x;
  int id = ids[t];
  if (id < 0 || id >= vocab) { dev_error(err, DGDEV_BAD_INDEX); id = 0; }
  const bool add = sc != nullptr && (use_sc == nullptr || *use_sc != 0);
  const T* e = E + (long long)id * d;
  T* hr = h + t * d;
  float ss = 0.0f;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    float v = to_f(e[i]);
    if (add) v = __fadd_rn(v, to_f(sc[t * d + i]));
    const T hv = from_f<T>(v);
    hr[i] = hv;
    const float f = to_f(hv);
    ss = fmaf(f, f, ss);
  }
  rownorm_store<T>(hr, x + t * d, d, eps, ss, red);
}

// A given residual state as a layer's input: h[t] = h_in[t];  x[t] = RMSNorm(h[t]).
template <typename T>
__global__ void k_load_norm(const T* __restrict__ h_in, T* __restrict__ h, T* __restrict__ x, int d, float eps) {
  pdl_enter();
  __shared__ float red[32];
  const long long t = blockIdx.x;
  T* hr = h + t * d;
  float ss = 0.0f;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    const T hv = h_in[t * d + i];
    hr[i] = hv;
    const float f = to_f(hv);
    ss = fmaf(f, f, ss);
  }
  rownorm_store<T>(hr, x + t * d, d, eps, ss, red);
}

// Attention residual fused with the MoE RMSNorm:
// h = round(h + sum_s ws[s]);  x = RMSNorm(h).  One CTA per row.  Rows of up
// to 16 values per thread stay in registers, with every load issued before
// the first use; longer rows take the strided loop.
template <typename T>
__global__ void k_residual_norm(T* __restrict__ h, T* __restrict__ x, const float* __restrict__ ws,
                                long long split_stride, int splits, int d, float eps) {
  pdl_enter();
  __shared__ float red[32];
  const long long t = blockIdx.x;
  T* hr = h + t * d;
  const float* w = ws + t * d;
  constexpr int G = 4;
  if (d <= G * 4 * (int)blockDim.x) {
    float4 v[G], hv[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int i = (threadIdx.x + g * blockDim.x) * 4;
      if (i < d) { v[g] = *reinterpret_cast<const float4*>(w + i); hv[g] = load4<T>(hr + i); }
    }
    for (int s = 1; s < splits; ++s) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const int i = (threadIdx.x + g * blockDim.x) * 4;
        if (i < d) {
          const float4 u = *reinterpret_cast<const float4*>(w + s * split_stride + i);
          v[g].x += u.x; v[g].y += u.y; v[g].z += u.z; v[g].w += u.w;
        }
      }
    }
    float ss = 0.0f;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int i = (threadIdx.x + g * blockDim.x) * 4;
      if (i < d) {
        hv[g] = make_float4(to_f(from_f<T>(hv[g].x + v[g].x)), to_f(from_f<T>(hv[g].y + v[g].y)),
                            to_f(from_f<T>(hv[g].z + v[g].z)), to_f(from_f<T>(hv[g].w + v[g].w)));
        store4<T>(hr + i, hv[g].x, hv[g].y, hv[g].z, hv[g].w);
        ss = fmaf(hv[g].x, hv[g].x, ss);
        ss = fmaf(hv[g].y, hv[g].y, ss);
        ss = fmaf(hv[g].z, hv[g].z, ss);
        ss = fmaf(hv[g].w, hv[g].w, ss);
      }
    }
    const float tot = block_sum(ss, red);
    const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(tot, (float)d), eps)));
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int i = (threadIdx.x + g * blockDim.x) * 4;
      if (i < d) store4<T>(x + t * d + i, hv[g].x * r, hv[g].y * r, hv[g].z * r, hv[g].w * r);
    }
    return;
  }
  float ss = 0.0f;
  for (int i = threadIdx.x * 4; i < d; i += blockDim.x * 4) {
    float4 v = *reinterpret_cast<const float4*>(w + i);
    for (int s = 1; s < splits; ++s) {
      const float4 v2 = *reinterpret_cast<const float4*>(w + s * split_stride + i);
      v.x += v2.x; v.y += v2.y; v.z += v2.z; v.w += v2.w;
    }
    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const T hv = from_f<T>(to_f(hr[i + q]) + vv[q]);
      hr[i + q] = hv;
      const float f = to_f(hv);
      ss = fmaf(f, f, ss);
    }
  }
  rownorm_store4<T>(hr, x + t * d, d, eps, ss, red);
}

// MoE combine fused with the next RMSNorm (next layer's attention norm, or the
// final norm after the last layer -- all norms have unit gain):
// h[t] = round(h[t] + sum_slot gate[t][slot] * y[inv[t*k+slot]]) (slots in
// order);  x[t] = RMSNorm(h[t]).
// y holds `splits` partial slabs (split_stride apart; count read from the
// device) that are summed before weighting.  Vectorised by 4 (d % 64 == 0).
// Rows of up to kCombineG float4 per thread with up to kCombineK slots keep
// every value in registers, with all loads of the row issued before the
// first use (one round trip instead of one per chunk, and no re-read of h
// for the norm); the arithmetic and its order are those of the general loop.
constexpr int kCombineK = 8, kCombineG = 3;
template <typename T>
__global__ void __launch_bounds__(256, 2) k_moe_combine_norm(T* __restrict__ h, T* __restrict__ x, const float* __restrict__ y,
                                   const int* __restrict__ inv, const float* __restrict__ gate, int k, int d,
                                   float eps, const int* __restrict__ splits_dev, long long split_stride) {
  pdl_enter();
  __shared__ float red[32];
  __shared__ long long rows[64];
  __shared__ float gw[64];
  const long long t = blockIdx.x;
  const int ns = splits_dev ? *splits_dev : 1;
  if (threadIdx.x < k) {
    rows[threadIdx.x] = (long long)inv[t * k + threadIdx.x] * d;
    gw[threadIdx.x] = gate[t * k + threadIdx.x];
  }
  __syncthreads();
  T* hr = h + t * d;
  if (k <= kCombineK && d <= kCombineG * 4 * (int)blockDim.x) {
    // slots in two groups of kCombineK / 2: every load of a group is issued
    // before its first use, and the weighted sums run in slot order
    constexpr int kHalf = kCombineK / 2;
    float4 hv[kCombineG];
    float acc[kCombineG][4];
#pragma unroll
    for (int g = 0; g < kCombineG; ++g) {
      const int i = (threadIdx.x + g * blockDim.x) * 4;
      hv[g] = i < d ? load4<T>(hr + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      acc[g][0] = acc[g][1] = acc[g][2] = acc[g][3] = 0.0f;
    }
#pragma unroll
    for (int j0 = 0; j0 < kCombineK; j0 += kHalf) {
      if (j0 >= k) break;
      float4 v[kCombineG][kHalf];
#pragma unroll
      for (int g = 0; g < kCombineG; ++g) {
        const int i = (threadIdx.x + g * blockDim.x) * 4;
        if (i < d) {
#pragma unroll
          for (int jj = 0; jj < kHalf; ++jj)
            if (j0 + jj < k) v[g][jj] = *reinterpret_cast<const float4*>(y + rows[j0 + jj] + i);
        }
      }
      for (int s = 1; s < ns; ++s) {
#pragma unroll
        for (int g = 0; g < kCombineG; ++g) {
          const int i = (threadIdx.x + g * blockDim.x) * 4;
          if (i < d) {
#pragma unroll
            for (int jj = 0; jj < kHalf; ++jj)
              if (j0 + jj < k) {
                const float4 v2 = *reinterpret_cast<const float4*>(y + rows[j0 + jj] + i + s * split_stride);
                v[g][jj].x += v2.x; v[g][jj].y += v2.y; v[g][jj].z += v2.z; v[g][jj].w += v2.w;
              }
          }
        }
      }
#pragma unroll
      for (int g = 0; g < kCombineG; ++g)
#pragma unroll
        for (int jj = 0; jj < kHalf; ++jj)
          if (j0 + jj < k) {
            const float gj = gw[j0 + jj];
            acc[g][0] = fmaf(gj, v[g][jj].x, acc[g][0]);
            acc[g][1] = fmaf(gj, v[g][jj].y, acc[g][1]);
            acc[g][2] = fmaf(gj, v[g][jj].z, acc[g][2]);
            acc[g][3] = fmaf(gj, v[g][jj].w, acc[g][3]);
          }
    }
    float ss = 0.0f;
#pragma unroll
    for (int g = 0; g < kCombineG; ++g) {
      const int i = (threadIdx.x + g * blockDim.x) * 4;
      if (i < d) {
        hv[g] = make_float4(to_f(from_f<T>(hv[g].x + acc[g][0])), to_f(from_f<T>(hv[g].y + acc[g][1])),
                            to_f(from_f<T>(hv[g].z + acc[g][2])), to_f(from_f<T>(hv[g].w + acc[g][3])));
        store4<T>(hr + i, hv[g].x, hv[g].y, hv[g].z, hv[g].w);
        ss = fmaf(hv[g].x, hv[g].x, ss);
        ss = fmaf(hv[g].y, hv[g].y, ss);
        ss = fmaf(hv[g].z, hv[g].z, ss);
        ss = fmaf(hv[g].w, hv[g].w, ss);
      }
    }
    const float tot = block_sum(ss, red);
    const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(tot, (float)d), eps)));
#pragma unroll
    for (int g = 0; g < kCombineG; ++g) {
      const int i = (threadIdx.x + g * blockDim.x) * 4;
      if (i < d) store4<T>(x + t * d + i, hv[g].x * r, hv[g].y * r, hv[g].z * r, hv[g].w * r);
    }
    return;
  }
  float ss = 0.0f;
  for (int i = threadIdx.x * 4; i < d; i += blockDim.x * 4) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j0 = 0; j0 < k; j0 += 8) {
      // issue the loads of up to 8 slots before accumulating them in order
      float4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j0 + j < k) v[j] = *reinterpret_cast<const float4*>(y + rows[j0 + j] + i);
      for (int s = 1; s < ns; ++s) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j0 + j < k) {
            const float4 v2 = *reinterpret_cast<const float4*>(y + rows[j0 + j] + i + s * split_stride);
            v[j].x += v2.x; v[j].y += v2.y; v[j].z += v2.z; v[j].w += v2.w;
          }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j0 + j < k) {
          const float g = gw[j0 + j];
          acc[0] = fmaf(g, v[j].x, acc[0]);
          acc[1] = fmaf(g, v[j].y, acc[1]);
          acc[2] = fmaf(g, v[j].z, acc[2]);
          acc[3] = fmaf(g, v[j].w, acc[3]);
        }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const T hv = from_f<T>(to_f(hr[i + q]) + acc[q]);
      hr[i + q] = hv;
      const float f = to_f(hv);
      ss = fmaf(f, f, ss);
    }
  }
  rownorm_store4<T>(hr, x + t * d, d, eps, ss, red);
}

// ---------------------------------------------------------------------------
// After the QKV projection: sum split-K partials, rotate q and k by RoPE at
// their absolute positions, round, and scatter q -> Q[t][Hq][hd],
// k -> K cache [lbh][pos][hd], v -> V^T cache [lbh][hd][pos].
// Token t of the launch is canvas b = t / n_per, local i = t % n_per,
// position pos0 + i.
// ---------------------------------------------------------------------------
struct QkvPostArgs {
  const float* ws;
  long long split_stride;
  int splits;
  int Hq, Hkv, hd;
  int n_per;        // tokens per canvas in this launch
  int pos0;         // position of local token 0
  int b0;           // first canvas index of this launch
  int B;            // canvases in the KV cache
  int layer;
  int S;            // key slot stride of the cache
  const float2* rope;
};

// out = float(in) over n elements (diagnostic copies).
template <typename T>
__global__ void k_cast_f32(const T* __restrict__ in, float* __restrict__ out, long long n) {
  pdl_enter();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    out[i] = to_f(in[i]);
}

// QKV post-processing: sum the split-K partials of the fused QKV GEMM, apply
// rotate-half RoPE to q and k, store q (token-major) and k into the cache,
// and v transposed into V^T.  Flat grid over two ranges:
//   [0, n_qk):  thread = (token, q|k head, 4 rotation pairs c..c+3), float4
//               loads of both halves, 8-byte stores;
//   [n_qk, ..): thread = (v head, 4 channels, token), token fastest so each
//               V^T row segment is written by consecutive lanes.
// Partials are summed in split order.  hd % 8 == 0.
template <typename T>
__global__ void __launch_bounds__(256) k_qkv_post(QkvPostArgs a, int n_tok, T* __restrict__ Q,
                                                  T* __restrict__ Kc, T* __restrict__ Vt) {
  pdl_enter();
  const int hd = a.hd, half = hd / 2, q4 = half / 4;
  const int nq = a.Hq * hd, nk = a.Hkv * hd, ncol = nq + 2 * nk;
  const long long n_qk = (long long)n_tok * (a.Hq + a.Hkv) * q4;
  const long long n_v = (long long)a.Hkv * (hd / 4) * n_tok;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  auto load4 = [&](long long t, int c) {
    const float* w = a.ws + t * ncol + c;
    float4 v = *reinterpret_cast<const float4*>(w);
    for (int s = 1; s < a.splits; ++s) {
      const float4 u = *reinterpret_cast<const float4*>(w + s * a.split_stride);
      v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
    }
    return v;
  };
  if (i < n_qk) {
    const int c = (int)(i % q4) * 4;
    const long long r = i / q4;
    const int head = (int)(r % (a.Hq + a.Hkv));
    const long long t = r / (a.Hq + a.Hkv);
    const int b = a.b0 + (int)(t / a.n_per), pos = a.pos0 + (int)(t % a.n_per);
    const int base = head < a.Hq ? head * hd : nq + (head - a.Hq) * hd;
    const float4 x0 = load4(t, base + c), x1 = load4(t, base + c + half);
    const float4 r01 = *reinterpret_cast<const float4*>(a.rope + (long long)pos * half + c);
    const float4 r23 = *reinterpret_cast<const float4*>(a.rope + (long long)pos * half + c + 2);
    const float lo[4] = {x0.x, x0.y, x0.z, x0.w}, hi[4] = {x1.x, x1.y, x1.z, x1.w};
    const float cs[4] = {r01.x, r01.z, r23.x, r23.z}, sn[4] = {r01.y, r01.w, r23.y, r23.w};
    T* dst;
    if (head < a.Hq) {
      dst = Q + (t * a.Hq + head) * hd;
    } else {
      const long long lbh = ((long long)a.layer * a.B + b) * a.Hkv + (head - a.Hq);
      dst = Kc + (lbh * a.S + pos) * hd;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      dst[c + j] = from_f<T>(lo[j] * cs[j] - hi[j] * sn[j]);
      dst[c + half + j] = from_f<T>(lo[j] * sn[j] + hi[j] * cs[j]);
    }
  } else if (i < n_qk + n_v) {
    const long long iv = i - n_qk;
    const long long t = iv % n_tok;
    const long long r = iv / n_tok;
    const int c = (int)(r % (hd / 4)) * 4;
    const int g = (int)(r / (hd / 4));
    const int b = a.b0 + (int)(t / a.n_per), pos = a.pos0 + (int)(t % a.n_per);
    const float4 v = load4(t, nq + nk + g * hd + c);
    const long long lbh = ((long long)a.layer * a.B + b) * a.Hkv + g;
    T* dst = Vt + (lbh * hd + c) * a.S + pos;
    dst[0] = from_f<T>(v.x);
    dst[a.S] = from_f<T>(v.y);
    dst[2 * (long long)a.S] = from_f<T>(v.z);
    dst[3 * (long long)a.S] = from_f<T>(v.w);
  }
}

// out = round(sum_s ws[s]) over n elements.
template <typename T>
__global__ void k_sum_round(T* __restrict__ out, const float* __restrict__ ws, long long split_stride,
                            int splits, long long n) {
  pdl_enter();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    float v = ws[i];
    for (int s = 1; s < splits; ++s) v += ws[s * split_stride + i];
    out[i] = from_f<T>(v);
  }
}


// ---------------------------------------------------------------------------
// Router top-k on logits produced by the router GEMM: r_e = sum over the
// split-K partials of x . Wr[e] (fp32 accumulation) + b_e; the k largest
// (ties to the lower expert id) in descending order; gate weights = softmax
// over the k selected logits.  One warp per token.
// ---------------------------------------------------------------------------
__global__ void k_router_topk(const float* __restrict__ r, int splits, long long split_stride,
                              const float* __restrict__ bias, const float* __restrict__ tok_bias, int E, int k,
                              int n_tok, int* __restrict__ ids, float* __restrict__ gate) {
  pdl_enter();
  extern __shared__ float rt[];   // [warps][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long t = (long long)blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= n_tok) return;
  float* lg = rt + warp * E;
  for (int e = lane; e < E; e += 32) {
    float v = r[t * E + e];
    for (int s = 1; s < splits; ++s) v += r[s * split_stride + t * E + e];
    lg[e] = v + (bias ? bias[e] : 0.0f) + (tok_bias ? tok_bias[t * E + e] : 0.0f);
  }
  __syncwarp();
  float sel = 0.0f, top = 0.0f;
  int sid = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int e = lane; e < E; e += 32) {
      const float v = lg[e];
      if (v > bv || (v == bv && e < bi)) { bv = v; bi = e; }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if (j == 0) top = bv;
    if (lane == j) { sel = bv; sid = bi; }
    if (lane == 0) lg[bi] = -INFINITY;
    __syncwarp();
  }
  const float ex = lane < k ? expf(sel - top) : 0.0f;
  float den = ex;
#pragma unroll
  for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (lane < k) {
    ids[t * k + lane] = sid;
    gate[t * k + lane] = ex / den;
  }
}

// Router bias b_e = -s ln(e + 1) in fp32 (Zipf-skewed expert popularity).
__global__ void k_router_bias_f32(float* bias, int E, float s) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < E) bias[e] = s == 0.0f ? 0.0f : (float)(-(double)s * log((double)(e + 1)));
}

// ---------------------------------------------------------------------------
// Permute: stable counting sort of the T*k (token, slot) pairs by expert.
// perm[pos] = pair, inv[pair] = pos; work items (expert, first row, rows,
// first row) cover each expert's rows in tiles of `bn`.  One CTA; warp w
// places the pairs of experts w, w+32, ... in pair order (stable).
// ---------------------------------------------------------------------------
// Split-K factors of the two expert GEMMs, chosen here on the device from the
// number of work items: out[g] for g = 0 (gate|up) and 1 (down) from (m tiles,
// k blocks, cap); out[2] = rows of the largest work item.
struct SplitPlan {
  int mt[2], kb[2], cap[2];
  int fused0;   // the gate|up GEMM writes the SwiGLU output itself when it runs unsplit
  int* out;     // [0] gate|up split, [1] down split, [2] rows of the largest item
};

// Exclusive prefix sum of one int per thread over the block (blockDim a
// multiple of 32); *total receives the block sum.  Uses wsum[32].
__device__ __forceinline__ int block_scan_excl(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = lane < nw ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < nw) wsum[lane] = t;
  }
  __syncthreads();
  const int base = warp > 0 ? wsum[warp - 1] : 0;
  *total = wsum[nw - 1];
  __syncthreads();
  return base + x - v;
}

struct PermuteArgs {
  const int* ids;          // [n_pairs] expert of each (token, slot)
  int n_pairs, E, bn;
  int* perm;               // [n_pairs] pair at each expert-ordered position
  int* inv;                // [n_pairs] position of each pair
  int4* work;              // work items (expert, first row, rows, first row)
  int* work_count;
  int* counts_out;         // [E] rows per expert, or null
  SplitPlan plan;
  unsigned long long* touched_acc;   // running total of distinct experts, or null
  int* err;
};

// The permute by one CTA (any multiple of 32 threads); psm holds
// (warps x E + E + 1) ints.  ids are read through L2: they may have been
// written by other CTAs of the same kernel.  Only a `writer` CTA stores the
// results to global memory (perm, inv, work items, counts, split plan);
// perm_s (shared, n_pairs ints, or null) receives the permutation locally.
__device__ void permute_body(const PermuteArgs& a, int* psm, bool writer = true, int* perm_s = nullptr) {
  const int* __restrict__ ids = a.ids;
  const int n_pairs = a.n_pairs, E = a.E, bn = a.bn;
  int* __restrict__ perm = a.perm;
  int* __restrict__ inv = a.inv;
  int4* __restrict__ work = a.work;
  int* __restrict__ counts_out = a.counts_out;
  SplitPlan plan = a.plan;
  int* err = a.err;
  // Warp w owns the contiguous pair range [w*chunk, (w+1)*chunk).  A pair's
  // position is offs[e] (pairs of lower experts) + pairs of expert e in
  // earlier warps + pairs of e earlier in this warp's range, which keeps the
  // (token, slot) order within each expert.
  const int nwarps = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* hist = psm;                  // [nwarps][E]
  int* offs = psm + nwarps * E;     // [E + 1]
  for (int i = threadIdx.x; i < nwarps * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int chunk = (n_pairs + nwarps - 1) / nwarps;
  const int p_begin = min(n_pairs, warp * chunk), p_end = min(n_pairs, p_begin + chunk);
  const unsigned lt_mask = (1u << lane) - 1u;
  int* my = hist + warp * E;
  for (int p0 = p_begin; p0 < p_end; p0 += 32) {
    const int p = p0 + lane;
    int e = p < p_end ? __ldcg(ids + p) : -1;
    if (e >= E || (p < p_end && e < 0)) { dev_error(err, DGDEV_BAD_INDEX); e = -1; }
    const unsigned same = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (same & lt_mask) == 0) my[e] += __popc(same);
    __syncwarp();
  }
  __syncthreads();
  // per expert: exclusive prefix over warps; the total goes to offs[e]
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int acc = 0;
    for (int w = 0; w < nwarps; ++w) {
      const int c = hist[w * E + e];
      hist[w * E + e] = acc;
      acc += c;
    }
    offs[e] = acc;
  }
  __syncthreads();
  // expert offsets and work items: block-wide exclusive scans of the expert
  // row counts and item counts (chunks of blockDim experts, with carries)
  __shared__ int wsum[32], s_max_rows, s_touched;
  if (threadIdx.x == 0) { s_max_rows = 0; s_touched = 0; }
  int carry_rows = 0, carry_items = 0;
  for (int e0 = 0; e0 < E; e0 += blockDim.x) {
    const int e = e0 + threadIdx.x;
    const int c = e < E ? offs[e] : 0;
    const int it = (c + bn - 1) / bn;
    int tot_rows, tot_items;
    const int pr = block_scan_excl(c, wsum, &tot_rows);
    const int pi = block_scan_excl(it, wsum, &tot_items);
    if (e < E) {
      const int acc = carry_rows + pr, nw0 = carry_items + pi;
      offs[e] = acc;
      if (writer) {
        if (counts_out) counts_out[e] = c;
        for (int j = 0; j < it; ++j)
          work[nw0 + j] = make_int4(e, acc + j * bn, min(bn, c - j * bn), acc + j * bn);
        if (c > 0) { atomicMax(&s_max_rows, min(c, bn)); atomicAdd(&s_touched, 1); }
      }
    }
    carry_rows += tot_rows;
    carry_items += tot_items;
  }
  __syncthreads();
  if (threadIdx.x == 0) offs[E] = carry_rows;
  if (threadIdx.x == 0 && writer) {
    const int nw = carry_items;
    *a.work_count = nw;
    // running total of distinct experts this layer streamed (measurement)
    if (a.touched_acc) *a.touched_acc += (unsigned long long)s_touched;
    if (plan.out) {
      // Split-K factor per GEMM: the persistent kernel runs ceil(tiles / SMs)
      // waves of tiles that each take 1/s of a full-K tile, and every split
      // adds one fp32 partial slab (written, then read by the consumer).  In
      // units of the time to stream the group's weights once:
      //   cost(s) = ceil(mt * nw * s / SMs) / s + s * r,
      //   r = partial bytes (written and read) / weight bytes / 4.
      for (int g = 0; g < 2; ++g) {
        // partial slabs mostly stay in L2: charged at a quarter of the weight-stream rate
        const float r = (float)n_pairs / ((float)max(1, nw) * (float)(plan.kb[g] * 64));
        const int s_max = max(1, min(plan.cap[g], plan.kb[g] / 4));
        int best = 1;
        float best_cost = 3.4e38f;
        for (int s = 1; s <= s_max; ++s) {
          const int waves = (plan.mt[g] * nw * s + kSMs - 1) / kSMs;
          // an unsplit fused gate|up GEMM writes no fp32 partials at all
          const float cost = (float)waves / (float)s + ((g == 0 && plan.fused0 && s == 1) ? 0.0f : (float)s * r);
          if (cost < best_cost) { best_cost = cost; best = s; }
        }
        plan.out[g] = best;
      }
      plan.out[2] = s_max_rows;
    }
  }
  __syncthreads();
  for (int p0 = p_begin; p0 < p_end; p0 += 32) {
    const int p = p0 + lane;
    int e = p < p_end ? __ldcg(ids + p) : -1;
    if (e >= E) e = -1;
    const unsigned same = __match_any_sync(0xffffffffu, e);
    if (e >= 0) {
      const int pos = offs[e] + my[e] + __popc(same & lt_mask);
      if (writer) {
        perm[pos] = p;
        inv[p] = pos;
      }
      if (perm_s) perm_s[pos] = p;
    }
    __syncwarp();
    if (e >= 0 && (same & lt_mask) == 0) my[e] += __popc(same);
    __syncwarp();
  }
}

__global__ void k_permute(PermuteArgs a) {
  pdl_enter();
  extern __shared__ int psm[];
  permute_body(a, psm);
}

// Permute and gather in one kernel: every CTA sorts all (token, slot) pairs in
// shared memory (the same stable counting sort), CTA 0 publishes the
// permutation, work items and split plan, and each CTA copies its share of
// the expert-ordered rows xp[pos] = x[perm[pos] / k].  Dynamic shared memory:
// permute_smem(E) + n_pairs ints.
template <typename T>
__global__ void __launch_bounds__(1024) k_permute_gather(PermuteArgs a, const T* __restrict__ x, int k, int d,
                                                         T* __restrict__ xp) {
  pdl_enter();
  extern __shared__ int psm[];
  const int nwarps = blockDim.x >> 5;
  int* perm_s = psm + nwarps * a.E + a.E + 1;
  // positions of pairs with an invalid expert id (reported as an error) stay
  // unplaced: they copy row 0 rather than an undefined one
  for (int i = threadIdx.x; i < a.n_pairs; i += blockDim.x) perm_s[i] = 0;
  permute_body(a, psm, blockIdx.x == 0, perm_s);
  __syncthreads();
  const int per = (a.n_pairs + gridDim.x - 1) / gridDim.x;
  const int p0 = min(a.n_pairs, (int)blockIdx.x * per), p1 = min(a.n_pairs, p0 + per);
  const int nv = d * (int)sizeof(T) / 16;
  const long long n = (long long)(p1 - p0) * nv;
  for (long long i = threadIdx.x; i < n; i += blockDim.x) {
    const int pos = p0 + (int)(i / nv), c = (int)(i % nv);
    const long long src = perm_s[pos] / k;
    reinterpret_cast<uint4*>(xp + (long long)pos * d)[c] = reinterpret_cast<const uint4*>(x + src * d)[c];
  }
}

// Threads of the permute kernel: whole warps, with the per-warp histograms
// kept within 48 KB of shared memory.
inline int permute_threads(int E) { return 32 * std::max(1, std::min(32, 12288 / std::max(1, E) - 2)); }
inline size_t permute_smem(int E) { return ((size_t)(permute_threads(E) / 32) * E + E + 1) * sizeof(int); }

// xp[pos] = x[perm[pos] / k]: expert-ordered copy of the normalised rows.
template <typename T>
__global__ void k_gather(const T* __restrict__ x, const int* __restrict__ perm, int k, int d,
                         T* __restrict__ xp) {
  pdl_enter();
  const int pos = blockIdx.x;
  const long long src = perm[pos] / k;
  const uint4* s = reinterpret_cast<const uint4*>(x + src * d);
  uint4* o = reinterpret_cast<uint4*>(xp + (long long)pos * d);
  const int nv = d * (int)sizeof(T) / 16;
  for (int i = threadIdx.x; i < nv; i += blockDim.x) o[i] = s[i];
}

// SwiGLU: a = round(silu(g) * u) with g / u the gate and up columns of each
// row of the gate|up GEMM output, interleaved in blocks of 64 (columns
// [128 i, 128 i + 64) gate, the next 64 up), each summed over the split-K
// partials (count read from the device).  When `fused` is set and the GEMM ran
// with one split, its epilogue already wrote `a` and this kernel does nothing.
template <typename T>
__global__ void k_swiglu(const float* __restrict__ gu, int ff, long long n, T* __restrict__ a,
                         const int* __restrict__ splits_dev, long long split_stride, int fused) {
  pdl_enter();
  const int ns = splits_dev ? *splits_dev : 1;
  if (fused && ns == 1) return;
  const long long n4 = n / 4;   // ff is a multiple of 64
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    const long long e = i * 4, r = e / ff;
    const int c = (int)(e % ff);
    const float* gp = gu + r * 2 * ff + (c / 64) * 128 + c % 64;
    float4 g = *reinterpret_cast<const float4*>(gp);
    float4 u = *reinterpret_cast<const float4*>(gp + 64);
    for (int s = 1; s < ns; ++s) {
      const float4 g2 = *reinterpret_cast<const float4*>(gp + s * split_stride);
      const float4 u2 = *reinterpret_cast<const float4*>(gp + s * split_stride + 64);
      g.x += g2.x; g.y += g2.y; g.z += g2.z; g.w += g2.w;
      u.x += u2.x; u.y += u2.y; u.z += u2.z; u.w += u2.w;
    }
    a[e] = from_f<T>(g.x / (1.0f + expf(-g.x)) * u.x);
    a[e + 1] = from_f<T>(g.y / (1.0f + expf(-g.y)) * u.y);
    a[e + 2] = from_f<T>(g.z / (1.0f + expf(-g.z)) * u.z);
    a[e + 3] = from_f<T>(g.w / (1.0f + expf(-g.w)) * u.w);
  }
}

// ---------------------------------------------------------------------------
// Vocab sampler, one CTA per logit row (row = canvas * 256 + position).
//  pass 1: row max + argmax, Gumbel-max token at 1/T (Philox per 4 logits);
//  pass 2: e_v = exp(l_v - m); S, U summed exactly in Q40 int64;
//  pass 3: p_v = e_v * (1/S) stored for self-conditioning.
// H = ln(S) - U/S; all binary32 steps use the fixed-sequence math above.
// ---------------------------------------------------------------------------
struct SamplerArgs {
  const float* logits;
  int vocab;
  int positions;        // rows per canvas (256)
  uint64_t seed;
  float temp_start, temp_end;
  const DevState* state;
  int step_override;    // >= 0: use this round instead of state->step
  float t_override;     // used when step_override >= 0
  float* H;
  int* tok;
  int* amax;
  long long* s_q;       // optional
  long long* u_q;       // optional
};

struct ArgBest {
  float v;
  int i;
};
__device__ __forceinline__ ArgBest arg_better(ArgBest a, ArgBest b) {
  if (b.i < 0) return a;
  if (a.i < 0) return b;
  if (b.v > a.v || (b.v == a.v && b.i < a.i)) return b;
  return a;
}
__device__ __forceinline__ ArgBest warp_argmax(ArgBest x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    ArgBest y;
    y.v = __shfl_xor_sync(0xffffffffu, x.v, o);
    y.i = __shfl_xor_sync(0xffffffffu, x.i, o);
    x = arg_better(x, y);
  }
  return x;
}

// Vocab-wide sampler pass.  One cluster of NC CTAs per row (sampler_cluster:
// 1 or 2 up to a 65536-entry vocabulary, else 8); CTA r of the cluster owns the
// contiguous vocab slice [r V/NC, (r+1) V/NC).  The results do not depend on
// NC: the sums are exact integers, maxima break ties to the lower index, the
// Philox counters are vocabulary indices, and the Gumbel filter only skips
// values that cannot beat the running best of the thread that sees them.
// Partial results are exchanged through distributed shared memory and every
// CTA combines them in rank order (integer sums are exact, arg-maxima break
// ties to the lower index), so all CTAs hold the same row values.
//   pass 1: max / argmax of the logits, and the Gumbel-max key
//           argmax_v (l_v / T + g_v), g_v = -ln(-ln u_v).  Since
//           -ln u >= 1 - u, g_v <= -ln(1 - u_v) <= -E ln 2 with E the binary
//           exponent of 1 - u_v (exact in binary32); the exact g_v is
//           evaluated only where that bound plus a margin reaches the
//           thread's best key, so the winner is unchanged.
//   pass 2: e_v = exp(l_v - m) (own binary32 exp), S and U = sum e (l - m) as
//           truncated Q40 int64.
//   pass 3: probabilities e_v / S in the storage dtype (e_v recomputed).
// Passes 2 and 3 re-read the slice (from L2); nothing is staged in shared
// memory, so several clusters share an SM.  The arithmetic uses no
// conversion-unit instructions per element.
// ---------------------------------------------------------------------------
constexpr int kSampCta = 8;        // most CTAs per row (one thread-block cluster)
// CTAs per row: fewer, longer slices for small vocabularies, where each CTA's
// fixed work (reductions, cluster barriers) would otherwise dominate -- one
// CTA per row once the rows alone give every SM four CTAs, else two.
// Measured at V = 32768, 8192 rows: exact sampler 2.95 / 2.19 / 2.05 ms for
// 8 / 2 / 1 CTAs per row; at V = 262144, 256 rows: 0.495 / 0.518 / 0.502 ms
// for 8 / 4 / 2.
inline int sampler_cluster(int vocab, long long rows) {
  if (vocab > 65536) return kSampCta;
  return rows >= 4LL * kSMs ? 1 : 2;
}
constexpr int kSampThreads = 256;

struct SampPart {
  ArgBest m, g;
  long long s, u;
  float fl;   // top-k: this slice's candidate floor
  int cnt;    // top-k: this slice's buffered candidates
};

template <typename T, int NC>
__global__ void __cluster_dims__(NC, 1, 1) __launch_bounds__(kSampThreads)
k_sampler(SamplerArgs a, T* __restrict__ probs) {
  pdl_enter();
  __shared__ SampPart part;
  __shared__ ArgBest red_m[32], red_g[32];
  __shared__ long long red_s[32], red_u[32];
  uint32_t rank;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
  const long long row = blockIdx.x / NC;
  const int canvas = (int)(row / a.positions), pos = (int)(row % a.positions);
  const int step = a.step_override >= 0 ? a.step_override : a.state->step;
  const float t = a.step_override >= 0 ? a.t_override : a.state->t;
  const float temp = __fadd_rn(a.temp_end, __fmul_rn(__fsub_rn(a.temp_start, a.temp_end), t));
  const float inv_t = __fdiv_rn(1.0f, temp);
  const uint32_t k0 = (uint32_t)a.seed, k1 = (uint32_t)(a.seed >> 32) ^ (uint32_t)canvas;
  const int n4 = a.vocab / (4 * NC);        // float4 groups in this slice
  const int g0 = (int)rank * n4;                  // first global float4 group
  const float4* l4 = reinterpret_cast<const float4*>(a.logits + row * a.vocab) + g0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;

  // pass 1
  ArgBest bm{-INFINITY, -1}, bg{-INFINITY, -1};
  for (int i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 l = l4[i];
    const int v4 = g0 + i;
    const uint4 w = philox4x32_10(make_uint4((uint32_t)v4, (uint32_t)pos, (uint32_t)step, STREAM_GUMBEL), k0, k1);
    const float lv[4] = {l.x, l.y, l.z, l.w};
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int v = v4 * 4 + j;
      bm = arg_better(bm, ArgBest{lv[j], v});
      const float lt = __fmul_rn(lv[j], inv_t);
      // 1 - u, u = (2 (x >> 9) + 1) 2^-24, exactly in binary32 from f =
      // 1 + (x >> 9) 2^-23: (2 - f) - 2^-24.  Its binary exponent E (in
      // [-24, -1]) gives g <= -E ln 2 (-E as a float through the 2^23 trick).
      const float f = __uint_as_float(0x3F800000u | (wv[j] >> 9));
      const float omu = __fsub_rn(__fsub_rn(2.0f, f), 5.9604644775390625e-8f);
      const int negE = 127 - (int)(__float_as_uint(omu) >> 23);
      const float g_ub = __fmul_rn(__fsub_rn(__int_as_float(0x4B000000 + negE), 8388608.0f), 0.69314718f);
      if (bg.i < 0 || lt + g_ub + (1e-3f + 1e-5f * fabsf(bg.v)) >= bg.v) {
        const float key = __fadd_rn(lt, gumbel_of(wv[j]));
        bg = arg_better(bg, ArgBest{key, v});
      }
    }
  }
  bm = warp_argmax(bm);
  bg = warp_argmax(bg);
  if (lane == 0) { red_m[warp] = bm; red_g[warp] = bg; }
  __syncthreads();
  if (warp == 0) {
    ArgBest x = lane < nw ? red_m[lane] : ArgBest{-INFINITY, -1};
    ArgBest y = lane < nw ? red_g[lane] : ArgBest{-INFINITY, -1};
    x = warp_argmax(x);
    y = warp_argmax(y);
    if (lane == 0) { part.m = x; part.g = y; }
  }
  cluster_sync_all();
  ArgBest M{-INFINITY, -1}, G{-INFINITY, -1};
  for (int r = 0; r < NC; ++r) {
    const SampPart* pr = cluster_peer(&part, r);
    M = arg_better(M, ArgBest{pr->m.v, pr->m.i});
    G = arg_better(G, ArgBest{pr->g.v, pr->g.i});
  }
  if (rank == 0 && threadIdx.x == 0) {
    a.amax[row] = M.i;
    a.tok[row] = G.i;
  }
  const float m = M.v;

  // pass 2
  long long sq = 0, uq = 0;
  double sd = 0.0, ud = 0.0;
  for (int i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 l = l4[i];
    const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float dlt = __fsub_rn(lv[j], m);
      const float e = dg_expf(dlt);
      q40_add(e, sq, sd);
      q40_add(__fmul_rn(e, dlt), uq, ud);
    }
  }
  sq = q40_total(sq, sd);
  uq = q40_total(uq, ud);
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    sq += __shfl_xor_sync(0xffffffffu, sq, o);
    uq += __shfl_xor_sync(0xffffffffu, uq, o);
  }
  if (lane == 0) { red_s[warp] = sq; red_u[warp] = uq; }
  __syncthreads();
  if (threadIdx.x == 0) {
    long long S = 0, U = 0;
    for (int w = 0; w < nw; ++w) { S += red_s[w]; U += red_u[w]; }
    part.s = S;
    part.u = U;
  }
  cluster_sync_all();
  long long S = 0, U = 0;
  for (int r = 0; r < NC; ++r) {
    const SampPart* pr = cluster_peer(&part, r);
    S += pr->s;
    U += pr->u;
  }
  // no CTA may leave (or reuse `part`) while another still reads it
  cluster_sync_all();
  if (rank == 0 && threadIdx.x == 0) {
    const float sf = __ll2float_rn(S), uf = __ll2float_rn(U);
    a.H[row] = __fsub_rn(dg_logf(__fmul_rn(sf, 9.094947017729282e-13f)), __fdiv_rn(uf, sf));
    if (a.s_q) a.s_q[row] = S;
    if (a.u_q) a.u_q[row] = U;
  }

  // pass 3
  if (probs) {
    const float inv_s = __fdiv_rn(1.0f, __fmul_rn(__ll2float_rn(S), 9.094947017729282e-13f));
    T* pr = probs + row * a.vocab + (long long)g0 * 4;
    for (int i = threadIdx.x; i < n4; i += blockDim.x) {
      const float4 l = l4[i];
      store4<T>(pr + (long long)i * 4, __fmul_rn(dg_expf(__fsub_rn(l.x, m)), inv_s),
                __fmul_rn(dg_expf(__fsub_rn(l.y, m)), inv_s), __fmul_rn(dg_expf(__fsub_rn(l.z, m)), inv_s),
                __fmul_rn(dg_expf(__fsub_rn(l.w, m)), inv_s));
    }
  }
}

// Launch of the sampler over `rows` rows (vocab % (4 kSampCta) == 0).
// nc_want: CTAs per row (1, 2, 4 or 8 dividing the vocabulary into float4
// groups), 0 for sampler_cluster's choice.
inline int sampler_nc(int vocab, long long rows, int nc_want) {
  if ((nc_want == 1 || nc_want == 2 || nc_want == 4 || nc_want == 8) && vocab % (4 * nc_want) == 0) return nc_want;
  return sampler_cluster(vocab, rows);
}
template <typename T>
cudaError_t launch_sampler(const SamplerArgs& sa, T* probs, long long rows, cudaStream_t s, bool pdl,
                           int nc_want = 0) {
  const size_t smem = 0;
  const int nc = sampler_nc(sa.vocab, rows, nc_want);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(rows * nc));
  cfg.blockDim = dim3(kSampThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr_pdl[1];
  attr_pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr_pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr_pdl;
  cfg.numAttrs = pdl ? 1 : 0;
  switch (nc) {
    case 1: return cudaLaunchKernelEx(&cfg, k_sampler<T, 1>, sa, probs);
    case 2: return cudaLaunchKernelEx(&cfg, k_sampler<T, 2>, sa, probs);
    case 4: return cudaLaunchKernelEx(&cfg, k_sampler<T, 4>, sa, probs);
    default: return cudaLaunchKernelEx(&cfg, k_sampler<T, 8>, sa, probs);
  }
}

// ---------------------------------------------------------------------------
// Top-k-truncated sampler (the optimisation the DiffusionGemma technical-
// report explainer, section 九, names for large batches).  Per row: the K
// largest logits (value descending, ties to the lower index) are the
// candidates; the token is the Gumbel-max draw among them with the exact
// sampler's noise g_v (Philox counter (v>>2, position, round, stream 0));
// the candidate weights w_j = e_j (1/s), e_j = exp(l_j - m), s = e_0 + e_1 +
// ... in candidate order, feed self-conditioning.  Entropy, row argmax and
// the Q40 sums are those of the full row, as in k_sampler.
//
// Same cluster layout as k_sampler (NC CTAs per row).  Pass 1 keeps
// the slice's K best in a shared candidate buffer: every value above the
// current threshold (the K-th best so far) is appended; when the next
// iteration could overflow the buffer it is sorted and cut back to K.
// Iterations visit increasing indices, so a later value equal to the
// threshold can never displace a kept one and a strict comparison suffices.
// Rank 0 merges the NC lists through distributed shared memory and
// draws among the row's K candidates: Philox runs on K values per row, not V.
// ---------------------------------------------------------------------------
constexpr int kTopkMax = 256;      // largest supported truncation K
constexpr int kCandCap = 2048;     // candidate buffer per CTA (>= kSampCta * kTopkMax)

// Sort cv/ci[0, n) best first -- value descending, index ascending -- by a
// bitonic network over the next power of two (padding with (-inf, INT_MAX),
// which ranks after every real entry).  Block-wide; n <= kCandCap.
__device__ __forceinline__ void cand_sort(float* cv, int* ci, int n) {
  int n2 = 1;
  while (n2 < n) n2 <<= 1;
  for (int i = n + (int)threadIdx.x; i < n2; i += blockDim.x) { cv[i] = -INFINITY; ci[i] = 0x7fffffff; }
  __syncthreads();
  for (int k = 2; k <= n2; k <<= 1)
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n2; i += blockDim.x) {
        const int p = i ^ j;
        if (p > i) {
          const float va = cv[i], vb = cv[p];
          const int ia = ci[i], ib = ci[p];
          const bool b_ahead = vb > va || (vb == va && ib < ia);
          if (((i & k) == 0) == b_ahead) { cv[i] = vb; cv[p] = va; ci[i] = ib; ci[p] = ia; }
        }
      }
      __syncthreads();
    }
}

template <typename T, int NC>
__global__ void __cluster_dims__(NC, 1, 1) __launch_bounds__(kSampThreads)
k_sampler_topk(SamplerArgs a, int K, int* __restrict__ cand_ids, T* __restrict__ cand_w) {
  pdl_enter();
  __shared__ SampPart part;
  __shared__ ArgBest red_m[32], red_g[32];
  __shared__ long long red_s[32], red_u[32];
  __shared__ float cv[kCandCap];
  __shared__ int ci[kCandCap];
  __shared__ float ew[kTopkMax];
  __shared__ int s_cnt, s_have;
  __shared__ float s_tau, s_inv;
  uint32_t rank;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
  const long long row = blockIdx.x / NC;
  const int canvas = (int)(row / a.positions), pos = (int)(row % a.positions);
  const int step = a.step_override >= 0 ? a.step_override : a.state->step;
  const float t = a.step_override >= 0 ? a.t_override : a.state->t;
  const float temp = __fadd_rn(a.temp_end, __fmul_rn(__fsub_rn(a.temp_start, a.temp_end), t));
  const float inv_t = __fdiv_rn(1.0f, temp);
  const uint32_t k0 = (uint32_t)a.seed, k1 = (uint32_t)(a.seed >> 32) ^ (uint32_t)canvas;
  const int n4 = a.vocab / (4 * NC);
  const int g0 = (int)rank * n4;
  const float4* l4 = reinterpret_cast<const float4*>(a.logits + row * a.vocab) + g0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;

  // pass 1: row max / argmax and the row's K best.  First each thread's
  // maximum: the K-th largest of those maxima (K <= blockDim.x) is a floor
  // with at least K values of the slice at or above it, and the largest of
  // the cluster's floors F has at least K values of the row at or above it,
  // so every value of the row's K best -- ties included -- is at or above F.
  // Each CTA buffers its values >= F.  When the cluster's buffers together
  // fit one buffer, rank 0 gathers them and sorts once; otherwise every CTA
  // sorts its own down to its K best (by the threshold loop below when even
  // its own values >= F overflow, as on flat rows) and rank 0 merges the
  // lists.  Both ways the K best come out in the same order (value
  // descending, index ascending).
  ArgBest bm{-INFINITY, -1};
  {
    float tmax = -INFINITY;
    for (int i = threadIdx.x; i < n4; i += blockDim.x) {
      const float4 l = l4[i];
      const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        bm = arg_better(bm, ArgBest{lv[j], (g0 + i) * 4 + j});
        tmax = fmaxf(tmax, lv[j]);
      }
    }
    cv[threadIdx.x] = tmax;
    ci[threadIdx.x] = threadIdx.x;
    __syncthreads();
    cand_sort(cv, ci, blockDim.x);
  }
  const float floor_loc = cv[K - 1];
  bm = warp_argmax(bm);
  if (lane == 0) red_m[warp] = bm;
  __syncthreads();
  if (warp == 0) {
    ArgBest x = lane < nw ? red_m[lane] : ArgBest{-INFINITY, -1};
    x = warp_argmax(x);
    if (lane == 0) { part.m = x; part.fl = floor_loc; s_cnt = 0; }
  }
  cluster_sync_all();
  ArgBest M{-INFINITY, -1};
  float F = -INFINITY;
  for (int r = 0; r < NC; ++r) {
    const SampPart* pr = cluster_peer(&part, r);
    M = arg_better(M, ArgBest{pr->m.v, pr->m.i});
    F = fmaxf(F, pr->fl);
  }
  const float m = M.v;
  for (int i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 l = l4[i];
    const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (lv[j] >= F) {
        const int slot = atomicAdd(&s_cnt, 1);
        if (slot < kCandCap) { cv[slot] = lv[j]; ci[slot] = (g0 + i) * 4 + j; }
      }
  }
  __syncthreads();
  if (threadIdx.x == 0) part.cnt = s_cnt;
  cluster_sync_all();
  int total = 0;
  bool fits = true;
  for (int r = 0; r < NC; ++r) {
    const int c = cluster_peer(&part, r)->cnt;
    total += c;
    fits = fits && c <= kCandCap;
  }
  const bool one_sort = fits && total <= kCandCap;   // the same outcome in every CTA of the cluster
  if (!one_sort) {
    const bool bounded = s_cnt <= kCandCap;
    __syncthreads();
    if (threadIdx.x == 0) { s_cnt = bounded ? s_cnt : 0; s_have = 0; s_tau = -INFINITY; }
    __syncthreads();
    for (int base = 0; !bounded && base < n4; base += blockDim.x) {
      const int cnt = s_cnt;
      __syncthreads();                       // every thread has read cnt before any append
      if (cnt + 4 * (int)blockDim.x > kCandCap) {
        cand_sort(cv, ci, cnt);
        if (threadIdx.x == 0) {
          s_cnt = min(cnt, K);
          s_have = cnt >= K;
          s_tau = cnt >= K ? cv[K - 1] : -INFINITY;
        }
        __syncthreads();
      }
      const bool have = s_have != 0;
      const float tau = s_tau;
      const int i = base + (int)threadIdx.x;
      if (i < n4) {
        const float4 l = l4[i];
        const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int v = (g0 + i) * 4 + j;
          if (!have || lv[j] > tau) {
            const int slot = atomicAdd(&s_cnt, 1);
            if (slot < kCandCap) { cv[slot] = lv[j]; ci[slot] = v; }
          }
        }
      }
      __syncthreads();
    }
    {
      const int cnt = min(s_cnt, kCandCap);
      __syncthreads();
      cand_sort(cv, ci, cnt);
      if (threadIdx.x == 0) s_cnt = min(cnt, K);
    }
    cluster_sync_all();                      // every list is final before rank 0 reads it
  }

  if (rank == 0) {
    if (one_sort) {
      // every CTA's candidates after rank 0's own, then one sort
      int off = s_cnt;
      for (int r = 1; r < NC; ++r) {
        const float* pv = cluster_peer(cv, r);
        const int* pi = cluster_peer(ci, r);
        const int pc = cluster_peer(&part, r)->cnt;
        for (int j = threadIdx.x; j < pc; j += blockDim.x) {
          cv[off + j] = pv[j];
          ci[off + j] = pi[j];
        }
        off += pc;
      }
      for (int j = total + (int)threadIdx.x; j < K; j += blockDim.x) { cv[j] = -INFINITY; ci[j] = 0x7fffffff; }
      __syncthreads();
      cand_sort(cv, ci, max(total, K));
    } else {
      // merge the lists: rank r's K best go to [r K, (r+1) K)
      for (int r = 1; r < NC; ++r) {
        const float* pv = cluster_peer(cv, r);
        const int* pi = cluster_peer(ci, r);
        const int pc = *cluster_peer(&s_cnt, r);
        for (int j = threadIdx.x; j < K; j += blockDim.x) {
          cv[r * K + j] = j < pc ? pv[j] : -INFINITY;
          ci[r * K + j] = j < pc ? pi[j] : 0x7fffffff;
        }
      }
      for (int j = s_cnt + (int)threadIdx.x; j < K; j += blockDim.x) { cv[j] = -INFINITY; ci[j] = 0x7fffffff; }
      __syncthreads();
      cand_sort(cv, ci, NC * K);
    }
    // Gumbel-max among the candidates; candidate weights
    ArgBest bg{-INFINITY, -1};
    for (int j = threadIdx.x; j < K; j += blockDim.x) {
      const int v = ci[j];
      const uint4 w = philox4x32_10(make_uint4((uint32_t)v >> 2, (uint32_t)pos, (uint32_t)step, STREAM_GUMBEL),
                                    k0, k1);
      const uint32_t word = (v & 3) == 0 ? w.x : (v & 3) == 1 ? w.y : (v & 3) == 2 ? w.z : w.w;
      const float key = __fadd_rn(__fmul_rn(cv[j], inv_t), gumbel_of(word));
      bg = arg_better(bg, ArgBest{key, v});
      ew[j] = dg_expf(__fsub_rn(cv[j], m));
    }
    bg = warp_argmax(bg);
    if (lane == 0) red_g[warp] = bg;
    __syncthreads();
    if (threadIdx.x == 0) {
      ArgBest G{-INFINITY, -1};
      for (int w = 0; w < nw; ++w) G = arg_better(G, red_g[w]);
      a.tok[row] = G.i;
      a.amax[row] = M.i;
      float sum = 0.0f;
      for (int j = 0; j < K; ++j) sum = __fadd_rn(sum, ew[j]);
      s_inv = __fdiv_rn(1.0f, sum);
    }
    __syncthreads();
    for (int j = threadIdx.x; j < K; j += blockDim.x) {
      cand_ids[row * K + j] = ci[j];
      cand_w[row * K + j] = from_f<T>(__fmul_rn(ew[j], s_inv));
    }
  }

  // pass 2: S, U of the full row (as in k_sampler)
  long long sq = 0, uq = 0;
  double sd = 0.0, ud = 0.0;
  for (int i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 l = l4[i];
    const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float dlt = __fsub_rn(lv[j], m);
      const float e = dg_expf(dlt);
      q40_add(e, sq, sd);
      q40_add(__fmul_rn(e, dlt), uq, ud);
    }
  }
  sq = q40_total(sq, sd);
  uq = q40_total(uq, ud);
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    sq += __shfl_xor_sync(0xffffffffu, sq, o);
    uq += __shfl_xor_sync(0xffffffffu, uq, o);
  }
  if (lane == 0) { red_s[warp] = sq; red_u[warp] = uq; }
  __syncthreads();
  if (threadIdx.x == 0) {
    long long S = 0, U = 0;
    for (int w = 0; w < nw; ++w) { S += red_s[w]; U += red_u[w]; }
    part.s = S;
    part.u = U;
  }
  cluster_sync_all();
  long long S = 0, U = 0;
  for (int r = 0; r < NC; ++r) {
    const SampPart* pr = cluster_peer(&part, r);
    S += pr->s;
    U += pr->u;
  }
  // no CTA may leave while another still reads its shared memory
  cluster_sync_all();
  if (rank == 0 && threadIdx.x == 0) {
    const float sf = __ll2float_rn(S), uf = __ll2float_rn(U);
    a.H[row] = __fsub_rn(dg_logf(__fmul_rn(sf, 9.094947017729282e-13f)), __fdiv_rn(uf, sf));
    if (a.s_q) a.s_q[row] = S;
    if (a.u_q) a.u_q[row] = U;
  }
}

template <typename T>
cudaError_t launch_sampler_topk(const SamplerArgs& sa, int K, int* cand_ids, T* cand_w, long long rows,
                                cudaStream_t s, bool pdl, int nc_want = 0) {
  const int nc = sampler_nc(sa.vocab, rows, nc_want);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(rows * nc));
  cfg.blockDim = dim3(kSampThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr_pdl[1];
  attr_pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr_pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr_pdl;
  cfg.numAttrs = pdl ? 1 : 0;
  switch (nc) {
    case 1: return cudaLaunchKernelEx(&cfg, k_sampler_topk<T, 1>, sa, K, cand_ids, cand_w);
    case 2: return cudaLaunchKernelEx(&cfg, k_sampler_topk<T, 2>, sa, K, cand_ids, cand_w);
    case 4: return cudaLaunchKernelEx(&cfg, k_sampler_topk<T, 4>, sa, K, cand_ids, cand_w);
    default: return cudaLaunchKernelEx(&cfg, k_sampler_topk<T, 8>, sa, K, cand_ids, cand_w);
  }
}

// Self-conditioning input of a truncated distribution: u[t] = sum_j w[t][j]
// E[id[t][j]] (fp32, candidate order), stored in T.  One CTA per position.
template <typename T>
__global__ void k_sc_gather(const int* __restrict__ ids, const T* __restrict__ w, int K,
                            const T* __restrict__ emb, int d, T* __restrict__ u) {
  pdl_enter();
  __shared__ int s_id[kTopkMax];
  __shared__ float s_w[kTopkMax];
  const long long t = blockIdx.x;
  for (int j = threadIdx.x; j < K; j += blockDim.x) {
    s_id[j] = ids[t * K + j];
    s_w[j] = to_f(w[t * K + j]);
  }
  __syncthreads();
  for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) {
    float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
    for (int j = 0; j < K; ++j) {
      const float4 e = load4<T>(emb + (long long)s_id[j] * d + c);
      a0 = fmaf(s_w[j], e.x, a0);
      a1 = fmaf(s_w[j], e.y, a1);
      a2 = fmaf(s_w[j], e.z, a2);
      a3 = fmaf(s_w[j], e.w, a3);
    }
    store4<T>(u + t * d + c, a0, a1, a2, a3);
  }
}

// ---------------------------------------------------------------------------
// Commit / re-noise / stop, one CTA of 256 threads per canvas.
// Default: commit where H < bound.  Entropy-bounded: sort (trunc(H 2^32), i)
// ascending, commit the longest prefix with exact sum <= trunc(bound 2^32),
// at least one.  Stop: (mean mode) all committed or sum H < n * bound, or
// (EB mode) sum H < n * bound and argmax == previous argmax (not at round 0);
// the last round of the budget always stops.  Uncommitted positions get a
// fresh uniform token (Philox stream 1).
// In block-loop mode a stopped canvas is frozen: its outputs are written once.
// ---------------------------------------------------------------------------
struct CommitArgs {
  const float* H;
  const int* tok;
  const int* amax;
  int* prev_amax;          // [B*256] argmax of the previous round (updated)
  int vocab;
  uint64_t seed;
  int commit_mode;
  float commit_bound;
  int stop_mode;
  float stop_bound;
  int max_steps;
  DevState* state;
  int step_override;       // >= 0: single-step mode with this round
  // single-step outputs (any may be null)
  uint8_t* commit;
  int* canvas_next;
  int* stop;
  int* n_committed;
  // block-loop state (null in single-step mode)
  int* canvas_cur;         // [B*256] canvas fed to the next round
  int* done;               // [B]
  int* steps_used;         // [B]
  int* n_committed_out;    // [B]
  int* canvas_out;         // [B*256]
};

__global__ void __launch_bounds__(256) k_commit(CommitArgs a) {
  pdl_enter();
  const int b = blockIdx.x, i = threadIdx.x;
  const int n = 256;
  const int step = a.step_override >= 0 ? a.step_override : a.state->step;
  const bool loop = a.done != nullptr;
  if (loop && a.done[b]) return;
  const long long idx = (long long)b * n + i;
  const float h = a.H[idx];
  const long long hq = __float2ll_rz(__fmul_rn(h, 4294967296.0f));
  __shared__ long long key_h[256];
  __shared__ int key_i[256];
  __shared__ long long sum_red[8];
  __shared__ int cnt_red[8], same_red[8];
  __shared__ int commit_s[256];

  int committed;
  if (a.commit_mode == 0) {
    committed = h < a.commit_bound;
  } else {
    key_h[i] = hq;
    key_i[i] = i;
    __syncthreads();
    // bitonic sort of (hq, i) ascending
    for (int kk = 2; kk <= n; kk <<= 1) {
      for (int j = kk >> 1; j > 0; j >>= 1) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const bool up = (i & kk) == 0;
          const long long ha = key_h[i], hb = key_h[ixj];
          const int ia = key_i[i], ib = key_i[ixj];
          const bool gt = ha > hb || (ha == hb && ia > ib);
          if (gt == up) { key_h[i] = hb; key_h[ixj] = ha; key_i[i] = ib; key_i[ixj] = ia; }
        }
        __syncthreads();
      }
    }
    // inclusive prefix sum of sorted entropies (exact int64)
    const long long lim = __float2ll_rz(__fmul_rn(a.commit_bound, 4294967296.0f));
    if (i == 0) {
      long long acc = 0;
      for (int r = 0; r < n; ++r) {
        acc += key_h[r];
        commit_s[key_i[r]] = (r == 0 || acc <= lim) ? 1 : 0;
        if (r > 0 && acc > lim) {
          for (int q = r + 1; q < n; ++q) commit_s[key_i[q]] = 0;
          break;
        }
      }
    }
    __syncthreads();
    committed = commit_s[i];
  }

  // reductions: count, sum of fixed-point entropies, argmax unchanged
  const int same = (a.amax[idx] == a.prev_amax[idx]) ? 1 : 0;
  long long s = hq;
  int c = committed, sm = same;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    c += __shfl_xor_sync(0xffffffffu, c, o);
    sm += __shfl_xor_sync(0xffffffffu, sm, o);
  }
  if ((i & 31) == 0) { sum_red[i >> 5] = s; cnt_red[i >> 5] = c; same_red[i >> 5] = sm; }
  __syncthreads();
  long long hsum = 0;
  int ncom = 0, nsame = 0;
  for (int w = 0; w < 8; ++w) { hsum += sum_red[w]; ncom += cnt_red[w]; nsame += same_red[w]; }
  const long long bound_q = __float2ll_rz(__fmul_rn(a.stop_bound, 4294967296.0f));
  const bool low = hsum < (long long)n * bound_q;
  bool stop;
  if (step >= a.max_steps - 1) stop = true;
  else if (a.stop_mode == 0) stop = (ncom == n) || low;
  else stop = step > 0 && low && nsame == n;

  const uint32_t k0 = (uint32_t)a.seed, k1 = (uint32_t)(a.seed >> 32) ^ (uint32_t)b;
  const uint4 w = philox4x32_10(make_uint4(0u, (uint32_t)i, (uint32_t)step, STREAM_RENOISE), k0, k1);
  const int nxt = committed ? a.tok[idx] : token_from_word(w.x, a.vocab);

  __syncthreads();
  if (a.commit) a.commit[idx] = (uint8_t)committed;
  if (a.canvas_next) a.canvas_next[idx] = nxt;
  a.prev_amax[idx] = a.amax[idx];
  if (i == 0) {
    if (a.stop) a.stop[b] = stop ? 1 : 0;
    if (a.n_committed) a.n_committed[b] = ncom;
  }
  if (loop) {
    a.canvas_cur[idx] = nxt;
    if (stop) {
      a.canvas_out[idx] = a.tok[idx];
      if (i == 0) {
        a.done[b] = 1;
        a.steps_used[b] = step + 1;
        a.n_committed_out[b] = ncom;
        atomicSub(&a.state->active, 1);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Block-loop control.
// ---------------------------------------------------------------------------
// Start of a round: t = 1 - s/(N-1) in binary32 (t = 1 when N = 1).
__global__ void k_round_begin(DevState* st) {
  pdl_enter();
  const int s = st->step, N = st->n_steps;
  st->t = N <= 1 ? 1.0f : __fsub_rn(1.0f, __fdiv_rn((float)s, (float)(N - 1)));
  st->use_selfcond = s > 0 ? 1 : 0;
}

// Single-step mode: set the round and time given by the caller.
__global__ void k_set_round(DevState* st, int step, float t, int use_sc) {
  pdl_enter();
  st->step = step;
  st->t = t;
  st->use_selfcond = use_sc;
}

// Block-loop start: initial canvases from Philox stream 2, counters reset.
__global__ void k_loop_init(DevState* st, int n_steps, int n_canvas, int* canvas_cur, int* done,
                            int* steps_used, int* n_committed_out, int* prev_amax, uint64_t seed,
                            int vocab) {
  const int b = blockIdx.x, i = threadIdx.x;
  const uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32) ^ (uint32_t)b;
  const uint4 w = philox4x32_10(make_uint4(0u, (uint32_t)i, 0u, STREAM_INIT_CANVAS), k0, k1);
  canvas_cur[b * 256 + i] = token_from_word(w.x, vocab);
  prev_amax[b * 256 + i] = -1;
  if (i == 0) { done[b] = 0; steps_used[b] = 0; n_committed_out[b] = 0; }
  if (b == 0 && i == 0) {
    st->step = 0;
    st->n_steps = n_steps;
    st->active = n_canvas;
    st->cond = 1;
  }
}

// End of a round: advance and set the loop's while-condition on the device.
__global__ void k_round_end_cond(DevState* st, cudaGraphConditionalHandle handle) {
  pdl_enter();
  st->step += 1;
  const int c = (st->active > 0 && st->step < st->n_steps && st->err == 0) ? 1 : 0;
  st->cond = c;
  cudaGraphSetConditional(handle, c);
}
