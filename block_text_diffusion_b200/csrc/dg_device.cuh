// Device building blocks: fixed-sequence binary32 numerics, Philox, bf16
// helpers, and thin PTX wrappers for mbarriers, TMA and tcgen05 (sm_100a).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

typedef __nv_bfloat16 bf16;

// ---------------------------------------------------------------------------
// Error word written by device code (first error wins); read by the host.
// ---------------------------------------------------------------------------
enum : int {
  DGDEV_OK = 0,
  DGDEV_TIMEOUT_TMA = 1,
  DGDEV_TIMEOUT_MMA = 2,
  DGDEV_TIMEOUT_EPI = 3,
  DGDEV_BAD_INDEX = 4,
};

__device__ __forceinline__ void dev_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// Programmatic dependent launch: every kernel of the step lets the next
// kernel in the stream be scheduled at once, and waits for the previous
// kernel (and its memory) before it touches global memory the previous
// kernels write.  Kernels with a prologue (barriers, tensor memory, weight
// tiles, which no kernel of the step writes) run it before the wait.
// Without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_enter() {
  pdl_launch();
  pdl_wait();
}

// ---------------------------------------------------------------------------
// dtype helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

// Four consecutive values as floats (p 16-byte aligned for float, 8-byte for bf16).
template <typename T> __device__ __forceinline__ float4 load4(const T* p);
template <> __device__ __forceinline__ float4 load4<float>(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
template <> __device__ __forceinline__ float4 load4<bf16>(const bf16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
  const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
  return make_float4(__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi));
}

// Four consecutive values (p 16-byte aligned for float, 8-byte for bf16).
template <typename T> __device__ __forceinline__ void store4(T* p, float a, float b, float c, float d);
template <> __device__ __forceinline__ void store4<float>(float* p, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
template <> __device__ __forceinline__ void store4<bf16>(bf16* p, float a, float b, float c, float d) {
  const __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
  uint2 u;
  u.x = *reinterpret_cast<const uint32_t*>(&lo);
  u.y = *reinterpret_cast<const uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(p) = u;
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11, section 3.2): ten rounds
// of the multiply-xor S-box with the Weyl key schedule.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
    const uint32_t lo0 = c.x * 0xD2511F53u, hi0 = __umulhi(c.x, 0xD2511F53u);
    const uint32_t lo1 = c.z * 0xCD9E8D57u, hi1 = __umulhi(c.z, 0xCD9E8D57u);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

// Philox counter word 3: which random stream a draw belongs to.
enum : uint32_t { STREAM_GUMBEL = 0, STREAM_RENOISE = 1, STREAM_INIT_CANVAS = 2, STREAM_WEIGHTS = 3 };

// uint32 -> (0,1): ((x >> 9)*2 + 1) * 2^-24, exact in binary32.
__device__ __forceinline__ float uniform_open(uint32_t x) {
  return __fmul_rn(__uint2float_rn((x >> 9) * 2u + 1u), 5.9604644775390625e-08f);
}

// floor(x * vocab / 2^32): a uniform token id.
__device__ __forceinline__ int token_from_word(uint32_t x, int vocab) {
  return (int)(((uint64_t)x * (uint64_t)vocab) >> 32);
}

// ---------------------------------------------------------------------------
// Binary32 math with a fixed operation sequence (every op an explicit IEEE
// round-to-nearest intrinsic, nothing fused), so the result is the same bits
// on any faithful IEEE implementation of the same sequence.
// Constants are the binary32 roundings of: ln2 cut to 16 significant bits
// (Cody-Waite high part), ln2 minus that part, 1/ln2, 2*pi, and 1/n or
// +-1/n! Taylor coefficients.
// ---------------------------------------------------------------------------
#define DG_F(bits) __uint_as_float(bits)

// ln x for positive normal x: x = 2^e m, m in [sqrt(1/2), sqrt(2)],
// ln m = 2 atanh(s) = 2 s (1 + s^2/3 + ... + s^10/11), s = (m-1)/(m+1).
__device__ __forceinline__ float dg_logf(float x) {
  const uint32_t b = __float_as_uint(x);
  int e = (int)(b >> 23) - 127;
  uint32_t mb = (b & 0x007FFFFFu) | 0x3F800000u;
  if (mb > 0x3FB504F3u) { mb -= 0x00800000u; e += 1; }
  const float m = __uint_as_float(mb);
  const float s = __fdiv_rn(__fsub_rn(m, 1.0f), __fadd_rn(m, 1.0f));
  const float z = __fmul_rn(s, s);
  float p = DG_F(0x3DBA2E8Cu);                            // 1/11
  p = __fadd_rn(__fmul_rn(p, z), DG_F(0x3DE38E39u));      // 1/9
  p = __fadd_rn(__fmul_rn(p, z), DG_F(0x3E124925u));      // 1/7
  p = __fadd_rn(__fmul_rn(p, z), DG_F(0x3E4CCCCDu));      // 1/5
  p = __fadd_rn(__fmul_rn(p, z), DG_F(0x3EAAAAABu));      // 1/3
  p = __fadd_rn(__fmul_rn(p, z), 1.0f);
  const float lnm = __fmul_rn(__fadd_rn(s, s), p);
  const float ef = __int2float_rn(e);
  return __fadd_rn(__fmul_rn(ef, DG_F(0x3F317200u)),
                   __fadd_rn(__fmul_rn(ef, DG_F(0x35BFBE8Eu)), lnm));
}

// e^x for x <= 0: k = rint(x/ln2), r = (x - k ln2_hi) - k ln2_lo,
// e^r by Taylor through r^7/7!, times 2^k; 0 below -86.
__device__ __forceinline__ float dg_expf(float x) {
  if (x < -86.0f) return 0.0f;
  const float t = __fmul_rn(x, DG_F(0x3FB8AA3Bu));
  // rint(t) for |t| < 2^22: adding 1.5 * 2^23 rounds to an integer (ties to
  // even) in the low mantissa bits; subtracting it back is exact.  Integer
  // arithmetic only: no conversion unit.
  const float tk = __fadd_rn(t, 12582912.0f);
  const float k = __fsub_rn(tk, 12582912.0f);
  const float r = __fsub_rn(__fsub_rn(x, __fmul_rn(k, DG_F(0x3F317200u))),
                            __fmul_rn(k, DG_F(0x35BFBE8Eu)));
  float p = DG_F(0x39500D01u);                            // 1/7!
  p = __fadd_rn(__fmul_rn(p, r), DG_F(0x3AB60B61u));      // 1/6!
  p = __fadd_rn(__fmul_rn(p, r), DG_F(0x3C088889u));      // 1/5!
  p = __fadd_rn(__fmul_rn(p, r), DG_F(0x3D2AAAABu));      // 1/4!
  p = __fadd_rn(__fmul_rn(p, r), DG_F(0x3E2AAAABu));      // 1/3!
  p = __fadd_rn(__fmul_rn(p, r), 0.5f);
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);
  const int ki = __float_as_int(tk) - 0x4B400000;   // == (int)k
  return __fmul_rn(p, __uint_as_float((uint32_t)(ki + 127) << 23));
}

// 2^x by the hardware approximation (flushes denormals; 2^-inf = 0); used
// where a few ulps do not matter (attention probabilities).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// trunc(x * 2^40) as int64 for |x| < 2^23, by exponent and mantissa shifts
// (bit-identical to converting the exact product x * 2^40 toward zero).
__device__ __forceinline__ long long q40_trunc(float x) {
  const uint32_t b = __float_as_uint(x);
  const int e = (int)((b >> 23) & 0xFFu);
  if (e == 0) return 0;                               // zero (no subnormal inputs here)
  const uint64_t m = (uint64_t)((b & 0x007FFFFFu) | 0x00800000u);
  const int sh = e - 127 - 23 + 40;                   // x * 2^40 = m * 2^sh
  const uint64_t v = sh >= 0 ? (m << sh) : (sh > -64 ? (m >> -sh) : 0ull);
  return (b >> 31) ? -(long long)v : (long long)v;
}

// Adds trunc(x * 2^40) to a Q40 sum kept in two parts.  A binary32 x with
// |x| >= 2^-17 is a multiple of 2^-40, so trunc(x 2^40) = x 2^40 exactly and
// a float64 sum of such x is exact while it stays below 2^13 in magnitude
// (a thread adds at most a few hundred terms of magnitude <= 1); smaller
// terms take the integer truncation.  q40_total joins the parts exactly.
__device__ __forceinline__ void q40_add(float x, long long& iq, double& dq) {
  if (fabsf(x) >= 7.62939453125e-06f) dq += (double)x;
  else iq += q40_trunc(x);
}
__device__ __forceinline__ long long q40_total(long long iq, double dq) {
  return iq + (long long)(dq * 1099511627776.0);   // dq 2^40 is an integer below 2^53
}

// cos(2 pi u) for u in (0,1): fold to b in [0,1/8] by the cosine symmetries,
// then the Taylor series of cos (through x^10) or sin (through x^11).
__device__ __forceinline__ float dg_cos2pif(float u) {
  float a = u > 0.5f ? __fsub_rn(1.0f, u) : u;
  const bool neg = a > 0.25f;
  if (neg) a = __fsub_rn(0.5f, a);
  const bool use_sin = a > 0.125f;
  const float b = use_sin ? __fsub_rn(0.25f, a) : a;
  const float x = __fmul_rn(b, DG_F(0x40C90FDBu));
  const float z = __fmul_rn(x, x);
  float r;
  if (use_sin) {
    float q = DG_F(0xB2D7322Bu);                          // -1/11!
    q = __fadd_rn(__fmul_rn(q, z), DG_F(0x3638EF1Du));    // 1/9!
    q = __fadd_rn(__fmul_rn(q, z), DG_F(0xB9500D01u));    // -1/7!
    q = __fadd_rn(__fmul_rn(q, z), DG_F(0x3C088889u));    // 1/5!
    q = __fadd_rn(__fmul_rn(q, z), DG_F(0xBE2AAAABu));    // -1/3!
    q = __fadd_rn(__fmul_rn(q, z), 1.0f);
    r = __fmul_rn(x, q);
  } else {
    float q = DG_F(0xB493F27Eu);                          // -1/10!
    q = __fadd_rn(__fmul_rn(q, z), DG_F(0x37D00D01u));    // 1/8!
    q = __fadd_rn(__fmul_rn(q, z), DG_F(0xBAB60B61u));    // -1/6!
    q = __fadd_rn(__fmul_rn(q, z), DG_F(0x3D2AAAABu));    // 1/4!
    q = __fadd_rn(__fmul_rn(q, z), -0.5f);
    r = __fadd_rn(__fmul_rn(q, z), 1.0f);
  }
  return neg ? -r : r;
}

// Gumbel noise -ln(-ln u).
__device__ __forceinline__ float gumbel_of(uint32_t word) {
  return -dg_logf(-dg_logf(uniform_open(word)));
}

// Thread-block clusters: barrier over every thread of every CTA of the
// cluster (release / acquire), and distributed shared memory addressing.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}

// Address of `p` (this CTA's shared memory) in the shared memory of cluster CTA `rank`.
template <typename P>
__device__ __forceinline__ const P* cluster_peer(const P* p, int rank) {
  uint64_t out;
  asm volatile("mapa.u64 %0, %1, %2;" : "=l"(out) : "l"((uint64_t)p), "r"(rank));
  return reinterpret_cast<const P*>(out);
}

// ---------------------------------------------------------------------------
// Bounded waiting: every spin gives up after ~2 s of wall time (globaltimer)
// and reports failure instead of hanging the GPU.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
constexpr int kSMs = 148;   // streaming multiprocessors of a B200


constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Returns false (and records `code`) if the phase did not complete in time.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err, int code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0 && global_ns() - t0 > kWaitLimitNs) {
      dev_error(err, code);
      return false;
    }
  }
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// ---------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor), no multicast.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"((uint64_t)map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"((uint64_t)map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)map) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: TMEM allocation, MMA issue, commit, loads/stores, fences.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  const uint32_t z = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(z), "r"(z), "r"(z), "r"(z)
      : "memory");
}
// Arrive on `bar` once every previously issued tcgen05.mma of this thread is done.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor for a K-major tile stored by TMA with
// 128-byte swizzle: rows of 128 B, 8-row atoms 1024 B apart (SBO), start
// address 1024-aligned for the tile; +32 B per 16-element K step.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;             // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;   // stride byte offset
  d |= (uint64_t)1 << 46;             // descriptor version for sm_100
  d |= (uint64_t)2 << 61;             // 128-byte swizzle
  return d;
}

// 32 lanes x 32-bit, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// Issue-only variants: several loads (or stores) in flight, then one wait.
__device__ __forceinline__ void tmem_ld16_nw(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st16_nw(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
