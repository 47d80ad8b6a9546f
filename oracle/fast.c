/* Plain-C twins of the oracle's slowest numpy loops (weight generation and
 * the per-row sampler pass), for the workloads the numpy versions cannot
 * finish in seconds.
 *
 * TEST INFRASTRUCTURE ONLY: built and loaded by oracle/_native.py for the
 * tests, the smoke check and the bench's CPU-baseline leg.  Shares no code
 * with the CUDA library.  Every function repeats, operation for operation,
 * the binary32 sequence of its numpy definition in oracle/numerics.py and
 * oracle/sampler.py (tests assert bit equality), compiled with
 * -ffp-contract=off so no multiply-add is fused.
 *
 * Definitions: Philox4x32-10 (Salmon et al., SC'11, section 3.2); log by
 * exponent split + atanh series; exp by Cody-Waite reduction + Taylor
 * series; cos(2 pi u) by octant folding + Taylor series; Box-Muller normals.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static inline float bits_f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static inline uint32_t f_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static void philox(uint32_t c[4], uint32_t k0, uint32_t k1) {
  for (int r = 0; r < 10; ++r) {
    if (r) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
    uint64_t p0 = (uint64_t)c[0] * 0xD2511F53u;
    uint64_t p1 = (uint64_t)c[2] * 0xCD9E8D57u;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0; c[1] = lo1; c[2] = n2; c[3] = lo0;
  }
}

static inline float uniform_open(uint32_t x) {
  return (float)((x >> 9) * 2u + 1u) * 5.9604644775390625e-08f; /* 2^-24 */
}

/* Constants: each is the binary32 rounding of the stated real number. */
static float LN2_HI, LN2_LO, INV_LN2, TWO_PI;
static float AT[5], EC[6], CC[5], SC[5];
static int consts_ready = 0;

static void init_consts(void) {
  if (consts_ready) return;
  double ln2 = log(2.0);
  LN2_HI = bits_f(f_bits((float)ln2) & 0xFFFFFF00u);
  LN2_LO = (float)(ln2 - (double)LN2_HI);
  INV_LN2 = (float)(1.0 / ln2);
  TWO_PI = (float)(2.0 * 3.14159265358979323846);
  const int at[5] = {11, 9, 7, 5, 3};
  for (int i = 0; i < 5; ++i) AT[i] = (float)(1.0 / at[i]);
  double f = 1.0; double fact[12]; fact[0] = 1.0;
  for (int n = 1; n < 12; ++n) { f *= n; fact[n] = f; }
  const int en[6] = {7, 6, 5, 4, 3, 2};
  for (int i = 0; i < 6; ++i) EC[i] = (float)(1.0 / fact[en[i]]);
  CC[0] = (float)(-1.0 / fact[10]); CC[1] = (float)(1.0 / fact[8]); CC[2] = (float)(-1.0 / fact[6]);
  CC[3] = (float)(1.0 / fact[4]); CC[4] = -0.5f;
  SC[0] = (float)(-1.0 / fact[11]); SC[1] = (float)(1.0 / fact[9]); SC[2] = (float)(-1.0 / fact[7]);
  SC[3] = (float)(1.0 / fact[5]); SC[4] = (float)(-1.0 / 6.0);
  consts_ready = 1;
}

static float log_f32(float x) {
  uint32_t b = f_bits(x);
  int e = (int)(b >> 23) - 127;
  uint32_t mb = (b & 0x007FFFFFu) | 0x3F800000u;
  if (mb > 0x3FB504F3u) { mb -= 0x00800000u; e += 1; }
  float m = bits_f(mb);
  float s = (m - 1.0f) / (m + 1.0f);
  float z = s * s;
  float p = AT[0];
  for (int i = 1; i < 5; ++i) p = p * z + AT[i];
  p = p * z + 1.0f;
  float lnm = (s + s) * p;
  float ef = (float)e;
  return ef * LN2_HI + (ef * LN2_LO + lnm);
}

static float exp_f32(float x) {
  if (x < -86.0f) return 0.0f;
  float t = x * INV_LN2;
  float k = rintf(t);
  float r = (x - k * LN2_HI) - k * LN2_LO;
  float p = EC[0];
  for (int i = 1; i < 6; ++i) p = p * r + EC[i];
  p = p * r + 1.0f;
  p = p * r + 1.0f;
  int ki = (int)k;
  return p * bits_f((uint32_t)(ki + 127) << 23);
}

static float cos2pi_f32(float u) {
  float a = u > 0.5f ? 1.0f - u : u;
  int neg = a > 0.25f;
  if (neg) a = 0.5f - a;
  int use_sin = a > 0.125f;
  float b = use_sin ? 0.25f - a : a;
  float x = b * TWO_PI;
  float z = x * x;
  float r;
  if (use_sin) {
    float q = SC[0];
    for (int i = 1; i < 5; ++i) q = q * z + SC[i];
    q = q * z + 1.0f;
    r = x * q;
  } else {
    float q = CC[0];
    for (int i = 1; i < 5; ++i) q = q * z + CC[i];
    r = q * z + 1.0f;
  }
  return neg ? -r : r;
}

static inline float round_bf16(float w) {
  uint32_t b = f_bits(w);
  uint32_t lsb = (b >> 16) & 1u;
  return bits_f((b + 0x7FFFu + lsb) & 0xFFFF0000u);
}

/* Weights of one tensor: elements [start, start+count) of its row-major
 * order; see oracle/model.py for the definition. */
void oc_weights(uint64_t seed, uint32_t tensor_id, uint64_t start, uint64_t count, int bf16,
                float* out) {
  init_consts();
  uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < (int64_t)count; ++i) {
    uint64_t j = start + (uint64_t)i;
    uint32_t c[4] = {(uint32_t)j, (uint32_t)(j >> 32), tensor_id, 3u};
    philox(c, k0, k1);
    float u1 = uniform_open(c[0]), u2 = uniform_open(c[1]);
    float r = sqrtf(log_f32(u1) * -2.0f);
    float z = r * cos2pi_f32(u2);
    float w = 0.02f * z;
    out[i] = bf16 ? round_bf16(w) : w;
  }
}

/* One sampler pass over `rows` logit rows of one canvas (row i = position
 * pos0 + i): decision-precision entropy, argmax, Gumbel-max token at 1/T =
 * inv_t, and optionally the untempered probabilities.  Mirrors
 * oracle/sampler.py row_stats + gumbel_argmax. */
void oc_sampler_rows(const float* logits, int64_t rows, int64_t vocab, uint64_t seed,
                     uint32_t canvas_id, uint32_t pos0, uint32_t step, float inv_t,
                     float* H, int32_t* amax, int32_t* tok, int64_t* s_q, int64_t* u_q,
                     float* probs) {
  init_consts();
  uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32) ^ canvas_id;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < rows; ++r) {
    const float* l = logits + r * vocab;
    float m = l[0]; int32_t am = 0;
    for (int64_t v = 1; v < vocab; ++v) if (l[v] > m) { m = l[v]; am = (int32_t)v; }
    int64_t sq = 0, uq = 0;
    float best = 0.0f; int32_t bt = -1;
    uint32_t w[4] = {0, 0, 0, 0};
    for (int64_t v = 0; v < vocab; ++v) {
      float d = l[v] - m;
      float e = exp_f32(d);
      sq += (int64_t)(e * 1099511627776.0f);          /* 2^40, truncation */
      uq += (int64_t)((e * d) * 1099511627776.0f);
      if ((v & 3) == 0) {
        w[0] = (uint32_t)(v >> 2); w[1] = pos0 + (uint32_t)r; w[2] = step; w[3] = 0u;
        philox(w, k0, k1);
      }
      float u = uniform_open(w[v & 3]);
      float key = l[v] * inv_t + -log_f32(-log_f32(u));
      if (bt < 0 || key > best) { best = key; bt = (int32_t)v; }
    }
    float sf = (float)sq, uf = (float)uq;
    float h = log_f32(sf * 9.094947017729282e-13f) - uf / sf;  /* 2^-40 */
    H[r] = h; amax[r] = am; tok[r] = bt; s_q[r] = sq; u_q[r] = uq;
    if (probs) {
      float inv_s = 1.0f / (sf * 9.094947017729282e-13f);
      for (int64_t v = 0; v < vocab; ++v) probs[r * vocab + v] = exp_f32(l[v] - m) * inv_s;
    }
  }
}
