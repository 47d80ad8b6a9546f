/*
 * dg.h -- C ABI of the B200 block-text-diffusion denoising step.
 *
 * What the library computes (DiffusionGemma technical-report explainer,
 * mlqm.cn, sections 一, 二 and 四; "谷歌都下场了：扩散语言模型的四倍速与六倍错",
 * bohuyeshan.top, section 一):
 *   - a prompt is encoded with CAUSAL attention into a cached KV;
 *   - a 256-token canvas of uniform-noise tokens is refined round after round
 *     by the same weights with BIDIRECTIONAL attention over [prompt ; canvas],
 *     a top-k Mixture-of-Experts SwiGLU FFN, and a self-conditioning input
 *     carrying the previous round's predicted distribution;
 *   - an entropy-bounded sampler follows each round: per-position entropy,
 *     Gumbel-max sampling at a temperature falling linearly 0.8 -> 0.4,
 *     commit of low-entropy positions, uniform re-noising of the rest, and an
 *     adaptive stop.
 *
 * Conventions (every entry point):
 *   - Device pointers are raw CUDA device addresses on the current device;
 *     host pointers are marked "host".  The caller owns every buffer it
 *     passes; the library owns the weights and its workspace (dg_model).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     enqueued asynchronously and return at once; argument errors are
 *     returned immediately, device-side errors (a bad token id, a wait that
 *     ran out) are latched in the model and returned by dg_sync_status.
 *   - No C++ exception crosses this boundary.  A call that returns an error
 *     leaves the model usable unless it returns DG_ERR_CUDA.
 *   - Token ids are int32 in [0, vocab).  Layouts are row-major.
 *   - One model must not be used from two streams at the same time.
 */
#ifndef DG_H
#define DG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DG_OK = 0,
  DG_ERR_INVALID_ARG = 1, /* a pointer, size or config field is out of range */
  DG_ERR_OOM = 2,         /* device allocation failed (nothing is leaked)     */
  DG_ERR_CUDA = 3,        /* a CUDA call failed; the context may be unusable  */
  DG_ERR_TIMEOUT = 4,     /* a bounded device wait gave up                    */
  DG_ERR_STATE = 5,       /* wrong call order, or a device-side index error   */
  DG_ERR_UNSUPPORTED = 6  /* shape or feature this build does not handle      */
} dg_status;

enum { DG_FP32 = 0, DG_BF16 = 1 };
enum { DG_COMMIT_THRESH = 0, DG_COMMIT_EB = 1 };
enum { DG_STOP_MEAN = 0, DG_STOP_EB = 1 };

/* Architecture + sampler.  Requirements checked by dg_init_weights:
 * canvas_len == 256; head_dim in {64, 128} (128 for DG_BF16); n_heads a
 * multiple of n_kv_heads with 128 % (n_heads / n_kv_heads) == 0;
 * d_model, d_ff multiples of 64; vocab a multiple of 64; top_k <= n_experts
 * <= 1024, top_k <= 64; 1 <= max_canvases; max_prompt >= 1;
 * 0 <= sample_topk <= min(256, vocab); expert_fp8 in {0, 1}, 1 only with
 * DG_BF16. */
typedef struct dg_config {
  int32_t n_layers, d_model, n_heads, n_kv_heads, head_dim;
  int32_t n_experts, top_k, d_ff, vocab;
  int32_t dtype;          /* DG_FP32 or DG_BF16: storage of weights/activations */
  float logit_scale;      /* multiplier on the final logits                      */
  float rope_theta;       /* RoPE base (rotate-half pairs i, i + head_dim/2)     */
  float rms_eps;          /* RMSNorm epsilon (unit gains)                        */
  float zipf_s;           /* router bias -zipf_s * ln(e + 1); 0 = none           */
  float temp_start;       /* temperature at the first round (0.8)                */
  float temp_end;         /* temperature at the last round (0.4)                 */
  int32_t max_steps;      /* round budget N of dg_generate_block                 */
  int32_t commit_mode;    /* DG_COMMIT_THRESH (entropy < bound) or DG_COMMIT_EB  */
  float commit_bound;     /* 0.5 nats (THRESH) or cumulative 0.1 (EB)            */
  int32_t stop_mode;      /* DG_STOP_MEAN or DG_STOP_EB                          */
  float stop_bound;       /* mean-entropy bound: 0.1 (MEAN) or 0.005 (EB)        */
  int32_t canvas_len;     /* must be 256                                         */
  int32_t max_canvases;   /* largest batch B passed to any call                  */
  int32_t max_prompt;     /* largest prompt length P passed to any call          */
  uint64_t sample_seed;   /* Philox key of all sampling draws                    */
  int32_t sample_topk;    /* 0: exact sampling over the vocabulary.  K > 0: top-k
                             truncation (DiffusionGemma technical-report
                             explainer, section 九: the large-batch sampler
                             optimisation) -- the token is the Gumbel-max draw
                             among the K largest logits (same noise per token id
                             as the exact draw), self-conditioning uses the
                             untempered probabilities renormalised over those K;
                             entropy, argmax, commit and stop are unchanged.    */
  int32_t expert_fp8;     /* 1: expert weights (gate, up, down) stored as OCP E4M3
                             codes with one power-of-two scale per 128 inputs of
                             each row, s = 2^ceil(log2(amax / 448)), q = RNE(w/s)
                             (a reading of the FP8 deployment in the release news,
                             section "速度数据"); the model computes with q s,
                             exactly a bf16 value.  DG_BF16 only.                */
} dg_config;

typedef struct dg_model dg_model;

/* Outputs of one denoising round for B canvases.  Every pointer is a device
 * buffer owned by the caller; any may be NULL except `tokens`. */
typedef struct dg_step_out {
  float* logits;          /* fp32 [B,256,vocab]: logit_scale * RMSNorm(h) E^T      */
  float* entropy;         /* fp32 [B,256]: entropy (nats) of softmax(logits)       */
  int32_t* tokens;        /* int32 [B,256]: Gumbel-max sample at the round's T     */
  int32_t* argmax;        /* int32 [B,256]: argmax of the logits                   */
  uint8_t* commit;        /* uint8 [B,256]: 1 where the position graduates         */
  int32_t* canvas_next;   /* int32 [B,256]: sample where committed, else fresh noise */
  void* selfcond_next;    /* model dtype [B,256,d_model]: next round's input       */
  int32_t* stop;          /* int32 [B]: 1 when the stop rule fires this round      */
  int32_t* n_committed;   /* int32 [B]: committed positions this round             */
} dg_step_out;

/* Allocate a model and fill every weight on the device from the counter-based
 * generator: w = round(0.02 * sqrt(-2 ln u1) * cos(2 pi u2)), u1/u2 from
 * Philox4x32-10 keyed by `seed`, counter (element index, tensor id, 3)
 * (Salmon et al., SC'11).  `cfg` (host) is copied.  On success *out owns all
 * device memory; free it with dg_free.  Errors: DG_ERR_INVALID_ARG (config),
 * DG_ERR_OOM, DG_ERR_CUDA. */
dg_status dg_init_weights(const dg_config* cfg, uint64_t seed, void* stream, dg_model** out);

/* Release everything the model owns (synchronises its stream).  NULL is a no-op. */
dg_status dg_free(dg_model* model);

/* Bytes of the KV-cache buffer for B canvases with P-token prompts: keys
 * [L][B][Hkv][S][hd] followed by transposed values [L][B][Hkv][hd][S],
 * S = round_up(P + 256, 64), model dtype.  0 if B or P is out of range. */
size_t dg_kv_bytes(const dg_model* model, int32_t B, int32_t P);

/* Causal encode (explainer section 二: the prompt is read with causal
 * attention and cached): prompt = device int32 [B,P]; writes the keys/values
 * of positions 0..P-1 of every layer into `kv` (device, dg_kv_bytes bytes,
 * owned by the caller; it is zeroed first).  No logits are produced. */
dg_status dg_encode_prompt(dg_model* model, const int32_t* prompt, int32_t B, int32_t P, void* kv,
                           void* stream);

/* One denoising round (explainer sections 二 and 四) for B canvases against
 * the encoded prompt `kv` (canvas keys/values are written into it):
 *   canvas    device int32 [B,256] current tokens;
 *   selfcond  device [B,256,d_model] in the model dtype, or NULL for zeros
 *             (the first round);
 *   step      round index s in [0, max_steps) (Philox counter, last-round
 *             stop, EB stop at s = 0);
 *   t         diffusion time in [0,1]; temperature T = temp_end +
 *             (temp_start - temp_end) * t.
 * Outputs as described in dg_step_out.  The EB stop rule compares with the
 * argmax of the previous dg_denoise_step call on the same model. */
dg_status dg_denoise_step(dg_model* model, void* kv, int32_t B, int32_t P, const int32_t* canvas,
                          const void* selfcond, int32_t step, float t, const dg_step_out* out,
                          void* stream);

/* A full block (explainer section 四): canvases start from uniform noise
 * (Philox stream 2), rounds run on the device until every canvas stops or
 * max_steps is reached, t_s = 1 - s/(max_steps - 1).  The loop is one CUDA
 * graph with a device-side while condition; a stopped canvas is frozen.
 * Outputs (device, caller-owned): canvas_out int32 [B,256] = sampled tokens
 * of the stopping round; steps_used int32 [B]; n_committed int32 [B]. */
dg_status dg_generate_block(dg_model* model, void* kv, int32_t B, int32_t P, int32_t* canvas_out,
                            int32_t* steps_used, int32_t* n_committed, void* stream);

/* Block-autoregressive generation (release news "不是逐词写，而是整块去噪";
 * "谷歌都下场了：扩散语言模型的四倍速与六倍错", section 一): the prompt is encoded
 * causally, then n_blocks canvases are generated one after another, each as
 * dg_generate_block does; a finished canvas joins the context by a causal
 * encode of its 256 tokens at positions P + 256 i, so block i attends to
 * [prompt ; blocks 0 .. i-1 ; its own canvas].  Block i samples with seed
 * sample_seed + i.
 *   prompt      device int32 [B, P].
 *   kv          caller buffer of dg_kv_bytes(model, B, P + 256 (n_blocks - 1))
 *               bytes; holds the whole context on return.
 *   tokens_out  device int32 [B, n_blocks, 256]: each block's sampled tokens.
 *   steps_used, n_committed  device int32 [B, n_blocks].
 * P + 256 (n_blocks - 1) must not exceed max_prompt, 1 <= B <= max_canvases
 * and n_blocks >= 1 (DG_ERR_INVALID_ARG otherwise, nothing enqueued).
 * Asynchronous on `stream`; a device-side wait that ran out is reported by the
 * next call or dg_sync_status.  The block loop's graph is re-captured for each
 * block (the canvas positions and the seed change). */
dg_status dg_generate(dg_model* model, const int32_t* prompt, int32_t B, int32_t P, int32_t n_blocks, void* kv,
                      int32_t* tokens_out, int32_t* steps_used, int32_t* n_committed, void* stream);

/* Wait for the model's stream and return the first latched device error
 * (DG_ERR_TIMEOUT, DG_ERR_STATE) or DG_OK; clears the latch. */
dg_status dg_sync_status(dg_model* model, void* stream);

/* Static text for a status code. */
const char* dg_status_string(dg_status status);

/* Number of kernels one dg_denoise_step launches for B canvases (the graph
 * body of one dg_generate_block round has the same count plus one). */
int32_t dg_kernels_per_step(const dg_model* model, int32_t B, int32_t P);

/* Split-K GEMM that allocates nothing.  The method pages have no counterpart
 * of this call; it is a deployment aid.  Some callers cannot allocate device
 * memory: serving loops that reserve all device memory up front, and code
 * that must not block other streams (cudaMalloc/cudaFree can synchronise the
 * device and fail under memory pressure).  For them this call keeps its
 * split-K partial sums in a fixed 64 MiB file-scope device array (every GPU
 * that loads the library holds it until the process exits) instead of a
 * workspace.
 *   out[n][m] = sum_k A[m][k] B[n][k]: A device bf16 [M,K], B device bf16
 *   [N,K] (row-major, K a multiple of 8), out device fp32 [N,M]; k_splits
 *   >= 1 is capped at ceil(K/64).  Inputs and outputs are the caller's.
 * Returns DG_ERR_INVALID_ARG when min(k_splits, ceil(K/64)) * N * M exceeds
 * 16 Mi floats (the array's size) or an argument is out of range.  The first
 * call on a device looks up the array's device address (once per device,
 * with that device current); make it before any stream capture.  The call
 * returns after the result is in `out` (it synchronises `stream`).  Every
 * call shares the one array, so calls that overlap on the GPU (other
 * streams, other host threads) race and must be serialised by the caller. */
dg_status dg_gemm_splitk_noalloc(const void* A, const void* B, float* out, int32_t M, int32_t N, int32_t K,
                                 int32_t k_splits, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DG_H */
