/*
 * dg_test.h -- kernel-level entry points of the denoising-step library, used
 * by the parity tests and the benchmark.  Same conventions as dg.h: device
 * pointers unless marked "host", caller-owned buffers, asynchronous on
 * `stream`, status codes, no exceptions.  Hooks marked "allocates" take
 * temporary device memory and synchronise `stream` before returning.
 */
#ifndef DG_TEST_H
#define DG_TEST_H

#include "dg.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Fixed-sequence binary32 math of the sampler and the weight generator,
 * elementwise over n values:
 *   which 0: natural log of positive normal float `in`
 *   which 1: e^x for float x <= 0 (0 below -86)
 *   which 2: cos(2 pi u) for float u in (0,1)
 *   which 3: Gumbel noise -ln(-ln u(w)) of uint32 words w
 *   which 4: weight value 0.02 * BoxMuller(Philox(seed, (j, tensor_id, 3)))
 *            for uint64 indices j in `in` (seed = aux0, tensor_id = aux1). */
dg_status dg_test_math(int32_t which, const void* in, float* out, int64_t n, uint64_t aux0, uint32_t aux1,
                       void* stream);

/* The top-k-truncated sampler kernel (DiffusionGemma technical-report
 * explainer, section 九): as dg_test_sampler for H, argmax and S_q/U_q; the
 * token is the Gumbel-max draw among the K largest logits of the row (value
 * descending, ties to the lower index; noise as in the exact sampler);
 * cand_ids int32 [rows, K] lists them best first and cand_w [rows, K] (bf16
 * if w_bf16 else fp32) holds w_j = e_j (1/s), e_j = exp(l_j - max),
 * s = e_0 + ... + e_{K-1} summed in that order.  vocab a multiple of 32,
 * 1 <= K <= min(256, vocab) (DG_ERR_INVALID_ARG otherwise).  Asynchronous. */
dg_status dg_test_sampler_topk(const float* logits, int32_t rows, int32_t vocab, int32_t positions, uint64_t seed,
                               int32_t step, float t, float temp_start, float temp_end, int32_t K, float* H,
                               int32_t* tok, int32_t* amax, int64_t* s_q, int64_t* u_q, int32_t* cand_ids,
                               void* cand_w, int32_t w_bf16, void* stream);

/* Self-conditioning gather of a truncated distribution (the previous
 * round's prediction fed back, DiffusionGemma technical-report explainer,
 * section 二, restricted to the top-k candidates of section 九): u [rows, d] =
 * sum_j cand_w[r][j] emb[cand_ids[r][j]] (fp32 in candidate order, stored
 * bf16 if bf16 else fp32; emb [*, d] in the same dtype).  d a multiple of
 * 64, 1 <= K <= 256.  Asynchronous. */
dg_status dg_test_sc_gather(const int32_t* cand_ids, const void* cand_w, int32_t rows, int32_t K, const void* emb,
                            int32_t d, int32_t bf16, void* u, void* stream);

/* Philox4x32-10 of n (counter[4], key[2]) records: in uint32 [n,6] ->
 * out uint32 [n,4] (Salmon et al., SC'11). */
dg_status dg_test_philox(const uint32_t* in, uint32_t* out, int64_t n, void* stream);

/* The vocab sampler kernel on caller logits fp32 [rows, vocab] (row = canvas
 * * positions + position; canvas = row / positions keys the Philox stream):
 * entropy H, Gumbel-max token at T = temp_end + (temp_start - temp_end) t,
 * argmax, exact fixed-point sums S_q/U_q (2^-40 units, may be NULL) and the
 * probabilities (bf16 if probs_bf16 else fp32; may be NULL).  vocab must be
 * a multiple of 32 (DG_ERR_INVALID_ARG otherwise). */
dg_status dg_test_sampler(const float* logits, int32_t rows, int32_t vocab, int32_t positions, uint64_t seed,
                          int32_t step, float t, float temp_start, float temp_end, float* H, int32_t* tok,
                          int32_t* amax, int64_t* s_q, int64_t* u_q, void* probs, int32_t probs_bf16,
                          void* stream);

/* The commit / re-noise / stop kernel for B canvases of 256 positions.
 * prev_amax (in/out) holds the previous round's argmax and is overwritten. */
dg_status dg_test_commit(const float* H, const int32_t* tok, const int32_t* amax, int32_t* prev_amax, int32_t B,
                         int32_t vocab, uint64_t seed, int32_t step, int32_t max_steps, int32_t commit_mode,
                         float commit_bound, int32_t stop_mode, float stop_bound, uint8_t* commit,
                         int32_t* canvas_next, int32_t* stop, int32_t* n_committed, void* stream);

/* Dense GEMM out[split][n][m] = alpha * sum_{k in split} A[m][k] B[n][k]
 * (A [M,K], B [N,K] row-major, bf16 through tcgen05 when bf16 != 0, else
 * fp32 SIMT); out holds k_splits partial slabs of N*M floats; bn in
 * {32,64,128,256} is the token tile (bf16 only); flags bit 0 selects the
 * persistent tile-walking kernel, bit 1 (bn 256, not persistent) 256-row
 * tiles with two accumulators.  Allocates (a 32-byte error word). */
dg_status dg_test_gemm(const void* A, const void* B, float* out, int32_t M, int32_t N, int32_t K, int32_t bf16,
                       float alpha, int32_t k_splits, int32_t bn, int32_t flags, void* stream);

/* The bf16 router kernel: logits r = x Wr^T (+ bias, fp32, may be NULL) for
 * x bf16 [T, d] and Wr bf16 [E, d] (E <= 128, d % 64 == 0), then per token
 * the k <= 32 largest logits (ties to the lower expert id) in descending
 * order -> ids int32 [T, k], and their softmax -> gate fp32 [T, k]
 * (Mixture-of-Experts FFN, DiffusionGemma technical-report explainer,
 * section 二).  Allocates (a 32-byte error word); synchronises. */
dg_status dg_test_router(const void* x, const void* wr, const float* bias, const float* tok_bias, int32_t T,
                         int32_t d, int32_t E, int32_t k, int32_t* ids, float* gate, void* stream);

/* Structured per-token router bias for the canvas passes (routing-locality
 * workloads: a stand-in for the expert locality of a trained router, which
 * the DiffusionGemma technical-report explainer, section 五, puts at about
 * 84 of 128 experts per round).  bias: device fp32 [L][n_tok][E], owned by
 * the caller and read by every later canvas round until replaced; row
 * b*256 + i biases canvas b, position i; the router adds it to the logits
 * (selection and gates).  n_tok = 0 (bias may be NULL) removes it.  n_tok
 * must be a multiple of 256 and at most max_canvases*256, and a later round
 * over more canvases than n_tok/256 fails with DG_ERR_INVALID_ARG.  Drops
 * the captured block loop (the next block recaptures it).  Host-only. */
dg_status dg_set_routing_bias(dg_model* m, const float* bias, int32_t n_tok);

/* Grouped GEMM as used by the experts: A [groups*M, K], B [rows, K] with
 * rows ordered by group (counts host int32 [groups]); out [rows, M] fp32,
 * out[r][m] = sum_k A[g(r)*M + m][k] B[r][k]; flags bit 0 as dg_test_gemm,
 * bit 1 (persistent only) sizes the ring stages from the largest item, bit 2
 * (persistent, bf16, M % 128 == 0) applies SwiGLU in the epilogue: A rows
 * interleave gate / up in blocks of 64 and out receives bf16 [rows][M/2],
 * out[r][f] = round(silu(g) u) with g, u the rows 128 (f/64) + f%64 (+64);
 * bit 3 (persistent, bn 256) uses 256-row tiles (two accumulators per CTA).
 * Allocates. */
dg_status dg_test_grouped_gemm(const void* A, const void* B, const int32_t* counts, int32_t groups, int32_t M,
                               int32_t K, int32_t bf16, int32_t bn, int32_t flags, float* out, void* stream);

/* Split-KV plan of the bf16 attention kernel (host only, no device call):
 * out int32[5] = {query tiles per (canvas, KV head), key splits, 64-key
 * blocks per split, CTAs, 1 if the splits of a query-tile pair merge inside
 * the kernel as one thread-block cluster (at most 8 splits) else 0} for n_q
 * queries per canvas, G query heads per KV head, n_keys keys, rows = query
 * rows of the launch and part_rows_cap = rows the partial-output buffer
 * holds per split sum (binding only when the splits merge through it). */
/* Launch choices of the step that depend only on the shape (host only, no
 * device call).  out int32[2]: out[0] = CTAs per row of the vocab samplers
 * for a vocabulary of `vocab` entries and `rows` logit rows (one
 * thread-block cluster per row: 8 above 65536 entries; else 1 when the rows
 * alone give every SM four CTAs, 2 otherwise); out[1] = 1 when the permute
 * and the expert-row gather run as one kernel for `n_pairs` (token, slot)
 * pairs over `n_experts` experts (the permutation fits 96 KB of shared
 * memory), else 0.  DG_ERR_INVALID_ARG for a null out or non-positive
 * sizes. */
dg_status dg_test_launch_shape(int32_t vocab, int64_t rows, int32_t n_experts, int32_t n_pairs, int32_t* out);

/* Thread-block clusters of the bf16 attention kernel that the device can
 * hold at once, per cluster size (the capacity the split-KV plan is given):
 * out int32[9], out[c] for c = 1..8, out[0] = 0; 0 where the device refuses
 * the query.  Host memory; needs a device; does not synchronise. */
dg_status dg_test_attn_capacity(int32_t* out);

dg_status dg_test_attn_plan(int64_t n_q, int32_t G, int32_t Hkv, int32_t n_canvas, int32_t n_keys, int64_t rows,
                            int64_t part_rows_cap, int32_t* out);

/* FP8 expert-weight quantisation (OCP E4M3, one power-of-two scale per 128
 * inputs of each row: s = 2^ceil(log2(amax / 448)), q = RNE(w / s); a
 * reading of the FP8 deployment in the DiffusionGemma release news, section
 * "速度数据"): w bf16 [rows, K] -> codes uint8 [rows, K], scales fp32
 * [rows, ceil(K / 128)].  Asynchronous. */
dg_status dg_test_quant_fp8(const void* w, int64_t rows, int32_t K, uint8_t* codes, float* scales, void* stream);

/* Grouped GEMM over FP8 weights (the experts of the Mixture-of-Experts FFN,
 * explainer section 二, stored as in dg_test_quant_fp8): A8 codes [groups*M, K] with scales
 * [groups*M, ceil(K/128)], B bf16 [rows, K] ordered by group (counts host
 * int32 [groups]); out fp32 [k_splits][rows][M], the split-K partials
 * (K chunks of 128 divided evenly, the last split taking the rest):
 * out[s][r][m] = sum over the split's inputs of (q s)[g(r)*M + m][k] B[r][k].
 * K a multiple of 16; bn in {32, 64, 128, 256}.  Allocates; synchronises. */
dg_status dg_test_grouped_gemm_fp8(const uint8_t* A8, const float* scales, const void* B, const int32_t* counts,
                                   int32_t groups, int32_t M, int32_t K, int32_t bn, int32_t k_splits, float* out,
                                   void* stream);

/* Attention kernels (tcgen05 for bf16, SIMT for fp32) plus the split
 * merge, on plain layouts: q [n_canvas*n_q, Hq, hd], k and v
 * [n_canvas, Hkv, n_keys, hd] -> out fp32 [n_canvas*n_q, Hq*hd].  Query i of
 * a canvas sits at position q_pos0 + i; causal != 0 hides keys after it.
 * force_path (bf16): 0 = the plan's choice, 1 = split partials in global
 * memory merged by the combine kernel, 2 = merge inside the kernel across a
 * cluster of at most 8 splits (bf16 output, widened to fp32 here); path_out
 * (host, may be NULL) receives the path taken (1 or 2; 1 for fp32).
 * Allocates. */
dg_status dg_test_attention(const void* q, const void* k, const void* v, int32_t n_canvas, int32_t n_q,
                            int32_t q_pos0, int32_t n_keys, int32_t causal, int32_t Hq, int32_t Hkv,
                            int32_t head_dim, int32_t bf16, int32_t force_path, int32_t* path_out, float* out,
                            void* stream);

/* Copy weight tensor `tensor_id` (0 = E [V,d], 1 = W_sc [d,d]; layer l:
 * 16+16l + {0 Wq,1 Wk,2 Wv,3 Wo,4 Wr,5 Wg [E,ff,d],6 Wu,7 Wd [E,d,ff]})
 * into dst in its logical row-major layout, model dtype. */
dg_status dg_read_weight(const dg_model* model, int32_t tensor_id, void* dst, void* stream);

/* Store prompt keys/values k, v [L, B, Hkv, P, hd] (model dtype; keys
 * already rotated) into the library's cache layout inside `kv`. */
dg_status dg_load_kv(dg_model* model, void* kv, int32_t B, int32_t P, const void* k, const void* v, void* stream);

/* Run `reps` single denoising rounds (step 0, t = 1, self-conditioning on)
 * with a CUDA event pair around every kernel launch on `stream`; returns
 * per-phase total milliseconds and launch counts (host arrays of n_phases;
 * phase names from dg_phase_name).  Synchronises. */
dg_status dg_profile_step(dg_model* model, void* kv, int32_t B, int32_t P, int32_t reps, float* phase_ms,
                          int32_t* phase_launches, int32_t n_phases, void* stream);

/* Name of profile phase i, or NULL past the last one. */
const char* dg_phase_name(int32_t i);

/* Per-layer, per-expert row counts of the most recent call (device int32
 * [n_layers][n_experts]); the nonzero entries of row l are the distinct
 * experts layer l streamed. */
dg_status dg_expert_counts(const dg_model* model, int32_t* counts, void* stream);

/* Distinct experts each layer streamed, summed over every canvas pass (one
 * per layer per denoising round, in single steps and in the block loop; the
 * prompt encode is not counted) since the model was created or last reset:
 * per_layer host uint64 [n_layers] (may be NULL when only resetting);
 * reset != 0 zeroes the sums afterwards.  Synchronises when reading. */
dg_status dg_touched_experts_sum(dg_model* model, uint64_t* per_layer, int32_t reset, void* stream);

/* Diagnostic trace of later eager calls (dg_denoise_step, dg_encode_prompt):
 * for every layer l, h after the attention residual -> h_trace[l][0][T][d]
 * and after the MoE -> h_trace[l][1][T][d], then the final RMSNorm(h) ->
 * h_trace[L][0][T][d] (fp32; the buffer holds 2L+1 slabs of T*d), and the
 * routing ids -> ids_trace[l][T][top_k] (T = tokens of the call).  Both NULL turns it off;
 * the block-loop graph never traces.  Buffers are the caller's. */
dg_status dg_debug_trace(dg_model* model, float* h_trace, int32_t* ids_trace);

/* One transformer layer of the canvas pass from a given residual state
 * (DiffusionGemma technical-report explainer, section 二: a pre-norm block
 * of bidirectional attention over [prompt KV ; canvas] and the top-k MoE
 * FFN).  h_in: device [B*256][d] in the model dtype, the residual stream
 * entering layer `layer`; the layer normalises it, attends with the canvas
 * at positions P..P+255 over the prompt keys/values the caller stored in
 * `kv` (dg_load_kv) plus its own, and writes the canvas keys/values of that
 * layer into `kv`.  Outputs (device, caller-owned): h_trace fp32
 * [3][B*256][d] = h after the attention residual, h after the MoE, and
 * RMSNorm of the latter; ids int32 [B*256][top_k] = the routing (slot order).
 * A per-token router bias set by dg_set_routing_bias applies.  Synchronises;
 * DG_ERR_INVALID_ARG for a bad layer or shape, a device error code otherwise. */
dg_status dg_test_layer(dg_model* model, void* kv, int32_t B, int32_t P, int32_t layer, const void* h_in,
                        float* h_trace, int32_t* ids, void* stream);

/* The MoE half of one layer of the canvas pass from a given state
 * (DiffusionGemma technical-report explainer, section 二: the top-k MoE FFN
 * after the attention residual).  h_attn: device [B*256][d] in the model
 * dtype, the residual stream after the layer's attention; the call
 * normalises it, routes each token to its top-k experts (a router bias set
 * by dg_set_routing_bias applies), runs the experts and adds the gated sum
 * to the stream.  Outputs (device, caller-owned): h_trace fp32 [3][B*256][d]
 * whose rows [1] = h after the MoE and [2] = RMSNorm of it (rows [0] are not
 * written); ids int32 [B*256][top_k] = the routing (slot order).
 * Synchronises; DG_ERR_INVALID_ARG for a bad layer or B, a device error code
 * otherwise. */
dg_status dg_test_moe(dg_model* model, int32_t B, int32_t layer, const void* h_attn, float* h_trace,
                      int32_t* ids, void* stream);

/* Kernel launches recorded in one captured block-loop round (graph body). */
int32_t dg_launches_per_round(const dg_model* model);

#ifdef __cplusplus
}
#endif

#endif /* DG_TEST_H */
