/*
 * dg.h -- C-ABI of libdg: the denoising pass of a block-diffusion ("uniform-state")
 * MoE language model on one B200 (sm_100a).
 *
 * What the calls compute (page title -- section):
 *   "DiffusionGemma" video explainer -- "The fix: a 256-token canvas": a canvas of
 *       token slots is refined in parallel over several denoising passes;
 *   same page -- "Uniform State Diffusion": noise is random vocabulary tokens, every
 *       position is updated in parallel, low-confidence tokens are re-noised with
 *       fresh random tokens, and passes repeat until the canvas converges;
 *   same page -- "Two modes, one model": prefill mode reads tokens with causal
 *       attention and writes the KV cache; denoising mode lets every canvas token
 *       attend to all canvas tokens and to the KV cache;
 *   same page -- "Long-form text: chaining canvases": each completed canvas is
 *       appended to the KV cache by a prefill step before the next canvas opens;
 *   "Module 12. Diffusion Language Models" exercises -- prefix/block mask solution:
 *       prefix rows causal, block rows see prefix and block; prefix K/V is reused
 *       across denoising steps unchanged;
 *   same page -- MoE remark: one pass reads the union of the experts its canvas
 *       positions route to.
 *
 * Conventions for every call:
 *   - All device pointers are owned by the caller; the library never frees them and
 *     allocates no device memory of its own.  Host structs are read during the call
 *     only (dg_model_create copies what it needs).
 *   - Work is enqueued asynchronously on the given stream (NULL = legacy default
 *     stream); the return code covers argument validation and launch errors only.
 *     Device-side failures (a bounded wait that timed out) are recorded in the
 *     workspace's error word and reported by dg_device_status.
 *   - On any error no kernel has been launched unless the code is DG_ERR_CUDA.
 *   - dg_last_error() returns a thread-local message for the last non-OK status.
 *
 * Data layouts (row-major; "bf16" = IEEE bfloat16 bits; the fp32 model uses float):
 *   weights, all [out_features][in_features] (y = x W^T):
 *     embed, w_out   [V][H]
 *     w_qkv          [(nq + 2 nkv) d][H]    rows of W_q, then W_k, then W_v
 *     w_o            [H][nq d]
 *     w_router       [E][H]                 always fp32
 *     w_gate, w_up   [E][F][H]              SwiGLU expert: h = silu(x W_gate^T) * (x W_up^T)
 *     w_down         [E][H][F]
 *   KV cache, per layer:  K [nkv][capacity][d],  V transposed: Vt [nkv][d][capacity]
 *   canvas / tokens int32 [n];  logits fp32 [C][V]
 */
#ifndef DG_H
#define DG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dg_stream; /* a cudaStream_t */

typedef enum dg_status {
  DG_OK = 0,
  DG_ERR_INVALID_ARG = -1, /* null pointer, bad size, unsupported shape for the dtype    */
  DG_ERR_CAPACITY = -2,    /* KV cache or workspace too small; nothing was changed        */
  DG_ERR_CUDA = -3,        /* a CUDA call failed; see dg_last_error()                      */
  DG_ERR_TIMEOUT = -4,     /* a device-side bounded wait gave up (from dg_device_status)   */
  DG_ERR_UNSUPPORTED = -5  /* valid shape that this build does not implement               */
} dg_status;

typedef enum dg_dtype { DG_DTYPE_BF16 = 0, DG_DTYPE_F32 = 1 } dg_dtype;

typedef struct dg_config {
  int32_t n_layers, hidden, n_q_heads, n_kv_heads, head_dim;
  int32_t n_experts, top_k, expert_ffn, vocab;
  float rope_theta; /* RoPE base (rotate-half pairs, absolute positions)             */
  float rms_eps;    /* RMSNorm epsilon (unit gain)                                   */
  int32_t dtype;    /* dg_dtype of weights, activations and KV cache                 */
} dg_config;
/* Shape rules.  Both dtypes: n_q_heads % n_kv_heads == 0, top_k <= min(16, n_experts),
 * n_experts <= 256, hidden % 64 == 0, expert_ffn % 64 == 0, vocab % 4 == 0,
 * head_dim even and <= 128.  bf16 additionally: head_dim == 128, hidden % 128 == 0. */

typedef struct dg_layer_weights {
  const void* w_qkv;
  const void* w_o;
  const float* w_router;
  const void* w_gate;
  const void* w_up;
  const void* w_down;
} dg_layer_weights;

typedef struct dg_weights {
  const void* embed;
  const void* w_out;
  const dg_layer_weights* layers; /* host array of n_layers */
} dg_weights;

typedef struct dg_kv_cache {
  void* const* k;   /* host array [n_layers] of device pointers, K  [nkv][capacity][d] */
  void* const* vt;  /* host array [n_layers] of device pointers, Vt [nkv][d][capacity] */
  int32_t capacity; /* positions per layer, multiple of 8                               */
  int32_t len;      /* valid positions [0, len); dg_prefill_append advances it          */
} dg_kv_cache;

typedef struct dg_model dg_model;

/* Validate the config, copy it and the weight pointers, and pre-encode the weight
 * tensor maps.  The weights must stay alive and unchanged while the model exists.
 * Every weight pointer must be 16-byte aligned (DG_ERR_INVALID_ARG otherwise): the
 * kernels read embedding and router rows with 16-byte loads and TMA needs aligned bases. */
dg_status dg_model_create(const dg_config* cfg, const dg_weights* w, dg_model** out);
void dg_model_destroy(dg_model* m);

/* Bytes of device workspace for calls on up to max_tokens tokens per call (canvas or
 * prefill length).  The caller allocates it (256-byte aligned), zero-fills it once, and
 * passes it to every call; its first 4 bytes are the device error word.  Calls that
 * share a workspace must be ordered on one stream (they reuse its buffers). */
size_t dg_workspace_bytes(const dg_config* cfg, int32_t max_tokens);
/* Workspace bytes dg_canvas_update needs on its own for a C x V logits matrix. */
size_t dg_update_workspace_bytes(int32_t C, int32_t V);

/* Prefill mode.  Runs the T tokens at positions len..len+T-1 through the stack with
 * causal attention over [0, len + i] and writes their K/V into every layer's cache at
 * [len, len + T); then cache->len += T.  No logits are produced.
 * DG_ERR_CAPACITY if len + T > capacity (cache and len unchanged). */
dg_status dg_prefill_append(dg_model* m, dg_kv_cache* cache, const int32_t* d_tokens, int32_t T, void* d_ws,
                            size_t ws_bytes, dg_stream stream);

/* Denoising mode.  One pass over the canvas at positions len..len+C-1: every canvas
 * query attends to cached keys [0, len) and all C canvas keys.  Writes
 * d_logits[C][V] (fp32).  The canvas K/V are written to cache slots [len, len+C) as
 * scratch; cache->len and slots [0, len) are never modified.
 * DG_ERR_CAPACITY if len + C > capacity. */
dg_status dg_denoise_pass(dg_model* m, const dg_kv_cache* cache, const int32_t* d_canvas, int32_t C,
                          float* d_logits, void* d_ws, size_t ws_bytes, dg_stream stream);

/* Canvas update.  For each row i of d_logits[C][V]: argmax (lowest id on ties) and
 * confidence = largest softmax probability.  Every position takes its argmax, then
 * the n_renoise lowest-confidence positions (lower position first on ties) take a
 * fresh token: SplitMix64 draw number (step << 32 | i) of the stream seeded with
 * `seed`, mapped to [0, V) as (draw >> 32) * V >> 32.  Writes d_canvas[C]; writes
 * d_conf[C] if not NULL.  C <= 1024, V % 4 == 0, 0 <= n_renoise <= C. */
dg_status dg_canvas_update(const float* d_logits, int32_t C, int32_t V, int32_t n_renoise, uint64_t seed,
                           uint32_t step, int32_t* d_canvas, float* d_conf, void* d_ws, size_t ws_bytes,
                           dg_stream stream);

/* One denoising pass and its canvas update without materialising the logits (bf16
 * models; DG_ERR_UNSUPPORTED for fp32): the vocabulary projection's epilogue emits the
 * update's statistics per (token, 128-id tile) -- the largest logit, the sum of exp(l -
 * max), the candidate id and its logit -- which are merged per token in id order and
 * selected as dg_canvas_update (mask_id < 0: n = n_renoise, with seed and step) or
 * dg_canvas_update_masked (mask_id >= 0: n = n_keep; seed and step unused) would on the
 * logits.  d_canvas[C] is the pass's input and receives the update; d_conf[C] as those
 * calls (nullable).  The 4 C V bytes of logits are neither written nor read.  Results
 * equal the two-call path's up to fp32 summation order.  C <= 1024, 0 <= n <= C. */
dg_status dg_denoise_update(dg_model* m, const dg_kv_cache* cache, int32_t* d_canvas, int32_t C, int32_t n,
                            uint64_t seed, uint32_t step, int32_t mask_id, float* d_conf, void* d_ws, size_t ws_bytes,
                            dg_stream stream);

/* S denoising passes with re-noising, then (if append) the canvas is appended to the
 * cache by dg_prefill_append.  After pass s (0-based) the number of re-noised
 * positions is floor(C * f_s + 1e-9), f_s = (r_start (S-1-s) + r_end s) / (S-1)
 * (f_0 = r_start when S == 1); the update of pass s uses step = s.  d_canvas holds
 * the initial noise on entry and the result on return.  d_logits ([C][V], 16-byte
 * aligned) receives the last pass's logits.  C <= 1024.  Every argument the passes,
 * updates and append would check is checked before the first launch. */
dg_status dg_generate_canvas(dg_model* m, dg_kv_cache* cache, int32_t* d_canvas, int32_t C, int32_t S,
                             float r_start, float r_end, uint64_t seed, int32_t append, float* d_logits,
                             void* d_ws, size_t ws_bytes, dg_stream stream);

/* Masked-diffusion variant of the update ("DiffusionGemma" video explainer -- "First
 * attempt: masked diffusion": noise is a [MASK] placeholder that the model fills in,
 * and a filled position stays fixed).  For each row i of d_logits[C][V]: a position
 * holding any token other than mask_id is locked and keeps it; a masked position's
 * candidate is its argmax over every token except mask_id (lowest id on ties), its
 * confidence that token's softmax probability over all V logits.  Of the M masked
 * positions the min(n_keep, M) least confident (lower position first on ties) keep
 * mask_id; the others take their candidates.  Writes d_canvas[C] in place; d_conf[C]
 * (every position's candidate confidence) if not NULL.  Workspace as for
 * dg_canvas_update.  C <= 1024, V % 4 == 0, 0 <= mask_id < V, 0 <= n_keep <= C. */
dg_status dg_canvas_update_masked(const float* d_logits, int32_t C, int32_t V, int32_t n_keep, int32_t mask_id,
                                  int32_t* d_canvas, float* d_conf, void* d_ws, size_t ws_bytes, dg_stream stream);

/* S masked-diffusion passes from an all-mask_id canvas (written by this call into
 * d_canvas[C]): pass s keeps n_s = dg_renoise_count(C, S, s, keep_start, keep_end)
 * positions masked at most (keep_start = (S-1)/S, keep_end = 0 unmasks C/S per pass and
 * ends with none), then appends the canvas by prefill if `append`.  Same workspace,
 * logits buffer and errors as dg_generate_canvas. */
dg_status dg_generate_canvas_masked(dg_model* m, dg_kv_cache* cache, int32_t* d_canvas, int32_t C, int32_t S,
                                    float keep_start, float keep_end, int32_t mask_id, int32_t append,
                                    float* d_logits, void* d_ws, size_t ws_bytes, dg_stream stream);

/* Several canvases in one call.  Canvas b (0 <= b < B) is a separate request with its
 * own KV cache caches[b] (host array of B caches that share no buffers; each must have
 * room for C more positions) and its own positions caches[b].len ..; it attends only to
 * its own cache and its own canvas.  Row-wise buffers hold the canvases one after
 * another: tokens / canvases int32 [B][C], logits fp32 [B][C][V].  Each canvas's result
 * is the one the single-canvas call gives it (up to fp32 summation order: split-K factors
 * follow the row count); the router, the expert GEMMs and the vocabulary projection run
 * once over all B C rows, so each used expert's weights are read once per batch instead
 * of once per canvas (Hacker News discussion of DiffusionGemma, the comment on batching:
 * batched requests share the reads of common weights).  Workspace:
 * dg_workspace_bytes(cfg, B * C).  B * C <= 2^20. */
dg_status dg_prefill_append_batched(dg_model* m, dg_kv_cache* caches, int32_t B, const int32_t* d_tokens, int32_t T,
                                    void* d_ws, size_t ws_bytes, dg_stream stream);
dg_status dg_denoise_pass_batched(dg_model* m, const dg_kv_cache* caches, int32_t B, const int32_t* d_canvases,
                                  int32_t C, float* d_logits, void* d_ws, size_t ws_bytes, dg_stream stream);
/* dg_generate_canvas for B canvases at once: the same schedule for all, canvas b
 * re-noised from the stream seeded with seeds[b] (host array [B]); the append (if any)
 * writes canvas b into caches[b].  C <= 1024; every argument is checked before the first
 * launch. */
dg_status dg_generate_canvases(dg_model* m, dg_kv_cache* caches, int32_t B, int32_t* d_canvases, int32_t C, int32_t S,
                               float r_start, float r_end, const uint64_t* seeds, int32_t append, float* d_logits,
                               void* d_ws, size_t ws_bytes, dg_stream stream);
/* dg_generate_canvas_masked for B canvases at once (each from an all-mask_id canvas,
 * written by this call into d_canvases[B][C]; the same keep schedule for all). */
dg_status dg_generate_canvases_masked(dg_model* m, dg_kv_cache* caches, int32_t B, int32_t* d_canvases, int32_t C,
                                      int32_t S, float keep_start, float keep_end, int32_t mask_id, int32_t append,
                                      float* d_logits, void* d_ws, size_t ws_bytes, dg_stream stream);

/* 8-bit expert weights (MX-FP8 storage: E4M3 codes with one E8M0 power-of-two scale per
 * 32 consecutive K elements of a row; see dg_debug_gemm_mx8 in dg_debug.h for the byte
 * layouts and limits).  The pages name FP8 and NVFP4 deployments of the model without a
 * format ("Module 12. Diffusion Language Models" exercises, the MoE remark); these are the
 * OCP MX and NVFP4-style block formats, weight-only.  Errors (for these and the output-
 * matrix setters below): DG_ERR_INVALID_ARG for a NULL model, an fp32 model, NULL or
 * misaligned pointers or a non-finite tensor scale; DG_ERR_CUDA if a tensor map cannot be
 * encoded; on any error the model keeps its previous weights.  Per layer:
 *   gate, up     codes [E][F][H],  scales [E][H / 64][F][2]
 *   down         codes [E][H][F],  scales [E][F / 64][H][2]
 * all device pointers, 16-byte aligned, alive and unchanged while set.  Each weight is
 * value(code) * 2^(scale - 127), decoded exactly to bf16 inside the expert GEMMs, so the
 * model computes with exactly those weights at the bf16 path's precision; the expert
 * weight stream is half the bytes of bf16. */
typedef struct dg_expert_weights_mx8 {
  const void* gate;
  const void* gate_scales;
  const void* up;
  const void* up_scales;
  const void* down;
  const void* down_scales;
} dg_expert_weights_mx8;
/* Run the experts of every layer from these 8-bit weights (host array [n_layers]; NULL
 * returns to the bf16 experts given at creation).  bf16 models only.  Applies to the
 * batched calls (dg_denoise_pass_batched, dg_prefill_append_batched,
 * dg_generate_canvases; B = 1 is one canvas); the single-canvas calls keep the bf16
 * experts. */
dg_status dg_model_set_experts_mx8(dg_model* m, const dg_expert_weights_mx8* layers);
/* The same with 4-bit expert weights (E2M1 codes two per byte with one E4M3 scale per 16
 * consecutive K elements and an fp32 scale per weight tensor; see dg_debug_gemm_nv4 in
 * dg_debug.h for the byte layouts).  Per layer, in the same struct:
 *   gate, up     codes [E][F][H / 2],  scales [E][H / 64][F][4]
 *   down         codes [E][H][F / 2],  scales [E][F / 64][H][4]
 * tensor_scales: host array [n_layers][3] (gate, up, down), finite.  Each weight is
 * e2m1(code) * e4m3(block scale) * tensor scale; the expert weight stream is about a
 * quarter of bf16's. */
dg_status dg_model_set_experts_nv4(dg_model* m, const dg_expert_weights_mx8* layers, const float* tensor_scales);

/* Project to the vocabulary from an 8-bit output matrix (NULL codes returns to the bf16
 * W_out given at creation).  bf16 models only; applies to the batched calls, like the
 * low-precision experts.  codes: E4M3 [V][H] (row v = vocabulary id v); scales: E8M0
 * [H / 64][V][2], entry [j][v][b] the scale of elements 64 j + 32 b .. + 31 of row v, each
 * in [0, 134] (block scale 2^(s - 127) <= 2^7); codes 0x7F / 0xFF (NaN) must not occur.
 * Each weight is value(code) * 2^(scale - 127), decoded exactly to bf16 for s >= 9.  The
 * output matrix's stream is about half of bf16's.  Both pointers device, 16-byte aligned,
 * caller-owned and kept alive while the model uses them. */
dg_status dg_model_set_vocab_mx8(dg_model* m, const void* codes, const void* scales);
/* The same from a 4-bit output matrix: codes E2M1 two per byte [V][H / 2] (element 2 i in
 * the low nibble of byte i), scales E4M3 [H / 64][V][4] (non-negative, not NaN), one finite
 * tensor scale; each weight is e2m1(code) * e4m3(scale) * tensor_scale. */
dg_status dg_model_set_vocab_nv4(dg_model* m, const void* codes, const void* scales, float tensor_scale);

/* The re-noise count dg_generate_canvas uses after pass `step` of S (pure host arithmetic). */
int32_t dg_renoise_count(int32_t C, int32_t S, int32_t step, float r_start, float r_end);

/* Synchronize the stream, read and clear the workspace error word.  DG_OK or
 * DG_ERR_TIMEOUT (a kernel's bounded wait gave up; its outputs are not valid). */
dg_status dg_device_status(void* d_ws, dg_stream stream);

const char* dg_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* DG_H */
