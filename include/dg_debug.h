/*
 * dg_debug.h -- inspection entry points of libdg: per-layer taps of the denoising
 * pass (for layer-by-layer comparison with an independent implementation) and
 * per-kernel timing with CUDA events.  None of these change what the pass computes.
 */
#ifndef DG_DEBUG_H
#define DG_DEBUG_H

#include "dg.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Per-layer copies taken during dg_denoise_pass and dg_prefill_append, for calls of at
 * most `rows` tokens (a call with more tokens takes none; C below is the call's token
 * count).  Each member is a host array of n_layers device pointers (the array itself or
 * any entry may be NULL = not taken), each sized for `rows` tokens.
 *   x_attn   fp32 [C][H]   residual after the attention block
 *   x_out    fp32 [C][H]   residual after the MoE block
 *   topk_idx int32 [C][k]  routed experts, descending router logit
 *   topk_w   fp32 [C][k]   combine weights (softmax over the k chosen logits)
 *   counts   int32 [E]     rows routed to each expert
 *   perm     int32 [C k]   perm[p] = t*k + j of the p-th row in expert order
 *   unions   device int32 [n_layers] (single pointer): experts with at least one row */
typedef struct dg_taps {
  float* const* x_attn;
  float* const* x_out;
  int32_t* const* topk_idx;
  float* const* topk_w;
  int32_t* const* counts;
  int32_t* const* perm;
  int32_t* unions;
  int32_t rows;
} dg_taps;

/* Copy the tap pointers into the model (NULL turns taps off). */
dg_status dg_set_taps(dg_model* m, const dg_taps* taps);

/* Kernel kinds timed by the profiler. */
typedef enum dg_kernel_kind {
  DG_K_EMBED_NORM = 0,
  DG_K_RMS_NORM,
  DG_K_GEMM_QKV,
  DG_K_ROPE_KV,
  DG_K_ATTENTION,
  DG_K_ATTN_MERGE,
  DG_K_GEMM_O,
  DG_K_ROUTER,
  DG_K_TOPK,
  DG_K_PERMUTE,
  DG_K_GATHER,
  DG_K_GEMM_GATE_UP,
  DG_K_SWIGLU,
  DG_K_GEMM_DOWN,
  DG_K_COMBINE,
  DG_K_GEMM_VOCAB,
  DG_K_UPDATE_PARTIAL,
  DG_K_UPDATE_SELECT,
  DG_K_COUNT
} dg_kernel_kind;

/* When on, every kernel launch of the library is bracketed by a pair of CUDA events
 * recorded on the launching stream.  Off by default. */
dg_status dg_profile_enable(int32_t on);
/* Wait for the recorded events and return, for one kind, the summed device time (ms)
 * and the number of launches since the last reset. */
dg_status dg_profile_read(int32_t kind, double* total_ms, int32_t* launches);
void dg_profile_reset(void);
const char* dg_kernel_name(int32_t kind);

/* One launch of the persistent tcgen05 GEMM alone (bf16):
 *   acc[r][f] = sum_k W[g][f][k] * (X[r][k] + X_lo[r][k])   (X_lo NULL: X alone)
 * for rows r of group g = [group_off[g], group_off[g+1]) (group_off: device int32
 * [n_groups + 1], or NULL for one group of x_rows rows).  W is [n_groups][rows][K].
 * W2 NULL: out (fp32, row stride ld_out) = acc.  W2 given (same shape as W): out / out_lo
 * (bf16 hi / lo, out_lo nullable) = silu(acc) * acc2, acc2 the same sum over W2.
 * Groups are cut into work items of at most 128 rows, as in the pass's expert GEMMs;
 * offsets that decrease or leave [0, x_rows] launch no tile and set the error word to 5.
 * K % 64 == 0, rows >= 1.  d_scratch: 256-byte aligned,
 * dg_debug_gemm_scratch_bytes(x_rows, n_groups) bytes (the work list).  d_err: device
 * int32 error word. */
size_t dg_debug_gemm_scratch_bytes(int32_t x_rows, int32_t n_groups);
dg_status dg_debug_gemm_bf16(const void* W, const void* W2, int32_t rows, int32_t n_groups, const void* X,
                             const void* X_lo, int32_t x_rows, int32_t K, const int32_t* group_off, void* out,
                             void* out_lo, int32_t ld_out, void* d_scratch, size_t scratch_bytes,
                             int32_t* d_err, dg_stream stream);

/* The same GEMM over 8-bit weights (MX-FP8 storage: OCP E4M3 elements with one E8M0
 * power-of-two scale per 32 consecutive K elements of a row): every weight is
 * value(code) * 2^(scale - 127), decoded exactly to bf16 in the kernel, so
 *   acc[r][f] = sum_k dec(W)[g][f][k] * (X[r][k] + X_lo[r][k])
 * with everything else (groups, W2 / SwiGLU epilogue, outputs, errors, scratch) as
 * dg_debug_gemm_bf16, except that groups are cut into work items of at most 64 rows.
 * W (and W2): codes uint8 [n_groups][rows][K] (E4M3: sign, 4 exponent bits with bias 7,
 * 3 mantissa bits; codes 0x7F and 0xFF must not occur).  W_scales (and W2_scales): uint8
 * [n_groups][K / 64][rows][2], entry [g][j][f][h] the E8M0 scale of elements
 * 64 j + 32 h .. + 31 of row f; every scale <= 134 (block scale <= 2^7); decoding is exact
 * for scales >= 9 (below, subnormal codes round to bf16's subnormals).  rows % 8 == 0,
 * K % 64 == 0; every pointer 16-byte aligned. */
dg_status dg_debug_gemm_mx8(const void* W, const void* W_scales, const void* W2, const void* W2_scales, int32_t rows,
                            int32_t n_groups, const void* X, const void* X_lo, int32_t x_rows, int32_t K,
                            const int32_t* group_off, void* out, void* out_lo, int32_t ld_out, void* d_scratch,
                            size_t scratch_bytes, int32_t* d_err, dg_stream stream);

/* The same GEMM over 4-bit weights (NVFP4-style storage: E2M1 elements -- sign, 2 exponent
 * bits with bias 1, 1 mantissa bit -- with one E4M3 scale per 16 consecutive K elements of
 * a row and one fp32 scale g per weight tensor): every weight is
 * e2m1(code) * e4m3(block scale) * g.  Code times block scale is decoded exactly to bf16
 * in the kernel and g multiplies the fp32 accumulator, so
 *   acc[r][f] = g * sum_k dec(W)[g][f][k] * (X[r][k] + X_lo[r][k]).
 * W (and W2): uint8 [n_groups][rows][K / 2], element 2 i of a row in the low nibble of
 * byte i.  W_scales (and W2_scales): E4M3 codes uint8 [n_groups][K / 64][rows][4], entry
 * [g][j][f][b] the scale of elements 64 j + 16 b .. + 15 of row f (non-negative, not NaN).
 * g (and g2 for W2): finite.  Everything else as dg_debug_gemm_mx8. */
dg_status dg_debug_gemm_nv4(const void* W, const void* W_scales, float g, const void* W2, const void* W2_scales,
                            float g2, int32_t rows, int32_t n_groups, const void* X, const void* X_lo,
                            int32_t x_rows, int32_t K, const int32_t* group_off, void* out, void* out_lo,
                            int32_t ld_out, void* d_scratch, size_t scratch_bytes, int32_t* d_err, dg_stream stream);

/* One attention launch (bf16, head_dim 128) through the single-head kernel (one query
 * head x 128 rows per CTA, two S buffers in TMEM), as in the pass: q [nq][n_q][128],
 * K [nkv][cap][128], Vt [nkv][128][cap]; queries at positions pos0.. over keys
 * [0, n_keys), causal or not.  out bf16 [n_q][nq * 128] (hi part); out_lo (nullable)
 * receives the lo part, out + out_lo = the fp32 attention output to ~16 bits.  d_ws: a
 * workspace sized by dg_workspace_bytes for a config with these heads, hidden 128 and
 * >= n_q tokens.  As in the pass, the keys from the multiple of 128 at or below pos0 up
 * to n_keys are read as the call's own (with zero low terms here); they must fit the
 * workspace's window of ceil(n_q / 128) * 128 + 128 rows, which pos0 + n_q == n_keys
 * always does.  0 <= pos0 <= n_keys.  Violations: DG_ERR_INVALID_ARG, nothing launched. */
dg_status dg_debug_attention_bf16(const void* q, const void* k, const void* vt, int32_t cap, int32_t n_q, int32_t pos0,
                                  int32_t n_keys, int32_t causal, int32_t nq, int32_t nkv, void* out, void* out_lo,
                                  void* d_ws, size_t ws_bytes, dg_stream stream);

/* The same attention through the head-pair kernel: two query heads of one KV head per CTA
 * (one when nq / nkv is odd, or when single heads fill at least a quarter more SMs in the
 * one wave of CTAs), 128-key chunks, the same precision terms, outputs, workspace and
 * errors as dg_debug_attention_bf16.  The bf16 pass's attention runs the single-head kernel
 * of dg_debug_attention_bf16; setting DG_ATTN_PAIR=1 in the environment (read once per
 * process) routes it through this kernel instead. */
dg_status dg_debug_attention_pair_bf16(const void* q, const void* k, const void* vt, int32_t cap, int32_t n_q,
                                       int32_t pos0, int32_t n_keys, int32_t causal, int32_t nq, int32_t nkv,
                                       void* out, void* out_lo, void* d_ws, size_t ws_bytes, dg_stream stream);

/* Failure-detection self-test: launches one kernel whose thread waits, with the
 * library's bounded wait, on an mbarrier that nothing completes.  After timeout_ms
 * the wait gives up, records a timeout code in the workspace error word and the
 * kernel returns normally (no trap, the context stays usable); dg_device_status then
 * returns DG_ERR_TIMEOUT.  timeout_ms in [1, 10000]. */
dg_status dg_debug_bounded_wait(void* d_ws, int32_t timeout_ms, dg_stream stream);

/* Failure-detection control: sets the limit of every bounded wait in the tensor-core
 * kernels (GEMMs, attention, fused vocabulary/update) to limit_ns, for every later
 * launch on the current device, until set again; the default is 2 s (2000000000).  A
 * limit of 0 makes a wait that is not already satisfied give up at once, so the next
 * launch records a timeout code in its error word and winds down (no trap, no hang):
 * the failure tests use it to show that each kernel's abort path returns.  Not for use
 * while kernels run.  DG_ERR_INVALID_ARG above 2 s; DG_ERR_CUDA if a copy fails. */
dg_status dg_debug_set_wait_limit(uint64_t limit_ns);

/* Tensor-pipe rate probe: `blocks` CTAs (one per SM), each with one thread issuing
 * `count` tcgen05 MMAs of 128 x n x 16 (bf16 inputs, fp32 accumulation in TMEM) back to
 * back on operands it zeroes first -- A from shared memory (a_tmem = 0) or from TMEM
 * (a_tmem = 1), B from shared memory -- then waiting for them (bounded wait, 1 s).
 * *cycles_out (host): block 0's clock64 cycles from the first issue to the completion;
 * *ms_out (host): the launch's CUDA-event time.  n in {64, 128, 256}, count in
 * [1, 1048576], blocks in [1, 1024].  The work is the probe's only output; it measures
 * the rate the attention kernel's 128 x 128 x 16 instructions can reach.
 * DG_ERR_INVALID_ARG on a bad argument (nothing launched); DG_ERR_TIMEOUT if the wait gave up. */
dg_status dg_debug_mma_rate(int32_t a_tmem, int32_t n, int32_t count, int32_t blocks, uint64_t* cycles_out,
                            float* ms_out, dg_stream stream);

/* Kernels launched by the library since it was loaded (all kinds, profiling or not). */
int64_t dg_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* DG_DEBUG_H */
