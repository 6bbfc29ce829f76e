// Host-side launchers of the device kernels (internal to libdg; not part of the C-ABI).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dg {

// ---------------------------------------------------------------- tcgen05 GEMM
// out[row][feature] (op)= sum_k W[g][feature][k] * X[row][k]
// W comes from a 3-D tensor map (K, rows per group, groups), box 64 x 128 x 1; X from
// 2-D maps (K, rows) with boxes of 64 x 16 and 64 x 64 rows.  With two_terms, X = X_hi + X_lo (maps B and B2);
// with dual_a, a second weight tensor (map A2, same shape) accumulates into a second
// TMEM region and the epilogue writes silu(W x) * (W2 x) as bf16 hi (+ lo).
// Work: dense -- rows [0, n_tokens) in chunks of n_max, times k_splits (split s reduces
// K range [s K/k_splits, (s+1) K/k_splits) into out + s * split_stride); grouped -- the
// device list items[0 .. *n_items).
enum TcEpilogue { EPI_STORE_F32 = 0, EPI_SWIGLU_BF16 = 2 };

struct TcWorkItem {
  int group, row0, rows, pad;
};

struct TcGemmParams {
  int K;                 // reduction length, multiple of 64 * k_splits
  int a_rows_per_group;  // output features per group (rows of W[g])
  int m_tiles;           // ceil(a_rows_per_group / 128)
  int n_max;             // token rows per tile, multiple of 16, <= 256
  int n_tokens;          // dense: token rows
  int k_splits;          // dense only
  size_t split_stride;   // elements between split outputs
  const TcWorkItem* items;  // grouped: device work list (null: dense)
  const int* n_items;       // grouped: device count
  int dual_a;
  int m_pair;            // a tile = two consecutive 128-row weight tiles (m_tiles counts pairs)
  int two_terms;
  void* out;
  void* out_lo;
  int ld_out;            // elements per output row
  int smem_budget;       // bytes for pipeline stages
  int* err;              // device error word
};

// grid = min(max_tiles, SMs); max_tiles bounds the tile count (exact for dense GEMMs)
// B / B2: token maps with 16-row boxes; Bb / B2b: the same tensors with 64-row boxes
cudaError_t launch_tc_gemm(int epi, const CUtensorMap& A, const CUtensorMap& A2, const CUtensorMap& B,
                           const CUtensorMap& B2, const CUtensorMap& Bb, const CUtensorMap& B2b, const TcGemmParams& p,
                           int max_tiles, cudaStream_t st);
// The same GEMM over low-precision weights decoded exactly to bf16 (token maps, work list
// and epilogues as launch_tc_gemm; n_max <= 64 with two weight matrices, <= 128 with one;
// k_splits == 1; dense tiles always weight tile first).  A / A2: weight codes,
// S / S2: their block scales, as byte tensors.
//   FMT_MX8: E4M3 codes, 3-D maps (K bytes, rows, groups), box 64 x 128 x 1, 64-byte swizzle;
//            E8M0 scales [groups][K / 64][rows][2], 3-D maps (2 rows, K / 64, groups), box 256 x 1 x 1.
//   FMT_NV4: E2M1 codes two per byte, 3-D maps (K / 2 bytes, rows, groups), box 32 x 128 x 1,
//            32-byte swizzle; E4M3 scales [groups][K / 64][rows][4] as 3-D maps
//            (16 bytes = 4 rows, rows / 4, groups * K / 64), box 16 x 32 x 1; the epilogue
//            multiplies the accumulators by the tensor scales g_a (and g_a2 for A2).
enum LowpFormat { FMT_MX8 = 0, FMT_NV4 = 1 };
cudaError_t launch_tc_gemm_lowp(int fmt, int epi, const CUtensorMap& A, const CUtensorMap& A2, const CUtensorMap& S,
                                const CUtensorMap& S2, const CUtensorMap& B, const CUtensorMap& B2,
                                const CUtensorMap& Bb, const CUtensorMap& B2b, const TcGemmParams& p, float g_a,
                                float g_a2, int max_tiles, cudaStream_t st);
// grouped work list from group offsets off[E + 1] over `rows` token rows (checked on the
// device: bad offsets give no items and DG_DEVERR_BAD_COUNT in *err)
cudaError_t launch_build_items(const int32_t* off, int E, int n_max, int rows, TcWorkItem* items, int* n_items,
                               int* err, cudaStream_t st);
int num_sms();

// ---------------------------------------------------------------- tcgen05 attention
// Q [nq][n_q][128] bf16, K cache [nkv][cap][128] bf16, V^T cache [nkv][128][cap] bf16.
struct TcAttnParams {
  int n_q;             // query rows per head
  int q_pos0;          // absolute position of query row 0
  int n_keys;          // keys [0, n_keys) exist in the cache
  int causal;          // 1: key j visible to query i iff j <= q_pos0 + i
  int group;           // query heads per kv head
  int nq;              // query heads
  int chunks_per_split;
  int n_splits;
  float scale_log2;    // log2(e) / sqrt(d)
  int has_lo;          // query and current K/V carry low terms (bf16 model)
  int base;            // 128-aligned start of the low-term window (<= q_pos0)
  __nv_bfloat16* out;     // [n_q][nq * 128] when n_splits == 1 (hi part)
  __nv_bfloat16* out_lo;  // lo part, or null
  float* part_o;       // [n_splits][nq][n_q][128]
  float* part_lse;     // [n_splits][nq][n_q], log2 domain
  int* err;
};
// Single-head kernel (chunks_per_split counts 128-key chunks; with n_splits > 1 the
// partials go to part_o / part_lse for launch_attn_merge2).  Q / Ql: the query hi / lo
// [nq][n_q][128]; K / Vt: the cache; Kl / Vtl: low terms of the current K/V, rows (keys)
// counted from `base`; every map with 64 x 128 boxes.
cudaError_t launch_tc_attention(const CUtensorMap& Q, const CUtensorMap& Ql, const CUtensorMap& K,
                                const CUtensorMap& Vt, const CUtensorMap& Kl, const CUtensorMap& Vtl,
                                const TcAttnParams& p, cudaStream_t st);
// Head-pair variant (same parameters and outputs; chunks_per_split counts 128-key chunks):
// K / Kl maps with 128-row boxes (64 d wide), Vt / Vtl as above.  pair_heads = 1: two heads of one KV
// head per CTA where the group is even; 0: one head per CTA.  Grid y =
// attn2_head_groups(nq, group, pair_heads).
cudaError_t launch_tc_attention2(const CUtensorMap& Q, const CUtensorMap& Ql, const CUtensorMap& K,
                                 const CUtensorMap& Vt, const CUtensorMap& Kl, const CUtensorMap& Vtl,
                                 const TcAttnParams& p, int pair_heads, cudaStream_t st);
int attn2_head_groups(int nq, int group, int pair_heads);
// the head-pair path's split merge, one warp per (row, head) over the GPU, d = 128,
// n_splits <= 16
cudaError_t launch_attn_merge2(const float* part_o, const float* part_lse, int n_splits, int nq, int n_q,
                               __nv_bfloat16* out, __nv_bfloat16* out_lo, cudaStream_t st);
// ---------------------------------------------------------------- SIMT kernels (any dtype)
// T = float (fp32 model) or __nv_bfloat16; an activation for a bf16 GEMM is written as
// hi + lo bf16 tensors (lo pointers may be null: single term).
template <typename T>
cudaError_t launch_embed_norm(const int32_t* tokens, const T* embed, int n, int V, int H, float eps, float* x, T* xn,
                              T* xn_lo, int* err, cudaStream_t st);
// q / K / V^T hi parts (the cache holds K and V^T); with q_lo set (bf16 model) also the
// low parts: q_lo like q, k_lo [nkv][lo_rows][d] and vt_lo [nkv][d][lo_rows] at row
// (position - lo_base), rows [0, pos0 - lo_base) zeroed
template <typename T>
cudaError_t launch_rope_scatter(const float* qkv, int n_parts, size_t part_stride, int n, int nq, int nkv, int d,
                                int pos0, float theta, T* q, T* kcache, T* vtcache, int cap, T* q_lo, T* k_lo,
                                T* vt_lo, int lo_base, int lo_rows, cudaStream_t st);
cudaError_t launch_simt_gemm_f32(int epi_add, const float* W, const float* X, const int* group_off, int n_groups,
                                 int max_rows_per_group, int n_tokens, int M, int K, float* out, int ld_out,
                                 cudaStream_t st);
cudaError_t launch_simt_attention_f32(const float* q, const float* kcache, const float* vtcache, int cap, int n_q,
                                      int q_pos0, int n_keys, int causal, int nq, int nkv, int d, float* out,
                                      cudaStream_t st);
template <typename T>
cudaError_t launch_router_fused(float* x, const float* parts, int n_parts, size_t part_stride, const float* w_router,
                                int n, int H, int E, int k, float eps, float* logits, int32_t* topk_idx, float* topk_w,
                                T* xn, T* xn_lo, cudaStream_t st);
cudaError_t launch_permute(const int32_t* idx, int n, int k, int E, int32_t* counts, int32_t* offsets,
                           int32_t* perm, int32_t* inv, int32_t* union_out, int item_rows, TcWorkItem* items,
                           int* n_items, cudaStream_t st);
template <typename T>
cudaError_t launch_gather_rows(const T* xn, const T* xn_lo, const int32_t* perm, int rows, int k, int H, T* xs,
                               T* xs_lo, cudaStream_t st);
cudaError_t launch_swiglu_f32(const float* g, const float* u, int rows, int F, float* h, cudaStream_t st);
template <typename T>
cudaError_t launch_combine_norm(const float* ys, const int32_t* inv, const float* w, int n, int k, int H, float eps,
                                float* x, T* xn, T* xn_lo, cudaStream_t st);

// ---------------------------------------------------------------- canvas update
struct UpdPart {
  float m;    // row max over the slice
  float s;    // sum of exp(l - m) over the slice
  int a;      // first index of the largest logit among the candidate ids
  float m2;   // that logit (the ids other than an excluded one; m when nothing is excluded)
};
int update_splits(int C, int V);

// The vocabulary projection with the update's statistics as its epilogue (no logits):
// part[token][tile] for tokens [0, n_tokens) and 128-id tiles [0, m_tiles) of the output
// matrix (A: 3-D map (K, V, 1), box 64 x 128 x 1; B / Bb: the final normed state, 2-D maps
// with 16- and 64-row boxes); excl >= 0 makes every record's candidate skip that id.
struct VuParams {
  int K;            // hidden size
  int V;            // vocabulary
  int m_tiles;      // ceil(V / 128)
  int n_max;        // tokens per tile, multiple of 16, <= 256
  int n_tokens;
  int excl;
  UpdPart* part;    // [n_tokens][m_tiles]
  int smem_budget;
  int* err;
};
cudaError_t launch_vocab_update(const CUtensorMap& A, const CUtensorMap& B, const CUtensorMap& Bb, const VuParams& p,
                                cudaStream_t st);
// each token's tile records merged in id order into out[token]
cudaError_t launch_upd_merge_rows(const UpdPart* part, int C, int tiles, UpdPart* out, cudaStream_t st);
// excl >= 0: the candidate skips that id
cudaError_t launch_update_partial(const float* logits, int C, int V, int splits, int excl, UpdPart* part,
                                  cudaStream_t st);
// mask_id < 0: the re-noising update; mask_id >= 0: the masked-diffusion update
cudaError_t launch_update_select(const UpdPart* part, int C, int V, int splits, int n_renoise, uint64_t seed,
                                 uint32_t step, int32_t* canvas, float* conf, int mask_id, cudaStream_t st);
cudaError_t launch_fill_i32(int32_t* p, int n, int32_t v, cudaStream_t st);

cudaError_t launch_bounded_wait_selftest(int* err, uint64_t limit_ns, cudaStream_t st);
// tensor-pipe rate probe (k_probe.cu): `blocks` CTAs, each issuing `count` MMAs of
// 128 x n x 16 (A from TMEM when a_tmem), n in {64, 128, 256}; block 0's cycles to *cycles
cudaError_t launch_mma_rate(int a_tmem, int n, int count, int blocks, unsigned long long* cycles, int* err,
                            cudaStream_t st);

// the bounded-wait limit of each kernel file (default DG_WAIT_NS; failure tests shorten it)
cudaError_t set_wait_limit_attn(uint64_t ns);
cudaError_t set_wait_limit_attn2(uint64_t ns);
cudaError_t set_wait_limit_gemm(uint64_t ns);
cudaError_t set_wait_limit_gemm_lowp(uint64_t ns);
cudaError_t set_wait_limit_vocab_update(uint64_t ns);

}  // namespace dg
