// Host-side launchers of the device kernels (internal to libdg; not part of the C-ABI).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dg {

// ---------------------------------------------------------------- tcgen05 GEMM
// out[token][feature] (op)= sum_k W[feature][k] * X[token][k]
// W rows come from tensor map A (bf16, K-major, box 64 x 128), X rows from tensor map
// B (bf16, K-major, box 64 x 16).  With two_terms, X = X_hi + X_lo is given as two
// bf16 tensors (maps B and B2) and both products accumulate into the same fp32 tile.
// Group g (an expert) owns token rows [group_off[g], group_off[g+1]) of X and W rows
// [g * a_rows_per_group, ...).  With k_splits > 1 (one group only), split s reduces
// K range [s K/k_splits, (s+1) K/k_splits) and stores to out + s * split_stride.
enum TcEpilogue { EPI_STORE_F32 = 0, EPI_ADD_F32 = 1, EPI_SWIGLU_BF16 = 2 };

struct TcGemmParams {
  int K;                 // reduction length, multiple of 64 * k_splits
  int a_rows_per_group;  // W rows per group, multiple of 128
  const int* group_off;  // device [n_groups + 1], or nullptr for one group of n_tokens rows
  int n_tokens;
  void* out;             // EPI_SWIGLU_BF16: bf16 h_hi; h_lo follows at out_lo
  void* out_lo;
  int ld_out;            // elements per output row
  int two_terms;         // X given as hi + lo
  int k_splits;
  size_t split_stride;   // elements between split outputs
  int smem_budget;       // bytes for pipeline stages
  int* err;              // device error word
};

cudaError_t launch_tc_gemm(int epi, const CUtensorMap& A, const CUtensorMap& B, const CUtensorMap& B2,
                           const TcGemmParams& p, int m_tiles, int n_groups, int max_rows_per_group, cudaStream_t st);

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
  __nv_bfloat16* out;     // [n_q][nq * 128] when n_splits == 1 (hi part)
  __nv_bfloat16* out_lo;  // lo part, or null
  float* part_o;       // [n_splits][nq][n_q][128]
  float* part_lse;     // [n_splits][nq][n_q], log2 domain
  int* err;
};
cudaError_t launch_tc_attention(const CUtensorMap& Q, const CUtensorMap& K, const CUtensorMap& Vt,
                                const TcAttnParams& p, cudaStream_t st);
cudaError_t launch_attn_merge(const float* part_o, const float* part_lse, int n_splits, int nq, int n_q, int d,
                              __nv_bfloat16* out, __nv_bfloat16* out_lo, cudaStream_t st);

// ---------------------------------------------------------------- SIMT kernels (any dtype)
// T = float (fp32 model) or __nv_bfloat16; an activation for a bf16 GEMM is written as
// hi + lo bf16 tensors (lo pointers may be null: single term).
template <typename T>
cudaError_t launch_embed_norm(const int32_t* tokens, const T* embed, int n, int V, int H, float eps, float* x, T* xn,
                              T* xn_lo, int* err, cudaStream_t st);
template <typename T>
cudaError_t launch_rope_scatter(const float* qkv, int n_parts, size_t part_stride, int n, int nq, int nkv, int d,
                                int pos0, float theta, T* q, T* kcache, T* vtcache, int cap, cudaStream_t st);
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
                           int32_t* perm, int32_t* inv, int32_t* union_out, cudaStream_t st);
template <typename T>
cudaError_t launch_gather_rows(const T* xn, const T* xn_lo, const int32_t* perm, int rows, int k, int H, T* xs,
                               T* xs_lo, cudaStream_t st);
cudaError_t launch_swiglu_packed_f32(const float* gu, int rows, int F, float* h, cudaStream_t st);
template <typename T>
cudaError_t launch_combine_norm(const float* ys, const int32_t* inv, const float* w, int n, int k, int H, float eps,
                                float* x, T* xn, T* xn_lo, cudaStream_t st);
cudaError_t launch_pack_gate_up(const void* gate, const void* up, void* out, int E, int F, int H, int elem_bytes,
                                cudaStream_t st);

// ---------------------------------------------------------------- canvas update
struct UpdPart {
  float m;    // row max over the slice
  float s;    // sum of exp(l - m) over the slice
  int a;      // first index attaining m
  int pad;
};
int update_splits(int C, int V);
cudaError_t launch_update_partial(const float* logits, int C, int V, int splits, UpdPart* part, cudaStream_t st);
cudaError_t launch_update_select(const UpdPart* part, int C, int V, int splits, int n_renoise, uint64_t seed,
                                 uint32_t step, int32_t* canvas, float* conf, cudaStream_t st);

cudaError_t launch_bounded_wait_selftest(int* err, uint64_t limit_ns, cudaStream_t st);

}  // namespace dg
