// Non-tensor-core kernels of the pass: embedding + RMSNorm, RoPE and KV-cache
// writes, the router and its top-k, the expert histogram / stable permutation /
// row gather, the weighted combine, the canvas update (softmax confidence,
// argmax, lowest-confidence re-noising), and fp32 GEMM / attention used by the
// fp32 model (tcgen05 has no fp32 operand kind).
#include <math.h>

#include <cooperative_groups.h>

#include "dg_common.cuh"
#include "dg_kernels.h"

namespace cg = cooperative_groups;

namespace dg {

// ---------------------------------------------------------------- block reductions
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = (threadIdx.x < nw) ? red[threadIdx.x] : 0.0f;
  if (warp == 0) t = warp_sum(t);
  if (threadIdx.x == 0) red[0] = t;
  __syncthreads();
  return red[0];
}

// ---------------------------------------------------------------- embedding + RMSNorm
// An fp32 activation v handed to a bf16 GEMM is stored as hi = bf16(v) and
// lo = bf16(v - hi); the GEMM accumulates W hi + W lo, which carries ~16 significant
// bits of v.  For the fp32 model T = float and there is no lo part.
template <typename T>
__device__ __forceinline__ void store_act(T* hi, T* lo, size_t i, float v) {
  const T h = from_f32<T>(v);
  hi[i] = h;
  if (lo) lo[i] = from_f32<T>(v - to_f32(h));
}

// x[t] = embed[tokens[t]] (fp32), xn[t] = x[t] / sqrt(mean(x[t]^2) + eps)
template <typename T>
__global__ void embed_norm_kernel(const int32_t* __restrict__ tokens, const T* __restrict__ embed, int V, int H,
                                  float eps, float* __restrict__ x, T* __restrict__ xn, T* __restrict__ xn_lo,
                                  int* __restrict__ err) {
  griddep_sync();
  __shared__ float red[32];
  const int t = blockIdx.x;
  int tok = tokens[t];
  if (tok < 0 || tok >= V) {  // never read outside the table: flag and use token 0
    if (threadIdx.x == 0) atomicCAS(err, 0, DG_DEVERR_BAD_TOKEN);
    tok = 0;
  }
  const T* e = embed + (size_t)tok * H;
  float* xr = x + (size_t)t * H;
  constexpr int VE = 16 / sizeof(T);  // elements per 16-byte vector
  float ss = 0.0f;
  for (int v = threadIdx.x; v < H / VE; v += blockDim.x) {
    const uint4 raw = reinterpret_cast<const uint4*>(e)[v];
    const T* el = reinterpret_cast<const T*>(&raw);
#pragma unroll
    for (int j = 0; j < VE; ++j) {
      const float f = to_f32(el[j]);
      xr[v * VE + j] = f;
      ss += f * f;
    }
  }
  ss = block_sum(ss, red);
  const float inv = 1.0f / sqrtf(ss / (float)H + eps);
  for (int h = threadIdx.x; h < H; h += blockDim.x) store_act(xn, xn_lo, (size_t)t * H + h, xr[h] * inv);
}

template <typename T>
cudaError_t launch_embed_norm(const int32_t* tokens, const T* embed, int n, int V, int H, float eps, float* x, T* xn,
                              T* xn_lo, int* err, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  return launch_k(embed_norm_kernel<T>, dim3(n), dim3(256), 0, st, tokens, embed, V, H, eps, x, xn, xn_lo, err);
}

// ---------------------------------------------------------------- RoPE + KV cache write
// qkv[t] = [q heads | k heads | v heads] (fp32).  Rotate-half RoPE at position pos0 + t
// (angles in double precision), then q -> q[h][t][:], k -> K[kvh][pos][:],
// v -> V^T[kvh][:][pos], all in the activation dtype.
// most split-K partial slabs a consumer sums (the projections' split-K factors are at
// most 4 and 8; launches with more are refused)
constexpr int kMaxSumParts = 8;

template <typename T>
__global__ void rope_scatter_kernel(const float* __restrict__ qkv, int n_parts, size_t part_stride, int nq, int nkv,
                                    int d, int pos0, float theta, int n, T* __restrict__ q, T* __restrict__ kc,
                                    T* __restrict__ vtc, int cap, T* __restrict__ q_lo, T* __restrict__ k_lo,
                                    T* __restrict__ vt_lo, int lo_base, int lo_rows) {
  griddep_sync();
  extern __shared__ float cs[];  // [d/2] cos, [d/2] sin, then the summed qkv row
  const int t = blockIdx.x;
  const int half = d / 2;
  const int pos = pos0 + t;
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    const double inv_freq = pow((double)theta, -2.0 * (double)i / (double)d);
    double sn, cn;
    sincos((double)pos * inv_freq, &sn, &cn);
    cs[i] = (float)cn;
    cs[half + i] = (float)sn;
  }
  const int W = (nq + 2 * nkv) * d;
  float* row = cs + d;  // qkv row = sum of the split-K partials, in a fixed order
  for (int i = threadIdx.x; i < W / 4; i += blockDim.x) {
    // every partial's load issued before the first add (the sum keeps its fixed order)
    float4 a[kMaxSumParts];
#pragma unroll
    for (int s = 0; s < kMaxSumParts; ++s)
      if (s < n_parts) a[s] = reinterpret_cast<const float4*>(qkv + s * part_stride + (size_t)t * W)[i];
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < kMaxSumParts; ++s)
      if (s < n_parts) {
        v.x += a[s].x;
        v.y += a[s].y;
        v.z += a[s].z;
        v.w += a[s].w;
      }
    reinterpret_cast<float4*>(row)[i] = v;
  }
  __syncthreads();
  // q and k heads: pairs (i, i + d/2)
  for (int idx = threadIdx.x; idx < (nq + nkv) * half; idx += blockDim.x) {
    const int hh = idx / half, i = idx % half;
    const float x1 = row[hh * d + i], x2 = row[hh * d + i + half];
    const float c = cs[i], s = cs[half + i];
    const float o1 = x1 * c - x2 * s, o2 = x2 * c + x1 * s;
    if (hh < nq) {
      const size_t o = ((size_t)hh * n + t) * d;
      store_act(q, q_lo, o + i, o1);
      store_act(q, q_lo, o + i + half, o2);
    } else {
      const int kh = hh - nq;
      T* dst = kc + ((size_t)kh * cap + pos) * d;
      const T a = from_f32<T>(o1), b = from_f32<T>(o2);
      dst[i] = a;
      dst[i + half] = b;
      if (k_lo) {
        T* dl = k_lo + ((size_t)kh * lo_rows + (pos - lo_base)) * d;
        dl[i] = from_f32<T>(o1 - to_f32(a));
        dl[i + half] = from_f32<T>(o2 - to_f32(b));
      }
    }
  }
  for (int idx = threadIdx.x; idx < nkv * d; idx += blockDim.x) {
    const int hh = idx / d, dd = idx % d;
    const float v = row[(nq + nkv) * d + idx];
    const T a = from_f32<T>(v);
    vtc[((size_t)hh * d + dd) * cap + pos] = a;
    if (vt_lo) vt_lo[((size_t)hh * d + dd) * lo_rows + (pos - lo_base)] = from_f32<T>(v - to_f32(a));
  }
  // the window rows before the first current position hold cached keys: no low part
  if (k_lo) {
    for (int r = t; r < pos0 - lo_base; r += n)
      for (int idx = threadIdx.x; idx < nkv * d; idx += blockDim.x) {
        const int hh = idx / d, dd = idx % d;
        k_lo[((size_t)hh * lo_rows + r) * d + dd] = from_f32<T>(0.0f);
        vt_lo[((size_t)hh * d + dd) * lo_rows + r] = from_f32<T>(0.0f);
      }
  }
}

template <typename T>
cudaError_t launch_rope_scatter(const float* qkv, int n_parts, size_t part_stride, int n, int nq, int nkv, int d,
                                int pos0, float theta, T* q, T* kcache, T* vtcache, int cap, T* q_lo, T* k_lo,
                                T* vt_lo, int lo_base, int lo_rows, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  if (n_parts < 1 || n_parts > kMaxSumParts) return cudaErrorInvalidValue;
  const size_t smem = (size_t)(d + (nq + 2 * nkv) * d) * sizeof(float);
  return launch_k(rope_scatter_kernel<T>, dim3(n), dim3(256), smem, st, qkv, n_parts, part_stride, nq, nkv, d, pos0,
                  theta, n, q, kcache, vtcache, cap, q_lo, k_lo, vt_lo, lo_base, lo_rows);
}

// ---------------------------------------------------------------- fp32 GEMM (fp32 model)
// out[row][feat] (+)= sum_k W[g*M + feat][k] * X[row][k] for rows of group g
constexpr int SG_BT = 32, SG_BF = 64, SG_BK = 32;
__global__ void simt_gemm_f32_kernel(int epi_add, const float* __restrict__ W, const float* __restrict__ X,
                                     const int* __restrict__ group_off, int n_tokens, int M, int K,
                                     float* __restrict__ out, int ld_out) {
  griddep_sync();
  __shared__ float sx[SG_BT][SG_BK + 1];
  __shared__ float sw[SG_BF][SG_BK + 1];
  const int g = blockIdx.y;
  int r_begin = 0, r_end = n_tokens;
  if (group_off) {
    r_begin = group_off[g];
    r_end = group_off[g + 1];
  }
  const int r0 = r_begin + blockIdx.z * SG_BT;
  if (r0 >= r_end) return;
  const int f0 = blockIdx.x * SG_BF;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;  // 16 x 16 threads: 2 rows x 4 features each
  float acc[2][4] = {};
  const float* Wg = W + (size_t)g * M * K;
  for (int k0 = 0; k0 < K; k0 += SG_BK) {
    for (int i = threadIdx.x; i < SG_BT * SG_BK; i += blockDim.x) {
      const int r = i / SG_BK, kk = i % SG_BK;
      sx[r][kk] = (r0 + r < r_end && k0 + kk < K) ? X[(size_t)(r0 + r) * K + k0 + kk] : 0.0f;
    }
    for (int i = threadIdx.x; i < SG_BF * SG_BK; i += blockDim.x) {
      const int f = i / SG_BK, kk = i % SG_BK;
      sw[f][kk] = (f0 + f < M && k0 + kk < K) ? Wg[(size_t)(f0 + f) * K + k0 + kk] : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < SG_BK; ++kk) {
      float a[2], b[4];
#pragma unroll
      for (int i = 0; i < 2; ++i) a[i] = sx[ty * 2 + i][kk];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = sw[tx + 16 * j][kk];
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = r0 + ty * 2 + i;
    if (r >= r_end) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int f = f0 + tx + 16 * j;
      if (f >= M) continue;
      float* dst = out + (size_t)r * ld_out + f;
      if (epi_add)
        *dst += acc[i][j];
      else
        *dst = acc[i][j];
    }
  }
}

cudaError_t launch_simt_gemm_f32(int epi_add, const float* W, const float* X, const int* group_off, int n_groups,
                                 int max_rows_per_group, int n_tokens, int M, int K, float* out, int ld_out,
                                 cudaStream_t st) {
  if (max_rows_per_group <= 0 || n_groups <= 0) return cudaSuccess;
  dim3 grid((M + SG_BF - 1) / SG_BF, n_groups, (max_rows_per_group + SG_BT - 1) / SG_BT);
  return launch_k(simt_gemm_f32_kernel, dim3(grid), dim3(256), 0, st, epi_add, W, X, group_off, n_tokens, M, K, out, ld_out);
}

// ---------------------------------------------------------------- fp32 attention (fp32 model)
// one warp per (query row, head); lane = key within a 32-key chunk, online softmax
__global__ void simt_attention_f32_kernel(const float* __restrict__ q, const float* __restrict__ kc,
                                          const float* __restrict__ vtc, int cap, int n_q, int q_pos0, int n_keys,
                                          int causal, int nq, int nkv, int d, float* __restrict__ out) {
  griddep_sync();
  __shared__ float sq[128];
  const int qrow = blockIdx.x, h = blockIdx.y, lane = threadIdx.x;
  const int kvh = h / (nq / nkv);
  for (int i = lane; i < d; i += 32) sq[i] = q[((size_t)h * n_q + qrow) * d + i];
  __syncwarp();
  const int lim = causal ? min(n_keys, q_pos0 + qrow + 1) : n_keys;
  const float scale = 1.0f / sqrtf((float)d);
  float m = -INFINITY, l = 0.0f;
  float o[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  const float* K = kc + (size_t)kvh * cap * d;
  const float* Vt = vtc + (size_t)kvh * d * cap;
  for (int k0 = 0; k0 < lim; k0 += 32) {
    const int key = k0 + lane;
    float s = -INFINITY;
    if (key < lim) {
      float acc = 0.0f;
      for (int i = 0; i < d; ++i) acc = fmaf(sq[i], K[(size_t)key * d + i], acc);
      s = acc * scale;
    }
    const float cm = warp_max(s);
    const float mn = fmaxf(m, cm);
    const float alpha = (m == -INFINITY) ? 0.0f : expf(m - mn);
    const float p = (key < lim) ? expf(s - mn) : 0.0f;
    l = l * alpha + warp_sum(p);
#pragma unroll
    for (int j = 0; j < 4; ++j) o[j] *= alpha;
    const int nk = min(32, lim - k0);
    for (int kk = 0; kk < nk; ++kk) {
      const float pk = __shfl_sync(0xffffffffu, p, kk);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int dd = lane + 32 * j;
        if (dd < d) o[j] = fmaf(pk, Vt[(size_t)dd * cap + k0 + kk], o[j]);
      }
    }
    m = mn;
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int dd = lane + 32 * j;
    if (dd < d) out[(size_t)qrow * nq * d + (size_t)h * d + dd] = o[j] / l;
  }
}

cudaError_t launch_simt_attention_f32(const float* q, const float* kcache, const float* vtcache, int cap, int n_q,
                                      int q_pos0, int n_keys, int causal, int nq, int nkv, int d, float* out,
                                      cudaStream_t st) {
  if (n_q <= 0) return cudaSuccess;
  return launch_k(simt_attention_f32_kernel, dim3(n_q, nq), dim3(32), 0, st, q, kcache, vtcache, cap, n_q, q_pos0, n_keys,
           causal, nq, nkv, d, out);
}

// ---------------------------------------------------------------- residual + RMSNorm + router + top-k
// Per token: x += sum of the output-projection partials (fixed order); xn = x / rms(x)
// in fp32; router logits l[e] = xn . w_router[e] (fp32); the k largest (ties to the
// lower expert id) and their softmax weights.  xn is also stored (hi/lo) as the expert
// input.
//
// A cluster of RT_G CTAs takes RT_TOK tokens and splits the experts among its CTAs, so
// each CTA streams only E / RT_G rows of the router matrix: CTA r adds the residual and
// normalises its own RT_TOK / RT_G tokens, the normalised rows are shared through
// distributed shared memory, every CTA computes its experts' logits for all RT_TOK
// tokens (four experts per warp at once, each token row read from shared memory once per
// four experts, sixteen float4 weight loads per lane in flight), and CTA r runs
// the top-k of its own tokens over the logits of all CTAs.  Each logit is one lane-
// strided fp32 dot product followed by a warp sum, as in a single-CTA version.
// Four tokens per cluster (one per CTA): the kernel is bound by its own latencies, not by
// bandwidth, so twice the CTAs with half the work each (the router matrix is read from
// L2 twice as often, 1.4 MB per cluster at the large model) finish sooner.
constexpr int RT_G = 4;
constexpr int RT_TOK = 4;
constexpr int RT_OWN = RT_TOK / RT_G;
constexpr int RT_THREADS = 256;
constexpr int RT_EB = 4;   // experts per warp at once
constexpr int RT_PF = 4;   // float4 steps of the weights loaded ahead (RT_PF * RT_EB loads)
template <typename T>
__global__ void __launch_bounds__(RT_THREADS) router_fused_kernel(
    float* __restrict__ x, const float* __restrict__ parts, int n_parts, size_t part_stride,
    const float* __restrict__ wr, int n, int H, int E, int k, float eps, float* __restrict__ logits_out,
    int32_t* __restrict__ topk_idx, float* __restrict__ topk_w, T* __restrict__ xn, T* __restrict__ xn_lo) {
  griddep_sync();
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int Eg = E / RT_G;
  extern __shared__ float sm[];
  float* own = sm;                  // [RT_OWN][H] this CTA's normalised rows
  float* xs = own + RT_OWN * H;     // [RT_TOK][H] the cluster's normalised rows
  float* lg = xs + RT_TOK * H;      // [RT_TOK][Eg] this CTA's experts' logits
  __shared__ float inv_s[RT_OWN];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NW = RT_THREADS / 32;
  const int t0 = (int)(blockIdx.x / RT_G) * RT_TOK;
  const int nt = min(RT_TOK, n - t0);
  const int o0 = t0 + rank * RT_OWN;
  const int no = max(0, min(RT_OWN, n - o0));
  const int H4 = H / 4;
  // residual add of the partials for the owned tokens
  {
    float4* x4 = reinterpret_cast<float4*>(x + (size_t)o0 * H);
    const float4* p4 = reinterpret_cast<const float4*>(parts + (size_t)o0 * H);
    const size_t ps4 = part_stride / 4;
    float4* own4 = reinterpret_cast<float4*>(own);
    // two elements per thread and step: every partial's load of both issued before the
    // first add (each sum keeps its fixed order)
    for (int i0 = threadIdx.x; i0 < no * H4; i0 += 2 * RT_THREADS) {
      float4 a[2][kMaxSumParts], v[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = i0 + e * RT_THREADS;
        if (i < no * H4) {
#pragma unroll
          for (int s = 0; s < kMaxSumParts; ++s)
            if (s < n_parts) a[e][s] = p4[s * ps4 + i];
          v[e] = x4[i];
        }
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = i0 + e * RT_THREADS;
        if (i < no * H4) {
#pragma unroll
          for (int s = 0; s < kMaxSumParts; ++s)
            if (s < n_parts) {
              v[e].x += a[e][s].x;
              v[e].y += a[e][s].y;
              v[e].z += a[e][s].z;
              v[e].w += a[e][s].w;
            }
          x4[i] = v[e];
          own4[i] = v[e];
        }
      }
    }
  }
  __syncthreads();
  if (warp < no) {
    float ss = 0.0f;
    for (int h = lane; h < H; h += 32) ss += own[warp * H + h] * own[warp * H + h];
    ss = warp_sum(ss);
    if (lane == 0) inv_s[warp] = 1.0f / sqrtf(ss / (float)H + eps);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < no * H; i += RT_THREADS) {
    const float v = own[i] * inv_s[i / H];
    own[i] = v;
    store_act(xn, xn_lo, (size_t)o0 * H + i, v);
  }
  cl.sync();  // every CTA's rows are normalised
  // the cluster's rows into this CTA's shared memory: eight remote loads in flight per
  // thread before their stores (rank r's rows land at r * RT_OWN)
  {
    const float4* src[RT_G];
#pragma unroll
    for (int r = 0; r < RT_G; ++r) src[r] = reinterpret_cast<const float4*>(cl.map_shared_rank(own, r));
    float4* dst = reinterpret_cast<float4*>(xs);
    const int per = RT_OWN * H4;  // float4 of one rank's rows
    const int total = nt * H4;
    constexpr int CB = 8;
    for (int i0 = threadIdx.x; i0 < total; i0 += CB * RT_THREADS) {
      float4 v[CB];
#pragma unroll
      for (int c = 0; c < CB; ++c) {
        const int i = i0 + c * RT_THREADS;
        if (i < total) v[c] = src[i / per][i % per];
      }
#pragma unroll
      for (int c = 0; c < CB; ++c) {
        const int i = i0 + c * RT_THREADS;
        if (i < total) dst[i] = v[c];
      }
    }
  }
  __syncthreads();
  const float4* xs4 = reinterpret_cast<const float4*>(xs);
  // RT_EB experts per warp at once: each token row read from shared memory serves all of
  // them (shared-memory reads, not FMAs, bound a one-expert-per-warp loop)
  for (int j0 = warp * RT_EB; j0 < Eg; j0 += NW * RT_EB) {
    const float4* w4[RT_EB];
#pragma unroll
    for (int b = 0; b < RT_EB; ++b) w4[b] = reinterpret_cast<const float4*>(wr + (size_t)(rank * Eg + min(j0 + b, Eg - 1)) * H);
    float acc[RT_EB][RT_TOK] = {};
    for (int i0 = lane; i0 < H4; i0 += 32 * RT_PF) {
      float4 u[RT_PF][RT_EB];
#pragma unroll
      for (int q = 0; q < RT_PF; ++q) {
        const int i = i0 + 32 * q;
#pragma unroll
        for (int b = 0; b < RT_EB; ++b) u[q][b] = i < H4 ? w4[b][i] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int q = 0; q < RT_PF; ++q) {
        const int i = i0 + 32 * q;
        if (i < H4) {
#pragma unroll
          for (int a = 0; a < RT_TOK; ++a) {
            if (a < nt) {
              const float4 v = xs4[a * H4 + i];
#pragma unroll
              for (int b = 0; b < RT_EB; ++b)
                acc[b][a] = fmaf(u[q][b].x, v.x, fmaf(u[q][b].y, v.y, fmaf(u[q][b].z, v.z, fmaf(u[q][b].w, v.w, acc[b][a]))));
            }
          }
        }
      }
    }
#pragma unroll
    for (int b = 0; b < RT_EB; ++b)
#pragma unroll
      for (int a = 0; a < RT_TOK; ++a) {
        const float r = warp_sum(acc[b][a]);
        if (lane == 0 && j0 + b < Eg) lg[a * Eg + j0 + b] = r;
      }
  }
  cl.sync();  // every CTA's logits are in place
  // top-k: warp w < no selects for owned token w; lane takes experts lane + 32 i
  if (warp < no) {
    const int a = rank * RT_OWN + warp;  // token within the cluster
    float l[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      l[i] = -INFINITY;
      if (e < E) l[i] = cl.map_shared_rank(lg, e / Eg)[a * Eg + e % Eg];
    }
    if (logits_out)
      for (int i = 0; i < 8; ++i)
        if (lane + 32 * i < E) logits_out[(size_t)(t0 + a) * E + lane + 32 * i] = l[i];
    float chosen[16];
    int chosen_id[16];
    unsigned taken = 0u;  // bit i: entry lane + 32 i already chosen
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !((taken >> i) & 1u) && (bi == 0x7fffffff || l[i] > bv || (l[i] == bv && e < bi))) {
          bv = l[i];
          bi = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi))) {
          bv = ov;
          bi = oi;
        }
      }
      chosen[j] = bv;
      chosen_id[j] = bi;
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    }
    if (lane == 0) {
      float den = 0.0f;
      for (int j = 0; j < k; ++j) den += expf(chosen[j] - chosen[0]);
      for (int j = 0; j < k; ++j) {
        topk_idx[(size_t)(t0 + a) * k + j] = chosen_id[j];
        topk_w[(size_t)(t0 + a) * k + j] = expf(chosen[j] - chosen[0]) / den;
      }
    }
  }
  cl.sync();  // no CTA leaves while another still reads its shared memory
}

template <typename T>
cudaError_t launch_router_fused(float* x, const float* parts, int n_parts, size_t part_stride, const float* w_router,
                                int n, int H, int E, int k, float eps, float* logits, int32_t* topk_idx, float* topk_w,
                                T* xn, T* xn_lo, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  if (E > 256 || E % RT_G != 0 || k > 16 || k > E || (H % 4) != 0) return cudaErrorInvalidValue;
  if (n_parts < 0 || n_parts > kMaxSumParts) return cudaErrorInvalidValue;
  const size_t smem = ((size_t)(RT_OWN + RT_TOK) * H + (size_t)RT_TOK * (E / RT_G)) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(router_fused_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int clusters = (n + RT_TOK - 1) / RT_TOK;
  return launch_k_cluster(router_fused_kernel<T>, dim3(clusters * RT_G), dim3(RT_THREADS), smem, st, RT_G, x, parts,
                          n_parts, part_stride, w_router, n, H, E, k, eps, logits, topk_idx, topk_w, xn, xn_lo);
}

// ---------------------------------------------------------------- expert histogram + stable permutation
// counts[e], offsets[e] (exclusive scan, offsets[E] = n*k), perm[p] = flattened (t*k + j)
// of the p-th row when assignments are ordered by (expert, t, j); inv = inverse of perm;
// union_out = number of experts with at least one row.  One CTA of 1024 threads.
constexpr int PM_EMAX = 256;
__global__ void __launch_bounds__(1024) permute_kernel(const int32_t* __restrict__ idx, int total, int E,
                                                       int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                       int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                       int32_t* __restrict__ union_out, int item_rows,
                                                       TcWorkItem* __restrict__ items, int* __restrict__ n_items) {
  griddep_sync();
  __shared__ int cnt[PM_EMAX], base[PM_EMAX], run[PM_EMAX], ibase[PM_EMAX];
  __shared__ int wcnt[32][PM_EMAX];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0, run[e] = 0;
  __syncthreads();
  for (int a = tid; a < total; a += blockDim.x) {
    const int e = idx[a];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  if (warp == 0) {
    // exclusive scans of the counts and of the work items per expert: lane l holds
    // experts 8l .. 8l + 7
    constexpr int PER = PM_EMAX / 32;
    int c[PER], rows_l = 0, items_l = 0, used_l = 0;
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      const int e = lane * PER + q;
      c[q] = e < E ? cnt[e] : 0;
      rows_l += c[q];
      items_l += (c[q] + item_rows - 1) / item_rows;
      used_l += c[q] > 0;
    }
    int rows_x = rows_l, items_x = items_l;  // inclusive scans over lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int r2 = __shfl_up_sync(0xffffffffu, rows_x, o);
      const int i2 = __shfl_up_sync(0xffffffffu, items_x, o);
      if (lane >= o) rows_x += r2, items_x += i2;
    }
    int acc = rows_x - rows_l, iacc = items_x - items_l;
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      const int e = lane * PER + q;
      if (e < E) {
        base[e] = acc;
        ibase[e] = iacc;
        offsets[e] = acc;
        counts[e] = c[q];
      }
      acc += c[q];
      iacc += (c[q] + item_rows - 1) / item_rows;
    }
    const int used = warp_sum((float)used_l) + 0.5f;
    if (lane == 31) {
      offsets[E] = rows_x;
      *n_items = items_x;
    }
    if (lane == 0) *union_out = used;
  }
  __syncthreads();
  // work list of the grouped expert GEMMs: each expert's rows in items of <= item_rows
  for (int e = tid; e < E; e += blockDim.x)
    for (int r = 0, i = ibase[e]; r < cnt[e]; r += item_rows, ++i) {
      TcWorkItem it;
      it.group = e;
      it.row0 = base[e] + r;
      it.rows = min(item_rows, cnt[e] - r);
      it.pad = 0;
      items[i] = it;
    }
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int c0 = 0; c0 < total; c0 += blockDim.x) {
    const int a = c0 + tid;
    const int e = (a < total) ? idx[a] : -1;
    for (int i = tid; i < 32 * E; i += blockDim.x) wcnt[i / E][i % E] = 0;
    __syncthreads();
    const unsigned match = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(match & lt_mask);
    if (e >= 0 && e < E && rank == 0) wcnt[warp][e] = __popc(match);
    __syncthreads();
    if (e >= 0 && e < E) {
      int pre = 0;
      for (int w2 = 0; w2 < warp; ++w2) pre += wcnt[w2][e];
      const int pos = base[e] + run[e] + pre + rank;
      perm[pos] = a;
      inv[a] = pos;
    }
    __syncthreads();
    for (int e2 = tid; e2 < E; e2 += blockDim.x) {
      int s = 0;
      for (int w2 = 0; w2 < 32; ++w2) s += wcnt[w2][e2];
      run[e2] += s;
    }
    __syncthreads();
  }
}

cudaError_t launch_permute(const int32_t* idx, int n, int k, int E, int32_t* counts, int32_t* offsets,
                           int32_t* perm, int32_t* inv, int32_t* union_out, int item_rows, TcWorkItem* items,
                           int* n_items, cudaStream_t st) {
  if (E > PM_EMAX || item_rows < 1) return cudaErrorInvalidValue;
  return launch_k(permute_kernel, dim3(1), dim3(1024), 0, st, idx, n * k, E, counts, offsets, perm, inv, union_out, item_rows, items, n_items);
}

// xs[p] = xn[perm[p] / k] for the hi and (if present) lo parts; 16-byte vector copies
template <typename T>
__global__ void gather_rows_kernel(const T* __restrict__ xn, const T* __restrict__ xn_lo,
                                   const int32_t* __restrict__ perm, int k, int H, T* __restrict__ xs,
                                   T* __restrict__ xs_lo) {
  griddep_sync();
  const int p = blockIdx.x;
  const int t = perm[p] / k;
  const int nv = H * (int)sizeof(T) / 16;
  const uint4* src = reinterpret_cast<const uint4*>(xn + (size_t)t * H);
  const uint4* src_lo = xn_lo ? reinterpret_cast<const uint4*>(xn_lo + (size_t)t * H) : nullptr;
  uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)p * H);
  uint4* dst_lo = xn_lo ? reinterpret_cast<uint4*>(xs_lo + (size_t)p * H) : nullptr;
  // four 16-byte loads of each term in flight per thread before the stores
  constexpr int U = 4;
  for (int i0 = threadIdx.x; i0 < nv; i0 += U * blockDim.x) {
    uint4 a[U], b[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < nv) {
        a[u] = src[i];
        if (src_lo) b[u] = src_lo[i];
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < nv) {
        dst[i] = a[u];
        if (src_lo) dst_lo[i] = b[u];
      }
    }
  }
}

template <typename T>
cudaError_t launch_gather_rows(const T* xn, const T* xn_lo, const int32_t* perm, int rows, int k, int H, T* xs,
                               T* xs_lo, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  return launch_k(gather_rows_kernel<T>, dim3(rows), dim3(128), 0, st, xn, xn_lo, perm, k, H, xs, xs_lo);
}

// fp32 model: h = silu(g) * u
__global__ void swiglu_f32_kernel(const float* __restrict__ g, const float* __restrict__ u, int F,
                                  float* __restrict__ h) {
  griddep_sync();
  const size_t base = (size_t)blockIdx.x * F;
  for (int f = threadIdx.x; f < F; f += blockDim.x) {
    const float a = g[base + f];
    h[base + f] = a / (1.0f + expf(-a)) * u[base + f];
  }
}
cudaError_t launch_swiglu_f32(const float* g, const float* u, int rows, int F, float* h, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  return launch_k(swiglu_f32_kernel, dim3(rows), dim3(256), 0, st, g, u, F, h);
}

constexpr int kCombineBatch = 8;  // slot rows loaded together

// x[t] += sum_j w[t][j] * ys[inv[t*k + j]] (slots in order j = 0..k-1), then
// xn[t] = x[t] / rms(x[t]) for the next consumer (next layer's QKV, or the vocabulary
// projection with xn_lo = null).
template <typename T>
__global__ void combine_norm_kernel(const float* __restrict__ ys, const int32_t* __restrict__ inv,
                                    const float* __restrict__ w, int k, int H, float eps, float* __restrict__ x,
                                    T* __restrict__ xn, T* __restrict__ xn_lo) {
  griddep_sync();
  const int t = blockIdx.x;
  __shared__ int rows[16];
  __shared__ float ws[16];
  __shared__ float red[32];
  if (threadIdx.x < k) {
    rows[threadIdx.x] = inv[t * k + threadIdx.x];
    ws[threadIdx.x] = w[t * k + threadIdx.x];
  }
  __syncthreads();
  float4* xr = reinterpret_cast<float4*>(x + (size_t)t * H);
  float ss = 0.0f;
  for (int i = threadIdx.x; i < H / 4; i += blockDim.x) {
    // up to eight slots' row loads issued before their multiply-adds (slots still added in
    // order)
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < k; j0 += kCombineBatch) {
      float4 y[kCombineBatch];
#pragma unroll
      for (int j = 0; j < kCombineBatch; ++j)
        if (j0 + j < k) y[j] = reinterpret_cast<const float4*>(ys + (size_t)rows[j0 + j] * H)[i];
#pragma unroll
      for (int j = 0; j < kCombineBatch; ++j)
        if (j0 + j < k) {
          acc.x = fmaf(ws[j0 + j], y[j].x, acc.x);
          acc.y = fmaf(ws[j0 + j], y[j].y, acc.y);
          acc.z = fmaf(ws[j0 + j], y[j].z, acc.z);
          acc.w = fmaf(ws[j0 + j], y[j].w, acc.w);
        }
    }
    float4 v = xr[i];
    v.x += acc.x;
    v.y += acc.y;
    v.z += acc.z;
    v.w += acc.w;
    xr[i] = v;
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = block_sum(ss, red);
  const float invr = 1.0f / sqrtf(ss / (float)H + eps);
  for (int i = threadIdx.x; i < H / 4; i += blockDim.x) {
    const float4 v = xr[i];
    const size_t o = (size_t)t * H + 4 * i;
    store_act(xn, xn_lo, o + 0, v.x * invr);
    store_act(xn, xn_lo, o + 1, v.y * invr);
    store_act(xn, xn_lo, o + 2, v.z * invr);
    store_act(xn, xn_lo, o + 3, v.w * invr);
  }
}
template <typename T>
cudaError_t launch_combine_norm(const float* ys, const int32_t* inv, const float* w, int n, int k, int H, float eps,
                                float* x, T* xn, T* xn_lo, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  if (k > 16 || (H % 4) != 0) return cudaErrorInvalidValue;
  return launch_k(combine_norm_kernel<T>, dim3(n), dim3(256), 0, st, ys, inv, w, k, H, eps, x, xn, xn_lo);
}

// ---------------------------------------------------------------- canvas update
// (m, s): the largest logit and the sum of exp(l - m) over the ids seen
__device__ __forceinline__ void ms_merge(float& m, float& s, float om, float os) {
  if (om == -INFINITY) return;
  if (m == -INFINITY) {
    m = om, s = os;
    return;
  }
  if (om > m) {
    s = s * expf(m - om) + os;
    m = om;
  } else if (om < m) {
    s += os * expf(om - m);
  } else {
    s += os;
  }
}
// (m2, a): the largest logit among the ids other than an excluded one and its first
// index; merged by value, ties to the lower index
__device__ __forceinline__ void cand_merge(float& m2, int& a, float om2, int oa) {
  if (om2 > m2 || (om2 == m2 && oa < a)) {
    m2 = om2;
    a = oa;
  }
}

int update_splits(int C, int V) {
  // about four CTAs per SM over the canvas, slices of at least 4096 logits
  int s = (4 * 148 + C - 1) / (C > 0 ? C : 1);
  const int max_s = (V + 4095) / 4096;
  if (s > max_s) s = max_s;
  if (s < 1) s = 1;
  return s;
}

// per (row, slice): max, first argmax and sum exp(l - max), one streaming pass
// excl >= 0: the candidate (a, m2) skips that id (the masked-diffusion update never fills
// with the mask token); excl < 0: the candidate is the plain first argmax (m2 = m)
__global__ void update_partial_kernel(const float* __restrict__ logits, int V, int splits, int excl,
                                      UpdPart* __restrict__ part) {
  griddep_sync();
  __shared__ float sm[32], ss[32], sm2[32];
  __shared__ int sa[32];
  const int row = blockIdx.x, sp = blockIdx.y;
  const int slice = ((V + splits - 1) / splits + 3) & ~3;
  const int lo = sp * slice, hi = min(V, lo + slice);
  const float* lg = logits + (size_t)row * V;
  float m = -INFINITY, s = 0.0f, m2 = -INFINITY;
  int a = 0x7fffffff;
  const int stride = blockDim.x * 4;
  constexpr int VEC = 8;  // float4 loads in flight per thread
  for (int i0 = lo + threadIdx.x * 4; i0 < hi; i0 += VEC * stride) {
    float4 v4[VEC];
#pragma unroll
    for (int u = 0; u < VEC; ++u) {
      const int i = i0 + u * stride;
      v4[u] = (i < hi) ? *reinterpret_cast<const float4*>(lg + i) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    }
    // this chunk's max and first argmax (elements in index order), then its sum of exp
    float cm = -INFINITY;
    int ca = 0x7fffffff;
#pragma unroll
    for (int u = 0; u < VEC; ++u) {
      const float v[4] = {v4[u].x, v4[u].y, v4[u].z, v4[u].w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (v[q] > cm) {
          cm = v[q];
          ca = i0 + u * stride + q;
        }
    }
    if (cm == -INFINITY) continue;
    float cs = 0.0f;
#pragma unroll
    for (int u = 0; u < VEC; ++u) {
      cs += __expf(v4[u].x - cm) + __expf(v4[u].y - cm);
      cs += __expf(v4[u].z - cm) + __expf(v4[u].w - cm);
    }
    float cm2 = cm;
    int ca2 = ca;
    if (excl >= 0 && excl >= i0 && excl < i0 + VEC * stride && (excl - i0) % stride < 4) {
      // the excluded id lies in this chunk: its best other element, in index order
      cm2 = -INFINITY;
      ca2 = 0x7fffffff;
#pragma unroll
      for (int u = 0; u < VEC; ++u) {
        const float v[4] = {v4[u].x, v4[u].y, v4[u].z, v4[u].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int id = i0 + u * stride + q;
          if (id != excl && v[q] > cm2) {
            cm2 = v[q];
            ca2 = id;
          }
        }
      }
    }
    ms_merge(m, s, cm, cs);  // over every id
    cand_merge(m2, a, cm2, ca2);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, m, o);
    const float os = __shfl_xor_sync(0xffffffffu, s, o);
    const float om2 = __shfl_xor_sync(0xffffffffu, m2, o);
    const int oa = __shfl_xor_sync(0xffffffffu, a, o);
    ms_merge(m, s, om, os);
    cand_merge(m2, a, om2, oa);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) sm[warp] = m, ss[warp] = s, sm2[warp] = m2, sa[warp] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w2 = 1; w2 < (int)(blockDim.x >> 5); ++w2) {
      ms_merge(m, s, sm[w2], ss[w2]);
      cand_merge(m2, a, sm2[w2], sa[w2]);
    }
    UpdPart r;
    r.m = m;
    r.s = s;
    r.a = a;
    r.m2 = m2;
    part[(size_t)row * splits + sp] = r;
  }
}

__device__ __forceinline__ uint64_t splitmix64_out(uint64_t seed, uint64_t n) {
  uint64_t z = seed + (n + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// merge slices, confidence = 1 / sum exp(l - max); every position takes its argmax, then
// the n_renoise lowest-confidence positions (ties: lower position first) take a fresh
// token: SplitMix64(seed) draw number (step << 32 | position), multiply-shift onto [0, V).
// Masked mode (mask_id >= 0): positions holding a token other than mask_id keep it; a
// masked position's candidate is its best token other than mask_id, with confidence
// exp(m2 - m) / sum; of the M masked positions the min(n_renoise, M) least confident
// (ties: lower position first) stay mask_id and the others take their candidates.
__global__ void update_select_kernel(const UpdPart* __restrict__ part, int C, int V, int splits, int n_renoise,
                                     uint64_t seed, uint32_t step, int32_t* __restrict__ canvas,
                                     float* __restrict__ conf, int mask_id) {
  griddep_sync();
  extern __shared__ float den[];  // [C] sums (uniform) or confidences (masked), then [C] masked flags
  int* is_m = reinterpret_cast<int*>(den + C);
  __shared__ int n_masked;
  const int i = threadIdx.x;
  float m = -INFINITY, s = 0.0f, m2 = -INFINITY;
  int a = 0x7fffffff;
  if (i == 0) n_masked = 0;
  __syncthreads();
  if (i < C) {
    for (int sp0 = 0; sp0 < splits; sp0 += 8) {  // eight slices' partials in flight, merged in order
      UpdPart q[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (sp0 + u < splits) q[u] = part[(size_t)i * splits + sp0 + u];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (sp0 + u < splits) {
          ms_merge(m, s, q[u].m, q[u].s);
          cand_merge(m2, a, q[u].m2, q[u].a);
        }
    }
    if (mask_id < 0) {
      den[i] = s;
    } else {
      den[i] = expf(m2 - m) / s;
      is_m[i] = canvas[i] == mask_id;
      if (is_m[i]) atomicAdd(&n_masked, 1);
    }
  }
  __syncthreads();
  if (i < C) {
    if (mask_id < 0) {
      int rank = 0;
      for (int j = 0; j < C; ++j) {
        const float dj = den[j];
        rank += (dj > s) || (dj == s && j < i);
      }
      int tok = a;
      if (rank < n_renoise) {
        const uint64_t x = splitmix64_out(seed, ((uint64_t)step << 32) | (uint64_t)i);
        tok = (int)(((x >> 32) * (uint64_t)V) >> 32);
      }
      canvas[i] = tok;
      if (conf) conf[i] = 1.0f / s;
    } else {
      const float ci = den[i];
      if (is_m[i]) {
        int rank = 0;  // among the masked positions, by confidence, ties to the lower position
        for (int j = 0; j < C; ++j) rank += is_m[j] && (den[j] < ci || (den[j] == ci && j < i));
        const int keep = min(n_renoise, n_masked);
        canvas[i] = rank < keep ? mask_id : a;
      }
      if (conf) conf[i] = ci;
    }
  }
}

cudaError_t launch_update_partial(const float* logits, int C, int V, int splits, int excl, UpdPart* part,
                                  cudaStream_t st) {
  if (C <= 0) return cudaSuccess;
  return launch_k(update_partial_kernel, dim3(C, splits), dim3(256), 0, st, logits, V, splits, excl, part);
}
cudaError_t launch_update_select(const UpdPart* part, int C, int V, int splits, int n_renoise, uint64_t seed,
                                 uint32_t step, int32_t* canvas, float* conf, int mask_id, cudaStream_t st) {
  if (C <= 0) return cudaSuccess;
  if (C > 1024) return cudaErrorInvalidValue;
  const int threads = (C + 31) & ~31;
  return launch_k(update_select_kernel, dim3(1), dim3(threads), 2 * C * sizeof(float), st, part, C, V, splits,
                  n_renoise, seed, step, canvas, conf, mask_id);
}

// ---------------------------------------------------------------- int32 fill
__global__ void fill_i32_kernel(int32_t* p, int n, int32_t v) {
  griddep_sync();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = v;
}
cudaError_t launch_fill_i32(int32_t* p, int n, int32_t v, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  return launch_k(fill_i32_kernel, dim3((n + 255) / 256), dim3(256), 0, st, p, n, v);
}

// ---------------------------------------------------------------- timeout self-test
// One thread waits on an mbarrier that nothing will complete; the bounded wait gives
// up after limit_ns, records the error code and the kernel returns normally.
__global__ void bounded_wait_selftest_kernel(int* err, uint64_t limit_ns) {
  griddep_sync();
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    mbar_wait_ns(&bar, 0, limit_ns, err, DG_DEVERR_TIMEOUT_FULL);
  }
}
cudaError_t launch_bounded_wait_selftest(int* err, uint64_t limit_ns, cudaStream_t st) {
  return launch_k(bounded_wait_selftest_kernel, dim3(1), dim3(32), 0, st, err, limit_ns);
}

// ---------------------------------------------------------------- explicit instantiations
#define DG_INST(T)                                                                                                \
  template cudaError_t launch_embed_norm<T>(const int32_t*, const T*, int, int, int, float, float*, T*, T*, int*, \
                                            cudaStream_t);                                                        \
  template cudaError_t launch_rope_scatter<T>(const float*, int, size_t, int, int, int, int, int, float, T*, T*,  \
                                              T*, int, T*, T*, T*, int, int, cudaStream_t);                       \
  template cudaError_t launch_router_fused<T>(float*, const float*, int, size_t, const float*, int, int, int, int, \
                                              float, float*, int32_t*, float*, T*, T*, cudaStream_t);             \
  template cudaError_t launch_gather_rows<T>(const T*, const T*, const int32_t*, int, int, int, T*, T*,          \
                                             cudaStream_t);                                                       \
  template cudaError_t launch_combine_norm<T>(const float*, const int32_t*, const float*, int, int, int, float,   \
                                              float*, T*, T*, cudaStream_t);
DG_INST(float)
DG_INST(bf16)

}  // namespace dg
