// tcgen05 flash attention over the KV cache, both attention modes of the pass:
//   denoising mode: every canvas query sees all cached prefix keys and all canvas
//                   keys (bidirectional block rows of the prefix/block mask);
//   prefill mode:   new tokens see keys up to their own position (causal rows).
// One CTA = one query head x 128 query rows x a contiguous range of 128-key chunks
// (split-KV; partial results merged by attn_merge_kernel).  S = Q K^T and
// O += P V both run on the tensor core with fp32 accumulators in TMEM (S: columns
// 0..127, O: columns 128..255); softmax runs one query row per thread.  V is kept
// transposed in the cache ([d][position]) so both MMAs read K-major operands.
// The running max is only raised when it grows by more than 2^8 (log2 domain), so
// O in TMEM is rescaled rarely; P and l use the same (possibly stale) max, which
// leaves O / l exact.  P is carried as two bf16 terms, hi = bf16(p) and
// lo = bf16(p - hi), and O accumulates hi V + lo V: the probabilities keep about 16
// significant bits instead of 8, which keeps the attention output within a few
// fp32-accumulation ulps of exact softmax attention.
#include <math.h>

#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

constexpr int AT_BQ = 128;
constexpr int AT_BKEYS = 128;
constexpr int AT_D = 128;
constexpr uint32_t AT_HALF = 128 * 128;  // one [128 rows][64 bf16] swizzled block: 16 KB
constexpr int AT_SMEM = 1024 + 14 * AT_HALF;  // Q (2 blocks), K[2] (4), Vt[2] (4), P hi (2), P lo (2)

__global__ void __launch_bounds__(128, 1)
    tc_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmVt, const TcAttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_bar;
  __shared__ __align__(8) uint64_t kv_bar[2];
  __shared__ __align__(8) uint64_t s_bar;
  __shared__ __align__(8) uint64_t pv_bar;
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int abort_s;
  __shared__ int kv_issued_s, kv_consumed_s, q_consumed_s;

  const int tid = threadIdx.x, warp = tid >> 5;
  const int qt = blockIdx.x, h = blockIdx.y, sp = blockIdx.z;
  const int kvh = h / p.group;
  const int q_row0 = qt * AT_BQ;
  const int rows_here = min(AT_BQ, p.n_q - q_row0);
  int kv_end = p.n_keys;
  if (p.causal) kv_end = min(p.n_keys, p.q_pos0 + q_row0 + rows_here);
  const int nch_total = (kv_end + AT_BKEYS - 1) / AT_BKEYS;
  const int c_begin = sp * p.chunks_per_split;
  const int nck = min(nch_total, c_begin + p.chunks_per_split) - c_begin;
  const int qrow = q_row0 + tid;
  const int qpos = p.q_pos0 + qrow;

  if (nck <= 0) {
    // this split sees no key of the tile: an empty partial (weight 0 in the merge)
    griddep_sync();
    if (qrow < p.n_q) {
      float* po = p.part_o + (((size_t)sp * p.nq + h) * p.n_q + qrow) * AT_D;
      for (int i = 0; i < AT_D; ++i) po[i] = 0.0f;
      p.part_lse[((size_t)sp * p.nq + h) * p.n_q + qrow] = -INFINITY;
    }
    return;
  }

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                    // 2 blocks: d 0..63, d 64..127
  uint8_t* sK = smem + 2 * AT_HALF;      // [buf][2 blocks]
  uint8_t* sV = smem + 6 * AT_HALF;      // [buf][2 blocks]: V^T rows = d, K = keys 0..63 / 64..127
  uint8_t* sP = smem + 10 * AT_HALF;     // P hi, 2 blocks: keys 0..63, 64..127
  uint8_t* sPl = smem + 12 * AT_HALF;    // P lo, same layout

  if (warp == 0) tmem_alloc(&tmem_base_s, 256);
  if (tid == 32) {
    mbar_init(&q_bar, 1);
    mbar_init(&kv_bar[0], 1);
    mbar_init(&kv_bar[1], 1);
    mbar_init(&s_bar, 1);
    mbar_init(&pv_bar, 1);
    mbar_init(&drain_bar, 1);
    abort_s = 0;
    kv_issued_s = 0;
    kv_consumed_s = 0;
    q_consumed_s = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_sync();  // the previous kernel wrote q and this layer's canvas K/V
  const uint32_t tmem_S = tmem_base_s;
  const uint32_t tmem_O = tmem_base_s + 128;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

  auto load_kv = [&](int buf, int chunk) {
    const int key0 = chunk * AT_BKEYS;
    uint8_t* k = sK + buf * 2 * AT_HALF;
    uint8_t* v = sV + buf * 2 * AT_HALF;
    mbar_arrive_expect_tx(&kv_bar[buf], 4 * AT_HALF);
    tma_load_3d(k, &tmK, 0, key0, kvh, &kv_bar[buf]);
    tma_load_3d(k + AT_HALF, &tmK, 64, key0, kvh, &kv_bar[buf]);
    tma_load_3d(v, &tmVt, key0, 0, kvh, &kv_bar[buf]);
    tma_load_3d(v + AT_HALF, &tmVt, key0 + 64, 0, kvh, &kv_bar[buf]);
  };

  if (tid == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmVt);
    mbar_arrive_expect_tx(&q_bar, 2 * AT_HALF);
    tma_load_3d(sQ, &tmQ, 0, q_row0, h, &q_bar);
    tma_load_3d(sQ + AT_HALF, &tmQ, 64, q_row0, h, &q_bar);
    for (int i = 0; i < 2 && i < nck; ++i) load_kv(i, c_begin + i);
    kv_issued_s = min(2, nck);
  }

  const uint32_t idesc = idesc_bf16_f32(AT_BQ, AT_BKEYS);
  float m_used = -INFINITY, l = 0.0f;
  const int key_lim = p.causal ? min(p.n_keys, qpos + 1) : p.n_keys;

  for (int j = 0; j < nck; ++j) {
    const int buf = j & 1;
    if (tid == 0) {
      bool ok = true;
      if (j == 0) {
        ok = mbar_wait(&q_bar, 0, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
        if (ok) q_consumed_s = 1;
      }
      ok = ok && mbar_wait(&kv_bar[buf], (uint32_t)(j >> 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
      if (ok) {
        kv_consumed_s = j + 1;
        tc_fence_after();
        const uint32_t q = smem_u32(sQ), k = smem_u32(sK + buf * 2 * AT_HALF);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma(tmem_S, sw128_kmajor_desc(q + kb * AT_HALF + kk * 32),
                   sw128_kmajor_desc(k + kb * AT_HALF + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
      }
      tc_commit(&s_bar);
    }
    __syncwarp();
    mbar_wait(&s_bar, (uint32_t)j & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
    tc_fence_after();

    float s[AT_BKEYS];
#pragma unroll
    for (int c = 0; c < AT_BKEYS / 16; ++c) {
      uint32_t r[16];
      tmem_ld16(tmem_S + lane_off + c * 16, r);
      tc_wait_ld();
#pragma unroll
      for (int i = 0; i < 16; ++i) s[c * 16 + i] = __uint_as_float(r[i]) * p.scale_log2;
    }
    const int key0 = (c_begin + j) * AT_BKEYS;
    float rmax = -INFINITY;
#pragma unroll
    for (int i = 0; i < AT_BKEYS; ++i) {
      if (key0 + i >= key_lim) s[i] = -INFINITY;
      rmax = fmaxf(rmax, s[i]);
    }

    // PV of the previous chunk done: O is stable, P smem and the other KV buffer are free
    if (j > 0) mbar_wait(&pv_bar, (uint32_t)(j - 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
    if (tid == 0 && j >= 1 && j + 1 < nck && !abort_s) {
      load_kv((j + 1) & 1, c_begin + j + 1);
      kv_issued_s = j + 2;
    }
    const bool upd = rmax > m_used + 8.0f;
    const float alpha = upd ? exp2f(m_used - rmax) : 1.0f;  // 0 while nothing was visible yet
    // tcgen05.ld/st are warp-collective: the whole warp rescales if any of its rows must
    if (__any_sync(0xffffffffu, upd && j > 0)) {
      {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < AT_D / 16; ++c) {
          uint32_t r[16];
          tmem_ld16(tmem_O + lane_off + c * 16, r);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st16(tmem_O + lane_off + c * 16, r);
        }
        tc_wait_st();
      }
    }
    if (upd) {
      l *= alpha;
      m_used = rmax;
    }
    // P = exp2(s - m_used) as hi + lo bf16 terms, written as K-major A operands of the PV MMAs
#pragma unroll
    for (int blk = 0; blk < 2; ++blk) {
      uint8_t* pb = sP + blk * AT_HALF;
      uint8_t* pl = sPl + blk * AT_HALF;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t wh[4], wl[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i0 = blk * 64 + c * 8 + 2 * e;
          const float p0 = (s[i0] == -INFINITY) ? 0.0f : exp2f(s[i0] - m_used);
          const float p1 = (s[i0 + 1] == -INFINITY) ? 0.0f : exp2f(s[i0 + 1] - m_used);
          l += p0 + p1;
          const __nv_bfloat162 hi = __floats2bfloat162_rn(p0, p1);
          const __nv_bfloat162 lo = __floats2bfloat162_rn(p0 - __low2float(hi), p1 - __high2float(hi));
          wh[e] = *reinterpret_cast<const uint32_t*>(&hi);
          wl[e] = *reinterpret_cast<const uint32_t*>(&lo);
        }
        *reinterpret_cast<uint4*>(pb + sw128_offset(tid, c)) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
        *reinterpret_cast<uint4*>(pl + sw128_offset(tid, c)) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      if (!abort_s) {
        tc_fence_after();
        const uint32_t pp = smem_u32(sP), pl = smem_u32(sPl), v = smem_u32(sV + buf * 2 * AT_HALF);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t vd = sw128_kmajor_desc(v + kb * AT_HALF + kk * 32);
            tc_mma(tmem_O, sw128_kmajor_desc(pp + kb * AT_HALF + kk * 32), vd, idesc,
                   (j > 0 || (kb | kk) != 0) ? 1u : 0u);
            tc_mma(tmem_O, sw128_kmajor_desc(pl + kb * AT_HALF + kk * 32), vd, idesc, 1u);
          }
      }
      tc_commit(&pv_bar);
    }
    __syncwarp();
  }
  mbar_wait(&pv_bar, (uint32_t)(nck - 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
  __syncthreads();
  const bool run = (abort_s == 0);
  tc_fence_after();
  if (run) {
    const bool valid = qrow < p.n_q;
    const float inv_l = (l > 0.0f) ? 1.0f / l : 0.0f;
    if (p.n_splits == 1) {
      const size_t base = (size_t)qrow * p.nq * AT_D + (size_t)h * AT_D;
#pragma unroll
      for (int c = 0; c < AT_D / 16; ++c) {
        uint32_t r[16];
        tmem_ld16(tmem_O + lane_off + c * 16, r);
        tc_wait_ld();
        if (valid) {
          uint32_t w[8], wl[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float a = __uint_as_float(r[2 * e]) * inv_l, b = __uint_as_float(r[2 * e + 1]) * inv_l;
            const __nv_bfloat162 hi = __floats2bfloat162_rn(a, b);
            const __nv_bfloat162 lo = __floats2bfloat162_rn(a - __low2float(hi), b - __high2float(hi));
            w[e] = *reinterpret_cast<const uint32_t*>(&hi);
            wl[e] = *reinterpret_cast<const uint32_t*>(&lo);
          }
          uint4* dst = reinterpret_cast<uint4*>(p.out + base + c * 16);
          dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
          dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
          if (p.out_lo) {
            uint4* dl = reinterpret_cast<uint4*>(p.out_lo + base + c * 16);
            dl[0] = make_uint4(wl[0], wl[1], wl[2], wl[3]);
            dl[1] = make_uint4(wl[4], wl[5], wl[6], wl[7]);
          }
        }
      }
    } else {
      float* po = p.part_o + (((size_t)sp * p.nq + h) * p.n_q + qrow) * AT_D;
#pragma unroll
      for (int c = 0; c < AT_D / 16; ++c) {
        uint32_t r[16];
        tmem_ld16(tmem_O + lane_off + c * 16, r);
        tc_wait_ld();
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(po + c * 16);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_float4(__uint_as_float(r[4 * e]) * inv_l, __uint_as_float(r[4 * e + 1]) * inv_l,
                                 __uint_as_float(r[4 * e + 2]) * inv_l, __uint_as_float(r[4 * e + 3]) * inv_l);
        }
      }
      if (valid)
        p.part_lse[((size_t)sp * p.nq + h) * p.n_q + qrow] = (l > 0.0f) ? m_used + log2f(l) : -INFINITY;
    }
  } else if (tid == 0) {
    if (!q_consumed_s) mbar_wait_drain(&q_bar, 0);
    for (int c = kv_consumed_s; c < kv_issued_s; ++c) mbar_wait_drain(&kv_bar[c & 1], (uint32_t)(c >> 1) & 1u);
    tc_commit(&drain_bar);
    mbar_wait_drain(&drain_bar, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem_base_s, 256);
}

__global__ void attn_merge_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse, int n_splits,
                                  int nq, int n_q, int d, __nv_bfloat16* out, __nv_bfloat16* out_lo) {
  griddep_sync();
  const int qrow = blockIdx.x, h = blockIdx.y, t = threadIdx.x;
  float mx = -INFINITY;
  for (int s = 0; s < n_splits; ++s) mx = fmaxf(mx, part_lse[((size_t)s * nq + h) * n_q + qrow]);
  for (int dd = t; dd < d; dd += blockDim.x) {
    float num = 0.0f, den = 0.0f;
    if (mx != -INFINITY) {
      for (int s = 0; s < n_splits; ++s) {
        const float lse = part_lse[((size_t)s * nq + h) * n_q + qrow];
        if (lse == -INFINITY) continue;
        const float w = exp2f(lse - mx);
        num += w * part_o[(((size_t)s * nq + h) * n_q + qrow) * d + dd];
        den += w;
      }
    }
    const float v = den > 0.0f ? num / den : 0.0f;
    const size_t o = (size_t)qrow * nq * d + (size_t)h * d + dd;
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    out[o] = hi;
    if (out_lo) out_lo[o] = __float2bfloat16_rn(v - __bfloat162float(hi));
  }
}

cudaError_t launch_tc_attention(const CUtensorMap& Q, const CUtensorMap& K, const CUtensorMap& Vt,
                                const TcAttnParams& p, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(tc_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((p.n_q + AT_BQ - 1) / AT_BQ, p.nq, p.n_splits);
  return launch_k(tc_attn_kernel, dim3(grid), dim3(128), AT_SMEM, st, Q, K, Vt, p);
}

cudaError_t launch_attn_merge(const float* part_o, const float* part_lse, int n_splits, int nq, int n_q, int d,
                              __nv_bfloat16* out, __nv_bfloat16* out_lo, cudaStream_t st) {
  return launch_k(attn_merge_kernel, dim3(n_q, nq), dim3(128), 0, st, part_o, part_lse, n_splits, nq, n_q, d, out, out_lo);
}

}  // namespace dg
