// tcgen05 / TMEM / TMA GEMM for every dense contraction of the bf16 pass:
// QKV and output projections, the two grouped expert GEMMs and the vocabulary
// projection.  All of them stream a weight matrix once while the token operand
// (at most 256 rows per tile) is small, so weights sit on the 128-row M side of
// the MMA and tokens on N ("swap-AB"): one CTA owns a 128-row weight tile and
// all tokens of its group (an expert's routed rows, or the whole canvas).
//
// Roles (128 threads): thread 0 issues TMA loads into a ring of smem stages,
// thread 32 issues tcgen05.mma into a TMEM accumulator and frees stages with
// tcgen05.commit, then all four warps drain TMEM (warp w owns lanes 32w..32w+31)
// through the epilogue.  Stage count adapts to the token count at run time.
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

constexpr int TC_BM = 128;
constexpr int TC_BK = 64;
constexpr int TC_MAX_N = 256;
constexpr int TC_B_BOX = 16;
constexpr int TC_MAX_STAGES = 24;

template <int EPI>
__global__ void __launch_bounds__(128, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmB2, const TcGemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[TC_MAX_STAGES];
  __shared__ __align__(8) uint64_t empty_bar[TC_MAX_STAGES];
  __shared__ __align__(8) uint64_t accum_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int abort_s;
  __shared__ int n_issued_s, n_consumed_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.y;
  int tok_begin = 0, tok_end = p.n_tokens;
  if (p.group_off) {
    tok_begin = p.group_off[g];
    tok_end = p.group_off[g + 1];
  }
  const int split = (int)blockIdx.z % p.k_splits;
  const int chunk = (int)blockIdx.z / p.k_splits;
  const int t0 = tok_begin + chunk * TC_MAX_N;
  if (t0 >= tok_end) return;  // uniform across the CTA, before any allocation
  const int n = min(TC_MAX_N, tok_end - t0);
  const int n_pad = (n + 15) & ~15;
  const int terms = p.two_terms ? 2 : 1;
  const uint32_t a_bytes = TC_BM * TC_BK * 2;
  const uint32_t b_bytes = (uint32_t)n_pad * TC_BK * 2;  // one term
  const uint32_t stage_bytes = a_bytes + terms * b_bytes;
  int stages = p.smem_budget / (int)stage_bytes;
  if (stages > TC_MAX_STAGES) stages = TC_MAX_STAGES;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int a_row0 = g * p.a_rows_per_group + (int)blockIdx.x * TC_BM;
  const int nkb = p.K / TC_BK / p.k_splits;
  const int kb0 = split * nkb;
  uint32_t tmem_cols = 32;
  while (tmem_cols < (uint32_t)n_pad) tmem_cols <<= 1;

  if (warp == 0) tmem_alloc(&tmem_base_s, tmem_cols);
  if (tid == 32) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&accum_bar, 1);
    abort_s = 0;
    n_issued_s = 0;
    n_consumed_s = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;

  if (tid == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if (terms == 2) prefetch_tmap(&tmB2);
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % stages;
      const uint32_t ph = (uint32_t)(kb / stages) & 1u;
      if (!mbar_wait(&empty_bar[s], ph ^ 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_EMPTY)) break;
      uint8_t* sa = smem + (size_t)s * stage_bytes;
      uint8_t* sb = sa + a_bytes;
      const int kx = (kb0 + kb) * TC_BK;
      mbar_arrive_expect_tx(&full_bar[s], stage_bytes);
      tma_load_2d(sa, &tmA, kx, a_row0, &full_bar[s]);
      for (int r = 0; r < n_pad; r += TC_B_BOX) tma_load_2d(sb + r * 128, &tmB, kx, t0 + r, &full_bar[s]);
      if (terms == 2)
        for (int r = 0; r < n_pad; r += TC_B_BOX)
          tma_load_2d(sb + b_bytes + r * 128, &tmB2, kx, t0 + r, &full_bar[s]);
      n_issued_s = kb + 1;
    }
  } else if (tid == 32) {
    const uint32_t idesc = idesc_bf16_f32(TC_BM, n_pad);
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % stages;
      const uint32_t ph = (uint32_t)(kb / stages) & 1u;
      if (!mbar_wait(&full_bar[s], ph, &abort_s, p.err, DG_DEVERR_TIMEOUT_FULL)) break;
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + (size_t)s * stage_bytes);
      const uint32_t sb = sa + a_bytes;
#pragma unroll
      for (int kk = 0; kk < TC_BK / 16; ++kk) {
        const uint64_t ad = sw128_kmajor_desc(sa + kk * 32);
        tc_mma(tmem, ad, sw128_kmajor_desc(sb + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
        if (terms == 2) tc_mma(tmem, ad, sw128_kmajor_desc(sb + b_bytes + kk * 32), idesc, 1u);
      }
      tc_commit(&empty_bar[s]);
      n_consumed_s = kb + 1;
    }
    tc_commit(&accum_bar);
  }
  __syncwarp();

  mbar_wait(&accum_bar, 0, &abort_s, p.err, DG_DEVERR_TIMEOUT_ACCUM);
  __syncthreads();
  const bool run = (abort_s == 0);  // uniform across the CTA
  tc_fence_after();
  const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);
  if (run) {
    if (EPI == EPI_STORE_F32 || EPI == EPI_ADD_F32) {
      float* out = reinterpret_cast<float*>(p.out) + (size_t)split * p.split_stride;
      const int feat = (int)blockIdx.x * TC_BM + warp * 32 + lane;
      for (int c0 = 0; c0 < n_pad; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(t_lane + c0, r);
        tc_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (c0 + j < n) {
            float* dst = out + (size_t)(t0 + c0 + j) * p.ld_out + feat;
            const float v = __uint_as_float(r[j]);
            if (EPI == EPI_ADD_F32)
              *dst += v;
            else
              *dst = v;
          }
        }
      }
    } else {
      // packed gate/up tile: lanes 0..63 hold gate rows f0..f0+63, lanes 64..127 the up rows
      float* xch = reinterpret_cast<float*>(smem);  // [n_pad][64]; all loads were consumed
      if (warp >= 2) {
        for (int c0 = 0; c0 < n_pad; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(t_lane + c0, r);
          tc_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) xch[(c0 + j) * 64 + (warp - 2) * 32 + lane] = __uint_as_float(r[j]);
        }
      }
      __syncthreads();
      if (warp < 2) {
        bf16* out = reinterpret_cast<bf16*>(p.out);
        bf16* out_lo = reinterpret_cast<bf16*>(p.out_lo);
        const int f = (int)blockIdx.x * 64 + warp * 32 + lane;
        for (int c0 = 0; c0 < n_pad; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(t_lane + c0, r);
          tc_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (c0 + j < n) {
              const float gte = __uint_as_float(r[j]);
              const float up = xch[(c0 + j) * 64 + warp * 32 + lane];
              const float hv = gte / (1.0f + expf(-gte)) * up;
              const bf16 hi = __float2bfloat16_rn(hv);
              out[(size_t)(t0 + c0 + j) * p.ld_out + f] = hi;
              if (out_lo) out_lo[(size_t)(t0 + c0 + j) * p.ld_out + f] = __float2bfloat16_rn(hv - __bfloat162float(hi));
            }
          }
        }
      }
    }
  } else if (tid == 0) {
    // wind down: let issued loads and MMAs land before the smem / TMEM go away
    for (int kb = n_consumed_s; kb < n_issued_s; ++kb)
      mbar_wait_drain(&full_bar[kb % stages], (uint32_t)(kb / stages) & 1u);
    mbar_wait_drain(&accum_bar, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, tmem_cols);
}

cudaError_t launch_tc_gemm(int epi, const CUtensorMap& A, const CUtensorMap& B, const CUtensorMap& B2,
                           const TcGemmParams& p, int m_tiles, int n_groups, int max_rows_per_group, cudaStream_t st) {
  if (m_tiles <= 0 || n_groups <= 0 || max_rows_per_group <= 0) return cudaSuccess;
  if (p.k_splits < 1 || (p.K / TC_BK) % p.k_splits != 0 || (p.k_splits > 1 && n_groups != 1))
    return cudaErrorInvalidValue;
  const int smem = p.smem_budget + 1024;
  dim3 grid(m_tiles, n_groups, ((max_rows_per_group + TC_MAX_N - 1) / TC_MAX_N) * p.k_splits);
  cudaError_t e;
  switch (epi) {
    case EPI_STORE_F32:
      e = cudaFuncSetAttribute(tc_gemm_kernel<EPI_STORE_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      tc_gemm_kernel<EPI_STORE_F32><<<grid, 128, smem, st>>>(A, B, B2, p);
      break;
    case EPI_ADD_F32:
      e = cudaFuncSetAttribute(tc_gemm_kernel<EPI_ADD_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      tc_gemm_kernel<EPI_ADD_F32><<<grid, 128, smem, st>>>(A, B, B2, p);
      break;
    case EPI_SWIGLU_BF16:
      e = cudaFuncSetAttribute(tc_gemm_kernel<EPI_SWIGLU_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      tc_gemm_kernel<EPI_SWIGLU_BF16><<<grid, 128, smem, st>>>(A, B, B2, p);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace dg
