// The vocabulary projection fused with the first half of the canvas update: the same
// persistent weight-streaming tcgen05 GEMM as the bf16 path (output-matrix rows on M,
// canvas tokens on N, fp32 accumulators in TMEM), but the epilogue never stores the
// fp32 logits.  For every (token, 128-id tile) it writes the update's partial statistics
// -- the largest logit m, the sum of exp(l - m), and the candidate (the first largest
// id, or the first largest id other than an excluded one) with its logit -- the record
// the canvas-update kernels merge.  A row-merge kernel then reduces each token's tile
// records in id order to one record, and the selection runs on those.  The logits the
// pass would write and the update read back (4 C V bytes each way) are not moved.
//
// Roles (192 threads, one CTA per SM, tiles blockIdx.x, blockIdx.x + gridDim.x, ...):
// warp 0 TMA (weights 128 rows x 64, tokens in boxes of 64 then 16 rows, single term),
// warp 1 MMA into one of two TMEM accumulators, warps 2-5 the statistics epilogue of the
// other: each warp reduces its 32 ids for 32 token columns at a time with transposed
// shuffles (lane L ends with column L), the four warps' records are merged in id order
// through shared memory.  Every wait is bounded.
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

constexpr int VU_BM = 128;
constexpr int VU_BK = 64;
constexpr int VU_MAX_STAGES = 8;
constexpr int VU_THREADS = 192;
constexpr int VU_B_BOX = 16;
constexpr int VU_B_BOX_BIG = 64;

// the merges of the canvas-update kernels: (max, sum of exp) and (candidate logit, id),
// ties to the lower id
__device__ __forceinline__ void vu_ms_merge(float& m, float& s, float om, float os) {
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
__device__ __forceinline__ void vu_cand_merge(float& m2, int& a, float om2, int oa) {
  if (om2 > m2 || (om2 == m2 && oa < a)) {
    m2 = om2;
    a = oa;
  }
}

// Transposed warp reductions over 32 token columns: lane L enters with its id's value
// for each of the 32 columns and leaves with column L's result over the warp's 32 ids.
// At the stage with offset o each lane keeps one half of its current columns (the upper
// half when bit o of its lane is set), sends the other half to lane L ^ o and merges what
// it receives into what it keeps; after five stages the one column left is column L.
// 31 exchanges per value for 32 columns, all of a stage independent of each other.
__device__ __forceinline__ void vu_tr_argmax(float (&m)[32], int (&a)[32], int lane) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < o; ++j) {
      const float km = up ? m[j + o] : m[j], sm = up ? m[j] : m[j + o];
      const int ka = up ? a[j + o] : a[j], sa = up ? a[j] : a[j + o];
      const float rm = __shfl_xor_sync(0xffffffffu, sm, o);
      const int ra = __shfl_xor_sync(0xffffffffu, sa, o);
      const bool take = rm > km || (rm == km && ra < ka);  // ties to the lower id
      m[j] = take ? rm : km;
      a[j] = take ? ra : ka;
    }
  }
}
__device__ __forceinline__ void vu_tr_sum(float (&e)[32], int lane) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < o; ++j) {
      const float ke = up ? e[j + o] : e[j], se = up ? e[j] : e[j + o];
      e[j] = ke + __shfl_xor_sync(0xffffffffu, se, o);
    }
  }
}

__global__ void __launch_bounds__(VU_THREADS, 1)
    tc_vocab_update_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmBb, const VuParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[VU_MAX_STAGES];
  __shared__ __align__(8) uint64_t empty_bar[VU_MAX_STAGES];
  __shared__ __align__(8) uint64_t acc_full[2];
  __shared__ __align__(8) uint64_t acc_empty[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ UpdPart red[4][32];  // one 32-column group's records of the four epilogue warps
  __shared__ int epi_ok[4];       // each epilogue warp's wait result, so that all four leave together
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int abort_s;
  __shared__ int n_issued_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t a_bytes = VU_BM * VU_BK * 2;
  const uint32_t b_bytes = (uint32_t)p.n_max * 128;
  const uint32_t stage_bytes = a_bytes + b_bytes;
  int stages = p.smem_budget / (int)stage_bytes;
  if (stages > VU_MAX_STAGES) stages = VU_MAX_STAGES;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int acc_cols = p.n_max;
  uint32_t tmem_cols = 32;
  while (tmem_cols < (uint32_t)(2 * acc_cols)) tmem_cols <<= 1;
  const int nkb = p.K / VU_BK;
  // tile t = (id tile t / chunks, token chunk t % chunks): the CTAs that share an id tile's
  // weights run together, so the output matrix is read from DRAM once for all chunks
  const int chunks = (p.n_tokens + p.n_max - 1) / p.n_max;
  const int n_tiles = chunks * p.m_tiles;

  if (warp == 1) tmem_alloc(&tmem_base_s, tmem_cols);
  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(&drain_bar, 1);
    abort_s = 0;
    n_issued_s = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  griddep_sync();  // the final normed state comes from the previous kernel

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      prefetch_tmap(&tmBb);
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        const int m = t / chunks, row0 = (t % chunks) * p.n_max;
        const int rows = min(p.n_max, p.n_tokens - row0);
        const int n_pad = (rows + 15) & ~15;
        const uint32_t tx = a_bytes + (uint32_t)n_pad * 128u;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % stages;
          if (!mbar_wait(&empty_bar[s], ((uint32_t)(it / stages) & 1u) ^ 1u, &abort_s, p.err,
                         DG_DEVERR_TIMEOUT_EMPTY)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + (size_t)s * stage_bytes;
          uint8_t* sb = sa + a_bytes;
          const int kx = ((kb + t) % nkb) * VU_BK;  // tiles running together start at different k-blocks
          if (!DG_GUARD((kx * 2) % 16 == 0 && n_pad <= p.n_max &&
                            (uint32_t)(s + 1) * stage_bytes <= (uint32_t)p.smem_budget &&
                            (uint32_t)(2 * acc_cols) <= tmem_cols,
                        p.err)) {
            abort_s = 1;
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full_bar[s], tx);
          tma_load_3d(sa, &tmA, kx, m * VU_BM, 0, &full_bar[s]);
          int r = 0;
          for (; r + VU_B_BOX_BIG <= n_pad; r += VU_B_BOX_BIG) tma_load_2d(sb + r * 128, &tmBb, kx, row0 + r, &full_bar[s]);
          for (; r < n_pad; r += VU_B_BOX) tma_load_2d(sb + r * 128, &tmB, kx, row0 + r, &full_bar[s]);
          n_issued_s = it + 1;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int it = 0, j = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++j) {
        const int row0 = (t % chunks) * p.n_max;
        const int n_pad = (min(p.n_max, p.n_tokens - row0) + 15) & ~15;
        const int buf = j & 1;
        if (!mbar_wait(&acc_empty[buf], ((uint32_t)(j >> 1) & 1u) ^ 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ACCUM))
          break;
        tc_fence_after();
        const uint32_t d0 = tmem + (uint32_t)(buf * acc_cols);
        const uint32_t idesc = idesc_bf16_f32(VU_BM, n_pad);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % stages;
          if (!mbar_wait(&full_bar[s], (uint32_t)(it / stages) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + (size_t)s * stage_bytes);
          const uint32_t sb = sa + a_bytes;
#pragma unroll
          for (int kk = 0; kk < VU_BK / 16; ++kk)
            tc_mma(d0, sw128_kmajor_desc(sa + kk * 32), sw128_kmajor_desc(sb + kk * 32), idesc,
                   (kb != 0 || kk != 0) ? 1u : 0u);
          tc_commit(&empty_bar[s]);
        }
        if (ok) tc_commit(&acc_full[buf]);
      }
      tc_commit(&drain_bar);
    }
  } else {
    // ---------------- statistics epilogue, warps 2..5: TMEM lanes (warp % 4) * 32 .. + 31
    const int lg = warp & 3;
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    int j = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++j) {
      const int m = t / chunks, row0 = (t % chunks) * p.n_max;
      const int rows = min(p.n_max, p.n_tokens - row0);
      const int n_pad = (rows + 15) & ~15;
      const int buf = j & 1;
      // the four warps meet at named barriers below: they decide together whether to go on
      bool ok = mbar_wait(&acc_full[buf], (uint32_t)(j >> 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ACCUM);
      ok = __all_sync(0xffffffffu, ok);
      if (lane == 0) epi_ok[lg] = ok;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      const bool all_ok = epi_ok[0] && epi_ok[1] && epi_ok[2] && epi_ok[3];
      asm volatile("bar.sync 1, 128;" ::: "memory");  // epi_ok is rewritten at the next tile
      if (!all_ok) break;
      tc_fence_after();
      const uint32_t t0 = tmem + (uint32_t)(buf * acc_cols) + lane_off;
      const int id = m * VU_BM + lg * 32 + lane;  // this lane's vocabulary id
      const bool valid_id = id < p.V;
      // the excluded id's lane, when it lies in this warp's 32 ids (warp-uniform)
      const bool excl_here = p.excl >= 0 && p.excl >= m * VU_BM + lg * 32 && p.excl < m * VU_BM + lg * 32 + 32;
      for (int c0 = 0; c0 < n_pad; c0 += 32) {
        // this lane's id's logits for 32 token columns (16 when only 16 are left; the
        // others count as -inf and their records are not stored)
        float v[32], mm[32], e[32];
        int aa[32];
        {
          uint32_t r[16];
          tmem_ld16(t0 + c0, r);
          tc_wait_ld();
#pragma unroll
          for (int q = 0; q < 16; ++q) v[q] = valid_id ? __uint_as_float(r[q]) : -INFINITY;
          if (c0 + 16 < n_pad) {
            tmem_ld16(t0 + c0 + 16, r);
            tc_wait_ld();
#pragma unroll
            for (int q = 0; q < 16; ++q) v[16 + q] = valid_id ? __uint_as_float(r[q]) : -INFINITY;
          } else {
#pragma unroll
            for (int q = 0; q < 16; ++q) v[16 + q] = -INFINITY;
          }
        }
        // column lane: the largest logit over the warp's ids and its first id
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          mm[q] = v[q];
          aa[q] = valid_id ? id : 0x7fffffff;
        }
        vu_tr_argmax(mm, aa, lane);
        const float col_m = mm[0];
        const int col_a = aa[0];
        // sum of exp(l - column max) over the warp's ids
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const float cm = __shfl_sync(0xffffffffu, col_m, q);
          e[q] = (v[q] == -INFINITY) ? 0.0f : __expf(v[q] - cm);
        }
        vu_tr_sum(e, lane);
        // the candidate: the argmax, or where the excluded id is one of this warp's, the
        // argmax over the others
        float cand_m = col_m;
        int cand_a = col_a;
        if (excl_here) {
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            mm[q] = (id == p.excl) ? -INFINITY : v[q];
            aa[q] = (id == p.excl || !valid_id) ? 0x7fffffff : id;
          }
          vu_tr_argmax(mm, aa, lane);
          cand_m = mm[0];
          cand_a = aa[0];
        }
        red[lg][lane] = UpdPart{col_m, e[0], cand_a, cand_m};
        asm volatile("bar.sync 1, 128;" ::: "memory");  // the four epilogue warps
        if (lg == 0 && c0 + lane < rows &&
            DG_GUARD(row0 + c0 + lane < p.n_tokens && m < p.m_tiles && c0 + lane < n_pad, p.err)) {
          UpdPart o = red[0][lane];
#pragma unroll
          for (int w2 = 1; w2 < 4; ++w2) {  // warps in id order
            const UpdPart x = red[w2][lane];
            vu_ms_merge(o.m, o.s, x.m, x.s);
            vu_cand_merge(o.m2, o.a, x.m2, x.a);
          }
          p.part[(size_t)(row0 + c0 + lane) * p.m_tiles + m] = o;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");  // red is rewritten by the next group
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }

  __syncthreads();
  if (abort_s && tid == 0) {
    const int first = n_issued_s > stages ? n_issued_s - stages : 0;
    for (int i = first; i < n_issued_s; ++i) mbar_wait_drain(&full_bar[i % stages], (uint32_t)(i / stages) & 1u);
  }
  if (tid == 32) mbar_wait_drain(&drain_bar, 0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, tmem_cols);
}

// One CTA of UM_THREADS threads per token: thread t merges the token's tile records t,
// t + UM_THREADS, ... in id order (UM_BATCH loads in flight before the merges), each
// warp combines its lanes in a fixed butterfly, and thread 0 merges the warps' records
// in warp order: one record out.  (One warp per token, one load in flight per lane, left
// each lane 64 dependent loads at the large vocabulary.)
constexpr int UM_THREADS = 128;
constexpr int UM_BATCH = 8;
__global__ void __launch_bounds__(UM_THREADS) upd_merge_rows_kernel(const UpdPart* __restrict__ part, int C,
                                                                    int tiles, UpdPart* __restrict__ out) {
  griddep_sync();
  __shared__ UpdPart wrec[UM_THREADS / 32];
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (row >= C) return;
  const UpdPart* pr = part + (size_t)row * tiles;
  float m = -INFINITY, s = 0.0f, m2 = -INFINITY;
  int a = 0x7fffffff;
  for (int t0 = tid; t0 < tiles; t0 += UM_THREADS * UM_BATCH) {
    UpdPart x[UM_BATCH];
#pragma unroll
    for (int i = 0; i < UM_BATCH; ++i) {
      const int t = t0 + i * UM_THREADS;
      if (t < tiles) x[i] = pr[t];
    }
#pragma unroll
    for (int i = 0; i < UM_BATCH; ++i) {
      if (t0 + i * UM_THREADS < tiles) {
        vu_ms_merge(m, s, x[i].m, x[i].s);
        vu_cand_merge(m2, a, x[i].m2, x[i].a);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, m, o);
    const float os = __shfl_xor_sync(0xffffffffu, s, o);
    const float om2 = __shfl_xor_sync(0xffffffffu, m2, o);
    const int oa = __shfl_xor_sync(0xffffffffu, a, o);
    vu_ms_merge(m, s, om, os);
    vu_cand_merge(m2, a, om2, oa);
  }
  if (lane == 0) {
    UpdPart r;
    r.m = m;
    r.s = s;
    r.a = a;
    r.m2 = m2;
    wrec[warp] = r;
  }
  __syncthreads();
  if (tid == 0) {
    UpdPart r = wrec[0];
    for (int w = 1; w < UM_THREADS / 32; ++w) {
      vu_ms_merge(r.m, r.s, wrec[w].m, wrec[w].s);
      vu_cand_merge(r.m2, r.a, wrec[w].m2, wrec[w].a);
    }
    out[row] = r;
  }
}

cudaError_t launch_vocab_update(const CUtensorMap& A, const CUtensorMap& B, const CUtensorMap& Bb, const VuParams& p,
                                cudaStream_t st) {
  if (p.n_tokens <= 0) return cudaSuccess;
  if (p.K % VU_BK != 0 || p.K <= 0 || p.n_max < 16 || p.n_max > 256 || p.n_max % 16 != 0 || p.m_tiles < 1 ||
      p.smem_budget < VU_BM * VU_BK * 2 + p.n_max * 128)
    return cudaErrorInvalidValue;
  const int smem = p.smem_budget + 1024;
  const int tiles = ((p.n_tokens + p.n_max - 1) / p.n_max) * p.m_tiles;
  const int grid = tiles < num_sms() ? tiles : num_sms();
  cudaError_t e = cudaFuncSetAttribute(tc_vocab_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_k(tc_vocab_update_kernel, dim3(grid), dim3(VU_THREADS), smem, st, A, B, Bb, p);
}

cudaError_t launch_upd_merge_rows(const UpdPart* part, int C, int tiles, UpdPart* out, cudaStream_t st) {
  if (C <= 0) return cudaSuccess;
  return launch_k(upd_merge_rows_kernel, dim3(C), dim3(UM_THREADS), 0, st, part, C, tiles, out);
}

cudaError_t set_wait_limit_vocab_update(uint64_t ns) { return set_wait_limit_this_file(ns); }

}  // namespace dg
