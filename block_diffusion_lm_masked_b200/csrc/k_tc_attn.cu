// tcgen05 flash attention over the KV cache, both attention modes of the pass:
//   denoising mode: every canvas query sees all cached prefix keys and all canvas
//                   keys (bidirectional block rows of the prefix/block mask);
//   prefill mode:   new tokens see keys up to their own position (causal rows).
// One CTA = one query head x 128 query rows x a contiguous range of 128-key chunks
// (split-KV; partial results merged by attn_merge_kernel).  V is kept transposed in the
// cache ([d][position]) so the B operands of both MMAs are K-major in shared memory.
//
// Precision.  Cached keys/values are bf16 (the cache's storage format).  The query and
// the keys/values of the tokens the call itself processes are in flight at fp32
// precision, carried as bf16 hi + lo terms: S = Q_hi K^T + Q_lo K^T (+ Q_hi K_lo^T on
// the chunks holding current tokens), O += P_hi V + P_lo V (+ P_hi V_lo on those
// chunks).  The low parts of the current K/V live in a workspace window whose row 0 is
// the 128-aligned chunk start `base` at or below the first current position; rows
// before the first current position are zero there.
//
// Pipeline.  Warps 0-3 run the softmax (one query row per thread); warp 4 issues the
// TMA loads and the MMAs.  S (fp32) sits in TMEM columns 0..127; the softmax (max raised
// lazily by more than 2^8 so O is rescaled rarely) writes P as packed bf16 pairs, hi and
// lo, into one of two TMEM buffers (128..255 for even chunks, 384..511 for odd ones), and
// the PV MMAs read P from TMEM into O (256..383).  As soon as the softmax has read S of
// chunk j, the S MMA of chunk j + 1 runs, and the PV of chunk j runs beside the softmax of
// chunk j + 1.  Chunks of cached keys alternate between two 64 KB smem slots (the next one
// loads while this one is used); a chunk of current tokens takes both slots (hi K/V in
// one, lo in the other).  Hand-offs are mbarriers: S full, S read, and per P buffer P
// written and PV done.
#include <math.h>

#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

constexpr int AT_BQ = 128;
constexpr int AT_BKEYS = 128;
constexpr int AT_D = 128;
constexpr uint32_t AT_HALF = 128 * 128;                   // one [128 rows][64 bf16] swizzled block
constexpr uint32_t AT_SLOT = 4 * AT_HALF;                 // K (2 blocks) + V^T (2 blocks)
constexpr int AT_SMEM = 1024 + 4 * AT_HALF + 2 * AT_SLOT;  // Q hi, Q lo, two slots
// TMEM columns: S 0..127; P of even chunks 128..255, of odd chunks 384..511 (hi then lo,
// 64 packed columns each); O 256..383
constexpr uint32_t TM_S = 0, TM_O = 256;
__device__ __forceinline__ uint32_t tm_phi(int j) { return (j & 1) ? 384u : 128u; }
__device__ __forceinline__ uint32_t tm_plo(int j) { return tm_phi(j) + 64u; }
// warps 0-7: softmax, warp w takes query rows 32 (w % 4) .. + 31 (its TMEM lanes) and keys
// 64 (w / 4) .. + 63 of every chunk; warp 8: loads and MMAs
constexpr int AT_SM_WARPS = 8;
constexpr int AT_CTRL_WARP = AT_SM_WARPS;
constexpr int AT_THREADS = 32 * (AT_CTRL_WARP + 1);

// A operand from TMEM (P), B from shared memory (V^T), fp32 accumulate in TMEM
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__global__ void __launch_bounds__(AT_THREADS, 1)
    tc_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQl,
                   const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmVt,
                   const __grid_constant__ CUtensorMap tmKl, const __grid_constant__ CUtensorMap tmVtl,
                   const TcAttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_bar;
  __shared__ __align__(8) uint64_t kv_bar[2];  // K and V^T of the chunk in smem slot s have landed
  __shared__ __align__(8) uint64_t s_full;      // S of the chunk is in TMEM
  __shared__ __align__(8) uint64_t s_free;      // the softmax warps have read S
  __shared__ __align__(8) uint64_t p_ready[2];  // P of a chunk (buffer chunk & 1) is in TMEM
  __shared__ __align__(8) uint64_t pv_done[2];  // PV of a chunk (buffer chunk & 1) is complete
  __shared__ __align__(8) uint64_t x_bar[2];    // both halves of every row posted their chunk max
  __shared__ __align__(8) uint64_t l_bar;       // both halves posted their row sums
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ float x_max[2][2][AT_BQ];          // [chunk & 1][key half][row]
  __shared__ float x_sum[2][AT_BQ];             // [key half][row]
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int abort_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = blockIdx.x, h = blockIdx.y, sp = blockIdx.z;
  const int kvh = h / p.group;
  const int q_row0 = qt * AT_BQ;
  const int rows_here = min(AT_BQ, p.n_q - q_row0);
  int kv_end = p.n_keys;
  if (p.causal) kv_end = min(p.n_keys, p.q_pos0 + q_row0 + rows_here);
  const int nch_total = (kv_end + AT_BKEYS - 1) / AT_BKEYS;
  const int c_begin = sp * p.chunks_per_split;
  const int nck = min(nch_total, c_begin + p.chunks_per_split) - c_begin;
  const int qrow = q_row0 + tid;  // the empty-split path below: one query row per thread < 128

  if (nck <= 0) {
    // this split sees no key of the tile: an empty partial (weight 0 in the merge)
    griddep_sync();
    if (tid < AT_BQ && qrow < p.n_q) {
      float* po = p.part_o + (((size_t)sp * p.nq + h) * p.n_q + qrow) * AT_D;
      for (int i = 0; i < AT_D; ++i) po[i] = 0.0f;
      p.part_lse[((size_t)sp * p.nq + h) * p.n_q + qrow] = -INFINITY;
    }
    return;
  }

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                   // 2 blocks: d 0..63, 64..127
  uint8_t* sQl = smem + 2 * AT_HALF;    // low terms
  uint8_t* sSlot = smem + 4 * AT_HALF;  // [2 slots][K blk0, K blk1, Vt blk0, Vt blk1]

  if (warp == AT_CTRL_WARP) tmem_alloc(&tmem_base_s, 512);
  if (tid == AT_CTRL_WARP * 32) {
    mbar_init(&q_bar, 1);
    mbar_init(&kv_bar[0], 1);
    mbar_init(&kv_bar[1], 1);
    mbar_init(&s_full, 1);
    mbar_init(&s_free, AT_SM_WARPS);
    mbar_init(&p_ready[0], AT_SM_WARPS);
    mbar_init(&p_ready[1], AT_SM_WARPS);
    mbar_init(&x_bar[0], AT_SM_WARPS);
    mbar_init(&x_bar[1], AT_SM_WARPS);
    mbar_init(&l_bar, AT_SM_WARPS);
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(&drain_bar, 1);
    abort_s = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_sync();  // the previous kernel wrote q and this layer's current K/V
  const uint32_t tmem = tmem_base_s;

  // chunk j (0-based within this CTA) holds keys [key0, key0 + 128); "current" chunks
  // (key0 >= base) also carry low parts and take both slots; cached-key chunks
  // alternate slots j & 1
  auto is_cur = [&](int j) { return p.has_lo && (c_begin + j) * AT_BKEYS >= p.base; };
  const uint32_t idesc = idesc_bf16_f32(AT_BQ, AT_BKEYS);

  // ---- TMA / MMA issue bookkeeping (control thread only)
  int slot_loads[2] = {0, 0};             // loads issued into each slot so far
  int par_ring[2][2] = {{0, 0}, {0, 0}};  // [j & 1][slot]: parity of chunk j's load in that slot

  if (warp == AT_CTRL_WARP) {
    if (lane == 0) {
      // ================= control: TMA loads, S and PV MMAs
      int issued = 0;  // chunks whose loads were issued (in order)
      auto load_slot = [&](int slot, const CUtensorMap* mk, const CUtensorMap* mv, int krow, int vx) {
        uint8_t* k = sSlot + slot * AT_SLOT;
        uint8_t* v = k + 2 * AT_HALF;
        mbar_arrive_expect_tx(&kv_bar[slot], AT_SLOT);
        tma_load_3d(k, mk, 0, krow, kvh, &kv_bar[slot]);
        tma_load_3d(k + AT_HALF, mk, 64, krow, kvh, &kv_bar[slot]);
        tma_load_3d(v, mv, vx, 0, kvh, &kv_bar[slot]);
        tma_load_3d(v + AT_HALF, mv, vx + 64, 0, kvh, &kv_bar[slot]);
      };
      auto issue = [&](int j) {
        const int key0 = (c_begin + j) * AT_BKEYS;
        if (is_cur(j)) {
          par_ring[j & 1][0] = slot_loads[0]++ & 1;
          par_ring[j & 1][1] = slot_loads[1]++ & 1;
          load_slot(0, &tmK, &tmVt, key0, key0);
          load_slot(1, &tmKl, &tmVtl, key0 - p.base, key0 - p.base);
        } else {
          const int s = j & 1;
          par_ring[j & 1][s] = slot_loads[s]++ & 1;
          load_slot(s, &tmK, &tmVt, key0, key0);
        }
        issued = j + 1;
      };
      auto issue_pv = [&](int j) {
        const bool cur = is_cur(j);
        const int s_hi = cur ? 0 : (j & 1);
        const uint32_t v = smem_u32(sSlot + s_hi * AT_SLOT + 2 * AT_HALF);
        const uint32_t vl = smem_u32(sSlot + AT_SLOT + 2 * AT_HALF);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t pcol = kb * 32 + kk * 8;  // 16 keys = 8 packed columns
            const uint64_t vd = sw128_kmajor_desc(v + kb * AT_HALF + kk * 32);
            tc_mma_ts(tmem + TM_O, tmem + tm_phi(j) + pcol, vd, idesc, (j > 0 || (kb | kk) != 0) ? 1u : 0u);
            tc_mma_ts(tmem + TM_O, tmem + tm_plo(j) + pcol, vd, idesc, 1u);
            if (cur)
              tc_mma_ts(tmem + TM_O, tmem + tm_phi(j) + pcol, sw128_kmajor_desc(vl + kb * AT_HALF + kk * 32), idesc,
                        1u);
          }
        tc_commit(&pv_done[j & 1]);
      };

      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmQl);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmVt);
      if (p.has_lo) {
        prefetch_tmap(&tmKl);
        prefetch_tmap(&tmVtl);
      }
      mbar_arrive_expect_tx(&q_bar, 4 * AT_HALF);
      tma_load_3d(sQ, &tmQ, 0, q_row0, h, &q_bar);
      tma_load_3d(sQ + AT_HALF, &tmQ, 64, q_row0, h, &q_bar);
      tma_load_3d(sQl, &tmQl, 0, q_row0, h, &q_bar);
      tma_load_3d(sQl + AT_HALF, &tmQl, 64, q_row0, h, &q_bar);
      issue(0);
      if (nck > 1 && !is_cur(0) && !is_cur(1)) issue(1);

      bool ok = true;
      int pv_next = 0;  // the next chunk whose PV is to be issued
      // PV of chunk k once its P is in TMEM, then wait for it: the slot it read is free
      // afterwards.  (Barriers per P buffer: no waiter can fall two phases behind.)
      auto do_pv = [&](int k) {
        if (!mbar_wait(&p_ready[k & 1], (uint32_t)(k >> 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN))
          return false;
        tc_fence_after();
        issue_pv(k);
        pv_next = k + 1;
        return mbar_wait(&pv_done[k & 1], (uint32_t)(k >> 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
      };
      for (int j = 0; j < nck && ok; ++j) {
        const bool cur = is_cur(j);
        const int s_hi = cur ? 0 : (j & 1);
        if (issued <= j) {
          // chunk j was not prefetched: it needs a slot the previous chunk may still hold
          if (j >= 1 && pv_next == j - 1 && !(ok = do_pv(j - 1))) break;
          issue(j);
        }
        if (j == 0) ok = mbar_wait(&q_bar, 0, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
        if (ok) ok = mbar_wait(&kv_bar[s_hi], (uint32_t)par_ring[j & 1][s_hi], &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
        if (ok && cur) ok = mbar_wait(&kv_bar[1], (uint32_t)par_ring[j & 1][1], &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
        // S in TMEM was last read by the softmax of chunk j - 1
        if (ok && j >= 1) ok = mbar_wait(&s_free, (uint32_t)(j - 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
        if (!ok) break;
        tc_fence_after();
        {
          const uint32_t q = smem_u32(sQ), ql = smem_u32(sQl);
          const uint32_t k = smem_u32(sSlot + s_hi * AT_SLOT), kl = smem_u32(sSlot + AT_SLOT);
          const uint32_t d_s = tmem + TM_S;
#pragma unroll
          for (int kb = 0; kb < 2; ++kb)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t off = kb * AT_HALF + kk * 32;
              const uint64_t kd = sw128_kmajor_desc(k + off);
              tc_mma(d_s, sw128_kmajor_desc(q + off), kd, idesc, (kb | kk) != 0 ? 1u : 0u);
              tc_mma(d_s, sw128_kmajor_desc(ql + off), kd, idesc, 1u);
              if (cur) tc_mma(d_s, sw128_kmajor_desc(q + off), sw128_kmajor_desc(kl + off), idesc, 1u);
            }
          tc_commit(&s_full);
        }
        // the previous chunk's PV runs behind this S (and beside this chunk's softmax); then
        // the slot it held takes chunk j + 1
        if (j >= 1 && pv_next == j - 1 && !(ok = do_pv(j - 1))) break;
        if (issued == j + 1 && j + 1 < nck && !cur && !is_cur(j + 1)) issue(j + 1);
      }
      if (ok && pv_next == nck - 1) {
        ok = mbar_wait(&p_ready[(nck - 1) & 1], (uint32_t)((nck - 1) >> 1) & 1u, &abort_s, p.err,
                       DG_DEVERR_TIMEOUT_ATTN);
        if (ok) {
          tc_fence_after();
          issue_pv(nck - 1);
        }
      }
    }
    __syncwarp();
  } else {
    // ================= softmax warps: query row `row` (TMEM lane), keys 64 hf .. + 63 of each chunk.
    // Every bounded wait is voted on by the whole warp (__all_sync): the TMEM loads and
    // stores that follow are warp-collective, so no lane may go on alone after another
    // lane's wait gave up.
    const int row = (warp & 3) * 32 + lane, hf = warp >> 2;
    const int my_row = q_row0 + row;
    const int my_pos = p.q_pos0 + my_row;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    float m_used = -INFINITY, l = 0.0f;
    const int key_lim = p.causal ? min(p.n_keys, my_pos + 1) : p.n_keys;
    bool ok = true;
    for (int j = 0; j < nck && ok; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full, (uint32_t)j & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN));
      if (!ok) break;
      tc_fence_after();
      float s[AT_BKEYS / 2];
#pragma unroll
      for (int c = 0; c < AT_BKEYS / 32; ++c) {
        uint32_t r[16];
        tmem_ld16(tmem + TM_S + lane_off + hf * 64 + c * 16, r);
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) s[c * 16 + i] = __uint_as_float(r[i]) * p.scale_log2;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free);  // the control warp may write the next S
      const int key0 = (c_begin + j) * AT_BKEYS + hf * 64;
      float hmax = -INFINITY;
#pragma unroll
      for (int i = 0; i < AT_BKEYS / 2; ++i) {
        if (key0 + i >= key_lim) s[i] = -INFINITY;
        hmax = fmaxf(hmax, s[i]);
      }
      // the row max over both key halves
      x_max[j & 1][hf][row] = hmax;
      __syncwarp();
      if (lane == 0) mbar_arrive(&x_bar[j & 1]);
      ok = __all_sync(0xffffffffu, mbar_wait(&x_bar[j & 1], (uint32_t)(j >> 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN));
      if (!ok) break;
      const float rmax = fmaxf(hmax, x_max[j & 1][hf ^ 1][row]);
      const bool upd = rmax > m_used + 8.0f;
      const float alpha = upd ? exp2f(m_used - rmax) : 1.0f;  // 0 while nothing was visible yet
      // tcgen05.ld/st are warp-collective: the whole warp rescales its half of O if any of
      // its rows must, once the previous chunk's PV is complete (O stable)
      if (__any_sync(0xffffffffu, upd && j > 0)) {
        ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < AT_D / 32; ++c) {
          uint32_t r[16];
          tmem_ld16(tmem + TM_O + lane_off + hf * 64 + c * 16, r);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st16(tmem + TM_O + lane_off + hf * 64 + c * 16, r);
        }
      }
      if (upd) {
        l *= alpha;
        m_used = rmax;
      }
      // P buffer j & 1 was last read by the PV of chunk j - 2
      if (j >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[j & 1], (uint32_t)((j >> 1) - 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN));
        if (!ok) break;
        tc_fence_after();
      }
      // P = exp2(s - m_used) as packed bf16 pairs, hi and lo, into TMEM (this half's 32
      // packed columns)
#pragma unroll
      for (int c = 0; c < 2; ++c) {  // 32 keys -> 16 packed columns per store
        uint32_t wh[16], wl[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int i0 = c * 32 + 2 * e;
          const float p0 = (s[i0] == -INFINITY) ? 0.0f : exp2f(s[i0] - m_used);
          const float p1 = (s[i0 + 1] == -INFINITY) ? 0.0f : exp2f(s[i0 + 1] - m_used);
          l += p0 + p1;
          const __nv_bfloat162 hi = __floats2bfloat162_rn(p0, p1);
          const __nv_bfloat162 lo = __floats2bfloat162_rn(p0 - __low2float(hi), p1 - __high2float(hi));
          wh[e] = *reinterpret_cast<const uint32_t*>(&hi);
          wl[e] = *reinterpret_cast<const uint32_t*>(&lo);
        }
        tmem_st16(tmem + tm_phi(j) + lane_off + hf * 32 + c * 16, wh);
        tmem_st16(tmem + tm_plo(j) + lane_off + hf * 32 + c * 16, wl);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready[j & 1]);
    }
    if (ok)
      ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(nck - 1) & 1], (uint32_t)((nck - 1) >> 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN));
    if (ok) {
      // the row sum over both key halves
      x_sum[hf][row] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&l_bar);
      ok = __all_sync(0xffffffffu, mbar_wait(&l_bar, 0, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN));
    }
    if (ok) {
      l += x_sum[hf ^ 1][row];
      tc_fence_after();
      const bool valid = my_row < p.n_q;
      const float inv_l = (l > 0.0f) ? 1.0f / l : 0.0f;
      if (p.n_splits == 1) {
        const size_t base = (size_t)my_row * p.nq * AT_D + (size_t)h * AT_D + hf * 64;
#pragma unroll
        for (int c = 0; c < AT_D / 32; ++c) {
          uint32_t r[16];
          tmem_ld16(tmem + TM_O + lane_off + hf * 64 + c * 16, r);
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
        float* po = p.part_o + (((size_t)sp * p.nq + h) * p.n_q + my_row) * AT_D + hf * 64;
#pragma unroll
        for (int c = 0; c < AT_D / 32; ++c) {
          uint32_t r[16];
          tmem_ld16(tmem + TM_O + lane_off + hf * 64 + c * 16, r);
          tc_wait_ld();
          if (valid) {
            float4* dst = reinterpret_cast<float4*>(po + c * 16);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_float4(__uint_as_float(r[4 * e]) * inv_l, __uint_as_float(r[4 * e + 1]) * inv_l,
                                   __uint_as_float(r[4 * e + 2]) * inv_l, __uint_as_float(r[4 * e + 3]) * inv_l);
          }
        }
        if (valid && hf == 0)
          p.part_lse[((size_t)sp * p.nq + h) * p.n_q + my_row] = (l > 0.0f) ? m_used + log2f(l) : -INFINITY;
      }
    }
  }
  __syncthreads();
  if (abort_s && tid == AT_CTRL_WARP * 32) {
    // wind down: let issued loads and MMAs land before the smem / TMEM go away
    mbar_wait_drain(&q_bar, 0);
    for (int s2 = 0; s2 < 2; ++s2)
      if (slot_loads[s2] > 0) mbar_wait_drain(&kv_bar[s2], (uint32_t)(slot_loads[s2] - 1) & 1u);
    tc_commit(&drain_bar);
    mbar_wait_drain(&drain_bar, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == AT_CTRL_WARP) tmem_dealloc(tmem, 512);
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

cudaError_t launch_tc_attention(const CUtensorMap& Q, const CUtensorMap& Ql, const CUtensorMap& K,
                                const CUtensorMap& Vt, const CUtensorMap& Kl, const CUtensorMap& Vtl,
                                const TcAttnParams& p, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(tc_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((p.n_q + AT_BQ - 1) / AT_BQ, p.nq, p.n_splits);
  return launch_k(tc_attn_kernel, grid, dim3(AT_THREADS), AT_SMEM, st, Q, Ql, K, Vt, Kl, Vtl, p);
}

cudaError_t launch_attn_merge(const float* part_o, const float* part_lse, int n_splits, int nq, int n_q, int d,
                              __nv_bfloat16* out, __nv_bfloat16* out_lo, cudaStream_t st) {
  return launch_k(attn_merge_kernel, dim3(n_q, nq), dim3(128), 0, st, part_o, part_lse, n_splits, nq, n_q, d, out,
                  out_lo);
}

cudaError_t set_wait_limit_attn(uint64_t ns) { return set_wait_limit_this_file(ns); }

}  // namespace dg
