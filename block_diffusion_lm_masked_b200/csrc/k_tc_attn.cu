// tcgen05 flash attention over the KV cache, both attention modes of the pass:
//   denoising mode: every canvas query sees all cached prefix keys and all canvas
//                   keys (bidirectional block rows of the prefix/block mask);
//   prefill mode:   new tokens see keys up to their own position (causal rows).
// One CTA = one query head x 128 query rows x a contiguous range of 128-key chunks
// (split-KV; the last split of a tile and head to finish merges the partial results).
// V is kept transposed in the cache ([d][position]) so the B operands of both MMAs are
// K-major in shared memory.
//
// Precision.  Cached keys/values are bf16 (the cache's storage format).  The query and
// the keys/values of the tokens the call itself processes are in flight at fp32
// precision, carried as bf16 hi + lo terms: S = Q_hi K^T + Q_lo K^T (+ Q_hi K_lo^T on
// the chunks holding current tokens), O += P_hi V + P_lo V (+ P_hi V_lo on those
// chunks).  The low parts of the current K/V live in a workspace window whose row 0 is
// the 128-aligned chunk start `base` at or below the first current position; rows
// before the first current position are zero there.
//
// Layout.  The query tile lives in tensor memory for the whole CTA (the softmax warps
// load their rows from global memory and store them as packed bf16 pairs along d), so
// all of shared memory holds a ring of three 64 KB K/V slots (K [128 keys][128 d] and
// V^T [128 d][128 keys], 128-byte swizzled).  A chunk of cached keys takes one slot; a
// chunk of the call's own keys takes two (hi K/V in the first, lo in the second).
// TMEM (512 columns): Q hi 0..63 and lo 64..127, S 128..255 (fp32), O 256..383 (fp32),
// P hi 384..447 and lo 448..511 (packed bf16 pairs along the keys).
//
// Roles.  Warps 0-7 run the softmax (warp w: query rows 32 (w % 4) .. + 31, its TMEM
// lanes, and keys 64 (w / 4) .. + 63 of each chunk; the two warps of a row exchange their
// half-row maxima through shared memory); warp 8 issues the MMAs; warp 9 the TMA loads,
// running ahead as far as the ring's free slots allow.  The MMA warp issues S(j), then
// PV(j - 1) and a commit per slot of chunk j - 1 that frees it for the loads (where two
// chunks of own keys follow each other, chunk j cannot load until chunk j - 1's slots are
// free, so PV(j - 1) goes first there).  The softmax of chunk j reads S, lets S(j + 1)
// in, and writes P once PV(j - 1) has read the previous P.  Hand-offs are mbarriers.
#include <math.h>

#include "attn_merge.cuh"
#include "attn_softmax.cuh"
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

constexpr int AT_BQ = 128;
constexpr int AT_BKEYS = 128;
constexpr int AT_D = 128;
constexpr int AT_SLOTS = 3;
constexpr uint32_t AT_HALF = 128 * 128;                   // one [128 rows][64 bf16] swizzled block
constexpr uint32_t AT_SLOT = 4 * AT_HALF;                 // K (2 blocks) + V^T (2 blocks)
constexpr int AT_SMEM = 1024 + AT_SLOTS * AT_SLOT;
static_assert(AT_SMEM <= 227 * 1024 - 1024, "shared memory budget");
constexpr uint32_t TM_QHI = 0, TM_QLO = 64, TM_S = 128, TM_O = 256, TM_PHI = 384, TM_PLO = 448;
constexpr int AT_SM_WARPS = 8;
constexpr int AT_MMA_WARP = AT_SM_WARPS;
constexpr int AT_LOAD_WARP = AT_SM_WARPS + 1;
constexpr int AT_THREADS = 32 * (AT_LOAD_WARP + 1);

// A operand from TMEM (Q or P), B from shared memory (K or V^T), fp32 accumulate in TMEM
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The slot plan the load and the MMA warp both follow: chunk j takes the next one slot
// (cached keys) or two (own keys) of the ring, in order.
struct AtSlotPlan {
  int nxt = 0;
  int uses[AT_SLOTS] = {0, 0, 0};
  int slot[2][2], use[2][2], n[2];  // [j & 1][part]: slot, its use index; parts of chunk j
  __device__ void take(int j, bool cur) {
    const int b = j & 1;
    n[b] = cur ? 2 : 1;
    for (int i = 0; i < n[b]; ++i) {
      slot[b][i] = nxt;
      use[b][i] = uses[nxt]++;
      nxt = nxt + 1 == AT_SLOTS ? 0 : nxt + 1;
    }
  }
};

__global__ void __launch_bounds__(AT_THREADS, 1)
    tc_attn_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmVt,
                   const __grid_constant__ CUtensorMap tmKl, const __grid_constant__ CUtensorMap tmVtl,
                   const TcAttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_ready;           // the softmax warps stored the query tile in TMEM
  __shared__ __align__(8) uint64_t kv_full[AT_SLOTS];  // the slot's TMA loads have landed
  __shared__ __align__(8) uint64_t kv_free[AT_SLOTS];  // the MMAs reading the slot are complete
  __shared__ __align__(8) uint64_t s_full;             // S of the chunk is in TMEM
  __shared__ __align__(8) uint64_t s_free;             // the softmax warps have read S
  __shared__ __align__(8) uint64_t p_ready;            // P of the chunk is in TMEM
  __shared__ __align__(8) uint64_t pv_done;            // the PV of the chunk is complete
  __shared__ __align__(8) uint64_t x_bar[2];           // both halves of every row posted their chunk max
  __shared__ __align__(8) uint64_t l_bar;              // both halves posted their row sums
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ float x_max[2][2][AT_BQ];                 // [chunk & 1][key half][row]
  __shared__ float x_sum[2][AT_BQ];                    // [key half][row]
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

  if (nck <= 0) {
    // this split sees no key of the tile: an empty partial (weight 0 in the merge)
    griddep_sync();
    const int qrow = q_row0 + tid;
    if (tid < AT_BQ && qrow < p.n_q) {
      float* po = p.part_o + (((size_t)sp * p.nq + h) * p.n_q + qrow) * AT_D;
      for (int i = 0; i < AT_D; ++i) po[i] = 0.0f;
      p.part_lse[((size_t)sp * p.nq + h) * p.n_q + qrow] = -INFINITY;
    }
    if (p.n_splits > 1 && p.merge_cnt) merge_splits_if_last(p, qt, h, 1);
    return;
  }

  uint8_t* sSlot = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  if (warp == AT_MMA_WARP) tmem_alloc(&tmem_base_s, 512);
  if (tid == AT_LOAD_WARP * 32) {
    mbar_init(&q_ready, AT_SM_WARPS);
    for (int s = 0; s < AT_SLOTS; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_free[s], 1);
    }
    mbar_init(&s_full, 1);
    mbar_init(&s_free, AT_SM_WARPS);
    mbar_init(&p_ready, AT_SM_WARPS);
    mbar_init(&pv_done, 1);
    mbar_init(&x_bar[0], AT_SM_WARPS);
    mbar_init(&x_bar[1], AT_SM_WARPS);
    mbar_init(&l_bar, AT_SM_WARPS);
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
  // (key0 >= base) also carry low parts and take two slots
  auto is_cur = [&](int j) { return p.has_lo && (c_begin + j) * AT_BKEYS >= p.base; };
  const uint32_t idesc = idesc_bf16_f32(AT_BQ, AT_BKEYS);
  int loaded[AT_SLOTS] = {0, 0, 0};  // loads issued into each slot (for the wind-down)

  if (warp == AT_LOAD_WARP) {
    if (lane == 0) {
      // ================= loads: each chunk's slots in plan order, as slots free up
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmVt);
      if (p.has_lo) {
        prefetch_tmap(&tmKl);
        prefetch_tmap(&tmVtl);
      }
      AtSlotPlan lp;
      bool ok = true;
      for (int j = 0; j < nck && ok; ++j) {
        const int key0 = (c_begin + j) * AT_BKEYS;
        lp.take(j, is_cur(j));
        for (int i = 0; i < lp.n[j & 1] && ok; ++i) {
          const int s = lp.slot[j & 1][i], u = lp.use[j & 1][i];
          // the slot's previous chunk was freed by the MMAs that read it
          if (u >= 1 &&
              !(ok = mbar_wait(&kv_free[s], (uint32_t)(u - 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN)))
            break;
          const CUtensorMap* mk = (i == 0) ? &tmK : &tmKl;
          const CUtensorMap* mv = (i == 0) ? &tmVt : &tmVtl;
          const int krow = (i == 0) ? key0 : key0 - p.base;  // the low-term window starts at `base`
          if (!DG_GUARD(krow >= 0 && krow % AT_BKEYS == 0, p.err)) {
            ok = false;
            abort_s = 1;
            break;
          }
          uint8_t* k = sSlot + s * AT_SLOT;
          uint8_t* v = k + 2 * AT_HALF;
          loaded[s] += 1;
          mbar_arrive_expect_tx(&kv_full[s], AT_SLOT);
          tma_load_3d(k, mk, 0, krow, kvh, &kv_full[s]);
          tma_load_3d(k + AT_HALF, mk, 64, krow, kvh, &kv_full[s]);
          tma_load_3d(v, mv, krow, 0, kvh, &kv_full[s]);
          tma_load_3d(v + AT_HALF, mv, krow + 64, 0, kvh, &kv_full[s]);
        }
      }
    }
    __syncwarp();
  } else if (warp == AT_MMA_WARP) {
    if (lane == 0) {
      // ================= MMAs
      AtSlotPlan mp;
      auto slot_addr = [&](int s) { return smem_u32(sSlot + s * AT_SLOT); };
      auto issue_s = [&](int j) {
        const int b = j & 1;
        const bool cur = mp.n[b] == 2;
        const uint32_t k = slot_addr(mp.slot[b][0]);
        const uint32_t kl = cur ? slot_addr(mp.slot[b][1]) : 0u;
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t qc = kb * 32 + kk * 8;  // 16 d values = 8 packed Q columns
            const uint32_t off = kb * AT_HALF + kk * 32;
            const uint64_t kd = sw128_kmajor_desc(k + off);
            tc_mma_ts(tmem + TM_S, tmem + TM_QHI + qc, kd, idesc, (kb | kk) != 0 ? 1u : 0u);
            tc_mma_ts(tmem + TM_S, tmem + TM_QLO + qc, kd, idesc, 1u);
            if (cur) tc_mma_ts(tmem + TM_S, tmem + TM_QHI + qc, sw128_kmajor_desc(kl + off), idesc, 1u);
          }
        tc_commit(&s_full);
      };
      auto issue_pv = [&](int k) {
        const int b = k & 1;
        const bool cur = mp.n[b] == 2;
        const uint32_t v = slot_addr(mp.slot[b][0]) + 2 * AT_HALF;
        const uint32_t vl = cur ? slot_addr(mp.slot[b][1]) + 2 * AT_HALF : 0u;
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t pcol = kb * 32 + kk * 8;  // 16 keys = 8 packed P columns
            const uint64_t vd = sw128_kmajor_desc(v + kb * AT_HALF + kk * 32);
            tc_mma_ts(tmem + TM_O, tmem + TM_PHI + pcol, vd, idesc, (k > 0 || (kb | kk) != 0) ? 1u : 0u);
            tc_mma_ts(tmem + TM_O, tmem + TM_PLO + pcol, vd, idesc, 1u);
            if (cur)
              tc_mma_ts(tmem + TM_O, tmem + TM_PHI + pcol, sw128_kmajor_desc(vl + kb * AT_HALF + kk * 32), idesc,
                        1u);
          }
        tc_commit(&pv_done);
      };
      // PV of chunk k once its P is in TMEM; then chunk k's slots are freed for the loads
      // (the last chunk's slots are not reused: no commit that nobody waits for)
      auto pv_chunk = [&](int k) {
        if (!mbar_wait(&p_ready, (uint32_t)k & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN)) return false;
        tc_fence_after();
        issue_pv(k);
        if (k + 1 < nck)
          for (int i = 0; i < mp.n[k & 1]; ++i) tc_commit(&kv_free[mp.slot[k & 1][i]]);
        return true;
      };

      bool ok = mbar_wait(&q_ready, 0, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
      for (int j = 0; j < nck && ok; ++j) {
        mp.take(j, is_cur(j));
        const bool pv_first = j >= 1 && mp.n[(j - 1) & 1] + mp.n[j & 1] > AT_SLOTS;
        if (pv_first && !(ok = pv_chunk(j - 1))) break;
        for (int i = 0; i < mp.n[j & 1] && ok; ++i)
          ok = mbar_wait(&kv_full[mp.slot[j & 1][i]], (uint32_t)mp.use[j & 1][i] & 1u, &abort_s, p.err,
                         DG_DEVERR_TIMEOUT_ATTN);
        // S in TMEM was last read by the softmax of chunk j - 1
        if (ok && j >= 1) ok = mbar_wait(&s_free, (uint32_t)(j - 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
        if (!ok) break;
        tc_fence_after();
        issue_s(j);
        if (j >= 1 && !pv_first) ok = pv_chunk(j - 1);
      }
      if (ok) pv_chunk(nck - 1);
    }
    __syncwarp();
  } else {
    // ================= softmax warps: query row `row` (TMEM lane), keys 64 hf .. + 63 of each
    // chunk.  Every bounded wait is voted on by the whole warp (__all_sync): the TMEM loads
    // and stores that follow are warp-collective, so no lane may go on alone after another
    // lane's wait gave up.
    const int row = (warp & 3) * 32 + lane, hf = warp >> 2;
    const int my_row = q_row0 + row;
    const int my_pos = p.q_pos0 + my_row;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const bool valid = my_row < p.n_q;
    // the query row into TMEM: this warp's half of d, hi and lo, as packed bf16 pairs (the
    // pairs are the row's consecutive 32-bit words); rows past n_q are zero
    {
      const size_t qoff = ((size_t)h * p.n_q + (valid ? my_row : 0)) * AT_D + hf * 64;
      const uint4* qh = reinterpret_cast<const uint4*>(p.q + qoff);
      const uint4* ql = reinterpret_cast<const uint4*>(p.q_lo + qoff);
#pragma unroll
      for (int c = 0; c < 2; ++c) {  // 32 d values = 16 packed columns per store
        uint32_t wh[16], wl[16];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint4 a = valid ? qh[c * 4 + e] : make_uint4(0, 0, 0, 0);
          const uint4 b = (valid && p.has_lo) ? ql[c * 4 + e] : make_uint4(0, 0, 0, 0);
          wh[4 * e] = a.x, wh[4 * e + 1] = a.y, wh[4 * e + 2] = a.z, wh[4 * e + 3] = a.w;
          wl[4 * e] = b.x, wl[4 * e + 1] = b.y, wl[4 * e + 2] = b.z, wl[4 * e + 3] = b.w;
        }
        tmem_st16(tmem + TM_QHI + lane_off + hf * 32 + c * 16, wh);
        tmem_st16(tmem + TM_QLO + lane_off + hf * 32 + c * 16, wl);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&q_ready);
    }
    float m_used = -INFINITY, l = 0.0f;
    const int key_lim = p.causal ? min(p.n_keys, my_pos + 1) : p.n_keys;
    bool ok = true;
    for (int j = 0; j < nck && ok; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full, (uint32_t)j & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN));
      if (!ok) break;
      tc_fence_after();
      float s[AT_BKEYS / 2];
      {
        uint32_t r[4][16];
#pragma unroll
        for (int c = 0; c < AT_BKEYS / 32; ++c) tmem_ld16(tmem + TM_S + lane_off + hf * 64 + c * 16, r[c]);
        tc_wait_ld();
#pragma unroll
        for (int c = 0; c < AT_BKEYS / 32; ++c)
#pragma unroll
          for (int i = 0; i < 16; ++i) s[c * 16 + i] = __uint_as_float(r[c][i]) * p.scale_log2;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free);  // the MMA warp may write the next S
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
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&x_bar[j & 1], (uint32_t)(j >> 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN));
      if (!ok) break;
      const float rmax = fmaxf(hmax, x_max[j & 1][hf ^ 1][row]);
      const bool upd = rmax > m_used + 8.0f;
      const float alpha = upd ? exp2f(m_used - rmax) : 1.0f;  // 0 while nothing was visible yet
      if (upd) {
        l *= alpha;
        m_used = rmax;
      }
      // P = exp2(s - m_used) as packed bf16 pairs, hi and lo (this half's 32 packed columns:
      // keys 0..31 of the half in wh0 / wl0, 32..63 in wh1 / wl1)
      uint32_t wh0[16], wl0[16], wh1[16], wl1[16];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float p0 = (s[2 * e] == -INFINITY) ? 0.0f : ex2_approx(s[2 * e] - m_used);
        const float p1 = (s[2 * e + 1] == -INFINITY) ? 0.0f : ex2_approx(s[2 * e + 1] - m_used);
        l += p0 + p1;
        const __nv_bfloat162 hi = __floats2bfloat162_rn(p0, p1);
        const __nv_bfloat162 lo = __floats2bfloat162_rn(p0 - __low2float(hi), p1 - __high2float(hi));
        if (e < 16) {
          wh0[e] = *reinterpret_cast<const uint32_t*>(&hi);
          wl0[e] = *reinterpret_cast<const uint32_t*>(&lo);
        } else {
          wh1[e - 16] = *reinterpret_cast<const uint32_t*>(&hi);
          wl1[e - 16] = *reinterpret_cast<const uint32_t*>(&lo);
        }
      }
      // the previous chunk's PV has read P and added into O: P may be overwritten and O
      // rescaled (tcgen05.ld/st are warp-collective: the whole warp rescales its half of O
      // if any of its rows must)
      if (j >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(&pv_done, (uint32_t)(j - 1) & 1u, &abort_s, p.err,
                                               DG_DEVERR_TIMEOUT_ATTN));
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, upd)) {
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
      }
      tmem_st16(tmem + TM_PHI + lane_off + hf * 32, wh0);
      tmem_st16(tmem + TM_PHI + lane_off + hf * 32 + 16, wh1);
      tmem_st16(tmem + TM_PLO + lane_off + hf * 32, wl0);
      tmem_st16(tmem + TM_PLO + lane_off + hf * 32 + 16, wl1);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready);
    }
    if (ok)
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&pv_done, (uint32_t)(nck - 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN));
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
  // wind down: every MMA and commit the MMA thread issued has landed (also on the normal
  // path, so that no mbarrier arrive reaches this CTA's shared memory after it is gone),
  // and after an abort the loads the load thread issued have landed too
  if (tid == AT_MMA_WARP * 32) {
    tc_commit(&drain_bar);
    mbar_wait_drain(&drain_bar, 0);
  }
  if (abort_s && tid == AT_LOAD_WARP * 32)
    for (int s2 = 0; s2 < AT_SLOTS; ++s2)
      if (loaded[s2] > 0) mbar_wait_drain(&kv_full[s2], (uint32_t)(loaded[s2] - 1) & 1u);
  tc_fence_before();
  __syncthreads();
  if (warp == AT_MMA_WARP) tmem_dealloc(tmem, 512);
  if (p.n_splits > 1 && p.merge_cnt) merge_splits_if_last(p, qt, h, 1);
}

cudaError_t launch_tc_attention(const CUtensorMap& K, const CUtensorMap& Vt, const CUtensorMap& Kl,
                                const CUtensorMap& Vtl, const TcAttnParams& p, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(tc_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((p.n_q + AT_BQ - 1) / AT_BQ, p.nq, p.n_splits);
  return launch_k(tc_attn_kernel, grid, dim3(AT_THREADS), AT_SMEM, st, K, Vt, Kl, Vtl, p);
}

cudaError_t set_wait_limit_attn(uint64_t ns) { return set_wait_limit_this_file(ns); }

}  // namespace dg
