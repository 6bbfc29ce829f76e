// tcgen05 flash attention, head-pair kernel: the same attention as tc_attn_kernel (both
// modes, the same hi + lo precision terms, the same lazy rescale and split-KV partials),
// organised so that the tensor cores stay busy while the softmax runs.
//
// One CTA = two query heads of one KV head (one head when the GQA group is odd, or when
// the host asks for single heads because they fill more SMs) x 128 query rows x a
// contiguous range of 128-key chunks.  Each K/V chunk is loaded once for both heads.
// Warps 0-3 run the softmax of the first head and warps 4-7 that of the second, one query
// row per thread over the whole 128-key chunk, so no row statistics are exchanged between
// warps.  Warp 8 issues the TMA loads; warps 9 and 10 issue the MMAs, one per head.
//
// TMEM (512 columns): per head one S/P region of 128 columns and O (128 columns).  The
// softmax reads S (fp32, 128 keys) into registers and writes P over it as packed bf16
// pairs, hi in the first 64 columns and lo in the next 64; the PV MMAs read P from there.
// Shared memory: the query tiles (hi + lo, 64 KB per head) and a ring of three 32 KB
// half-slots, each holding one chunk's K [128 keys][128 d] or V^T [128 d][128 keys] (two
// 16 KB swizzled blocks); a chunk of the call's own keys also takes its K and V low terms.
// Ring order per chunk: K (and K lo), then V (and V lo).
//
// Each head's MMA thread, per chunk j: S(j) once PV(j-1) of its head has completed (which
// also means its softmax has read S(j-1) and written P(j-1)), a commit towards freeing the
// K half-slots, then PV(j) once its softmax has written P(j), and a commit towards freeing
// the V half-slots; a half-slot is free once both heads' commits have arrived.  The two
// threads run side by side: each bounded wait and commit costs a few hundred nanoseconds
// (measured), and with one issuing thread for both heads those costs, twelve per chunk,
// added up to about 2.4 of the chunk's 5.6 us.  While the softmax of one head works on
// S(j), the tensor cores run the other head's MMAs.
#include <math.h>

#include "attn_softmax.cuh"
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

constexpr int A2_BQ = 128;
constexpr int A2_W = 128;                       // keys per chunk
constexpr int A2_D = 128;
constexpr int A2_HSLOTS = 3;                    // half-slots of the K/V ring
constexpr uint32_t A2_BLK = 128 * 128;          // [128 rows][64 bf16] swizzled block: 16 KB
constexpr uint32_t A2_QHEAD = 4 * A2_BLK;       // Q hi (two d blocks) + Q lo: 64 KB
constexpr uint32_t A2_HSLOT = 2 * A2_BLK;       // K (two d blocks) or V^T (two key blocks): 32 KB
constexpr int A2_SMEM = 1024 + 2 * A2_QHEAD + A2_HSLOTS * A2_HSLOT;
constexpr int A2_LOAD_WARP = 8;
constexpr int A2_MMA_WARP = 9;   // the MMAs of the first head; warp 10 those of the second
constexpr int A2_THREADS = 32 * 11;
static_assert(A2_SMEM <= 227 * 1024 - 512, "shared memory budget");

// TMEM column offsets: head hl's S/P region and its O
__device__ __forceinline__ uint32_t a2_sp(int hl) { return (uint32_t)(hl * 256); }
__device__ __forceinline__ uint32_t a2_o(int hl) { return (uint32_t)(hl * 256 + 128); }

// A operand from TMEM (P), B from shared memory (V^T), fp32 accumulate in TMEM
__device__ __forceinline__ void a2_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The half-slot ring the load thread and both MMA threads follow, as plain arithmetic (no
// indexed arrays, so nothing spills to local memory): ring entries are taken in plan
// order, chunk j's K parts (one, or two for own keys: hi, lo), then as many V^T parts;
// entry e lives in half-slot e % A2_HSLOTS and is that half-slot's use e / A2_HSLOTS.
__device__ __forceinline__ int a2_slot(int e) { return e % A2_HSLOTS; }
__device__ __forceinline__ uint32_t a2_use_parity(int e) { return (uint32_t)(e / A2_HSLOTS) & 1u; }
// loads issued into half-slot s when the first n_entries entries were issued
__device__ __forceinline__ int a2_loads_into(int s, int n_entries) {
  return n_entries > s ? (n_entries - 1 - s) / A2_HSLOTS + 1 : 0;
}

__global__ void __launch_bounds__(A2_THREADS, 1)
    tc_attn2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQl,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmVt,
                    const __grid_constant__ CUtensorMap tmKl, const __grid_constant__ CUtensorMap tmVtl,
                    const TcAttnParams p, const int pair_heads) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_bar;
  __shared__ __align__(8) uint64_t hs_full[A2_HSLOTS];  // the half-slot's TMA loads have landed
  __shared__ __align__(8) uint64_t hs_free[A2_HSLOTS];  // the MMAs reading the half-slot are complete
  __shared__ __align__(8) uint64_t s_full[2];           // [head]: S of the chunk is in TMEM
  __shared__ __align__(8) uint64_t p_ready[2];          // [head]: P of the chunk is in TMEM (4 warps)
  __shared__ __align__(8) uint64_t pv_done[2];          // [head]: the PV of the chunk is complete
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int abort_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = blockIdx.x, sp = blockIdx.z;
  const int nh = (pair_heads && p.group % 2 == 0) ? 2 : 1;
  const int h0 = blockIdx.y * nh;
  const int kvh = h0 / p.group;
  const int q_row0 = qt * A2_BQ;
  const int rows_here = min(A2_BQ, p.n_q - q_row0);
  int kv_end = p.n_keys;
  if (p.causal) kv_end = min(p.n_keys, p.q_pos0 + q_row0 + rows_here);
  const int nch_total = (kv_end + A2_W - 1) / A2_W;
  const int c_begin = sp * p.chunks_per_split;
  const int nck = min(nch_total, c_begin + p.chunks_per_split) - c_begin;

  if (nck <= 0) {
    // this split sees no key of the tile: empty partials (weight 0 in the merge)
    griddep_sync();
    const int qrow = q_row0 + tid;
    if (tid < A2_BQ && qrow < p.n_q)
      for (int hl = 0; hl < nh; ++hl) {
        float* po = p.part_o + (((size_t)sp * p.nq + h0 + hl) * p.n_q + qrow) * A2_D;
        for (int i = 0; i < A2_D; ++i) po[i] = 0.0f;
        p.part_lse[((size_t)sp * p.nq + h0 + hl) * p.n_q + qrow] = -INFINITY;
      }
    return;
  }

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                   // [head][Q hi blk0, blk1, Q lo blk0, blk1]
  uint8_t* sHalf = smem + 2 * A2_QHEAD;  // [half-slot][blk0, blk1]

  if (warp == A2_MMA_WARP) tmem_alloc(&tmem_base_s, 512);
  if (tid == A2_LOAD_WARP * 32) {
    mbar_init(&q_bar, 1);
    for (int s = 0; s < A2_HSLOTS; ++s) {
      mbar_init(&hs_full[s], 1);
      mbar_init(&hs_free[s], nh);  // one commit per head's MMA thread
    }
    for (int hl = 0; hl < 2; ++hl) {
      mbar_init(&s_full[hl], 1);
      mbar_init(&p_ready[hl], 4);
      mbar_init(&pv_done[hl], 1);
    }
    mbar_init(&drain_bar, nh);
    abort_s = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_sync();  // the previous kernel wrote q and this layer's current K/V
  const uint32_t tmem = tmem_base_s;

  auto is_cur = [&](int j) { return p.has_lo && (c_begin + j) * A2_W >= p.base; };
  const uint32_t idesc = idesc_bf16_f32(A2_BQ, A2_W);  // S: 128 rows x 128 keys; PV: 128 rows x 128 d
  int issued = 0;  // ring entries the load thread issued loads for (for the wind-down)
  bool q_issued = false;

  if (warp == A2_LOAD_WARP) {
    if (lane == 0) {
      // ================= loads: the query tiles, then each chunk's K and V^T in plan order
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmQl);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmVt);
      if (p.has_lo) {
        prefetch_tmap(&tmKl);
        prefetch_tmap(&tmVtl);
      }
      mbar_arrive_expect_tx(&q_bar, nh * A2_QHEAD);
      for (int hl = 0; hl < nh; ++hl) {
        uint8_t* q = sQ + hl * A2_QHEAD;
        tma_load_3d(q, &tmQ, 0, q_row0, h0 + hl, &q_bar);
        tma_load_3d(q + A2_BLK, &tmQ, 64, q_row0, h0 + hl, &q_bar);
        tma_load_3d(q + 2 * A2_BLK, &tmQl, 0, q_row0, h0 + hl, &q_bar);
        tma_load_3d(q + 3 * A2_BLK, &tmQl, 64, q_row0, h0 + hl, &q_bar);
      }
      q_issued = true;
      bool ok = true;
      // ring entry e: wait until its half-slot's previous use was freed, then its two 16 KB blocks
      auto load_half = [&](int e, const CUtensorMap* map, bool is_v, int krow) {
        const int s = a2_slot(e);
        if (e >= A2_HSLOTS &&
            !mbar_wait(&hs_free[s], a2_use_parity(e - A2_HSLOTS), &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN))
          return false;
        if (!DG_GUARD(krow >= 0 && krow % A2_W == 0, p.err)) {
          abort_s = 1;
          return false;
        }
        uint8_t* dst = sHalf + s * A2_HSLOT;
        issued = e + 1;
        mbar_arrive_expect_tx(&hs_full[s], A2_HSLOT);
        if (is_v) {  // V^T [128 d][64 keys] blocks: keys krow .. +63, +64 .. +127
          tma_load_3d(dst, map, krow, 0, kvh, &hs_full[s]);
          tma_load_3d(dst + A2_BLK, map, krow + 64, 0, kvh, &hs_full[s]);
        } else {     // K [128 keys][64 d] blocks: d 0 .. 63, 64 .. 127
          tma_load_3d(dst, map, 0, krow, kvh, &hs_full[s]);
          tma_load_3d(dst + A2_BLK, map, 64, krow, kvh, &hs_full[s]);
        }
        return true;
      };
      for (int j = 0, e = 0; j < nck && ok; ++j) {
        const int key0 = (c_begin + j) * A2_W;
        const int n = is_cur(j) ? 2 : 1;
        // part 0: the cache's bf16 keys; part 1: the low terms, rows counted from `base`
        for (int i = 0; i < n && ok; ++i)
          ok = load_half(e + i, i == 0 ? &tmK : &tmKl, false, i == 0 ? key0 : key0 - p.base);
        for (int i = 0; i < n && ok; ++i)
          ok = load_half(e + n + i, i == 0 ? &tmVt : &tmVtl, true, i == 0 ? key0 : key0 - p.base);
        e += 2 * n;
      }
    }
    __syncwarp();
  } else if (warp == A2_MMA_WARP || warp == A2_MMA_WARP + 1) {
    const int hl = warp - A2_MMA_WARP;  // this warp's head
    if (lane == 0 && hl < nh) {
      // ================= MMAs of head hl: one issuing thread per head, so that each
      // head's waits, MMAs and commits run beside the other head's
      auto half_addr = [&](int e) { return smem_u32(sHalf + a2_slot(e) * A2_HSLOT); };
      // S(j): K parts at ring entries ek, ek + 1
      auto issue_s = [&](int ek, int n) {
        const uint32_t d = tmem + a2_sp(hl);
        const uint32_t q = smem_u32(sQ + hl * A2_QHEAD), ql = q + 2 * A2_BLK;
        const uint32_t k = half_addr(ek);
        const uint32_t kl = n == 2 ? half_addr(ek + 1) : 0u;
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t o = kb * A2_BLK + kk * 32;
            const uint64_t kd = sw128_kmajor_desc(k + o);
            tc_mma(d, sw128_kmajor_desc(q + o), kd, idesc, (kb | kk) != 0 ? 1u : 0u);
            tc_mma(d, sw128_kmajor_desc(ql + o), kd, idesc, 1u);
            if (n == 2) tc_mma(d, sw128_kmajor_desc(q + o), sw128_kmajor_desc(kl + o), idesc, 1u);
          }
        tc_commit(&s_full[hl]);
      };
      // PV(j): V^T parts at ring entries ev, ev + 1
      auto issue_pv = [&](int j, int ev, int n) {
        const uint32_t o = tmem + a2_o(hl), pp = tmem + a2_sp(hl);
        const uint32_t v = half_addr(ev);
        const uint32_t vl = n == 2 ? half_addr(ev + 1) : 0u;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // 16 keys = 8 packed P columns per MMA
          const uint32_t vo = (kk >> 2) * A2_BLK + (kk & 3) * 32;
          const uint64_t vd = sw128_kmajor_desc(v + vo);
          a2_mma_ts(o, pp + kk * 8, vd, idesc, (j > 0 || kk != 0) ? 1u : 0u);
          a2_mma_ts(o, pp + 64 + kk * 8, vd, idesc, 1u);
          if (n == 2) a2_mma_ts(o, pp + kk * 8, sw128_kmajor_desc(vl + vo), idesc, 1u);
        }
        tc_commit(&pv_done[hl]);
      };

      bool ok = mbar_wait(&q_bar, 0, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
      for (int j = 0, e = 0; j < nck && ok; ++j) {
        const int n = is_cur(j) ? 2 : 1;
        for (int i = 0; i < n && ok; ++i)
          ok = mbar_wait(&hs_full[a2_slot(e + i)], a2_use_parity(e + i), &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
        // the head's S/P region was last read by PV(j - 1)
        if (ok && j >= 1)
          ok = mbar_wait(&pv_done[hl], (uint32_t)(j - 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
        if (!ok) break;
        tc_fence_after();
        issue_s(e, n);
        // a K half-slot is free once both heads' S MMAs have read it (count: one per head)
        for (int i = 0; i < n; ++i) tc_commit(&hs_free[a2_slot(e + i)]);
        for (int i = 0; i < n && ok; ++i)
          ok = mbar_wait(&hs_full[a2_slot(e + n + i)], a2_use_parity(e + n + i), &abort_s, p.err,
                         DG_DEVERR_TIMEOUT_ATTN);
        if (ok) ok = mbar_wait(&p_ready[hl], (uint32_t)j & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
        if (!ok) break;
        tc_fence_after();
        issue_pv(j, e + n, n);
        for (int i = 0; i < n; ++i) tc_commit(&hs_free[a2_slot(e + n + i)]);
        e += 2 * n;
      }
    }
    __syncwarp();
  } else if ((warp >> 2) < nh) {
    // ================= softmax: head hl, query row `row` (TMEM lane), all 128 keys of a chunk
    const int hl = warp >> 2;
    const int h = h0 + hl;
    const int row = (warp & 3) * 32 + lane;
    const int my_row = q_row0 + row;
    const int my_pos = p.q_pos0 + my_row;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int key_lim = p.causal ? min(p.n_keys, my_pos + 1) : p.n_keys;
    const uint32_t spa = tmem + a2_sp(hl) + lane_off;
    float m_used = -INFINITY;
    uint64_t l2 = f2_pack(0.0f, 0.0f);  // the row sum as two partial sums (even and odd keys)
    const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
    bool ok = true;
    for (int j = 0; j < nck && ok; ++j) {
      // every wait's outcome is made warp-uniform: the tcgen05.ld / st that follow are
      // warp-collective, so a lane that gave up must take its whole warp with it
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&s_full[hl], (uint32_t)j & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN));
      if (!ok) break;
      tc_fence_after();
      // the chunk's raw scores, all eight loads in flight before the one wait
      uint32_t r[A2_W / 16][16];
#pragma unroll
      for (int c = 0; c < A2_W / 16; ++c) tmem_ld16(spa + c * 16, r[c]);
      tc_wait_ld();
      const int key0 = (c_begin + j) * A2_W;
      // keys at or past the row's limit (only in the chunk that holds the limit)
      if (__any_sync(0xffffffffu, key0 + A2_W > key_lim)) {
#pragma unroll
        for (int i = 0; i < A2_W; ++i)
          if (key0 + i >= key_lim) r[i / 16][i % 16] = __float_as_uint(-INFINITY);
      }
      // the row maximum of the raw scores (four independent chains), then scaled: the
      // scale is positive and rounding monotone, so this is the maximum of the scaled scores
      float cm4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int i = 0; i < A2_W; i += 8)
#pragma unroll
        for (int c = 0; c < 4; ++c)
          cm4[c] = max3f(cm4[c], __uint_as_float(r[(i + 2 * c) / 16][(i + 2 * c) % 16]),
                         __uint_as_float(r[(i + 2 * c) / 16][(i + 2 * c) % 16 + 1]));
      const float cmax = fmaxf(fmaxf(cm4[0], cm4[1]), fmaxf(cm4[2], cm4[3])) * p.scale_log2;
      const bool upd = cmax > m_used + 8.0f;
      const float alpha = upd ? ex2_approx(m_used - cmax) : 1.0f;  // 0 while nothing was visible yet
      // tcgen05.ld/st are warp-collective: the warp rescales its rows of O if any row must,
      // once the previous chunk's PV is complete (O stable; PV(j) waits for this P)
      if (__any_sync(0xffffffffu, upd && j > 0)) {
        ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[hl], (uint32_t)(j - 1) & 1u, &abort_s, p.err,
                                               DG_DEVERR_TIMEOUT_ATTN));
        if (!ok) break;
        tc_fence_after();
        const uint32_t oa = tmem + a2_o(hl) + lane_off;
        // (16 columns at a time: the chunk's 128 scores stay live in registers meanwhile)
#pragma unroll 1
        for (int c = 0; c < A2_D / 16; ++c) {
          uint32_t o[16];
          tmem_ld16(oa + c * 16, o);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st16(oa + c * 16, o);
        }
      }
      if (upd) {
        l2 = f2_mul(l2, f2_pack(alpha, alpha));
        m_used = cmax;
      }
      // P = 2^(s * scale - m_used) (one rounding), packed bf16 pairs over this row's S: hi
      // in columns 0..63, lo in 64..127.  A row that has seen no key has m_used = -inf and
      // only -inf scores: its offset is taken as 0, so that every P is 2^-inf = 0.
      const float neg_m = (m_used == -INFINITY) ? 0.0f : -m_used;
      const uint64_t nm2 = f2_pack(neg_m, neg_m);
#pragma unroll
      for (int c = 0; c < A2_W / 16; ++c) {  // 16 keys -> 8 packed columns per store
        uint32_t wh[8], wl[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int i0 = c * 16 + 2 * e;
          const uint64_t t = f2_fma(f2_pack(__uint_as_float(r[i0 / 16][i0 % 16]),
                                            __uint_as_float(r[i0 / 16][i0 % 16 + 1])), scale2, nm2);
          float t0, t1;
          f2_unpack(t, t0, t1);
          const float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
          const uint64_t pp = f2_pack(p0, p1);
          l2 = f2_add(l2, pp);
          const uint32_t hi = bf16x2_pack(p0, p1);
          float lo0, lo1;
          f2_unpack(f2_sub(pp, bf16x2_widen(hi)), lo0, lo1);
          wh[e] = hi;
          wl[e] = bf16x2_pack(lo0, lo1);
        }
        tmem_st8(spa + c * 8, wh);
        tmem_st8(spa + 64 + c * 8, wl);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready[hl]);
    }
    if (ok)
      ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[hl], (uint32_t)(nck - 1) & 1u, &abort_s, p.err,
                                             DG_DEVERR_TIMEOUT_ATTN));
    float l0, l1;
    f2_unpack(l2, l0, l1);
    const float l = l0 + l1;
    if (ok) {
      tc_fence_after();
      const bool valid = my_row < p.n_q;
      const float inv_l = (l > 0.0f) ? 1.0f / l : 0.0f;
      const uint32_t oa = tmem + a2_o(hl) + lane_off;
      if (p.n_splits == 1) {
        const size_t base = (size_t)my_row * p.nq * A2_D + (size_t)h * A2_D;
#pragma unroll
        for (int c = 0; c < A2_D / 16; ++c) {
          uint32_t r[16];
          tmem_ld16(oa + c * 16, r);
          tc_wait_ld();
          if (valid) {
            uint32_t w[8], wl[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float a = __uint_as_float(r[2 * e]) * inv_l, bb = __uint_as_float(r[2 * e + 1]) * inv_l;
              const __nv_bfloat162 hi = __floats2bfloat162_rn(a, bb);
              const __nv_bfloat162 lo = __floats2bfloat162_rn(a - __low2float(hi), bb - __high2float(hi));
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
        float* po = p.part_o + (((size_t)sp * p.nq + h) * p.n_q + my_row) * A2_D;
#pragma unroll
        for (int c = 0; c < A2_D / 16; ++c) {
          uint32_t r[16];
          tmem_ld16(oa + c * 16, r);
          tc_wait_ld();
          if (valid) {
            float4* dst = reinterpret_cast<float4*>(po + c * 16);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_float4(__uint_as_float(r[4 * e]) * inv_l, __uint_as_float(r[4 * e + 1]) * inv_l,
                                   __uint_as_float(r[4 * e + 2]) * inv_l, __uint_as_float(r[4 * e + 3]) * inv_l);
          }
        }
        if (valid) p.part_lse[((size_t)sp * p.nq + h) * p.n_q + my_row] = (l > 0.0f) ? m_used + log2f(l) : -INFINITY;
      }
    }
  }
  __syncthreads();
  // wind down: every MMA and commit the MMA thread issued has landed (also on the normal
  // path, so that no mbarrier arrive reaches this CTA's shared memory after it is gone),
  // and after an abort the loads the load thread issued have landed too
  if (lane == 0 && (warp == A2_MMA_WARP || (nh == 2 && warp == A2_MMA_WARP + 1))) tc_commit(&drain_bar);
  if (tid == A2_MMA_WARP * 32) mbar_wait_drain(&drain_bar, 0);
  if (abort_s && tid == A2_LOAD_WARP * 32) {
    if (q_issued) mbar_wait_drain(&q_bar, 0);
    for (int s = 0; s < A2_HSLOTS; ++s) {
      const int loads = a2_loads_into(s, issued);
      if (loads > 0) mbar_wait_drain(&hs_full[s], (uint32_t)(loads - 1) & 1u);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == A2_MMA_WARP) tmem_dealloc(tmem, 512);
}

// Split-KV merge in a kernel of its own (the head-pair kernel's splits write partials):
// one warp per (query row, head), spread over the whole GPU -- a merge by the last split
// of each tile would leave one CTA to read every split's partial rows (about 1 MB at the
// large model's nine splits), a tail of tens of microseconds.  Lane s < n_splits reads split s's
// log2-sum-exp, the warp takes their maximum and the weights exp2(lse_s - max) by
// shuffles, and each lane merges four of the 128 output columns over the splits (all the
// splits' loads issued before the first product), then writes the bf16 hi and lo parts.
// Rows with no visible key (every lse -inf) are written as zeros.
__global__ void __launch_bounds__(256) attn_merge2_kernel(const float* __restrict__ part_o,
                                                          const float* __restrict__ part_lse, int n_splits, int nq,
                                                          int n_q, __nv_bfloat16* out, __nv_bfloat16* out_lo) {
  griddep_sync();
  const int lane = threadIdx.x & 31;
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (w >= nq * n_q) return;
  const int h = w / n_q, row = w % n_q;
  const float lse = lane < n_splits ? part_lse[((size_t)lane * nq + h) * n_q + row] : -INFINITY;
  float mx = lse;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float wt = (lse == -INFINITY) ? 0.0f : exp2f(lse - mx);
  float den = wt;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  // every split's row slice loaded before the first product (same summation order)
  constexpr int MAXS = 16;
  float4 v[MAXS];
#pragma unroll
  for (int sp = 0; sp < MAXS; ++sp)
    if (sp < n_splits) v[sp] = reinterpret_cast<const float4*>(part_o + (((size_t)sp * nq + h) * n_q + row) * A2_D)[lane];
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int sp = 0; sp < MAXS; ++sp) {
    if (sp >= n_splits) break;
    const float ws = __shfl_sync(0xffffffffu, wt, sp);
    if (ws == 0.0f) continue;  // uniform across the warp
    acc.x += ws * v[sp].x;
    acc.y += ws * v[sp].y;
    acc.z += ws * v[sp].z;
    acc.w += ws * v[sp].w;
  }
  const float inv = den > 0.0f ? 1.0f / den : 0.0f;
  const float a[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
  uint32_t hw[2], lw[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const __nv_bfloat162 hi = __floats2bfloat162_rn(a[2 * e], a[2 * e + 1]);
    const __nv_bfloat162 lo = __floats2bfloat162_rn(a[2 * e] - __low2float(hi), a[2 * e + 1] - __high2float(hi));
    hw[e] = *reinterpret_cast<const uint32_t*>(&hi);
    lw[e] = *reinterpret_cast<const uint32_t*>(&lo);
  }
  const size_t o = (size_t)row * nq * A2_D + (size_t)h * A2_D + 4 * lane;
  *reinterpret_cast<uint2*>(out + o) = make_uint2(hw[0], hw[1]);
  if (out_lo) *reinterpret_cast<uint2*>(out_lo + o) = make_uint2(lw[0], lw[1]);
}

cudaError_t launch_attn_merge2(const float* part_o, const float* part_lse, int n_splits, int nq, int n_q,
                               __nv_bfloat16* out, __nv_bfloat16* out_lo, cudaStream_t st) {
  if (n_splits < 1 || n_splits > 16) return cudaErrorInvalidValue;
  const int warps = nq * n_q;
  return launch_k(attn_merge2_kernel, dim3((warps + 7) / 8), dim3(256), 0, st, part_o, part_lse, n_splits, nq, n_q,
                  out, out_lo);
}

int attn2_head_groups(int nq, int group, int pair_heads) { return (pair_heads && group % 2 == 0) ? nq / 2 : nq; }

cudaError_t launch_tc_attention2(const CUtensorMap& Q, const CUtensorMap& Ql, const CUtensorMap& K,
                                 const CUtensorMap& Vt, const CUtensorMap& Kl, const CUtensorMap& Vtl,
                                 const TcAttnParams& p, int pair_heads, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(tc_attn2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, A2_SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((p.n_q + A2_BQ - 1) / A2_BQ, attn2_head_groups(p.nq, p.group, pair_heads), p.n_splits);
  return launch_k(tc_attn2_kernel, grid, dim3(A2_THREADS), A2_SMEM, st, Q, Ql, K, Vt, Kl, Vtl, p, pair_heads);
}

cudaError_t set_wait_limit_attn2(uint64_t ns) { return set_wait_limit_this_file(ns); }

}  // namespace dg
