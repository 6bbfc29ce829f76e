// tcgen05 flash attention over the KV cache, single-head kernel, both attention modes of
// the pass:
//   denoising mode: every canvas query sees all cached prefix keys and all canvas keys
//                   (bidirectional block rows of the prefix/block mask);
//   prefill mode:   new tokens see keys up to their own position (causal rows).
// One CTA = one query head x 128 query rows x a contiguous range of 128-key chunks
// (split-KV: the splits write fp32 partials and log2-sum-exps, merged by
// attn_merge2_kernel).  V is kept transposed in the cache ([d][position]) so the B
// operands of both MMAs are K-major in shared memory.
//
// Precision.  Cached keys/values are bf16 (the cache's storage format).  The query and the
// keys/values of the tokens the call itself processes are in flight at fp32 precision,
// carried as bf16 hi + lo terms: S = Q_hi K^T + Q_lo K^T (+ Q_hi K_lo^T on the chunks
// holding current tokens), O += P_hi V + P_lo V (+ P_hi V_lo on those chunks).  The low
// parts of the current K/V live in a workspace window whose row 0 is the 128-aligned chunk
// start `base` at or below the first current position; rows before the first current
// position are zero there.
//
// Layout.  Shared memory: the query tile (hi + lo, 64 KB, TMA), a ring of three 32 KB
// half-slots for K [128 keys][128 d] and one of two for V^T [128 d][128 keys] (two 16 KB
// blocks each, 128-byte swizzled); a chunk of the call's own keys takes two entries of
// each ring (hi, then lo).
// TMEM (512 columns): two S buffers (fp32, 128 keys) at 0 and 128, O at 256, and P at 384
// (packed bf16 pairs along the keys: hi in 384..447, lo in 448..511).  Chunk j uses S
// buffer j & 1.
//
// Roles.  Warps 0-3 run the softmax, one query row per thread (its TMEM lane) over the
// whole 128-key chunk, so no row statistics are exchanged between warps; warps 4 and 7
// issue the TMA loads of the K ring (and the query tile) and of the V^T ring, each ring in
// its own order, so that a K load never waits behind a V^T half-slot still being read;
// warps 5 and 6 issue the MMAs, one thread each: warp 5 the S MMAs, S(j) once
// chunk j's K has landed and the softmax has read S(j - 2) out of the same buffer, then a
// commit freeing the K half-slots; warp 6 the PV MMAs, PV(j) once chunk j's V^T has landed
// and the softmax has written P(j), then a commit freeing the V^T half-slots.  Each issuing
// thread's waits and commits (a few hundred nanoseconds each, measured) then run while the
// tensor cores execute the other thread's MMAs, and the tensor cores compute S(j + 1) and
// PV(j - 1) while the softmax works on S(j).  The softmax of chunk j computes P(j) in
// registers, then, once PV(j - 1) is complete, rescales O (lazily, when its row maximum
// grew by more than 2^8) and writes P(j) over P(j - 1).  Hand-offs are mbarriers with
// bounded waits.
#include <math.h>

#include "attn_softmax.cuh"
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

constexpr int AT_BQ = 128;
constexpr int AT_W = 128;                       // keys per chunk
constexpr int AT_D = 128;
constexpr int AT_KSLOTS = 3;                    // half-slots of the K ring
constexpr int AT_VSLOTS = 2;                    // half-slots of the V^T ring (after the K ring's)
constexpr int AT_HSLOTS = AT_KSLOTS + AT_VSLOTS;
constexpr uint32_t AT_BLK = 128 * 128;          // [128 rows][64 bf16] swizzled block: 16 KB
constexpr uint32_t AT_QTILE = 4 * AT_BLK;       // Q hi (two d blocks) + Q lo (two d blocks): 64 KB
constexpr uint32_t AT_HSLOT = 2 * AT_BLK;       // K (two d blocks) or V^T (two key blocks): 32 KB
constexpr int AT_SMEM = 1024 + AT_QTILE + AT_HSLOTS * AT_HSLOT;
constexpr int AT_SM_WARPS = 4;
constexpr int AT_LOAD_WARP = 4;   // the query tile and the K ring
constexpr int AT_VLOAD_WARP = 7;  // the V^T ring
constexpr int AT_S_WARP = 5;    // issues the S MMAs (and holds the TMEM allocation)
constexpr int AT_PV_WARP = 6;   // issues the PV MMAs
constexpr int AT_THREADS = 32 * 8;
static_assert(AT_SMEM <= 227 * 1024 - 512, "shared memory budget");

// TMEM column offsets
__device__ __forceinline__ uint32_t at_s(int b) { return (uint32_t)(b * 128); }  // S buffer b
constexpr uint32_t AT_O = 256;                                                     // O
constexpr uint32_t AT_PHI = 384, AT_PLO = 448;                                     // P hi, P lo

// A operand from TMEM (P), B from shared memory (V^T), fp32 accumulate in TMEM
__device__ __forceinline__ void at_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The two half-slot rings, as plain arithmetic (no indexed arrays, so nothing spills to
// local memory).  Chunk j's K parts (one, or two for own keys: hi, lo) take the next
// entries of the K ring, its V^T parts those of the V^T ring; K entry e lives in half-slot
// e % AT_KSLOTS, V^T entry e in half-slot AT_KSLOTS + e % AT_VSLOTS, as that half-slot's
// use e / (ring size).  Each ring has one consumer (the S thread, the PV thread), which
// waits for its entries in order: so no wait can meet a half-slot whose previous use has
// not landed yet (a parity wait there would pass at once).
__device__ __forceinline__ int at_kslot(int e) { return e % AT_KSLOTS; }
__device__ __forceinline__ int at_vslot(int e) { return AT_KSLOTS + e % AT_VSLOTS; }
__device__ __forceinline__ uint32_t at_kparity(int e) { return (uint32_t)(e / AT_KSLOTS) & 1u; }
__device__ __forceinline__ uint32_t at_vparity(int e) { return (uint32_t)(e / AT_VSLOTS) & 1u; }
// loads issued into the ring's slot r (0-based within the ring) when its first n entries were issued
__device__ __forceinline__ int at_loads_into(int r, int n, int ring) { return n > r ? (n - 1 - r) / ring + 1 : 0; }

__global__ void __launch_bounds__(AT_THREADS, 1)
    tc_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQl,
                   const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmVt,
                   const __grid_constant__ CUtensorMap tmKl, const __grid_constant__ CUtensorMap tmVtl,
                   const TcAttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_bar;
  __shared__ __align__(8) uint64_t hs_full[AT_HSLOTS];  // the half-slot's TMA loads have landed
  __shared__ __align__(8) uint64_t hs_free[AT_HSLOTS];  // the MMAs reading the half-slot are complete
  __shared__ __align__(8) uint64_t s_full[2];           // [buffer]: S of the chunk is in TMEM
  __shared__ __align__(8) uint64_t s_free[2];           // [buffer]: the softmax warps have read S
  __shared__ __align__(8) uint64_t p_ready;             // P of the chunk is in TMEM
  __shared__ __align__(8) uint64_t pv_done;             // the PV of the chunk is complete
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int abort_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = blockIdx.x, h = blockIdx.y, sp = blockIdx.z;
  const int kvh = h / p.group;
  const int q_row0 = qt * AT_BQ;
  const int rows_here = min(AT_BQ, p.n_q - q_row0);
  int kv_end = p.n_keys;
  if (p.causal) kv_end = min(p.n_keys, p.q_pos0 + q_row0 + rows_here);
  const int nch_total = (kv_end + AT_W - 1) / AT_W;
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
    return;
  }

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                // [Q hi blk0, blk1, Q lo blk0, blk1]
  uint8_t* sHalf = smem + AT_QTILE;  // [half-slot][blk0, blk1]

  if (warp == AT_S_WARP) tmem_alloc(&tmem_base_s, 512);
  if (tid == AT_LOAD_WARP * 32) {
    mbar_init(&q_bar, 1);
    for (int s = 0; s < AT_HSLOTS; ++s) {
      mbar_init(&hs_full[s], 1);
      mbar_init(&hs_free[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], AT_SM_WARPS);
    }
    mbar_init(&p_ready, AT_SM_WARPS);
    mbar_init(&pv_done, 1);
    mbar_init(&drain_bar, 2);  // one commit per issuing thread
    abort_s = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_sync();  // the previous kernel wrote q and this layer's current K/V
  const uint32_t tmem = tmem_base_s;

  // chunk j (0-based within this CTA) holds keys [key0, key0 + 128); chunks of the call's
  // own keys (key0 >= base) also carry low terms and take two half-slots per operand
  auto is_cur = [&](int j) { return p.has_lo && (c_begin + j) * AT_W >= p.base; };
  const uint32_t idesc = idesc_bf16_f32(AT_BQ, AT_W);  // S: 128 rows x 128 keys; PV: 128 rows x 128 d
  int issued_k = 0, issued_v = 0;  // ring entries the load thread issued loads for (for the wind-down)
  bool q_issued = false;

  if (warp == AT_LOAD_WARP || warp == AT_VLOAD_WARP) {
    if (lane == 0) {
      // ================= loads: warp 4 the query tile, then each chunk's K in plan order;
      // warp 7 each chunk's V^T
      const bool is_v = warp == AT_VLOAD_WARP;
      if (!is_v) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmQl);
        prefetch_tmap(&tmK);
        if (p.has_lo) prefetch_tmap(&tmKl);
        mbar_arrive_expect_tx(&q_bar, AT_QTILE);
        tma_load_3d(sQ, &tmQ, 0, q_row0, h, &q_bar);
        tma_load_3d(sQ + AT_BLK, &tmQ, 64, q_row0, h, &q_bar);
        tma_load_3d(sQ + 2 * AT_BLK, &tmQl, 0, q_row0, h, &q_bar);
        tma_load_3d(sQ + 3 * AT_BLK, &tmQl, 64, q_row0, h, &q_bar);
        q_issued = true;
      } else {
        prefetch_tmap(&tmVt);
        if (p.has_lo) prefetch_tmap(&tmVtl);
      }
      const int ring = is_v ? AT_VSLOTS : AT_KSLOTS;
      const CUtensorMap* map_hi = is_v ? &tmVt : &tmK;
      const CUtensorMap* map_lo = is_v ? &tmVtl : &tmKl;
      bool ok = true;
      for (int j = 0, e = 0; j < nck && ok; ++j) {  // e: chunk j's first entry in this ring
        const int key0 = (c_begin + j) * AT_W;
        const int n = is_cur(j) ? 2 : 1;
        // part 0: the cache's bf16 keys; part 1: the low terms, rows counted from `base`
        for (int i = 0; i < n && ok; ++i, ++e) {
          // wait until the half-slot's previous use was freed, then its two 16 KB blocks
          const int s = is_v ? at_vslot(e) : at_kslot(e);
          if (e >= ring && !mbar_wait(&hs_free[s], is_v ? at_vparity(e - ring) : at_kparity(e - ring), &abort_s,
                                      p.err, DG_DEVERR_TIMEOUT_ATTN)) {
            ok = false;
            break;
          }
          const int krow = i == 0 ? key0 : key0 - p.base;
          if (!DG_GUARD(krow >= 0 && krow % AT_W == 0, p.err)) {
            abort_s = 1;
            ok = false;
            break;
          }
          uint8_t* dst = sHalf + s * AT_HSLOT;
          (is_v ? issued_v : issued_k) = e + 1;
          mbar_arrive_expect_tx(&hs_full[s], AT_HSLOT);
          const CUtensorMap* map = i == 0 ? map_hi : map_lo;
          if (is_v) {  // V^T [128 d][64 keys] blocks: keys krow .. +63, +64 .. +127
            tma_load_3d(dst, map, krow, 0, kvh, &hs_full[s]);
            tma_load_3d(dst + AT_BLK, map, krow + 64, 0, kvh, &hs_full[s]);
          } else {     // K [128 keys][64 d] blocks: d 0 .. 63, 64 .. 127
            tma_load_3d(dst, map, 0, krow, kvh, &hs_full[s]);
            tma_load_3d(dst + AT_BLK, map, 64, krow, kvh, &hs_full[s]);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == AT_S_WARP || warp == AT_PV_WARP) {
    if (lane == 0) {
      // ================= MMAs: warp 5 the S MMAs, warp 6 the PV MMAs, in chunk order
      auto half_addr = [&](int s) { return smem_u32(sHalf + s * AT_HSLOT); };
      const uint32_t q = smem_u32(sQ), ql = q + 2 * AT_BLK;
      // S(j): K parts at ring entries ek, ek + 1
      auto issue_s = [&](int j, int ek, int n) {
        const uint32_t d = tmem + at_s(j & 1);
        const uint32_t k = half_addr(at_kslot(ek));
        const uint32_t kl = n == 2 ? half_addr(at_kslot(ek + 1)) : 0u;
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // 16 d values per MMA
            const uint32_t o = kb * AT_BLK + kk * 32;
            const uint64_t kd = sw128_kmajor_desc(k + o);
            tc_mma(d, sw128_kmajor_desc(q + o), kd, idesc, (kb | kk) != 0 ? 1u : 0u);
            tc_mma(d, sw128_kmajor_desc(ql + o), kd, idesc, 1u);
            if (n == 2) tc_mma(d, sw128_kmajor_desc(q + o), sw128_kmajor_desc(kl + o), idesc, 1u);
          }
        tc_commit(&s_full[j & 1]);
      };
      // PV of chunk i once its V^T (ring entries ev, ev + 1) has landed and the softmax has
      // written P(i); then the commits that free its V half-slots
      auto do_pv = [&](int i, int ev, int n) {
        bool ok2 = true;
        for (int t = 0; t < n && ok2; ++t)
          ok2 = mbar_wait(&hs_full[at_vslot(ev + t)], at_vparity(ev + t), &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
        if (ok2) ok2 = mbar_wait(&p_ready, (uint32_t)i & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
        if (!ok2) return false;
        tc_fence_after();
        const uint32_t o = tmem + AT_O, ph = tmem + AT_PHI, pl = tmem + AT_PLO;
        const uint32_t v = half_addr(at_vslot(ev));
        const uint32_t vl = n == 2 ? half_addr(at_vslot(ev + 1)) : 0u;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // 16 keys = 8 packed P columns per MMA
          const uint32_t vo = (kk >> 2) * AT_BLK + (kk & 3) * 32;
          const uint64_t vd = sw128_kmajor_desc(v + vo);
          at_mma_ts(o, ph + kk * 8, vd, idesc, (i > 0 || kk != 0) ? 1u : 0u);
          at_mma_ts(o, pl + kk * 8, vd, idesc, 1u);
          if (n == 2) at_mma_ts(o, ph + kk * 8, sw128_kmajor_desc(vl + vo), idesc, 1u);
        }
        tc_commit(&pv_done);
        for (int t = 0; t < n; ++t) tc_commit(&hs_free[at_vslot(ev + t)]);
        return true;
      };

      if (warp == AT_S_WARP) {
        bool ok = mbar_wait(&q_bar, 0, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
        for (int j = 0, e = 0; j < nck && ok; ++j) {  // e: chunk j's first K entry
          const int n = is_cur(j) ? 2 : 1;
          for (int t = 0; t < n && ok; ++t)
            ok = mbar_wait(&hs_full[at_kslot(e + t)], at_kparity(e + t), &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
          // S buffer j & 1 was last read by the softmax of chunk j - 2
          if (ok && j >= 2)
            ok = mbar_wait(&s_free[j & 1], (uint32_t)((j - 2) >> 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN);
          if (!ok) break;
          tc_fence_after();
          issue_s(j, e, n);
          for (int t = 0; t < n; ++t) tc_commit(&hs_free[at_kslot(e + t)]);
          e += n;
        }
      } else {
        bool ok = true;
        for (int j = 0, e = 0; j < nck && ok; ++j) {  // e: chunk j's first V^T entry
          const int n = is_cur(j) ? 2 : 1;
          ok = do_pv(j, e, n);
          e += n;
        }
      }
    }
    __syncwarp();
  } else {
    // ================= softmax: query row `row` (TMEM lane), all 128 keys of a chunk.
    // Every bounded wait is voted on by the whole warp (__all_sync): the tcgen05.ld / st
    // that follow are warp-collective, so no lane may go on alone after another lane's
    // wait gave up.
    const int row = warp * 32 + lane;
    const int my_row = q_row0 + row;
    const int my_pos = p.q_pos0 + my_row;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const int key_lim = p.causal ? min(p.n_keys, my_pos + 1) : p.n_keys;
    float m_used = -INFINITY;
    uint64_t l2 = f2_pack(0.0f, 0.0f);  // the row sum as two partial sums (even and odd keys)
    const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
    bool ok = true;
    for (int j = 0; j < nck && ok; ++j) {
      const int b = j & 1;
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&s_full[b], (uint32_t)(j >> 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN));
      if (!ok) break;
      tc_fence_after();
      // the chunk's raw scores, all eight loads in flight before the one wait
      uint32_t r[AT_W / 16][16];
#pragma unroll
      for (int c = 0; c < AT_W / 16; ++c) tmem_ld16(tmem + at_s(b) + lane_off + c * 16, r[c]);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[b]);  // S(j + 2) may go into this buffer
      const int key0 = (c_begin + j) * AT_W;
      // keys at or past the row's limit (only in the chunk that holds the limit)
      if (__any_sync(0xffffffffu, key0 + AT_W > key_lim)) {
#pragma unroll
        for (int i = 0; i < AT_W; ++i)
          if (key0 + i >= key_lim) r[i / 16][i % 16] = __float_as_uint(-INFINITY);
      }
      // the row maximum of the raw scores (four independent chains), then scaled: the
      // scale is positive and rounding monotone, so this is the maximum of the scaled scores
      float cm4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int i = 0; i < AT_W; i += 8)
#pragma unroll
        for (int c = 0; c < 4; ++c)
          cm4[c] = max3f(cm4[c], __uint_as_float(r[(i + 2 * c) / 16][(i + 2 * c) % 16]),
                         __uint_as_float(r[(i + 2 * c) / 16][(i + 2 * c) % 16 + 1]));
      const float cmax = fmaxf(fmaxf(cm4[0], cm4[1]), fmaxf(cm4[2], cm4[3])) * p.scale_log2;
      const bool upd = cmax > m_used + 8.0f;
      const float alpha = upd ? ex2_approx(m_used - cmax) : 1.0f;  // 0 while nothing was visible yet
      if (upd) {
        l2 = f2_mul(l2, f2_pack(alpha, alpha));
        m_used = cmax;
      }
      // P = 2^(s * scale - m_used) (one rounding) as packed bf16 pairs, hi and lo, in
      // registers while the tensor cores finish PV(j - 1).  A row that has seen no key has
      // m_used = -inf and only -inf scores: its offset is taken as 0, so that every P is
      // 2^-inf = 0.
      const float neg_m = (m_used == -INFINITY) ? 0.0f : -m_used;
      const uint64_t nm2 = f2_pack(neg_m, neg_m);
      uint32_t wh[AT_W / 2], wl[AT_W / 2];
#pragma unroll
      for (int e = 0; e < AT_W / 2; ++e) {
        const int i0 = 2 * e;
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
      // PV(j - 1) is complete: O is stable and P(j - 1) read.  The warp rescales its rows of
      // O if any row must (16 columns at a time), then writes P(j).
      if (j > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&pv_done, (uint32_t)(j - 1) & 1u, &abort_s, p.err,
                                               DG_DEVERR_TIMEOUT_ATTN));
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, upd)) {
          const uint32_t oa = tmem + AT_O + lane_off;
#pragma unroll 1
          for (int c = 0; c < AT_D / 16; ++c) {
            uint32_t o[16];
            tmem_ld16(oa + c * 16, o);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16(oa + c * 16, o);
          }
        }
      }
#pragma unroll
      for (int c = 0; c < AT_W / 32; ++c) {  // 32 keys -> 16 packed columns per store
        uint32_t h16[16], l16[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) h16[e] = wh[c * 16 + e], l16[e] = wl[c * 16 + e];
        tmem_st16(tmem + AT_PHI + lane_off + c * 16, h16);
        tmem_st16(tmem + AT_PLO + lane_off + c * 16, l16);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready);
    }
    if (ok)
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&pv_done, (uint32_t)(nck - 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ATTN));
    float l0, l1;
    f2_unpack(l2, l0, l1);
    const float l = l0 + l1;
    if (ok) {
      tc_fence_after();
      const bool valid = my_row < p.n_q;
      const float inv_l = (l > 0.0f) ? 1.0f / l : 0.0f;
      const uint32_t oa = tmem + AT_O + lane_off;
      if (p.n_splits == 1) {
        const size_t base = (size_t)my_row * p.nq * AT_D + (size_t)h * AT_D;
#pragma unroll
        for (int c = 0; c < AT_D / 16; ++c) {
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
        float* po = p.part_o + (((size_t)sp * p.nq + h) * p.n_q + my_row) * AT_D;
#pragma unroll
        for (int c = 0; c < AT_D / 16; ++c) {
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
  if (lane == 0 && (warp == AT_S_WARP || warp == AT_PV_WARP)) tc_commit(&drain_bar);
  if (tid == AT_S_WARP * 32) mbar_wait_drain(&drain_bar, 0);
  if (abort_s && tid == AT_LOAD_WARP * 32) {
    if (q_issued) mbar_wait_drain(&q_bar, 0);
    for (int r = 0; r < AT_KSLOTS; ++r) {
      const int loads = at_loads_into(r, issued_k, AT_KSLOTS);
      if (loads > 0) mbar_wait_drain(&hs_full[r], (uint32_t)(loads - 1) & 1u);
    }
  }
  if (abort_s && tid == AT_VLOAD_WARP * 32) {
    for (int r = 0; r < AT_VSLOTS; ++r) {
      const int loads = at_loads_into(r, issued_v, AT_VSLOTS);
      if (loads > 0) mbar_wait_drain(&hs_full[AT_KSLOTS + r], (uint32_t)(loads - 1) & 1u);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == AT_S_WARP) tmem_dealloc(tmem, 512);
}

cudaError_t launch_tc_attention(const CUtensorMap& Q, const CUtensorMap& Ql, const CUtensorMap& K,
                                const CUtensorMap& Vt, const CUtensorMap& Kl, const CUtensorMap& Vtl,
                                const TcAttnParams& p, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(tc_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((p.n_q + AT_BQ - 1) / AT_BQ, p.nq, p.n_splits);
  return launch_k(tc_attn_kernel, grid, dim3(AT_THREADS), AT_SMEM, st, Q, Ql, K, Vt, Kl, Vtl, p);
}

cudaError_t set_wait_limit_attn(uint64_t ns) { return set_wait_limit_this_file(ns); }

}  // namespace dg
