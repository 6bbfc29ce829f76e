// Persistent tcgen05 GEMM with 8-bit weights for the expert contractions: the same
// weights-on-M / tokens-on-N tiling as the bf16 GEMM, but each weight row is stored as
// E4M3 codes with one power-of-two scale per 32 consecutive K elements (the OCP MX
// block format: E8M0 scale 2^(s - 127)).  The weight stream, which bounds these GEMMs,
// is half the bytes of bf16.
//
// Decoding is exact: an E4M3 value times a power of two has at most 4 significant bits,
// which bf16 holds, so the MMAs see exactly the weights the codes define and the pass
// keeps the precision model of the bf16 path (activations in one or two bf16 terms,
// fp32 accumulation).  Decoded tiles never touch shared memory: decoder warps read the
// 8-bit tile and its scales from shared memory, build the bf16 values in registers and
// store them to TMEM, and the MMA takes its A operand (the weights) from TMEM.
//
// Roles (448 threads, one CTA per SM, tiles blockIdx.x, blockIdx.x + gridDim.x, ...):
//   warp 0      TMA: 8-bit weight tiles (64-byte swizzle), scale tiles and token tiles
//               into a ring of shared-memory stages;
//   warp 1      TMEM allocation and tcgen05.mma (A from TMEM, B = tokens from smem) into
//               one of two accumulator buffers;
//   warps 2-5   epilogue of the other accumulator buffer (as the bf16 GEMM);
//   warps 6-13  decoders: shared-memory stage -> bf16 weights in a ring of TMEM stages.
//               Warp w covers TMEM lanes 32 (w % 4) .. + 31 (its weight rows) and one
//               32-element half of each 64-element k-block.
// Every wait is bounded; on a timeout the CTA winds down and the error word says which
// wait gave up.
//
// Decoding one code c (sign, 4 exponent bits e with bias 7, 3 mantissa bits m): the bf16
// bit pattern sign << 15 | (c & 0x7F) << 4 has exponent field e and mantissa m << 4, so it
// is value(c) * 2^-120 for normal codes (e > 0) and, as a bf16 subnormal, for the
// subnormal codes too (m * 2^-9 * 2^-120).  One bf16 multiply by 2^(s - 7) (exact: a
// power of two) gives value(c) * 2^(s - 127), exactly for every code when s >= 9 (below,
// subnormal codes round to bf16's subnormal grid).  Preconditions: s <= 134 (block scale
// <= 2^7, so the multiplier is a finite bf16), and codes 0x7F / 0xFF (NaN in E4M3) do
// not occur (they would decode as 480 times the scale).
//
// The 4-bit format (FMT_NV4) runs through the same kernel: E2M1 codes (sign, 2 exponent
// bits with bias 1, 1 mantissa bit; two per byte, the lower-indexed element in the low
// nibble), one E4M3 scale per 16 consecutive K elements, and one fp32 scale per weight
// tensor.  Code value times block scale has at most 6 significant bits, so the decoded
// bf16 weight is exact; the tensor scale multiplies the fp32 accumulator in the
// epilogue.  A code's bf16 bytes come from two 8-entry tables by byte permutes, its sign
// is merged with one select, and one bf16 multiply applies the block scale.
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

constexpr int MX_BM = 128;                    // weight rows per tile
constexpr int MX_BK = 64;                     // K elements per k-block
// per format: bytes of one weight tile (128 rows x 64 K) and of its scales
__host__ __device__ constexpr uint32_t mx_a_bytes(int fmt) { return fmt == FMT_NV4 ? MX_BM * MX_BK / 2 : MX_BM * MX_BK; }
__host__ __device__ constexpr uint32_t mx_s_bytes(int fmt) { return fmt == FMT_NV4 ? MX_BM * 4 : MX_BM * 2; }
constexpr int MX_T_STAGES = 4;                // TMEM stages of decoded weights
constexpr int MX_F_STAGES_MAX = 8;
constexpr int MX_DEC_WARPS = 8;
constexpr int MX_DEC_WARP0 = 6;
constexpr int MX_THREADS = 32 * (MX_DEC_WARP0 + MX_DEC_WARPS);
constexpr int MX_B_BOX = 16;
constexpr int MX_B_BOX_BIG = 64;

struct MxTile {
  int g, row0, rows, m;
};

__device__ __forceinline__ int mx_total_items(const TcGemmParams& p) {
  if (p.items) return *p.n_items;
  return (p.n_tokens + p.n_max - 1) / p.n_max;
}

// Grouped: tile t -> (work item t / m_tiles, weight tile t % m_tiles), so the tiles running
// together cover one item's weight rows.  Dense (one weight matrix, tokens in chunks of
// n_max): tile t -> (weight tile t / chunks, token chunk t % chunks), so the CTAs that share
// a weight tile run together and read it from DRAM once between them (L2 serves the rest).
__device__ __forceinline__ MxTile mx_decode_tile(const TcGemmParams& p, int t) {
  MxTile ti;
  if (p.items) {
    const TcWorkItem it = p.items[t / p.m_tiles];
    ti.m = t % p.m_tiles;
    ti.g = it.group;
    ti.row0 = it.row0;
    ti.rows = it.rows;
  } else {
    const int chunks = (p.n_tokens + p.n_max - 1) / p.n_max;
    ti.m = t / chunks;
    ti.g = 0;
    ti.row0 = (t % chunks) * p.n_max;
    ti.rows = min(p.n_max, p.n_tokens - ti.row0);
  }
  return ti;
}

struct MxWalk {
  int t, n_tiles;
  __device__ MxWalk(int n) : t(blockIdx.x), n_tiles(n) {}
  __device__ bool next(int& tile) {
    if (t >= n_tiles) return false;
    tile = t;
    t += gridDim.x;
    return true;
  }
};

__device__ __forceinline__ void mx_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// four codes (code i in byte i) -> two bf16x2 words (codes 0, 1 and codes 2, 3; the
// lower-indexed code in the low half), each value times the multiplier pair mm
__device__ __forceinline__ void mx8_decode4(uint32_t x, uint32_t mm, uint32_t& p01, uint32_t& p23) {
  const uint32_t mag = x & 0x7F7F7F7Fu;
  // bytes 0 and 1 to bits 8..15 and 24..31 (the sign lands on bits 15 and 31)
  const uint32_t s01 = __byte_perm(x, 0u, 0x1404), s23 = __byte_perm(x, 0u, 0x3424);
  const uint32_t m01 = __byte_perm(mag, 0u, 0x1404) >> 4, m23 = __byte_perm(mag, 0u, 0x3424) >> 4;
  p01 = bf16x2_mul((s01 & 0x80008000u) | m01, mm);
  p23 = bf16x2_mul((s23 & 0x80008000u) | m23, mm);
}

// bf16 bytes of the E2M1 magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 (high bytes, then low bytes)
constexpr uint32_t NV4_HI_A = 0x3F3F3F00u, NV4_HI_B = 0x40404040u;
constexpr uint32_t NV4_LO_A = 0xC0800000u, NV4_LO_B = 0xC0804000u;

// eight 4-bit codes (code i in bits 4i .. 4i+3) -> four bf16x2 words (codes 2j, 2j+1 in
// word j, the lower-indexed code in the low half), each value times the multiplier pair mm
__device__ __forceinline__ void nv4_decode8(uint32_t x, uint32_t mm, uint32_t (&w)[4]) {
  const uint32_t mags = x & 0x77777777u;  // table indices (the selector's replicate bits clear)
  const uint32_t h0 = __byte_perm(NV4_HI_A, NV4_HI_B, mags), h1 = __byte_perm(NV4_HI_A, NV4_HI_B, mags >> 16);
  const uint32_t l0 = __byte_perm(NV4_LO_A, NV4_LO_B, mags), l1 = __byte_perm(NV4_LO_A, NV4_LO_B, mags >> 16);
  const uint32_t xs = x << 4;  // byte j of xs carries code 2j's sign in bit 7; byte j of x, code 2j+1's
  const uint32_t m0 = __byte_perm(l0, h0, 0x5140), m1 = __byte_perm(l0, h0, 0x7362);
  const uint32_t m2 = __byte_perm(l1, h1, 0x5140), m3 = __byte_perm(l1, h1, 0x7362);
  w[0] = bf16x2_mul(m0 | (__byte_perm(xs, x, 0x4000) & 0x80008000u), mm);
  w[1] = bf16x2_mul(m1 | (__byte_perm(xs, x, 0x5010) & 0x80008000u), mm);
  w[2] = bf16x2_mul(m2 | (__byte_perm(xs, x, 0x6020) & 0x80008000u), mm);
  w[3] = bf16x2_mul(m3 | (__byte_perm(xs, x, 0x7030) & 0x80008000u), mm);
}

// bf16x2 pair of an E4M3 block scale (non-negative; exact: 4 significant bits, 2^-9..448)
__device__ __forceinline__ uint32_t e4m3_scale_pair(uint32_t sc) {
  const float f = __uint_as_float((sc & 0x7Fu) << 20) * 0x1p120f;  // the f32 bit trick, subnormal codes included
  const uint32_t h = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
  return h | (h << 16);
}

template <int EPI, int FMT>
__global__ void __launch_bounds__(MX_THREADS, 1)
    tc_gemm_lowp_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
                       const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmS2,
                       const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmB2,
                       const __grid_constant__ CUtensorMap tmBb, const __grid_constant__ CUtensorMap tmB2b,
                       const TcGemmParams p, const float g_a, const float g_a2) {
  constexpr uint32_t MX_A_BYTES = mx_a_bytes(FMT), MX_S_BYTES = mx_s_bytes(FMT);
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t f_full[MX_F_STAGES_MAX];   // a stage's TMA loads landed
  __shared__ __align__(8) uint64_t f_empty[MX_F_STAGES_MAX];  // decoders and MMAs are done with it
  __shared__ __align__(8) uint64_t t_full[MX_T_STAGES];       // decoded weights are in TMEM
  __shared__ __align__(8) uint64_t t_empty[MX_T_STAGES];      // the MMAs reading them completed
  __shared__ __align__(8) uint64_t acc_full[2];
  __shared__ __align__(8) uint64_t acc_empty[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int abort_s;
  __shared__ int n_issued_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int terms = p.two_terms ? 2 : 1;
  const int n_a = p.dual_a ? 2 : 1;
  // stage: token tiles (terms x n_max rows x 128 B, 1024-aligned for the 128-byte
  // swizzle), then the 8-bit weight tiles, then their scales
  const uint32_t b_bytes = (uint32_t)p.n_max * 128;
  const uint32_t a_off = (uint32_t)terms * b_bytes;
  const uint32_t s_off = a_off + (uint32_t)n_a * MX_A_BYTES;
  const uint32_t stage_bytes = (s_off + (uint32_t)n_a * MX_S_BYTES + 1023u) & ~1023u;
  int stages = p.smem_budget / (int)stage_bytes;
  if (stages > MX_F_STAGES_MAX) stages = MX_F_STAGES_MAX;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int acc_cols = p.n_max * n_a;
  const uint32_t a_col0 = 2u * (uint32_t)acc_cols;
  const uint32_t a_stage_cols = 32u * (uint32_t)n_a;  // 64 K elements = 32 packed columns per weight tile
  uint32_t tmem_cols = 32;
  while (tmem_cols < a_col0 + MX_T_STAGES * a_stage_cols) tmem_cols <<= 1;
  const int nkb = p.K / MX_BK;

  if (warp == 1) tmem_alloc(&tmem_base_s, tmem_cols);
  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&f_full[s], 1);
      mbar_init(&f_empty[s], MX_DEC_WARPS + 1);
    }
    for (int s = 0; s < MX_T_STAGES; ++s) {
      mbar_init(&t_full[s], MX_DEC_WARPS);
      mbar_init(&t_empty[s], 1);
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
  griddep_sync();  // the work list and the token operand come from the previous kernels
  const int n_tiles = mx_total_items(p) * p.m_tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmS);
      if (p.dual_a) {
        prefetch_tmap(&tmA2);
        prefetch_tmap(&tmS2);
      }
      prefetch_tmap(&tmB);
      prefetch_tmap(&tmBb);
      if (terms == 2) {
        prefetch_tmap(&tmB2);
        prefetch_tmap(&tmB2b);
      }
      int it = 0, t;
      bool ok = true;
      MxWalk walk(n_tiles);
      while (ok && walk.next(t)) {
        const MxTile ti = mx_decode_tile(p, t);
        const int n_pad = (ti.rows + 15) & ~15;
        const uint32_t tx = (uint32_t)terms * (uint32_t)n_pad * 128u + (uint32_t)n_a * (MX_A_BYTES + MX_S_BYTES);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % stages;
          if (!mbar_wait(&f_empty[s], ((uint32_t)(it / stages) & 1u) ^ 1u, &abort_s, p.err,
                         DG_DEVERR_TIMEOUT_EMPTY)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + (size_t)s * stage_bytes;
          const int kbx = (kb + t) % nkb;  // tiles running together start at different k-blocks
          const int kx = kbx * MX_BK;
          // the stage's TMA rules: x coordinates on 16-byte boundaries, every box inside the
          // stage, token rows within the ring's reservation, TMEM stages within the allocation
          if (!DG_GUARD(((FMT == FMT_NV4 ? kx / 2 : kx) % 16 == 0) && ((kx * 2) % 16 == 0) && n_pad <= p.n_max &&
                            s_off + (uint32_t)n_a * MX_S_BYTES <= stage_bytes &&
                            (uint32_t)(s + 1) * stage_bytes <= (uint32_t)p.smem_budget &&
                            a_col0 + MX_T_STAGES * a_stage_cols <= tmem_cols,
                        p.err)) {
            abort_s = 1;
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&f_full[s], tx);
          // codes: x in bytes along K; scales: MX8 (2 rows' bytes, k-block, group),
          // NV4 (16 bytes = 4 rows, rows / 4, group * k-blocks + k-block)
          const int ax = FMT == FMT_NV4 ? kx / 2 : kx;
          const int s0 = FMT == FMT_NV4 ? 0 : ti.m * MX_BM * 2;
          const int s1 = FMT == FMT_NV4 ? ti.m * (MX_BM / 4) : kbx;
          const int s2 = FMT == FMT_NV4 ? ti.g * nkb + kbx : ti.g;
          tma_load_3d(st + a_off, &tmA, ax, ti.m * MX_BM, ti.g, &f_full[s]);
          tma_load_3d(st + s_off, &tmS, s0, s1, s2, &f_full[s]);
          if (p.dual_a) {
            tma_load_3d(st + a_off + MX_A_BYTES, &tmA2, ax, ti.m * MX_BM, ti.g, &f_full[s]);
            tma_load_3d(st + s_off + MX_S_BYTES, &tmS2, s0, s1, s2, &f_full[s]);
          }
          int r = 0;
          for (; r + MX_B_BOX_BIG <= n_pad; r += MX_B_BOX_BIG) {
            tma_load_2d(st + r * 128, &tmBb, kx, ti.row0 + r, &f_full[s]);
            if (terms == 2) tma_load_2d(st + b_bytes + r * 128, &tmB2b, kx, ti.row0 + r, &f_full[s]);
          }
          for (; r < n_pad; r += MX_B_BOX) {
            tma_load_2d(st + r * 128, &tmB, kx, ti.row0 + r, &f_full[s]);
            if (terms == 2) tma_load_2d(st + b_bytes + r * 128, &tmB2, kx, ti.row0 + r, &f_full[s]);
          }
          n_issued_s = it + 1;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: A (decoded weights) from TMEM, B (tokens) from smem
      int it = 0, j = 0, t;
      bool ok = true;
      MxWalk walk(n_tiles);
      for (; ok && walk.next(t); ++j) {
        const MxTile ti = mx_decode_tile(p, t);
        const int n_pad = (ti.rows + 15) & ~15;
        const int buf = j & 1;
        if (!mbar_wait(&acc_empty[buf], ((uint32_t)(j >> 1) & 1u) ^ 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ACCUM))
          break;
        tc_fence_after();
        const uint32_t d0 = tmem + (uint32_t)(buf * acc_cols);
        const uint32_t d1 = d0 + (uint32_t)p.n_max;
        const uint32_t idesc = idesc_bf16_f32(MX_BM, n_pad);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % stages, ts = it % MX_T_STAGES;
          if (!mbar_wait(&t_full[ts], (uint32_t)(it / MX_T_STAGES) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_FULL) ||
              !mbar_wait(&f_full[s], (uint32_t)(it / stages) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sb = smem_u32(smem + (size_t)s * stage_bytes);
          const uint32_t a0 = tmem + a_col0 + (uint32_t)ts * a_stage_cols;
#pragma unroll
          for (int kk = 0; kk < MX_BK / 16; ++kk) {
            const uint32_t acc = (kb != 0 || kk != 0) ? 1u : 0u;
            const uint64_t bd = sw128_kmajor_desc(sb + kk * 32);
            const uint64_t bd2 = sw128_kmajor_desc(sb + b_bytes + kk * 32);
            const uint32_t ak = a0 + (uint32_t)kk * 8u;  // 16 K elements = 8 packed columns
            mx_mma_ts(d0, ak, bd, idesc, acc);
            if (terms == 2) mx_mma_ts(d0, ak, bd2, idesc, 1u);
            if (p.dual_a) {
              mx_mma_ts(d1, ak + 32u, bd, idesc, acc);
              if (terms == 2) mx_mma_ts(d1, ak + 32u, bd2, idesc, 1u);
            }
          }
          tc_commit(&t_empty[ts]);
          tc_commit(&f_empty[s]);
        }
        if (ok) tc_commit(&acc_full[buf]);
      }
      tc_commit(&drain_bar);  // completes once every MMA issued above has landed
    }
  } else if (warp < MX_DEC_WARP0) {
    // ---------------- epilogue warps 2..5: TMEM lanes (warp % 4) * 32 .. + 31
    const int lg = warp & 3;
    const int row = lg * 32 + lane;
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    int j = 0, t;
    MxWalk walk(n_tiles);
    for (; walk.next(t); ++j) {
      const MxTile ti = mx_decode_tile(p, t);
      const int n_pad = (ti.rows + 15) & ~15;
      const int buf = j & 1;
      // each wait's outcome is made warp-uniform: the tcgen05.ld below is warp-collective
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&acc_full[buf], (uint32_t)(j >> 1) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ACCUM)))
        break;
      tc_fence_after();
      const uint32_t t0 = tmem + (uint32_t)(buf * acc_cols) + lane_off;
      const int f = ti.m * MX_BM + row;  // weight row = output feature
      const bool fvalid = f < p.a_rows_per_group;
      for (int c0 = 0; c0 < n_pad; c0 += 16) {
        uint32_t ra[16], rb[16];
        tmem_ld16(t0 + c0, ra);
        if (EPI == EPI_SWIGLU_BF16) tmem_ld16(t0 + p.n_max + c0, rb);
        tc_wait_ld();
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int col = c0 + q;
          float a = __uint_as_float(ra[q]);
          float b = EPI == EPI_SWIGLU_BF16 ? __uint_as_float(rb[q]) : 0.0f;
          if (FMT == FMT_NV4) {  // the tensor scales
            a *= g_a;
            b *= g_a2;
          }
          if (!fvalid || col >= ti.rows) continue;
          const size_t o = (size_t)(ti.row0 + col) * p.ld_out + f;
          if (!DG_GUARD(ti.row0 + col < p.n_tokens && f < p.ld_out && c0 + q < n_pad, p.err)) continue;
          if (EPI == EPI_STORE_F32) {
            reinterpret_cast<float*>(p.out)[o] = a;
          } else {
            const float hv = a / (1.0f + expf(-a)) * b;
            const bf16 hi = __float2bfloat16_rn(hv);
            reinterpret_cast<bf16*>(p.out)[o] = hi;
            if (p.out_lo) reinterpret_cast<bf16*>(p.out_lo)[o] = __float2bfloat16_rn(hv - __bfloat162float(hi));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  } else {
    // ---------------- decoders: rows 32 (warp % 4) + lane, K half (warp - 6) / 4 of each k-block
    const int lq = warp & 3;
    const int half = (warp - MX_DEC_WARP0) >> 2;
    const int row = lq * 32 + lane;
    const uint32_t lane_off = (uint32_t)(lq * 32) << 16;
    // 16-byte chunk c of the row sits at c ^ swz: MX8 rows of 64 bytes, 64-byte swizzle;
    // NV4 rows of 32 bytes, 32-byte swizzle
    const int swz = FMT == FMT_NV4 ? (row >> 2) & 1 : (row >> 1) & 3;
    constexpr int row_bytes = FMT == FMT_NV4 ? MX_BK / 2 : MX_BK;
    int it = 0, t;
    bool ok = true;
    MxWalk walk(n_tiles);
    while (ok && walk.next(t)) {
      for (int kb = 0; kb < nkb; ++kb, ++it) {
        const int s = it % stages, ts = it % MX_T_STAGES;
        const bool got =
            mbar_wait(&f_full[s], (uint32_t)(it / stages) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_FULL) &&
            mbar_wait(&t_empty[ts], ((uint32_t)(it / MX_T_STAGES) & 1u) ^ 1u, &abort_s, p.err,
                      DG_DEVERR_TIMEOUT_EMPTY);
        if (!__all_sync(0xffffffffu, got)) {  // the tcgen05.st below is warp-collective
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* st = smem + (size_t)s * stage_bytes;
        const bool in_bounds = DG_GUARD(
            (uint32_t)row * row_bytes + row_bytes <= MX_A_BYTES / MX_BM * MX_BM && row < MX_BM &&
                a_col0 + (uint32_t)(ts + 1) * a_stage_cols <= tmem_cols,
            p.err);
        for (int a = 0; a < n_a && in_bounds; ++a) {
          const uint8_t* codes = st + a_off + (uint32_t)a * MX_A_BYTES + row * row_bytes;
          uint32_t w[16];
          if (FMT == FMT_NV4) {
            // 32 codes = one 16-byte chunk; block scales 2 half and 2 half + 1 (16 elements each)
            const uint8_t* sc = st + s_off + (uint32_t)a * MX_S_BYTES + row * 4 + 2 * half;
            const uint32_t mm0 = e4m3_scale_pair(sc[0]), mm1 = e4m3_scale_pair(sc[1]);
            const uint4 v = *reinterpret_cast<const uint4*>(codes + ((half ^ swz) << 4));
            uint32_t q[4];
            nv4_decode8(v.x, mm0, q);
            w[0] = q[0], w[1] = q[1], w[2] = q[2], w[3] = q[3];
            nv4_decode8(v.y, mm0, q);
            w[4] = q[0], w[5] = q[1], w[6] = q[2], w[7] = q[3];
            nv4_decode8(v.z, mm1, q);
            w[8] = q[0], w[9] = q[1], w[10] = q[2], w[11] = q[3];
            nv4_decode8(v.w, mm1, q);
            w[12] = q[0], w[13] = q[1], w[14] = q[2], w[15] = q[3];
          } else {
            const uint32_t e8 = st[s_off + (uint32_t)a * MX_S_BYTES + row * 2 + half];
            const uint32_t mh = (e8 + 120u) << 7;  // bf16 bits of 2^(e8 - 7)
            const uint32_t mm = mh | (mh << 16);
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
              const int c = 2 * half + c2;
              const uint4 v = *reinterpret_cast<const uint4*>(codes + ((c ^ swz) << 4));
              mx8_decode4(v.x, mm, w[c2 * 8 + 0], w[c2 * 8 + 1]);
              mx8_decode4(v.y, mm, w[c2 * 8 + 2], w[c2 * 8 + 3]);
              mx8_decode4(v.z, mm, w[c2 * 8 + 4], w[c2 * 8 + 5]);
              mx8_decode4(v.w, mm, w[c2 * 8 + 6], w[c2 * 8 + 7]);
            }
          }
          tmem_st16(tmem + lane_off + a_col0 + (uint32_t)ts * a_stage_cols + (uint32_t)a * 32u + (uint32_t)half * 16u,
                    w);
        }
        tc_wait_st();
        __syncwarp();
        if (lane == 0) mbar_arrive(&f_empty[s]);  // this warp's reads of the stage are done
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&t_full[ts]);
      }
    }
  }

  __syncthreads();
  if (abort_s && tid == 0) {
    // wind down: let the most recent load of every stage land before the smem goes away
    const int first = n_issued_s > stages ? n_issued_s - stages : 0;
    for (int i = first; i < n_issued_s; ++i) mbar_wait_drain(&f_full[i % stages], (uint32_t)(i / stages) & 1u);
  }
  if (tid == 32) mbar_wait_drain(&drain_bar, 0);  // every issued MMA has landed
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, tmem_cols);
}

template <int FMT>
static cudaError_t launch_fmt(int epi, const CUtensorMap& A, const CUtensorMap& A2, const CUtensorMap& S,
                              const CUtensorMap& S2, const CUtensorMap& B, const CUtensorMap& B2,
                              const CUtensorMap& Bb, const CUtensorMap& B2b, const TcGemmParams& p, float g_a,
                              float g_a2, int grid, int smem, cudaStream_t st) {
  cudaError_t e;
  if (epi == EPI_STORE_F32) {
    e = cudaFuncSetAttribute(tc_gemm_lowp_kernel<EPI_STORE_F32, FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem);
    if (e != cudaSuccess) return e;
    return launch_k(tc_gemm_lowp_kernel<EPI_STORE_F32, FMT>, dim3(grid), dim3(MX_THREADS), smem, st, A, A2, S, S2, B,
                    B2, Bb, B2b, p, g_a, g_a2);
  }
  if (epi == EPI_SWIGLU_BF16) {
    e = cudaFuncSetAttribute(tc_gemm_lowp_kernel<EPI_SWIGLU_BF16, FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem);
    if (e != cudaSuccess) return e;
    return launch_k(tc_gemm_lowp_kernel<EPI_SWIGLU_BF16, FMT>, dim3(grid), dim3(MX_THREADS), smem, st, A, A2, S, S2,
                    B, B2, Bb, B2b, p, g_a, g_a2);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_tc_gemm_lowp(int fmt, int epi, const CUtensorMap& A, const CUtensorMap& A2, const CUtensorMap& S,
                                const CUtensorMap& S2, const CUtensorMap& B, const CUtensorMap& B2,
                                const CUtensorMap& Bb, const CUtensorMap& B2b, const TcGemmParams& p, float g_a,
                                float g_a2, int max_tiles, cudaStream_t st) {
  if (max_tiles <= 0) return cudaSuccess;
  // TMEM: two accumulators of n_max columns per weight matrix and four decoded stages of 32
  // columns per matrix fit 512 columns for n_max <= 64 with two matrices, <= 128 with one
  if ((fmt != FMT_MX8 && fmt != FMT_NV4) || p.k_splits != 1 || p.K % MX_BK != 0 || p.K <= 0 || p.n_max < 16 ||
      p.n_max > (p.dual_a ? 64 : 128) || (p.n_max % 16) != 0 || p.m_tiles < 1 ||
      (epi == EPI_SWIGLU_BF16) != (p.dual_a != 0))
    return cudaErrorInvalidValue;
  const int n_a = p.dual_a ? 2 : 1;
  const int terms = p.two_terms ? 2 : 1;
  const int stage = ((terms * p.n_max * 128 + n_a * (int)(mx_a_bytes(fmt) + mx_s_bytes(fmt))) + 1023) & ~1023;
  if (p.smem_budget < 2 * stage) return cudaErrorInvalidValue;
  const int smem = p.smem_budget + 1024;
  const int sms = num_sms();
  const int grid = max_tiles < sms ? max_tiles : sms;
  return fmt == FMT_NV4 ? launch_fmt<FMT_NV4>(epi, A, A2, S, S2, B, B2, Bb, B2b, p, g_a, g_a2, grid, smem, st)
                        : launch_fmt<FMT_MX8>(epi, A, A2, S, S2, B, B2, Bb, B2b, p, g_a, g_a2, grid, smem, st);
}

cudaError_t set_wait_limit_gemm_lowp(uint64_t ns) { return set_wait_limit_this_file(ns); }

}  // namespace dg
