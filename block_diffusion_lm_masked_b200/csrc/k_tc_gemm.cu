// Persistent tcgen05 / TMEM / TMA GEMM for every dense contraction of the bf16 pass:
// the QKV and output projections, the two grouped expert GEMMs and the vocabulary
// projection.  All of them stream a weight matrix once while the token operand is
// small, so weights sit on the 128-row M side of the MMA and tokens on N: a tile is
// 128 weight rows x (up to n_max) token rows.
//
// One CTA per SM walks its share of the tiles (TileWalk: rounds of gridDim.x).  Roles
// (192 threads): warp 0 issues TMA loads into a ring of smem stages; warp 1 owns
// the TMEM allocation and issues tcgen05.mma into one of two accumulator buffers;
// warps 2-5 drain the other buffer through the epilogue, so the loads and MMAs of
// tile i+1 overlap the epilogue of tile i.  Every wait is bounded.
//
// Options: two_terms (tokens given as bf16 hi + lo, both accumulated: fp32-precision
// activations against bf16 weights; where a tile's padded token rows fit twice in its
// accumulator -- the expert tiles, 16-64 rows against 128 columns -- one MMA of N = 2 x rows
// takes the hi rows and the lo rows, which sit back to back in shared memory, into two
// column ranges that the epilogue adds: an MMA instruction costs about the same for any
// N up to 128 (measured: 96 cycles), so the small tiles issue half the instructions); dual_a (gate and up weight tiles accumulated
// into two TMEM regions, SwiGLU epilogue); m_pair (a tile is two consecutive 128-row
// weight tiles of one matrix sharing each token load: the dense projections, whose
// token operand is re-read once per weight tile, read it half as often); k_splits
// (split-K, one output slab per split).  Two accumulator buffers when they fit in the 512
// TMEM columns, else one (the loads of the next tile still run during the epilogue).
//
// Each tile starts its K walk at a different k-block (tile index mod k-blocks): tiles
// that run at the same time then read different k-blocks of the token operand, which
// all of them share, instead of hammering the same L2 lines in lockstep.
//
// The shared memory holds a ring of variable-size k-block buffers (KbRing): a k-block
// takes its weight boxes (16 KB each) and its token boxes of the tile's own padded row
// count, contiguously, so that an expert tile of 16 token rows takes 36 KB instead of a
// stage sized for the largest tile (64 KB): more weight bytes are in flight per SM when
// the tiles are small.  Up to 16 k-blocks are in flight, one pair of barriers each.
//
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

constexpr int TC_BM = 128;
constexpr int TC_BK = 64;
constexpr int TC_B_BOX = 16;      // token rows per small TMA box
constexpr int TC_B_BOX_BIG = 64;  // token rows per large TMA box
constexpr int TC_MAX_STAGES = 16;  // k-blocks in flight at most (barrier pairs)
constexpr int TC_THREADS = 192;

// The k-block buffers' offsets in the ring, in the order both the producer and the MMA
// warp walk the k-blocks: a buffer starts where the previous one ended, or at 0 when it
// would run past the end (the skipped tail then counts in its footprint).  Buffers are
// released in allocation order, so the bytes in use are the footprints of the k-blocks in
// flight, and a new buffer overlaps none of them exactly when that sum stays within the
// ring.  Sizes are multiples of 2 KB, so every buffer (and each box in it) starts on a
// 1024-byte swizzle atom.
struct KbRing {
  uint32_t cap, head;
  __device__ explicit KbRing(uint32_t c) : cap(c), head(0) {}
  __device__ uint32_t take(uint32_t bytes, uint32_t* foot) {
    if (head + bytes > cap) {
      *foot = cap - head + bytes;
      head = bytes;
      return 0u;
    }
    *foot = bytes;
    head += bytes;
    return head - bytes;
  }
};

struct TileInfo {
  int g, row0, rows, split, m;
};

__device__ __forceinline__ int total_items(const TcGemmParams& p) {
  if (p.items) return *p.n_items;
  const int chunks = (p.n_tokens + p.n_max - 1) / p.n_max;
  return chunks * p.k_splits;
}

// tile t -> (work item t / m_tiles, weight tile t % m_tiles)
__device__ __forceinline__ TileInfo decode_tile(const TcGemmParams& p, int t) {
  TileInfo ti;
  const int item = t / p.m_tiles;
  ti.m = t % p.m_tiles;
  if (p.items) {
    const TcWorkItem it = p.items[item];
    ti.g = it.group;
    ti.row0 = it.row0;
    ti.rows = it.rows;
    ti.split = 0;
  } else {
    const int chunk = item / p.k_splits;
    ti.split = item % p.k_splits;
    ti.g = 0;
    ti.row0 = chunk * p.n_max;
    ti.rows = min(p.n_max, p.n_tokens - ti.row0);
  }
  return ti;
}

// This CTA's tiles.  The tiles are dealt to the CTAs in rounds of gridDim.x, every other
// round in reverse CTA order (a serpentine), from a list with the whole weight tiles
// first and, when the weight rows are not a multiple of 128 (the expert FFN of 704
// rows), each work item's partial last weight tile at the end: the partial tiles, which
// stream fewer weight bytes, then even out the last rounds.  At the large model's
// gate/up GEMM (128 items x 5.5 weight tiles) the busiest CTA streams 5 tiles' weights
// instead of 6.
struct TileWalk {
  int r, n_tiles, m_tiles, full;
  __device__ TileWalk(const TcGemmParams& p, int n_tiles_) : r(0), n_tiles(n_tiles_), m_tiles(p.m_tiles) {
    const bool partial = p.m_tiles > 1 && p.a_rows_per_group % (p.m_pair ? 2 * TC_BM : TC_BM) != 0;
    full = partial ? n_tiles - n_tiles / p.m_tiles : n_tiles;
  }
  // the k-th tile of the list -> tile index (work item * m_tiles + weight tile)
  __device__ int order(int k) const {
    if (full == n_tiles) return k;
    if (k < full) return (k / (m_tiles - 1)) * m_tiles + k % (m_tiles - 1);
    return (k - full) * m_tiles + (m_tiles - 1);
  }
  __device__ bool next(int& tile) {
    while ((long long)r * gridDim.x < n_tiles) {
      const int c = (r & 1) ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x;
      const long long k = (long long)r * gridDim.x + c;
      ++r;
      if (k < n_tiles) {
        tile = order((int)k);
        return true;
      }
    }
    return false;
  }
};

template <int EPI>
__global__ void __launch_bounds__(TC_THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
                   const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmB2,
                   const __grid_constant__ CUtensorMap tmBb, const __grid_constant__ CUtensorMap tmB2b,
                   const TcGemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[TC_MAX_STAGES];
  __shared__ __align__(8) uint64_t empty_bar[TC_MAX_STAGES];
  __shared__ __align__(8) uint64_t acc_full[2];
  __shared__ __align__(8) uint64_t acc_empty[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int abort_s;
  __shared__ int n_issued_s, n_consumed_s;
  __shared__ uint32_t kb_foot[TC_MAX_STAGES];  // ring footprint of each k-block in flight (producer only)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int terms = p.two_terms ? 2 : 1;
  const int n_a = (p.dual_a || p.m_pair) ? 2 : 1;
  const uint32_t a_bytes = TC_BM * TC_BK * 2;  // one weight tile per k-block
  // a k-block buffer of a tile with n_pad token rows: weight boxes, then each token term
  auto kb_bytes = [&](int n_pad) { return n_a * a_bytes + (uint32_t)(terms * n_pad * 128); };
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int acc_cols = p.n_max * n_a;  // one accumulator buffer
  const int nbuf = 2 * acc_cols <= 512 ? 2 : 1;
  uint32_t tmem_cols = 32;
  while (tmem_cols < (uint32_t)(nbuf * acc_cols)) tmem_cols <<= 1;
  const int rows_per_tile = p.m_pair ? 2 * TC_BM : TC_BM;  // weight rows of one tile
  const int nkb = p.K / TC_BK / p.k_splits;

  if (warp == 1) tmem_alloc(&tmem_base_s, tmem_cols);
  if (tid == 0) {
    for (int s = 0; s < TC_MAX_STAGES; ++s) {
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
    n_consumed_s = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  griddep_sync();  // the work list and the token operand come from the previous kernels
  const int n_tiles = total_items(p) * p.m_tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      prefetch_tmap(&tmA);
      if (p.dual_a) prefetch_tmap(&tmA2);
      prefetch_tmap(&tmB);
      prefetch_tmap(&tmBb);
      if (terms == 2) {
        prefetch_tmap(&tmB2);
        prefetch_tmap(&tmB2b);
      }
      int it = 0, t;
      int released = 0;     // k-blocks whose buffers the MMAs have released (in order)
      uint32_t in_use = 0;  // ring bytes of the k-blocks released .. it - 1 (footprints)
      bool ok = true;
      KbRing ring((uint32_t)p.smem_budget);
      TileWalk walk(p, n_tiles);
      while (ok && walk.next(t)) {
        const TileInfo ti = decode_tile(p, t);
        const int n_pad = (ti.rows + 15) & ~15;
        const uint32_t tx = kb_bytes(n_pad);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % TC_MAX_STAGES;
          uint32_t foot;
          const uint32_t off = ring.take(tx, &foot);
          in_use += foot;
          // wait for the oldest k-blocks until this buffer fits beside those still in flight
          // and fewer than TC_MAX_STAGES are in flight
          while (released < it && (in_use > (uint32_t)p.smem_budget || it - released >= TC_MAX_STAGES)) {
            if (!mbar_wait(&empty_bar[released % TC_MAX_STAGES], (uint32_t)(released / TC_MAX_STAGES) & 1u, &abort_s,
                           p.err, DG_DEVERR_TIMEOUT_EMPTY)) {
              ok = false;
              break;
            }
            in_use -= kb_foot[released % TC_MAX_STAGES];
            ++released;
          }
          if (!ok) break;
          kb_foot[s] = foot;
          uint8_t* sa = smem + off;
          uint8_t* sb = sa + n_a * a_bytes;
          const int kx = (ti.split * nkb + (kb + t) % nkb) * TC_BK;
          mbar_arrive_expect_tx(&full_bar[s], tx);
          const int arow = ti.m * rows_per_tile;
          tma_load_3d(sa, &tmA, kx, arow, ti.g, &full_bar[s]);
          if (p.dual_a) tma_load_3d(sa + a_bytes, &tmA2, kx, arow, ti.g, &full_bar[s]);
          if (p.m_pair) tma_load_3d(sa + a_bytes, &tmA, kx, arow + TC_BM, ti.g, &full_bar[s]);
          int r = 0;
          for (; r + TC_B_BOX_BIG <= n_pad; r += TC_B_BOX_BIG) {
            tma_load_2d(sb + r * 128, &tmBb, kx, ti.row0 + r, &full_bar[s]);
            if (terms == 2) tma_load_2d(sb + n_pad * 128 + r * 128, &tmB2b, kx, ti.row0 + r, &full_bar[s]);
          }
          for (; r < n_pad; r += TC_B_BOX) {
            tma_load_2d(sb + r * 128, &tmB, kx, ti.row0 + r, &full_bar[s]);
            if (terms == 2) tma_load_2d(sb + n_pad * 128 + r * 128, &tmB2, kx, ti.row0 + r, &full_bar[s]);
          }
          n_issued_s = it + 1;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      int it = 0, j = 0, t;
      bool ok = true;
      KbRing ring((uint32_t)p.smem_budget);
      TileWalk walk(p, n_tiles);
      for (; ok && walk.next(t); ++j) {
        const TileInfo ti = decode_tile(p, t);
        const int n_pad = (ti.rows + 15) & ~15;
        const int buf = j % nbuf;
        if (!mbar_wait(&acc_empty[buf], ((uint32_t)(j / nbuf) & 1u) ^ 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_ACCUM))
          break;
        tc_fence_after();
        const uint32_t d0 = tmem + (uint32_t)(buf * acc_cols);
        const uint32_t d1 = d0 + (uint32_t)p.n_max;
        // both token terms in one MMA (columns 0 .. n_pad - 1: hi, n_pad .. 2 n_pad - 1: lo)
        const bool fuse = terms == 2 && 2 * n_pad <= p.n_max;
        const uint32_t idesc = idesc_bf16_f32(TC_BM, fuse ? 2 * n_pad : n_pad);
        const uint32_t tx = kb_bytes(n_pad);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % TC_MAX_STAGES;
          uint32_t foot;
          const uint32_t off = ring.take(tx, &foot);
          if (!mbar_wait(&full_bar[s], (uint32_t)(it / TC_MAX_STAGES) & 1u, &abort_s, p.err, DG_DEVERR_TIMEOUT_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + off);
          const uint32_t sb = sa + n_a * a_bytes;
#pragma unroll
          for (int kk = 0; kk < TC_BK / 16; ++kk) {
            const uint32_t acc = (kb != 0 || kk != 0) ? 1u : 0u;
            const uint64_t ad = sw128_kmajor_desc(sa + kk * 32);
            const uint64_t bd = sw128_kmajor_desc(sb + kk * 32);
            const uint64_t bd2 = sw128_kmajor_desc(sb + (uint32_t)n_pad * 128 + kk * 32);
            tc_mma(d0, ad, bd, idesc, acc);
            if (terms == 2 && !fuse) tc_mma(d0, ad, bd2, idesc, 1u);
            if (n_a == 2) {
              const uint64_t ad2 = sw128_kmajor_desc(sa + a_bytes + kk * 32);
              tc_mma(d1, ad2, bd, idesc, acc);
              if (terms == 2 && !fuse) tc_mma(d1, ad2, bd2, idesc, 1u);
            }
          }
          tc_commit(&empty_bar[s]);
          n_consumed_s = it + 1;
        }
        if (ok) tc_commit(&acc_full[buf]);
      }
      tc_commit(&drain_bar);  // completes once every MMA issued above has landed
    }
  } else {
    // ---------------- epilogue warps 2..5: TMEM lanes (warp % 4) * 32 .. + 31
    const int lg = warp & 3;
    const int row = lg * 32 + lane;  // row of the 128-row tile this thread drains
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    int j = 0, t;
    TileWalk walk(p, n_tiles);
    for (; walk.next(t); ++j) {
      const TileInfo ti = decode_tile(p, t);
      const int n_pad = (ti.rows + 15) & ~15;
      const int buf = j % nbuf;
      const bool fuse = terms == 2 && 2 * n_pad <= p.n_max;  // the lo term's columns follow the hi term's
      // the warp votes on the wait's outcome: tcgen05.ld below is warp-collective, so no lane
      // may go on alone after another gave up
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (uint32_t)(j / nbuf) & 1u, &abort_s, p.err,
                                             DG_DEVERR_TIMEOUT_ACCUM)))
        break;
      tc_fence_after();
      // paired weight tiles: the second accumulator holds weight rows 128 .. 255 of the tile
      for (int half = 0; half < (p.m_pair ? 2 : 1); ++half) {
        const uint32_t t0 = tmem + (uint32_t)(buf * acc_cols + half * p.n_max) + lane_off;
        const int f = ti.m * rows_per_tile + half * TC_BM + row;  // weight row = output feature
        const bool fvalid = f < p.a_rows_per_group;
        for (int c0 = 0; c0 < n_pad; c0 += 16) {
          uint32_t ra[16], rb[16], ra2[16], rb2[16];
          tmem_ld16(t0 + c0, ra);
          if (EPI == EPI_SWIGLU_BF16) tmem_ld16(t0 + p.n_max + c0, rb);
          if (fuse) {
            tmem_ld16(t0 + n_pad + c0, ra2);
            if (EPI == EPI_SWIGLU_BF16) tmem_ld16(t0 + p.n_max + n_pad + c0, rb2);
          }
          tc_wait_ld();
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int col = c0 + q;
            const float a = __uint_as_float(ra[q]) + (fuse ? __uint_as_float(ra2[q]) : 0.0f);
            const float b = EPI == EPI_SWIGLU_BF16 ? __uint_as_float(rb[q]) + (fuse ? __uint_as_float(rb2[q]) : 0.0f)
                                                   : 0.0f;
            if (!fvalid || col >= ti.rows) continue;
            const size_t o = (size_t)(ti.row0 + col) * p.ld_out + f;
            if (EPI == EPI_STORE_F32) {
              reinterpret_cast<float*>(p.out)[(size_t)ti.split * p.split_stride + o] = a;
            } else {
              const float hv = a / (1.0f + expf(-a)) * b;
              const bf16 hi = __float2bfloat16_rn(hv);
              reinterpret_cast<bf16*>(p.out)[o] = hi;
              if (p.out_lo) reinterpret_cast<bf16*>(p.out_lo)[o] = __float2bfloat16_rn(hv - __bfloat162float(hi));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }

  __syncthreads();
  if (abort_s && tid == 0) {
    // wind down: let issued loads land before the smem goes away
    for (int i = n_consumed_s; i < n_issued_s; ++i)
      mbar_wait_drain(&full_bar[i % TC_MAX_STAGES], (uint32_t)(i / TC_MAX_STAGES) & 1u);
  }
  if (tid == 32) mbar_wait_drain(&drain_bar, 0);  // every issued MMA has landed
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, tmem_cols);
}

// ---------------------------------------------------------------- work items of a grouped GEMM
// For each group g with rows [off[g], off[g+1]): items of at most n_max rows, in group
// order.  Written by one thread (E is small).  Offsets that decrease or leave [0, rows]
// are an input error: no item is emitted and the error word records DG_DEVERR_BAD_COUNT.
static __device__ void emit_work_items(const int32_t* off, int E, int n_max, int rows, TcWorkItem* items,
                                       int* n_items, int* err) {
  for (int e = 0; e < E; ++e) {
    if (off[e] < 0 || off[e + 1] < off[e] || off[e + 1] > rows) {
      atomicCAS(err, 0, DG_DEVERR_BAD_COUNT);
      *n_items = 0;
      return;
    }
  }
  int ni = 0;
  for (int e = 0; e < E; ++e) {
    const int c = off[e + 1] - off[e];
    for (int r = 0; r < c; r += n_max) {
      TcWorkItem it;
      it.group = e;
      it.row0 = off[e] + r;
      it.rows = min(n_max, c - r);
      it.pad = 0;
      items[ni++] = it;
    }
  }
  *n_items = ni;
}

__global__ void build_items_kernel(const int32_t* off, int E, int n_max, int rows, TcWorkItem* items, int* n_items,
                                   int* err) {
  griddep_sync();
  if (threadIdx.x == 0 && blockIdx.x == 0) emit_work_items(off, E, n_max, rows, items, n_items, err);
}

cudaError_t launch_build_items(const int32_t* off, int E, int n_max, int rows, TcWorkItem* items, int* n_items,
                               int* err, cudaStream_t st) {
  return launch_k(build_items_kernel, dim3(1), dim3(32), 0, st, off, E, n_max, rows, items, n_items, err);
}

static int g_num_sms = 0;

int num_sms() {
  if (g_num_sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      g_num_sms = 148;
  }
  return g_num_sms;
}

cudaError_t launch_tc_gemm(int epi, const CUtensorMap& A, const CUtensorMap& A2, const CUtensorMap& B,
                           const CUtensorMap& B2, const CUtensorMap& Bb, const CUtensorMap& B2b, const TcGemmParams& p,
                           int max_tiles, cudaStream_t st) {
  if (max_tiles <= 0) return cudaSuccess;
  if (p.k_splits < 1 || (p.K / TC_BK) % p.k_splits != 0 || (p.k_splits > 1 && p.items) || p.n_max < 16 ||
      p.n_max > 256 || (p.n_max % 16) != 0 || p.m_tiles < 1)
    return cudaErrorInvalidValue;
  const int n_a = (p.dual_a || p.m_pair) ? 2 : 1;
  const int stage = n_a * TC_BM * TC_BK * 2 + (p.two_terms ? 2 : 1) * p.n_max * 128;  // the largest k-block
  if (p.smem_budget < stage || p.smem_budget % 2048 != 0 || p.n_max * n_a > 512 || (epi == EPI_SWIGLU_BF16) != (p.dual_a != 0) ||
      (p.m_pair && (p.dual_a || epi != EPI_STORE_F32)))
    return cudaErrorInvalidValue;
  const int smem = p.smem_budget + 1024;
  const int sms = num_sms();
  const int grid = max_tiles < sms ? max_tiles : sms;
  cudaError_t e;
  switch (epi) {
    case EPI_STORE_F32:
      e = cudaFuncSetAttribute(tc_gemm_kernel<EPI_STORE_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      return launch_k(tc_gemm_kernel<EPI_STORE_F32>, dim3(grid), dim3(TC_THREADS), smem, st, A, A2, B, B2, Bb,
                      B2b, p);
    case EPI_SWIGLU_BF16:
      e = cudaFuncSetAttribute(tc_gemm_kernel<EPI_SWIGLU_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      return launch_k(tc_gemm_kernel<EPI_SWIGLU_BF16>, dim3(grid), dim3(TC_THREADS), smem, st, A, A2, B, B2, Bb,
                      B2b, p);
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t set_wait_limit_gemm(uint64_t ns) { return set_wait_limit_this_file(ns); }

}  // namespace dg
