// Split-KV merge inside the attention kernels, by the last split of a (query tile, head
// group) to finish: every split writes its partial output (already divided by its row
// sum) and its log2-sum-exp, then takes a ticket; the split whose ticket comes last
// combines all of them (weights 2^(lse_s - max), in split order) into the bf16 hi + lo
// output and resets the ticket for the next launch.  Block-wide; called by every CTA of
// the grid as it leaves.
#pragma once
#include <cuda_bf16.h>
#include <math.h>

#include "dg_kernels.h"

namespace dg {

constexpr int MG_BQ = 128;  // query rows per tile
constexpr int MG_D = 128;   // head dimension

// heads h0 .. h0 + nh - 1 of query tile qt; the ticket is p.merge_cnt[qt * p.nq + h0]
__device__ __forceinline__ void merge_splits_if_last(const TcAttnParams& p, int qt, int h0, int nh) {
  __shared__ int last_s;
  __threadfence();  // this CTA's partials are visible device-wide before its ticket
  __syncthreads();
  if (threadIdx.x == 0) last_s = atomicAdd(&p.merge_cnt[qt * p.nq + h0], 1) == p.n_splits - 1;
  __syncthreads();
  if (!last_s) return;
  __threadfence();
  const int q_row0 = qt * MG_BQ;
  const int rows = min(MG_BQ, p.n_q - q_row0);
  for (int idx = threadIdx.x; idx < nh * rows * (MG_D / 4); idx += blockDim.x) {
    const int h = h0 + idx / (rows * (MG_D / 4));
    const int rem = idx % (rows * (MG_D / 4));
    const int row = q_row0 + rem / (MG_D / 4), c4 = rem % (MG_D / 4);
    float mx = -INFINITY;
    for (int sp = 0; sp < p.n_splits; ++sp) mx = fmaxf(mx, __ldcg(&p.part_lse[((size_t)sp * p.nq + h) * p.n_q + row]));
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    float den = 0.0f;
    if (mx != -INFINITY) {
      for (int sp = 0; sp < p.n_splits; ++sp) {
        const float lse = __ldcg(&p.part_lse[((size_t)sp * p.nq + h) * p.n_q + row]);
        if (lse == -INFINITY) continue;
        const float w = exp2f(lse - mx);
        const float4 o =
            __ldcg(reinterpret_cast<const float4*>(p.part_o + (((size_t)sp * p.nq + h) * p.n_q + row) * MG_D) + c4);
        num.x += w * o.x;
        num.y += w * o.y;
        num.z += w * o.z;
        num.w += w * o.w;
        den += w;
      }
    }
    const float v[4] = {den > 0.f ? num.x / den : 0.f, den > 0.f ? num.y / den : 0.f, den > 0.f ? num.z / den : 0.f,
                        den > 0.f ? num.w / den : 0.f};
    uint32_t w[2], wl[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const __nv_bfloat162 hi = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
      const __nv_bfloat162 lo = __floats2bfloat162_rn(v[2 * e] - __low2float(hi), v[2 * e + 1] - __high2float(hi));
      w[e] = *reinterpret_cast<const uint32_t*>(&hi);
      wl[e] = *reinterpret_cast<const uint32_t*>(&lo);
    }
    const size_t o = (size_t)row * p.nq * MG_D + (size_t)h * MG_D + 4 * c4;
    *reinterpret_cast<uint2*>(p.out + o) = make_uint2(w[0], w[1]);
    if (p.out_lo) *reinterpret_cast<uint2*>(p.out_lo + o) = make_uint2(wl[0], wl[1]);
  }
  if (threadIdx.x == 0) p.merge_cnt[qt * p.nq + h0] = 0;  // ready for the next launch
}

}  // namespace dg
