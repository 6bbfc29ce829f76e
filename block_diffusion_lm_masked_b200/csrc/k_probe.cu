// Tensor-pipe rate probe: the rate at which one SM's tensor core completes tcgen05 MMA
// instructions of the shapes the pass issues, with nothing else running.  The attention
// kernel's roofline reading rests on it: its instructions are 128 x 128 x 16, and the
// probe shows what such instructions complete at on this part.
//
// One CTA per SM (launch bounds 1, 100 KB of shared memory, 512 TMEM columns): warp 0
// allocates TMEM, all threads zero the operands, then one thread issues `count` MMAs of
// 128 x n x 16 (bf16 inputs, fp32 accumulation into TMEM columns 0 .. n - 1) back to back
// -- A from shared memory, or from TMEM columns 256 .. 287 when a_tmem is set; B from
// shared memory, 128-byte swizzled K-major -- commits, and waits with a bounded wait.
// Block 0 records the clock64 cycles from before the first issue to the completion.
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

constexpr int PR_SMEM = 100 * 1024;

__global__ void __launch_bounds__(128, 1)
    mma_rate_kernel(int a_tmem, int n, int count, unsigned long long* cycles, int* err) {
  griddep_sync();
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t done;
  __shared__ uint32_t tmem_base_s;
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  if (warp == 0) tmem_alloc(&tmem_base_s, 512);
  if (threadIdx.x == 32) {
    mbar_init(&done, 1);
    fence_barrier_init();
  }
  // A: [128 rows][64 bf16] (16 KB) at 0; B: [n rows][64 bf16] (up to 32 KB) at 32 KB
  for (int i = threadIdx.x; i < 64 * 1024 / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(sm)[i] = 0u;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  {  // the A operand in TMEM: each warp zeroes columns 256 .. 287 of its own 32 lanes
    uint32_t z[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) z[i] = 0u;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    tmem_st16(tmem + lane_off + 256, z);
    tmem_st16(tmem + lane_off + 272, z);
    tc_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 32) {
    const uint32_t idesc = idesc_bf16_f32(128, n);
    const uint32_t a = smem_u32(sm), b = smem_u32(sm + 32768);
    const unsigned long long t0 = clock64();
    for (int i = 0; i < count; ++i) {
      const uint32_t kk = (uint32_t)(i & 3) * 32;  // the four 16-wide k-steps of a 64-wide block
      if (a_tmem) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem),
            "r"(tmem + 256u + (uint32_t)(i & 3) * 8u), "l"(sw128_kmajor_desc(b + kk)), "r"(idesc),
            "r"(i > 0 ? 1u : 0u)
            : "memory");
      } else {
        tc_mma(tmem, sw128_kmajor_desc(a + kk), sw128_kmajor_desc(b + kk), idesc, i > 0 ? 1u : 0u);
      }
    }
    tc_commit(&done);
    const bool ok = mbar_wait_ns(&done, 0, 1000000000ull, err, DG_DEVERR_TIMEOUT_FULL);
    const unsigned long long t1 = clock64();
    if (blockIdx.x == 0 && ok) *cycles = t1 - t0;
    if (!ok) mbar_wait_drain(&done, 0);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

cudaError_t launch_mma_rate(int a_tmem, int n, int count, int blocks, unsigned long long* cycles, int* err,
                            cudaStream_t st) {
  if (!(n == 64 || n == 128 || n == 256) || count < 1 || count > (1 << 20) || blocks < 1 || blocks > 1024)
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(mma_rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PR_SMEM);
  if (e != cudaSuccess) return e;
  return launch_k(mma_rate_kernel, dim3(blocks), dim3(128), PR_SMEM, st, a_tmem, n, count, cycles, err);
}

}  // namespace dg
