// The canvas update with its scratch in a fixed device array instead of a workspace.
//
// Callers that cannot give the library device memory -- a sampler inside another
// engine that owns all of it, or a loop that must not allocate or free once running
// because cudaFree synchronises the whole device -- still need the two-kernel update
// (per-slice max / sum / argmax, then the merge and selection), whose partials need
// somewhere to live between the kernels.  Here that is one file-scope __device__ array
// per device, in this library's device image; its address is looked up once per device
// and cached.  No device memory is allocated or freed and no allocating library is
// called.  Calls on one device share the array: concurrent calls race (ordering them is
// the caller's job), and after a call it holds that call's partials.
#include <atomic>
#include <cstdio>
#include <mutex>

#include "../../include/dg_noalloc.h"
#include "dg_kernels.h"

namespace dg {
dg_status set_error(dg_status s, const char* msg);  // records dg_last_error's message
}

namespace {

constexpr int kScratchParts = 2048;  // 32 KB; every C <= 1024 needs at most 592 + C
constexpr int kMaxDevices = 64;

std::mutex g_setup_mu;
std::atomic<dg::UpdPart*> g_scratch[kMaxDevices];

}  // namespace

static __device__ __align__(256) dg::UpdPart g_upd_scratch[kScratchParts];

// device address of g_upd_scratch on the current device, looked up on first use
static dg_status scratch_for_current_device(dg::UpdPart** out) {
  char msg[160];
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof msg, "cudaGetDevice: %s", cudaGetErrorString(e));
    return dg::set_error(DG_ERR_CUDA, msg);
  }
  if (dev < 0 || dev >= kMaxDevices) {
    snprintf(msg, sizeof msg, "device %d: the fixed scratch supports devices 0..%d", dev, kMaxDevices - 1);
    return dg::set_error(DG_ERR_UNSUPPORTED, msg);
  }
  dg::UpdPart* p = g_scratch[dev].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lk(g_setup_mu);
    p = g_scratch[dev].load(std::memory_order_relaxed);
    if (!p) {
      void* a = nullptr;
      e = cudaGetSymbolAddress(&a, g_upd_scratch);
      if (e != cudaSuccess) {
        snprintf(msg, sizeof msg, "cudaGetSymbolAddress of the update scratch: %s", cudaGetErrorString(e));
        return dg::set_error(DG_ERR_CUDA, msg);
      }
      p = static_cast<dg::UpdPart*>(a);
      g_scratch[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return DG_OK;
}

extern "C" dg_status dg_canvas_update_noalloc(const float* d_logits, int32_t C, int32_t V, int32_t n_renoise,
                                              uint64_t seed, uint32_t step, int32_t* d_canvas, float* d_conf,
                                              dg_stream stream) {
  char msg[160];
  if (!d_logits || !d_canvas) return dg::set_error(DG_ERR_INVALID_ARG, "logits / canvas is NULL");
  if (C <= 0 || C > 1024) return dg::set_error(DG_ERR_INVALID_ARG, "C must be in [1, 1024]");
  if (V <= 0 || V % 4 != 0) return dg::set_error(DG_ERR_INVALID_ARG, "V must be a positive multiple of 4");
  if (n_renoise < 0 || n_renoise > C) return dg::set_error(DG_ERR_INVALID_ARG, "n_renoise must be in [0, C]");
  if ((reinterpret_cast<uintptr_t>(d_logits) & 15) != 0)
    return dg::set_error(DG_ERR_INVALID_ARG, "logits must be 16-byte aligned");
  const int splits = dg::update_splits(C, V);
  if ((long long)C * splits > kScratchParts) {
    snprintf(msg, sizeof msg, "update of C=%d x V=%d needs %lld scratch records; the fixed array holds %d", C, V,
             (long long)C * splits, kScratchParts);
    return dg::set_error(DG_ERR_CAPACITY, msg);
  }
  dg::UpdPart* part = nullptr;
  dg_status s = scratch_for_current_device(&part);
  if (s != DG_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = dg::launch_update_partial(d_logits, C, V, splits, -1, part, st);
  if (e == cudaSuccess)
    e = dg::launch_update_select(part, C, V, splits, n_renoise, seed, step, d_canvas, d_conf, -1, st);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof msg, "canvas update launch: %s", cudaGetErrorString(e));
    return dg::set_error(DG_ERR_CUDA, msg);
  }
  return DG_OK;
}
