// The canvas update with its scratch in a fixed device array instead of a workspace.
//
// Callers that cannot give the library device memory -- a sampler inside another
// engine that owns all of it, or a loop that must not allocate or free once running
// because cudaFree synchronises the whole device -- still need the two-kernel update
// (per-slice max / sum / argmax, then the merge and selection), whose partials need
// somewhere to live between the kernels.  Here that is one file-scope __device__ array
// in this library's device image, which every context that loads the image holds once.
// Its address is looked up once per CUDA context and cached under the context's unique
// id (never reused within a process), so a device reset or a second context on the same
// device gets its own look-up instead of a stale address.  No device memory is
// allocated or freed and no allocating library is called.  Calls in one context share
// the array: concurrent calls race (ordering them is the caller's job), and after a
// call it holds that call's partials.
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>

#include "../../include/dg_debug.h"
#include "../../include/dg_noalloc.h"
#include "dg_kernels.h"

namespace dg {
dg_status set_error(dg_status s, const char* msg);  // records dg_last_error's message
dg_status launch_wrapped(int kind, cudaStream_t st, const char* what, cudaError_t (*fn)(void*), void* arg);
}

namespace {

constexpr int kScratchParts = 2048;  // 32 KB; every C <= 1024 needs at most 592 + C
constexpr int kCacheSlots = 64;      // contexts remembered; the oldest entry is replaced

struct Slot {
  unsigned long long ctx_id;
  dg::UpdPart* ptr;
};
std::mutex g_mu;
Slot g_slots[kCacheSlots];
int g_used = 0, g_next = 0;
PFN_cuCtxGetCurrent_v4000 g_get_current = nullptr;
PFN_cuCtxGetId_v12000 g_get_id = nullptr;

}  // namespace

static __device__ __align__(256) dg::UpdPart g_upd_scratch[kScratchParts];

static dg_status driver_fn(const char* name, void** fn) {
  char msg[160];
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint(name, fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || *fn == nullptr || q != cudaDriverEntryPointSuccess) {
    snprintf(msg, sizeof msg, "driver entry point %s unavailable", name);
    return dg::set_error(DG_ERR_CUDA, msg);
  }
  return DG_OK;
}

// unique id of the calling thread's current context (the runtime's primary context of
// the current device unless the caller made another one current)
static dg_status current_context_id(unsigned long long* id) {
  if (!g_get_current || !g_get_id) {
    void *a = nullptr, *b = nullptr;
    dg_status s = driver_fn("cuCtxGetCurrent", &a);
    if (s != DG_OK) return s;
    s = driver_fn("cuCtxGetId", &b);
    if (s != DG_OK) return s;
    g_get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(a);
    g_get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(b);
  }
  CUcontext ctx = nullptr;
  if (g_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
    return dg::set_error(DG_ERR_CUDA, "no current CUDA context (the caller's buffers live in one)");
  if (g_get_id(ctx, id) != CUDA_SUCCESS) return dg::set_error(DG_ERR_CUDA, "cuCtxGetId failed");
  return DG_OK;
}

// device address of g_upd_scratch in the current context, looked up on first use there
static dg_status scratch_for_current_context(dg::UpdPart** out) {
  char msg[160];
  std::lock_guard<std::mutex> lk(g_mu);
  unsigned long long id = 0;
  dg_status s = current_context_id(&id);
  if (s != DG_OK) return s;
  for (int i = 0; i < g_used; ++i)
    if (g_slots[i].ctx_id == id) {
      *out = g_slots[i].ptr;
      return DG_OK;
    }
  void* a = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&a, g_upd_scratch);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof msg, "cudaGetSymbolAddress of the update scratch: %s", cudaGetErrorString(e));
    return dg::set_error(DG_ERR_CUDA, msg);
  }
  Slot& slot = g_slots[g_used < kCacheSlots ? g_used++ : (g_next++ % kCacheSlots)];
  slot.ctx_id = id;
  slot.ptr = static_cast<dg::UpdPart*>(a);
  *out = slot.ptr;
  return DG_OK;
}

namespace {
struct UpdArgs {
  const float* logits;
  int C, V, splits, n_renoise;
  uint64_t seed;
  uint32_t step;
  int32_t* canvas;
  float* conf;
  dg::UpdPart* part;
  cudaStream_t st;
};
cudaError_t launch_partial(void* p) {
  auto* a = static_cast<UpdArgs*>(p);
  return dg::launch_update_partial(a->logits, a->C, a->V, a->splits, -1, a->part, a->st);
}
cudaError_t launch_select(void* p) {
  auto* a = static_cast<UpdArgs*>(p);
  return dg::launch_update_select(a->part, a->C, a->V, a->splits, a->n_renoise, a->seed, a->step, a->canvas,
                                  a->conf, -1, a->st);
}
}  // namespace

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
  dg_status s = scratch_for_current_context(&part);
  if (s != DG_OK) return s;
  UpdArgs a{d_logits, C, V, splits, n_renoise, seed, step, d_canvas, d_conf, part,
            reinterpret_cast<cudaStream_t>(stream)};
  s = dg::launch_wrapped(DG_K_UPDATE_PARTIAL, a.st, "update partial (no-alloc)", launch_partial, &a);
  if (s != DG_OK) return s;
  return dg::launch_wrapped(DG_K_UPDATE_SELECT, a.st, "update select (no-alloc)", launch_select, &a);
}
