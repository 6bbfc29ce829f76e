// C-ABI of libdg: validation, workspace carving, TMA tensor-map encoding and the
// launch sequences of the prefill, denoising pass, canvas update and canvas
// generation (declared in include/dg.h and include/dg_debug.h).
#include <cudaTypedefs.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>  // header-only; ranges reach a profiler only when one is attached

#include "../../include/dg.h"
#include "../../include/dg_debug.h"
#include "dg_common.cuh"
#include "dg_kernels.h"

using dg::bf16;

bool dg::pdl_enabled() {
  static const bool on = getenv("DG_NO_PDL") == nullptr;
  return on;
}

// ---------------------------------------------------------------- errors
static thread_local std::string g_err;
static dg_status fail(dg_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}
namespace dg {
// for entry points defined in other translation units
dg_status set_error(dg_status s, const char* msg) { return fail(s, "%s", msg); }
}  // namespace dg

#define DG_CHECK_ARG(cond, ...) \
  do {                          \
    if (!(cond)) return fail(DG_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)

// ---------------------------------------------------------------- profiling
extern "C" const char* dg_kernel_name(int32_t kind);
namespace {
struct ProfPair {
  cudaEvent_t a, b;
  int kind;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfPair> g_prof_pending;
std::vector<ProfPair> g_prof_free;
double g_prof_ms[DG_K_COUNT];
int g_prof_n[DG_K_COUNT];
int64_t g_launches = 0;

void prof_flush_locked() {
  for (auto& p : g_prof_pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(p.b) == cudaSuccess && cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) {
      g_prof_ms[p.kind] += ms;
      g_prof_n[p.kind] += 1;
    }
    g_prof_free.push_back(p);
  }
  g_prof_pending.clear();
}

// DG_NVTX set in the environment: every launch sits in an NVTX range named after its kind
// (for filtering ncu / nsys captures)
bool nvtx_on() {
  static const bool on = getenv("DG_NVTX") != nullptr;
  return on;
}

struct ProfScope {
  ProfPair pair{};
  bool on = false;
  bool nvtx = false;
  cudaStream_t st;
  ProfScope(int kind, cudaStream_t s) : st(s) {
    if (nvtx_on()) {
      nvtxRangePushA(dg_kernel_name(kind));
      nvtx = true;
    }
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_launches++;
    if (!g_prof_on) return;
    if (g_prof_pending.size() >= 8192) prof_flush_locked();
    if (!g_prof_free.empty()) {
      pair = g_prof_free.back();
      g_prof_free.pop_back();
    } else {
      if (cudaEventCreate(&pair.a) != cudaSuccess || cudaEventCreate(&pair.b) != cudaSuccess) return;
    }
    pair.kind = kind;
    on = cudaEventRecord(pair.a, st) == cudaSuccess;
  }
  ~ProfScope() {
    if (nvtx) nvtxRangePop();
    if (!on) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (cudaEventRecord(pair.b, st) == cudaSuccess) g_prof_pending.push_back(pair);
  }
};
}  // namespace

// Host-side fault injection: DG_FAULT_INJECT=launch:N makes the N-th kernel launch of the
// process (1-based, every kind) fail on the host without launching, as a failed launch
// would, so that the error paths can be exercised without faulting a GPU.
namespace {
long long fault_launch_index() {
  static const long long n = [] {
    const char* v = getenv("DG_FAULT_INJECT");
    long long k = 0;
    if (v && sscanf(v, "launch:%lld", &k) == 1 && k > 0) return k;
    return 0LL;
  }();
  return n;
}
std::atomic<long long> g_launch_seq{0};
bool inject_launch_fault() {
  const long long n = fault_launch_index();
  return n > 0 && g_launch_seq.fetch_add(1) + 1 == n;
}
}  // namespace

#define LAUNCH(kind, st, call)                                                                          \
  do {                                                                                                  \
    if (inject_launch_fault()) return fail(DG_ERR_CUDA, "%s: injected launch failure", #call);        \
    cudaError_t _e;                                                                                     \
    {                                                                                                   \
      ProfScope _ps((kind), (st));                                                                      \
      _e = (call);                                                                                      \
    }                                                                                                   \
    if (_e != cudaSuccess) return fail(DG_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(_e));          \
  } while (0)

namespace dg {
// one launch through the same wrapper as every other entry point (fault injection,
// launch count, NVTX range, per-kind event timing), for entry points in other files
dg_status launch_wrapped(int kind, cudaStream_t st, const char* what, cudaError_t (*fn)(void*), void* arg) {
  if (inject_launch_fault()) return fail(DG_ERR_CUDA, "%s: injected launch failure", what);
  cudaError_t e;
  {
    ProfScope ps(kind, st);
    e = fn(arg);
  }
  if (e != cudaSuccess) return fail(DG_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return DG_OK;
}
}  // namespace dg

// ---------------------------------------------------------------- tensor maps
static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> g_encode{nullptr};
static std::mutex g_encode_mu;
static dg_status get_encoder() {
  if (g_encode.load(std::memory_order_acquire)) return DG_OK;
  std::lock_guard<std::mutex> lk(g_encode_mu);
  if (g_encode.load(std::memory_order_relaxed)) return DG_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || fn == nullptr || q != cudaDriverEntryPointSuccess)
    return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(e));
  g_encode.store(reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn), std::memory_order_release);
  return DG_OK;
}

// bf16 tensor, up to 3 dims (dims[0] innermost), 128-byte swizzle
static dg_status encode_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                             const uint64_t* strides_bytes /* rank-1 entries */, const uint32_t* box) {
  if (get_encoder() != DG_OK) return DG_ERR_CUDA;
  cuuint64_t gd[3], gs[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) gd[i] = dims[i], bx[i] = box[i];
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = g_encode.load(std::memory_order_acquire)(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), gd, gs, bx,
                        es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return DG_OK;
}
// byte tensor (8-bit weight codes or their scales), up to 3 dims (dims[0] innermost)
static dg_status encode_u8(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                           const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle) {
  if (get_encoder() != DG_OK) return DG_ERR_CUDA;
  cuuint64_t gd[3], gs[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) gd[i] = dims[i], bx[i] = box[i];
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = g_encode.load(std::memory_order_acquire)(
      map, CU_TENSOR_MAP_DATA_TYPE_UINT8, (cuuint32_t)rank, const_cast<void*>(base), gd, gs, bx, es,
      CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled (u8) failed (%d)", (int)r);
  return DG_OK;
}
// 8-bit weight codes [groups][rows][cols] as a 3-D map, box (64 cols, 128 rows, 1 group),
// 64-byte swizzle; rows past a group's end read as zero codes
static dg_status map_codes(CUtensorMap* m, const void* base, uint64_t groups, uint64_t rows, uint64_t cols) {
  const uint64_t dims[3] = {cols, rows, groups};
  const uint64_t strides[2] = {cols, rows * cols};
  const uint32_t box[3] = {64, 128, 1};
  return encode_u8(m, base, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_64B);
}
// their scales [groups][cols / 64][rows][2] as a 3-D map, box (256 bytes = 128 rows, 1, 1)
static dg_status map_scales(CUtensorMap* m, const void* base, uint64_t groups, uint64_t rows, uint64_t cols) {
  const uint64_t dims[3] = {rows * 2, cols / 64, groups};
  const uint64_t strides[2] = {rows * 2, (cols / 64) * rows * 2};
  const uint32_t box[3] = {256, 1, 1};
  return encode_u8(m, base, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}
// 4-bit weight codes [groups][rows][cols / 2] (two per byte) as a 3-D map, box (32 bytes =
// 64 cols, 128 rows, 1 group), 32-byte swizzle
static dg_status map_codes4(CUtensorMap* m, const void* base, uint64_t groups, uint64_t rows, uint64_t cols) {
  const uint64_t dims[3] = {cols / 2, rows, groups};
  const uint64_t strides[2] = {cols / 2, rows * cols / 2};
  const uint32_t box[3] = {32, 128, 1};
  return encode_u8(m, base, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_32B);
}
// their E4M3 scales [groups][cols / 64][rows][4], viewed as 16-byte rows of 4 weight rows:
// dims (16, rows / 4, groups * cols / 64), box (16, 32, 1) = one 128-row tile's scales
static dg_status map_scales4(CUtensorMap* m, const void* base, uint64_t groups, uint64_t rows, uint64_t cols) {
  const uint64_t dims[3] = {16, rows / 4, groups * (cols / 64)};
  const uint64_t strides[2] = {16, rows * 4};
  const uint32_t box[3] = {16, 32, 1};
  return encode_u8(m, base, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}
// row-major [rows][cols] bf16 matrix as a 2-D map with box (64 cols, box_rows rows)
static dg_status map_rows(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t strides[1] = {cols * 2};
  const uint32_t box[2] = {64, box_rows};
  return encode_bf16(m, base, 2, dims, strides, box);
}
// weights [groups][rows][cols] bf16 as a 3-D map with box (64 cols, 128 rows, 1 group);
// rows past the end of a group read as zeros instead of the next group's rows
static dg_status map_weights(CUtensorMap* m, const void* base, uint64_t groups, uint64_t rows, uint64_t cols) {
  const uint64_t dims[3] = {cols, rows, groups};
  const uint64_t strides[2] = {cols * 2, rows * cols * 2};
  const uint32_t box[3] = {64, 128, 1};
  return encode_bf16(m, base, 3, dims, strides, box);
}

// ---------------------------------------------------------------- model
struct LayerMaps {
  CUtensorMap qkv, o, gate, up, down;
};
// low-precision experts of one layer: codes and block scales of gate, up and down, the
// format (dg::FMT_MX8 / dg::FMT_NV4) and the 4-bit tensor scales
struct LowpMaps {
  CUtensorMap gate, gate_s, up, up_s, down, down_s;
  int fmt;
  float g_gate, g_up, g_down;
};
// the output matrix in low precision: codes and block scales of W_out [V][H], the format
// and the 4-bit tensor scale
struct VocabLowp {
  CUtensorMap codes, scales;
  int fmt = 0;
  float g = 1.0f;
  bool on = false;
};
struct dg_model {
  dg_config cfg;
  const void* embed;
  const void* w_out;
  std::vector<dg_layer_weights> layers;
  std::vector<LayerMaps> maps;
  CUtensorMap out_map;
  std::vector<LowpMaps> lowp;  // non-empty: the batched calls run the experts from low-precision weights
  VocabLowp vocab_lowp;        // on: the batched calls project to the vocabulary from low-precision weights
  bool taps_on = false;
  std::vector<float*> tap_x_attn, tap_x_out, tap_topk_w;
  std::vector<int32_t*> tap_topk_idx, tap_counts, tap_perm;
  int32_t* tap_unions = nullptr;
  int tap_rows = 0;
};

static bool is_bf16(const dg_config& c) { return c.dtype == DG_DTYPE_BF16; }
static size_t act_bytes(const dg_config& c) { return is_bf16(c) ? 2 : 4; }
static int qkv_rows(const dg_config& c) { return (c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim; }

static dg_status validate_config(const dg_config* c) {
  DG_CHECK_ARG(c, "config is NULL");
  DG_CHECK_ARG(c->n_layers >= 1 && c->hidden > 0 && c->n_q_heads > 0 && c->n_kv_heads > 0 && c->head_dim > 0 &&
                   c->n_experts > 0 && c->top_k > 0 && c->expert_ffn > 0 && c->vocab > 0,
               "config sizes must be positive");
  DG_CHECK_ARG(c->dtype == DG_DTYPE_BF16 || c->dtype == DG_DTYPE_F32, "dtype must be DG_DTYPE_BF16 or DG_DTYPE_F32");
  DG_CHECK_ARG(c->n_q_heads % c->n_kv_heads == 0, "n_q_heads %% n_kv_heads != 0");
  DG_CHECK_ARG(c->top_k <= c->n_experts && c->top_k <= 16, "top_k must be <= min(16, n_experts)");
  DG_CHECK_ARG(c->n_experts <= 256, "n_experts must be <= 256");
  DG_CHECK_ARG(c->hidden % 64 == 0 && c->expert_ffn % 64 == 0, "hidden and expert_ffn must be multiples of 64");
  DG_CHECK_ARG(c->head_dim % 2 == 0 && c->head_dim <= 128, "head_dim must be even and <= 128");
  DG_CHECK_ARG(c->vocab % 4 == 0, "vocab must be a multiple of 4");
  DG_CHECK_ARG(c->rms_eps >= 0.f && c->rope_theta > 0.f, "bad rms_eps / rope_theta");
  if (is_bf16(*c)) {
    DG_CHECK_ARG(c->head_dim == 128, "bf16 model: head_dim must be 128");
    DG_CHECK_ARG(c->vocab % 128 == 0, "bf16 model: vocab must be a multiple of 128");
    DG_CHECK_ARG(qkv_rows(*c) % 128 == 0 && c->hidden % 128 == 0, "bf16 model: hidden must be a multiple of 128");
  }
  return DG_OK;
}

extern "C" dg_status dg_model_create(const dg_config* cfg, const dg_weights* w, dg_model** out) {
  dg_status s = validate_config(cfg);
  if (s != DG_OK) return s;
  DG_CHECK_ARG(w && out && w->embed && w->w_out && w->layers, "weights / out pointer is NULL");
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  DG_CHECK_ARG(a16(w->embed) && a16(w->w_out), "embed / w_out must be 16-byte aligned");
  for (int l = 0; l < cfg->n_layers; ++l) {
    const dg_layer_weights& L = w->layers[l];
    DG_CHECK_ARG(L.w_qkv && L.w_o && L.w_router && L.w_gate && L.w_up && L.w_down, "layer %d has a NULL weight", l);
    DG_CHECK_ARG(a16(L.w_qkv) && a16(L.w_o) && a16(L.w_router) && a16(L.w_gate) && a16(L.w_up) && a16(L.w_down),
                 "layer %d: weights must be 16-byte aligned", l);
  }
  dg_model* m = new (std::nothrow) dg_model();
  if (!m) return fail(DG_ERR_CUDA, "out of host memory");
  m->cfg = *cfg;
  m->embed = w->embed;
  m->w_out = w->w_out;
  try {
    m->layers.assign(w->layers, w->layers + cfg->n_layers);
    if (is_bf16(*cfg)) m->maps.resize(cfg->n_layers);
  } catch (...) {
    delete m;
    return fail(DG_ERR_CUDA, "out of host memory");
  }
  if (is_bf16(*cfg)) {
    const dg_config& c = *cfg;
    for (int l = 0; l < c.n_layers; ++l) {
      const dg_layer_weights& L = m->layers[l];
      LayerMaps& M = m->maps[l];
      const uint64_t E = c.n_experts, F = c.expert_ffn, H = c.hidden;
      if ((s = map_weights(&M.qkv, L.w_qkv, 1, qkv_rows(c), H)) != DG_OK ||
          (s = map_weights(&M.o, L.w_o, 1, H, (uint64_t)c.n_q_heads * c.head_dim)) != DG_OK ||
          (s = map_weights(&M.gate, L.w_gate, E, F, H)) != DG_OK ||
          (s = map_weights(&M.up, L.w_up, E, F, H)) != DG_OK ||
          (s = map_weights(&M.down, L.w_down, E, H, F)) != DG_OK) {
        delete m;
        return s;
      }
    }
    if ((s = map_weights(&m->out_map, m->w_out, 1, c.vocab, c.hidden)) != DG_OK) {
      delete m;
      return s;
    }
  }
  *out = m;
  return DG_OK;
}

extern "C" void dg_model_destroy(dg_model* m) { delete m; }

// ---------------------------------------------------------------- workspace layout
namespace {
constexpr int kMaxAttnSplits = 16;
constexpr int kMaxKsQkv = 4;   // split-K of the QKV projection
constexpr int kMaxKsO = 8;     // split-K of the output projection
constexpr int kSmemGemm = 200 * 1024;    // stage budget of the persistent GEMM (one CTA per SM)
inline size_t al(size_t x) { return (x + 255) & ~size_t(255); }

constexpr int kItemRows = 128;           // rows per work item of the grouped expert GEMMs
constexpr int kItemRowsMx8 = 64;         // the same for the 8-bit-weight expert GEMMs


struct WsLayout {
  size_t err, upd, x, xn, xn_lo, qkv, q, q_lo, k_lo, vt_lo, o, o_lo, part_o, part_lse, opart, topk_idx,
      topk_w, counts, offsets, perm, inv, uni, items, n_items, xs, xs_lo, h, h_lo, gu, ys, vtiles, total;
  int lo_rows;  // rows of the current-token K/V low-term window
};

size_t upd_bytes(int C, int V) { return al((size_t)C * dg::update_splits(C, V) * sizeof(dg::UpdPart)); }

WsLayout layout(const dg_config& c, int T) {
  WsLayout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t r = o;
    o += al(bytes);
    return r;
  };
  const bool bf = is_bf16(c);
  const size_t ab = act_bytes(c);
  const size_t H = c.hidden, k = c.top_k, F = c.expert_ffn, d = c.head_dim, E = c.n_experts;
  L.err = take(256);
  size_t upd_max = 0;
  for (int C = 1; C <= T; ++C) upd_max = upd_max > upd_bytes(C, c.vocab) ? upd_max : upd_bytes(C, c.vocab);
  L.upd = take(upd_max);
  L.x = take((size_t)T * H * 4);
  L.xn = take((size_t)T * H * ab);
  L.xn_lo = take(bf ? (size_t)T * H * 2 : 0);
  L.qkv = take((size_t)(bf ? kMaxKsQkv : 1) * T * qkv_rows(c) * 4);
  L.q = take((size_t)c.n_q_heads * T * d * ab);
  L.lo_rows = ((T + 127) / 128) * 128 + 128;
  L.q_lo = take(bf ? (size_t)c.n_q_heads * T * d * 2 : 0);
  L.k_lo = take(bf ? (size_t)c.n_kv_heads * L.lo_rows * d * 2 : 0);
  L.vt_lo = take(bf ? (size_t)c.n_kv_heads * L.lo_rows * d * 2 : 0);
  L.o = take((size_t)T * c.n_q_heads * d * ab);
  L.o_lo = take(bf ? (size_t)T * c.n_q_heads * d * 2 : 0);
  L.part_o = take(bf ? (size_t)kMaxAttnSplits * c.n_q_heads * T * d * 4 : 0);
  L.part_lse = take(bf ? (size_t)kMaxAttnSplits * c.n_q_heads * T * 4 : 0);
  L.opart = take((size_t)(bf ? kMaxKsO : 1) * T * H * 4);
  L.topk_idx = take((size_t)T * k * 4);
  L.topk_w = take((size_t)T * k * 4);
  L.counts = take(E * 4);
  L.offsets = take((E + 1) * 4);
  L.perm = take((size_t)T * k * 4);
  L.inv = take((size_t)T * k * 4);
  L.uni = take(4);
  L.items = take(((size_t)T * k / kItemRowsMx8 + E + 1) * sizeof(dg::TcWorkItem));
  L.n_items = take(4);
  L.xs = take((size_t)T * k * H * ab);
  L.xs_lo = take(bf ? (size_t)T * k * H * 2 : 0);
  L.h = take((size_t)T * k * F * ab);
  L.h_lo = take(bf ? (size_t)T * k * F * 2 : 0);
  L.gu = take(bf ? 0 : (size_t)T * k * 2 * F * 4);
  L.ys = take((size_t)T * k * H * 4);
  // the fused vocabulary/update path: one statistics record per (token, 128-id tile)
  L.vtiles = take((size_t)(T < 1024 ? T : 1024) * ((c.vocab + 127) / 128) * sizeof(dg::UpdPart));
  L.total = o;
  return L;
}

struct Ws {
  char* base;
  WsLayout L;
  template <typename P>
  P* at(size_t off) const {
    return reinterpret_cast<P*>(base + off);
  }
  int* err() const { return at<int>(L.err); }
};

int ceil_div(int a, int b) { return (a + b - 1) / b; }

// split-K factor: a divisor of the k-block count, at most max_ks, keeping >= 2 k-blocks
// per tile and the tile count within one wave of the persistent GEMM
int pick_ksplit(int m_tiles, int token_chunks, int nkb, int max_ks) {
  int best = 1;
  for (int ks = 1; ks <= max_ks; ++ks)
    if (nkb % ks == 0 && nkb / ks >= 2 && m_tiles * token_chunks * ks <= dg::num_sms()) best = ks;
  return best;
}
}  // namespace

extern "C" size_t dg_workspace_bytes(const dg_config* cfg, int32_t max_tokens) {
  if (validate_config(cfg) != DG_OK || max_tokens <= 0) return 0;
  return layout(*cfg, max_tokens).total;
}
extern "C" size_t dg_update_workspace_bytes(int32_t C, int32_t V) {
  if (C <= 0 || V <= 0) return 0;
  return 256 + upd_bytes(C, V);
}

// ---------------------------------------------------------------- the layer stack
namespace {

struct GemmCall {
  int kind, epi;
  const CUtensorMap* A;
  const CUtensorMap* A2;  // dual_a (gate / up) or null
  const void* X;
  const void* X_lo;       // null: single term
  int x_rows, K;
  int a_rows_per_group;   // output features per group
  const dg::TcWorkItem* items;  // grouped work list or null (dense)
  const int* n_items;
  int max_items;          // upper bound of the work-item count (sizes the grid)
  int n_max;              // token rows per tile
  void* out;
  void* out_lo;
  int ld_out;
  int k_splits;
  size_t split_stride;
  int smem_budget;
};

// dense projections (no work list, one weight matrix, fp32 store) of at least two weight
// tiles take them in pairs that share each token load
// weight tiles taken in pairs that share each token load: every fp32-store GEMM of at
// least 256 weight rows (the dense projections and the grouped expert down projection,
// whose short tiles -- 11 k-blocks of 16 token rows at the large model -- then halve their
// per-tile hand-offs and token loads); the gate/up GEMM already pairs its two matrices
bool pair_weight_tiles(int a_rows, bool grouped, bool dual, int epi) {
  (void)grouped;
  return !dual && epi == dg::EPI_STORE_F32 && a_rows >= 256;
}
// weight tiles of a dense projection as the GEMM walks them (pairs where they are paired)
int dense_weight_tiles(int a_rows) { return ceil_div(a_rows, pair_weight_tiles(a_rows, false, false,
                                                                                  dg::EPI_STORE_F32) ? 256 : 128); }

dg_status gemm_bf16(const GemmCall& g, int* err, cudaStream_t st) {
  CUtensorMap B, B2, Bb, B2b;
  dg_status s;
  if ((s = map_rows(&B, g.X, (uint64_t)g.x_rows, (uint64_t)g.K, 16)) != DG_OK) return s;
  if ((s = map_rows(&Bb, g.X, (uint64_t)g.x_rows, (uint64_t)g.K, 64)) != DG_OK) return s;
  if (g.X_lo) {
    if ((s = map_rows(&B2, g.X_lo, (uint64_t)g.x_rows, (uint64_t)g.K, 16)) != DG_OK) return s;
    if ((s = map_rows(&B2b, g.X_lo, (uint64_t)g.x_rows, (uint64_t)g.K, 64)) != DG_OK) return s;
  } else {
    B2 = B;
    B2b = Bb;
  }
  dg::TcGemmParams p{};
  p.K = g.K;
  p.a_rows_per_group = g.a_rows_per_group;
  p.m_pair = pair_weight_tiles(g.a_rows_per_group, g.items != nullptr, g.A2 != nullptr, g.epi) ? 1 : 0;
  p.m_tiles = ceil_div(g.a_rows_per_group, p.m_pair ? 256 : 128);
  p.n_max = g.n_max;
  p.n_tokens = g.x_rows;
  p.k_splits = g.k_splits;
  p.split_stride = g.split_stride;
  p.items = g.items;
  p.n_items = g.n_items;
  p.dual_a = g.A2 != nullptr;
  p.two_terms = g.X_lo != nullptr;
  p.out = g.out;
  p.out_lo = g.out_lo;
  p.ld_out = g.ld_out;
  p.smem_budget = g.smem_budget;
  p.err = err;
  const int items = g.items ? g.max_items : ceil_div(g.x_rows, g.n_max) * g.k_splits;
  LAUNCH(g.kind, st,
         dg::launch_tc_gemm(g.epi, *g.A, g.A2 ? *g.A2 : *g.A, B, B2, Bb, B2b, p, items * p.m_tiles, st));
  return DG_OK;
}

// a grouped expert GEMM over low-precision weights (A, S: codes and scales; A2, S2 for gate
// / up; g_a, g_a2: the 4-bit tensor scales)
dg_status gemm_lowp(const GemmCall& g, int fmt, const CUtensorMap* S, const CUtensorMap* S2, float g_a, float g_a2,
                   int* err, cudaStream_t st) {
  CUtensorMap B, B2, Bb, B2b;
  dg_status s;
  if ((s = map_rows(&B, g.X, (uint64_t)g.x_rows, (uint64_t)g.K, 16)) != DG_OK) return s;
  if ((s = map_rows(&Bb, g.X, (uint64_t)g.x_rows, (uint64_t)g.K, 64)) != DG_OK) return s;
  if (g.X_lo) {
    if ((s = map_rows(&B2, g.X_lo, (uint64_t)g.x_rows, (uint64_t)g.K, 16)) != DG_OK) return s;
    if ((s = map_rows(&B2b, g.X_lo, (uint64_t)g.x_rows, (uint64_t)g.K, 64)) != DG_OK) return s;
  } else {
    B2 = B;
    B2b = Bb;
  }
  dg::TcGemmParams p{};
  p.K = g.K;
  p.a_rows_per_group = g.a_rows_per_group;
  p.m_tiles = ceil_div(g.a_rows_per_group, 128);
  p.n_max = g.n_max;
  p.n_tokens = g.x_rows;
  p.k_splits = 1;
  p.items = g.items;
  p.n_items = g.n_items;
  p.dual_a = g.A2 != nullptr;
  p.two_terms = g.X_lo != nullptr;
  p.out = g.out;
  p.out_lo = g.out_lo;
  p.ld_out = g.ld_out;
  p.smem_budget = g.smem_budget;
  p.err = err;
  LAUNCH(g.kind, st,
         dg::launch_tc_gemm_lowp(fmt, g.epi, *g.A, g.A2 ? *g.A2 : *g.A, *S, S2 ? *S2 : *S, B, B2, Bb, B2b, p, g_a,
                                 g_a2, g.max_items * p.m_tiles, st));
  return DG_OK;
}

// split-KV factor: one wave of CTAs (the attention kernel holds a whole SM), at least two
// 128-key chunks per CTA
int attn_splits(int n_q, int nq, int n_keys, int* chunks_per_split) {
  const int nch = ceil_div(n_keys, 128);
  const int base = ceil_div(n_q, 128) * nq;
  int splits = dg::num_sms() / base;
  if (splits > kMaxAttnSplits) splits = kMaxAttnSplits;
  if (splits > nch / 2) splits = nch / 2;
  if (splits < 1) splits = 1;
  *chunks_per_split = ceil_div(nch, splits);
  splits = ceil_div(nch, *chunks_per_split);
  return splits;
}

// split-KV factor of the head-pair kernel: one wave of CTAs, at least two 128-key chunks
// per CTA (each CTA loads its query tiles once)
int attn_pair_splits(int n_q, int nq, int group, int pair_heads, int n_keys, int* chunks_per_split) {
  const int nch = ceil_div(n_keys, 128);
  const int base = ceil_div(n_q, 128) * dg::attn2_head_groups(nq, group, pair_heads);
  int splits = dg::num_sms() / base;
  if (splits > kMaxAttnSplits) splits = kMaxAttnSplits;
  if (splits > nch / 2) splits = nch / 2;
  if (splits < 1) splits = 1;
  *chunks_per_split = ceil_div(nch, splits);
  splits = ceil_div(nch, *chunks_per_split);
  return splits;
}

// The bf16 pass's attention runs the single-head kernel (tc_attn_kernel); DG_ATTN_PAIR=1
// routes it through the head-pair kernel (tc_attn2_kernel) instead
bool attn_pair_enabled() {
  static const bool pair = getenv("DG_ATTN_PAIR") != nullptr && getenv("DG_ATTN_PAIR")[0] == '1';
  return pair;
}

// The tensor maps both attention kernels read: the query hi / lo [nq][n_q][128], the
// cache's K [nkv][cap][128] and V^T [nkv][128][cap], the low terms of the current K / V^T
// (rows counted from `base`); every box is 64 x 128 (128-byte swizzled rows)
dg_status attn_maps(const dg_config& c, const Ws& ws, void* kc, void* vtc, int cap, int n_q, int n_keys, int base,
                    CUtensorMap* m) {
  const int nq = c.n_q_heads, nkv = c.n_kv_heads, d = c.head_dim;
  const int Lc = ws.L.lo_rows;
  const uint32_t box[3] = {64, 128, 1};
  dg_status s;
  {
    const uint64_t dims[3] = {(uint64_t)d, (uint64_t)n_q, (uint64_t)nq};
    const uint64_t str[2] = {(uint64_t)d * 2, (uint64_t)n_q * d * 2};
    if ((s = encode_bf16(&m[0], ws.at<void>(ws.L.q), 3, dims, str, box)) != DG_OK) return s;
    if ((s = encode_bf16(&m[1], ws.at<void>(ws.L.q_lo), 3, dims, str, box)) != DG_OK) return s;
  }
  {
    const uint64_t dims[3] = {(uint64_t)d, (uint64_t)n_keys, (uint64_t)nkv};
    const uint64_t str[2] = {(uint64_t)d * 2, (uint64_t)cap * d * 2};
    if ((s = encode_bf16(&m[2], kc, 3, dims, str, box)) != DG_OK) return s;
  }
  {
    const uint64_t dims[3] = {(uint64_t)n_keys, (uint64_t)d, (uint64_t)nkv};
    const uint64_t str[2] = {(uint64_t)cap * 2, (uint64_t)d * cap * 2};
    if ((s = encode_bf16(&m[3], vtc, 3, dims, str, box)) != DG_OK) return s;
  }
  {
    const uint64_t dims[3] = {(uint64_t)d, (uint64_t)(n_keys - base), (uint64_t)nkv};
    const uint64_t str[2] = {(uint64_t)d * 2, (uint64_t)Lc * d * 2};
    if ((s = encode_bf16(&m[4], ws.at<void>(ws.L.k_lo), 3, dims, str, box)) != DG_OK) return s;
  }
  {
    const uint64_t dims[3] = {(uint64_t)(n_keys - base), (uint64_t)d, (uint64_t)nkv};
    const uint64_t str[2] = {(uint64_t)Lc * 2, (uint64_t)d * Lc * 2};
    if ((s = encode_bf16(&m[5], ws.at<void>(ws.L.vt_lo), 3, dims, str, box)) != DG_OK) return s;
  }
  return DG_OK;
}

// the parameters both attention kernels share (the split layout is the caller's)
dg::TcAttnParams attn_params(const dg_config& c, const Ws& ws, int n_q, int pos0, int n_keys, int causal, int base) {
  const int nq = c.n_q_heads, d = c.head_dim;
  dg::TcAttnParams p;
  p.n_q = n_q;
  p.q_pos0 = pos0;
  p.n_keys = n_keys;
  p.causal = causal;
  p.group = nq / c.n_kv_heads;
  p.nq = nq;
  p.n_splits = 1;
  p.chunks_per_split = 1;
  p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)d));
  p.has_lo = 1;
  p.base = base;
  p.out = ws.at<bf16>(ws.L.o);
  p.out_lo = ws.at<bf16>(ws.L.o_lo);
  p.part_o = ws.at<float>(ws.L.part_o);
  p.part_lse = ws.at<float>(ws.L.part_lse);
  p.err = ws.err();
  return p;
}

// attention() through the head-pair kernel: the same inputs, outputs and workspace
dg_status attention_pair(const dg_config& c, const Ws& ws, void* kc, void* vtc, int cap, int n_q, int pos0,
                         int n_keys, int causal, cudaStream_t st) {
  const int nq = c.n_q_heads;
  const int base = (pos0 / 128) * 128;  // the low-term window starts here (a multiple of the 128-key chunk)
  CUtensorMap m[6];
  dg_status s;
  if ((s = attn_maps(c, ws, kc, vtc, cap, n_q, n_keys, base, m)) != DG_OK) return s;
  dg::TcAttnParams p = attn_params(c, ws, n_q, pos0, n_keys, causal, base);
  // head pairs share each K/V chunk and overlap one head's softmax with the other's MMAs;
  // single heads give twice the CTAs.  Take whichever fills more of the machine in one
  // wave (pairs unless single heads fill at least a quarter more SMs).
  int cps_pair = 0, cps_single = 0;
  const int sp_pair = attn_pair_splits(n_q, nq, p.group, 1, n_keys, &cps_pair);
  const int sp_single = attn_pair_splits(n_q, nq, p.group, 0, n_keys, &cps_single);
  const int q_tiles = ceil_div(n_q, 128);
  const int ctas_pair = q_tiles * dg::attn2_head_groups(nq, p.group, 1) * sp_pair;
  const int ctas_single = q_tiles * nq * sp_single;
  const int pair_heads = (p.group % 2 == 0 && 4 * ctas_single < 5 * ctas_pair) ? 1 : 0;
  p.n_splits = pair_heads ? sp_pair : sp_single;
  p.chunks_per_split = pair_heads ? cps_pair : cps_single;
  LAUNCH(DG_K_ATTENTION, st, dg::launch_tc_attention2(m[0], m[1], m[2], m[3], m[4], m[5], p, pair_heads, st));
  if (p.n_splits > 1)
    LAUNCH(DG_K_ATTN_MERGE, st,
           dg::launch_attn_merge2(p.part_o, p.part_lse, p.n_splits, nq, n_q, p.out, p.out_lo, st));
  return DG_OK;
}

// attention() through the single-head kernel: the same inputs, outputs and workspace
dg_status attention_single(const dg_config& c, const Ws& ws, void* kc, void* vtc, int cap, int n_q, int pos0,
                           int n_keys, int causal, cudaStream_t st) {
  const int nq = c.n_q_heads;
  const int base = (pos0 / 128) * 128;  // the low-term window starts at this chunk
  CUtensorMap m[6];
  dg_status s;
  if ((s = attn_maps(c, ws, kc, vtc, cap, n_q, n_keys, base, m)) != DG_OK) return s;
  dg::TcAttnParams p = attn_params(c, ws, n_q, pos0, n_keys, causal, base);
  p.n_splits = attn_splits(n_q, nq, n_keys, &p.chunks_per_split);
  LAUNCH(DG_K_ATTENTION, st, dg::launch_tc_attention(m[0], m[1], m[2], m[3], m[4], m[5], p, st));
  if (p.n_splits > 1)
    LAUNCH(DG_K_ATTN_MERGE, st,
           dg::launch_attn_merge2(p.part_o, p.part_lse, p.n_splits, nq, n_q, p.out, p.out_lo, st));
  return DG_OK;
}

// attention of n_q new rows at positions pos0.. over cache keys [0, n_keys) -> ws.o (+ ws.o_lo)
dg_status attention(const dg_config& c, const Ws& ws, void* kc, void* vtc, int cap, int n_q, int pos0, int n_keys,
                    int causal, cudaStream_t st) {
  if (is_bf16(c))
    return attn_pair_enabled() ? attention_pair(c, ws, kc, vtc, cap, n_q, pos0, n_keys, causal, st)
                               : attention_single(c, ws, kc, vtc, cap, n_q, pos0, n_keys, causal, st);
  LAUNCH(DG_K_ATTENTION, st,
         dg::launch_simt_attention_f32(ws.at<float>(ws.L.q), (const float*)kc, (const float*)vtc, cap, n_q, pos0,
                                       n_keys, causal, c.n_q_heads, c.n_kv_heads, c.head_dim, ws.at<float>(ws.L.o),
                                       st));
  return DG_OK;
}

// One transformer layer over n rows at positions pos0..  On entry ws.x holds the
// residual stream and ws.xn (+ xn_lo) its RMSNorm; on exit the same for the next layer
// (final: ws.xn single-term, the vocabulary projection's input).
// stop_after_kv: write this layer's K/V and return (last layer of a prefill).
template <typename T>
dg_status layer(dg_model* m, int l, const Ws& ws, void* kc, void* vtc, int cap, int n, int pos0, int causal,
                bool stop_after_kv, bool final_layer, cudaStream_t st) {
  const dg_config& c = m->cfg;
  const dg_layer_weights& W = m->layers[l];
  const int H = c.hidden, nq = c.n_q_heads, nkv = c.n_kv_heads, d = c.head_dim;
  const int E = c.n_experts, k = c.top_k, F = c.expert_ffn, QR = qkv_rows(c);
  const bool bf = is_bf16(c);
  int* err = ws.err();
  T* xn_lo = bf ? ws.at<T>(ws.L.xn_lo) : nullptr;
  dg_status s;
  // ---- attention block: QKV (split-K partials) -> RoPE + K/V into the cache -> attention -> output projection
  int ks_qkv = 1, ks_o = 1;
  if (bf) {
    ks_qkv = pick_ksplit(dense_weight_tiles(QR), ceil_div(n, 128), H / 64, kMaxKsQkv);
    GemmCall g{DG_K_GEMM_QKV, dg::EPI_STORE_F32, &m->maps[l].qkv, nullptr, ws.at<void>(ws.L.xn), xn_lo, n, H, QR,
               nullptr, nullptr, 0, 128, ws.at<float>(ws.L.qkv), nullptr, QR, ks_qkv, (size_t)n * QR, kSmemGemm};
    if ((s = gemm_bf16(g, err, st)) != DG_OK) return s;
  } else {
    LAUNCH(DG_K_GEMM_QKV, st,
           dg::launch_simt_gemm_f32(0, (const float*)W.w_qkv, ws.at<float>(ws.L.xn), nullptr, 1, n, n, QR, H,
                                    ws.at<float>(ws.L.qkv), QR, st));
  }
  LAUNCH(DG_K_ROPE_KV, st,
         dg::launch_rope_scatter<T>(ws.at<float>(ws.L.qkv), ks_qkv, (size_t)n * QR, n, nq, nkv, d, pos0, c.rope_theta,
                                    ws.at<T>(ws.L.q), (T*)kc, (T*)vtc, cap, bf ? ws.at<T>(ws.L.q_lo) : nullptr,
                                    bf ? ws.at<T>(ws.L.k_lo) : nullptr, bf ? ws.at<T>(ws.L.vt_lo) : nullptr,
                                    (pos0 / 128) * 128, ws.L.lo_rows, st));
  if (stop_after_kv) return DG_OK;
  if ((s = attention(c, ws, kc, vtc, cap, n, pos0, pos0 + n, causal, st)) != DG_OK) return s;
  if (bf) {
    ks_o = pick_ksplit(dense_weight_tiles(H), ceil_div(n, 128), nq * d / 64, kMaxKsO);
    GemmCall g{DG_K_GEMM_O, dg::EPI_STORE_F32, &m->maps[l].o, nullptr, ws.at<void>(ws.L.o), ws.at<void>(ws.L.o_lo),
               n, nq * d, H, nullptr, nullptr, 0, 128, ws.at<float>(ws.L.opart), nullptr, H, ks_o, (size_t)n * H,
               kSmemGemm};
    if ((s = gemm_bf16(g, err, st)) != DG_OK) return s;
  } else {
    LAUNCH(DG_K_GEMM_O, st,
           dg::launch_simt_gemm_f32(0, (const float*)W.w_o, ws.at<float>(ws.L.o), nullptr, 1, n, n, H, nq * d,
                                    ws.at<float>(ws.L.opart), H, st));
  }
  // ---- MoE block: residual + RMSNorm + router + top-k -> histogram / permutation -> experts -> combine + RMSNorm
  LAUNCH(DG_K_ROUTER, st,
         dg::launch_router_fused<T>(ws.at<float>(ws.L.x), ws.at<float>(ws.L.opart), ks_o, (size_t)n * H, W.w_router,
                                    n, H, E, k, c.rms_eps, nullptr, ws.at<int32_t>(ws.L.topk_idx),
                                    ws.at<float>(ws.L.topk_w), ws.at<T>(ws.L.xn), xn_lo, st));
  const bool taps = m->taps_on && n <= m->tap_rows;
  if (taps && !m->tap_x_attn.empty() && m->tap_x_attn[l])
    if (cudaMemcpyAsync(m->tap_x_attn[l], ws.at<float>(ws.L.x), (size_t)n * H * 4, cudaMemcpyDeviceToDevice, st) !=
        cudaSuccess)
      return fail(DG_ERR_CUDA, "tap copy failed");
  LAUNCH(DG_K_PERMUTE, st,
         dg::launch_permute(ws.at<int32_t>(ws.L.topk_idx), n, k, E, ws.at<int32_t>(ws.L.counts),
                            ws.at<int32_t>(ws.L.offsets), ws.at<int32_t>(ws.L.perm), ws.at<int32_t>(ws.L.inv),
                            ws.at<int32_t>(ws.L.uni), kItemRows, ws.at<dg::TcWorkItem>(ws.L.items),
                            ws.at<int>(ws.L.n_items), st));
  T* xs_lo = bf ? ws.at<T>(ws.L.xs_lo) : nullptr;
  LAUNCH(DG_K_GATHER, st,
         dg::launch_gather_rows<T>(ws.at<T>(ws.L.xn), xn_lo, ws.at<int32_t>(ws.L.perm), n * k, k, H,
                                   ws.at<T>(ws.L.xs), xs_lo, st));
  const int* off = ws.at<int>(ws.L.offsets);
  if (bf) {
    const dg::TcWorkItem* items = ws.at<dg::TcWorkItem>(ws.L.items);
    const int* n_items = ws.at<int>(ws.L.n_items);
    const int max_items = n * k / kItemRows + E;
    GemmCall gu{DG_K_GEMM_GATE_UP, dg::EPI_SWIGLU_BF16, &m->maps[l].gate, &m->maps[l].up, ws.at<void>(ws.L.xs), xs_lo,
                n * k, H, F, items, n_items, max_items, kItemRows, ws.at<void>(ws.L.h), ws.at<void>(ws.L.h_lo), F, 1, 0,
                kSmemGemm};
    if ((s = gemm_bf16(gu, err, st)) != DG_OK) return s;
    GemmCall dn{DG_K_GEMM_DOWN, dg::EPI_STORE_F32, &m->maps[l].down, nullptr, ws.at<void>(ws.L.h),
                ws.at<void>(ws.L.h_lo), n * k, F, H, items, n_items, max_items, kItemRows, ws.at<float>(ws.L.ys),
                nullptr, H, 1, 0, kSmemGemm};
    if ((s = gemm_bf16(dn, err, st)) != DG_OK) return s;
  } else {
    float* g = ws.at<float>(ws.L.gu);
    float* u = g + (size_t)n * k * F;
    LAUNCH(DG_K_GEMM_GATE_UP, st,
           dg::launch_simt_gemm_f32(0, (const float*)W.w_gate, ws.at<float>(ws.L.xs), off, E, n, n * k, F, H, g, F,
                                    st));
    LAUNCH(DG_K_GEMM_GATE_UP, st,
           dg::launch_simt_gemm_f32(0, (const float*)W.w_up, ws.at<float>(ws.L.xs), off, E, n, n * k, F, H, u, F,
                                    st));
    LAUNCH(DG_K_SWIGLU, st, dg::launch_swiglu_f32(g, u, n * k, F, ws.at<float>(ws.L.h), st));
    LAUNCH(DG_K_GEMM_DOWN, st,
           dg::launch_simt_gemm_f32(0, (const float*)W.w_down, ws.at<float>(ws.L.h), off, E, n, n * k, H, F,
                                    ws.at<float>(ws.L.ys), H, st));
  }
  LAUNCH(DG_K_COMBINE, st,
         dg::launch_combine_norm<T>(ws.at<float>(ws.L.ys), ws.at<int32_t>(ws.L.inv), ws.at<float>(ws.L.topk_w), n, k,
                                    H, c.rms_eps, ws.at<float>(ws.L.x), ws.at<T>(ws.L.xn),
                                    final_layer ? nullptr : xn_lo, st));
  if (taps) {
    auto cp = [&](void* dst, const void* src, size_t bytes) {
      return dst ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st) : cudaSuccess;
    };
    cudaError_t e = cudaSuccess;
    if (!m->tap_x_out.empty()) e = cp(m->tap_x_out[l], ws.at<float>(ws.L.x), (size_t)n * H * 4);
    if (e == cudaSuccess && !m->tap_topk_idx.empty())
      e = cp(m->tap_topk_idx[l], ws.at<int32_t>(ws.L.topk_idx), (size_t)n * k * 4);
    if (e == cudaSuccess && !m->tap_topk_w.empty())
      e = cp(m->tap_topk_w[l], ws.at<float>(ws.L.topk_w), (size_t)n * k * 4);
    if (e == cudaSuccess && !m->tap_counts.empty()) e = cp(m->tap_counts[l], ws.at<int32_t>(ws.L.counts), E * 4);
    if (e == cudaSuccess && !m->tap_perm.empty())
      e = cp(m->tap_perm[l], ws.at<int32_t>(ws.L.perm), (size_t)n * k * 4);
    if (e == cudaSuccess && m->tap_unions) e = cp(m->tap_unions + l, ws.at<int32_t>(ws.L.uni), 4);
    if (e != cudaSuccess) return fail(DG_ERR_CUDA, "tap copy failed: %s", cudaGetErrorString(e));
  }
  return DG_OK;
}

dg_status check_ws(const dg_config& c, void* d_ws, size_t ws_bytes, int n, Ws* ws) {
  DG_CHECK_ARG(d_ws, "workspace is NULL");
  DG_CHECK_ARG((reinterpret_cast<uintptr_t>(d_ws) & 255) == 0, "workspace must be 256-byte aligned");
  ws->base = static_cast<char*>(d_ws);
  ws->L = layout(c, n);
  if (ws_bytes < ws->L.total)
    return fail(DG_ERR_CAPACITY, "workspace too small: %zu < %zu bytes", ws_bytes, ws->L.total);
  return DG_OK;
}

dg_status check_cache(const dg_config& c, const dg_kv_cache* cache) {
  DG_CHECK_ARG(cache && cache->k && cache->vt, "cache is NULL");
  DG_CHECK_ARG(cache->capacity > 0 && cache->capacity % 8 == 0, "cache capacity must be a positive multiple of 8");
  DG_CHECK_ARG(cache->len >= 0 && cache->len <= cache->capacity, "cache len out of range");
  for (int l = 0; l < c.n_layers; ++l) {
    DG_CHECK_ARG(cache->k[l] && cache->vt[l], "cache layer %d is NULL", l);
    DG_CHECK_ARG((reinterpret_cast<uintptr_t>(cache->k[l]) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(cache->vt[l]) & 15) == 0,
                 "cache buffers must be 16-byte aligned");
  }
  return DG_OK;
}

// prefill: causal, the last layer stops after its K/V; denoise: bidirectional, the last
// layer leaves the vocabulary projection's input in ws.xn
template <typename T>
dg_status run_stack(dg_model* m, const dg_kv_cache* cache, const int32_t* tokens, int n, bool prefill, const Ws& ws,
                    cudaStream_t st) {
  const dg_config& c = m->cfg;
  const int pos0 = cache->len;
  T* xn_lo = is_bf16(c) ? ws.at<T>(ws.L.xn_lo) : nullptr;
  LAUNCH(DG_K_EMBED_NORM, st,
         dg::launch_embed_norm<T>(tokens, (const T*)m->embed, n, c.vocab, c.hidden, c.rms_eps, ws.at<float>(ws.L.x),
                                  ws.at<T>(ws.L.xn), xn_lo, ws.err(), st));
  for (int l = 0; l < c.n_layers; ++l) {
    const bool last = l == c.n_layers - 1;
    dg_status s = layer<T>(m, l, ws, cache->k[l], cache->vt[l], cache->capacity, n, pos0, prefill ? 1 : 0,
                           last && prefill, last && !prefill, st);
    if (s != DG_OK) return s;
  }
  return DG_OK;
}

// ---- several canvases in one pass
// Canvas b occupies rows [b C, (b + 1) C) of every row-wise buffer and reads and writes
// only its own cache; all rows share one router / permutation / expert GEMM / vocabulary
// projection, so an expert's weights are read once for the whole batch.
//
// layer_batched repeats layer()'s sequence with a loop over canvases around RoPE and
// attention, and the low-precision experts.  The copy is deliberate: the single-canvas
// sequence stays exactly as measured and validated until this one has run on a GPU;
// then layer() becomes layer_batched with one canvas and the copy goes.
struct Seg {
  void* kc;
  void* vtc;
  int cap;
  int pos0;  // the canvas's cache length
};

// A view of the workspace whose q / o buffers start at canvas b's slice: q is head-major
// [nq][C][d] per canvas, o row-major [C][nq d], so both slices are contiguous.
Ws canvas_view(const dg_config& c, const Ws& ws, int b, int C) {
  Ws wb = ws;
  const size_t qo = (size_t)b * c.n_q_heads * C * c.head_dim;  // elements before canvas b (q and o alike)
  wb.L.q += qo * act_bytes(c);
  wb.L.o += qo * act_bytes(c);
  if (is_bf16(c)) {
    wb.L.q_lo += qo * 2;
    wb.L.o_lo += qo * 2;
  }
  return wb;
}

template <typename T>
dg_status layer_batched(dg_model* m, int l, const Ws& ws, const std::vector<Seg>& segs, int C, int causal,
                        bool stop_after_kv, bool final_layer, cudaStream_t st) {
  const dg_config& c = m->cfg;
  const dg_layer_weights& W = m->layers[l];
  const int H = c.hidden, nq = c.n_q_heads, nkv = c.n_kv_heads, d = c.head_dim;
  const int E = c.n_experts, k = c.top_k, F = c.expert_ffn, QR = qkv_rows(c);
  const int n = (int)segs.size() * C;
  const bool bf = is_bf16(c);
  int* err = ws.err();
  T* xn_lo = bf ? ws.at<T>(ws.L.xn_lo) : nullptr;
  dg_status s;
  int ks_qkv = 1, ks_o = 1;
  if (bf) {
    ks_qkv = pick_ksplit(dense_weight_tiles(QR), ceil_div(n, 128), H / 64, kMaxKsQkv);
    GemmCall g{DG_K_GEMM_QKV, dg::EPI_STORE_F32, &m->maps[l].qkv, nullptr, ws.at<void>(ws.L.xn), xn_lo, n, H, QR,
               nullptr, nullptr, 0, 128, ws.at<float>(ws.L.qkv), nullptr, QR, ks_qkv, (size_t)n * QR, kSmemGemm};
    if ((s = gemm_bf16(g, err, st)) != DG_OK) return s;
  } else {
    LAUNCH(DG_K_GEMM_QKV, st,
           dg::launch_simt_gemm_f32(0, (const float*)W.w_qkv, ws.at<float>(ws.L.xn), nullptr, 1, n, n, QR, H,
                                    ws.at<float>(ws.L.qkv), QR, st));
  }
  // per canvas: RoPE at its own positions, K/V into its own cache, attention over its own
  // keys (the low-term window and the split-KV partials are reused canvas after canvas)
  for (int b = 0; b < (int)segs.size(); ++b) {
    const Seg& g = segs[b];
    const Ws wb = canvas_view(c, ws, b, C);
    LAUNCH(DG_K_ROPE_KV, st,
           dg::launch_rope_scatter<T>(ws.at<float>(ws.L.qkv) + (size_t)b * C * QR, ks_qkv, (size_t)n * QR, C, nq, nkv,
                                      d, g.pos0, c.rope_theta, wb.at<T>(wb.L.q), (T*)g.kc, (T*)g.vtc, g.cap,
                                      bf ? wb.at<T>(wb.L.q_lo) : nullptr, bf ? ws.at<T>(ws.L.k_lo) : nullptr,
                                      bf ? ws.at<T>(ws.L.vt_lo) : nullptr, (g.pos0 / 128) * 128, ws.L.lo_rows, st));
    if (stop_after_kv) continue;
    if ((s = attention(c, wb, g.kc, g.vtc, g.cap, C, g.pos0, g.pos0 + C, causal, st)) != DG_OK) return s;
  }
  if (stop_after_kv) return DG_OK;
  if (bf) {
    ks_o = pick_ksplit(dense_weight_tiles(H), ceil_div(n, 128), nq * d / 64, kMaxKsO);
    GemmCall g{DG_K_GEMM_O, dg::EPI_STORE_F32, &m->maps[l].o, nullptr, ws.at<void>(ws.L.o), ws.at<void>(ws.L.o_lo),
               n, nq * d, H, nullptr, nullptr, 0, 128, ws.at<float>(ws.L.opart), nullptr, H, ks_o, (size_t)n * H,
               kSmemGemm};
    if ((s = gemm_bf16(g, err, st)) != DG_OK) return s;
  } else {
    LAUNCH(DG_K_GEMM_O, st,
           dg::launch_simt_gemm_f32(0, (const float*)W.w_o, ws.at<float>(ws.L.o), nullptr, 1, n, n, H, nq * d,
                                    ws.at<float>(ws.L.opart), H, st));
  }
  LAUNCH(DG_K_ROUTER, st,
         dg::launch_router_fused<T>(ws.at<float>(ws.L.x), ws.at<float>(ws.L.opart), ks_o, (size_t)n * H, W.w_router,
                                    n, H, E, k, c.rms_eps, nullptr, ws.at<int32_t>(ws.L.topk_idx),
                                    ws.at<float>(ws.L.topk_w), ws.at<T>(ws.L.xn), xn_lo, st));
  const bool taps = m->taps_on && n <= m->tap_rows;
  if (taps && !m->tap_x_attn.empty() && m->tap_x_attn[l])
    if (cudaMemcpyAsync(m->tap_x_attn[l], ws.at<float>(ws.L.x), (size_t)n * H * 4, cudaMemcpyDeviceToDevice, st) !=
        cudaSuccess)
      return fail(DG_ERR_CUDA, "tap copy failed");
  const bool lowp = bf && !m->lowp.empty();
  const int item_rows = lowp ? kItemRowsMx8 : kItemRows;
  LAUNCH(DG_K_PERMUTE, st,
         dg::launch_permute(ws.at<int32_t>(ws.L.topk_idx), n, k, E, ws.at<int32_t>(ws.L.counts),
                            ws.at<int32_t>(ws.L.offsets), ws.at<int32_t>(ws.L.perm), ws.at<int32_t>(ws.L.inv),
                            ws.at<int32_t>(ws.L.uni), item_rows, ws.at<dg::TcWorkItem>(ws.L.items),
                            ws.at<int>(ws.L.n_items), st));
  T* xs_lo = bf ? ws.at<T>(ws.L.xs_lo) : nullptr;
  LAUNCH(DG_K_GATHER, st,
         dg::launch_gather_rows<T>(ws.at<T>(ws.L.xn), xn_lo, ws.at<int32_t>(ws.L.perm), n * k, k, H,
                                   ws.at<T>(ws.L.xs), xs_lo, st));
  const int* off = ws.at<int>(ws.L.offsets);
  if (lowp) {
    const dg::TcWorkItem* items = ws.at<dg::TcWorkItem>(ws.L.items);
    const int* n_items = ws.at<int>(ws.L.n_items);
    const int max_items = n * k / kItemRowsMx8 + E;
    const LowpMaps& X8 = m->lowp[l];
    GemmCall gu{DG_K_GEMM_GATE_UP, dg::EPI_SWIGLU_BF16, &X8.gate, &X8.up, ws.at<void>(ws.L.xs), xs_lo, n * k, H, F,
                items, n_items, max_items, kItemRowsMx8, ws.at<void>(ws.L.h), ws.at<void>(ws.L.h_lo), F, 1, 0,
                kSmemGemm};
    if ((s = gemm_lowp(gu, X8.fmt, &X8.gate_s, &X8.up_s, X8.g_gate, X8.g_up, err, st)) != DG_OK) return s;
    GemmCall dn{DG_K_GEMM_DOWN, dg::EPI_STORE_F32, &X8.down, nullptr, ws.at<void>(ws.L.h), ws.at<void>(ws.L.h_lo),
                n * k, F, H, items, n_items, max_items, kItemRowsMx8, ws.at<float>(ws.L.ys), nullptr, H, 1, 0,
                kSmemGemm};
    if ((s = gemm_lowp(dn, X8.fmt, &X8.down_s, nullptr, X8.g_down, 1.0f, err, st)) != DG_OK) return s;
  } else if (bf) {
    const dg::TcWorkItem* items = ws.at<dg::TcWorkItem>(ws.L.items);
    const int* n_items = ws.at<int>(ws.L.n_items);
    const int max_items = n * k / kItemRows + E;
    GemmCall gu{DG_K_GEMM_GATE_UP, dg::EPI_SWIGLU_BF16, &m->maps[l].gate, &m->maps[l].up, ws.at<void>(ws.L.xs), xs_lo,
                n * k, H, F, items, n_items, max_items, kItemRows, ws.at<void>(ws.L.h), ws.at<void>(ws.L.h_lo), F, 1, 0,
                kSmemGemm};
    if ((s = gemm_bf16(gu, err, st)) != DG_OK) return s;
    GemmCall dn{DG_K_GEMM_DOWN, dg::EPI_STORE_F32, &m->maps[l].down, nullptr, ws.at<void>(ws.L.h),
                ws.at<void>(ws.L.h_lo), n * k, F, H, items, n_items, max_items, kItemRows, ws.at<float>(ws.L.ys),
                nullptr, H, 1, 0, kSmemGemm};
    if ((s = gemm_bf16(dn, err, st)) != DG_OK) return s;
  } else {
    float* g = ws.at<float>(ws.L.gu);
    float* u = g + (size_t)n * k * F;
    LAUNCH(DG_K_GEMM_GATE_UP, st,
           dg::launch_simt_gemm_f32(0, (const float*)W.w_gate, ws.at<float>(ws.L.xs), off, E, n, n * k, F, H, g, F,
                                    st));
    LAUNCH(DG_K_GEMM_GATE_UP, st,
           dg::launch_simt_gemm_f32(0, (const float*)W.w_up, ws.at<float>(ws.L.xs), off, E, n, n * k, F, H, u, F,
                                    st));
    LAUNCH(DG_K_SWIGLU, st, dg::launch_swiglu_f32(g, u, n * k, F, ws.at<float>(ws.L.h), st));
    LAUNCH(DG_K_GEMM_DOWN, st,
           dg::launch_simt_gemm_f32(0, (const float*)W.w_down, ws.at<float>(ws.L.h), off, E, n, n * k, H, F,
                                    ws.at<float>(ws.L.ys), H, st));
  }
  LAUNCH(DG_K_COMBINE, st,
         dg::launch_combine_norm<T>(ws.at<float>(ws.L.ys), ws.at<int32_t>(ws.L.inv), ws.at<float>(ws.L.topk_w), n, k,
                                    H, c.rms_eps, ws.at<float>(ws.L.x), ws.at<T>(ws.L.xn),
                                    final_layer ? nullptr : xn_lo, st));
  if (taps) {
    auto cp = [&](void* dst, const void* src, size_t bytes) {
      return dst ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st) : cudaSuccess;
    };
    cudaError_t e = cudaSuccess;
    if (!m->tap_x_out.empty()) e = cp(m->tap_x_out[l], ws.at<float>(ws.L.x), (size_t)n * H * 4);
    if (e == cudaSuccess && !m->tap_topk_idx.empty())
      e = cp(m->tap_topk_idx[l], ws.at<int32_t>(ws.L.topk_idx), (size_t)n * k * 4);
    if (e == cudaSuccess && !m->tap_topk_w.empty())
      e = cp(m->tap_topk_w[l], ws.at<float>(ws.L.topk_w), (size_t)n * k * 4);
    if (e == cudaSuccess && !m->tap_counts.empty()) e = cp(m->tap_counts[l], ws.at<int32_t>(ws.L.counts), E * 4);
    if (e == cudaSuccess && !m->tap_perm.empty())
      e = cp(m->tap_perm[l], ws.at<int32_t>(ws.L.perm), (size_t)n * k * 4);
    if (e == cudaSuccess && m->tap_unions) e = cp(m->tap_unions + l, ws.at<int32_t>(ws.L.uni), 4);
    if (e != cudaSuccess) return fail(DG_ERR_CUDA, "tap copy failed: %s", cudaGetErrorString(e));
  }
  return DG_OK;
}

template <typename T>
dg_status run_stack_batched(dg_model* m, const dg_kv_cache* caches, int B, const int32_t* tokens, int C, bool prefill,
                            const Ws& ws, cudaStream_t st) {
  const dg_config& c = m->cfg;
  const int n = B * C;
  T* xn_lo = is_bf16(c) ? ws.at<T>(ws.L.xn_lo) : nullptr;
  LAUNCH(DG_K_EMBED_NORM, st,
         dg::launch_embed_norm<T>(tokens, (const T*)m->embed, n, c.vocab, c.hidden, c.rms_eps, ws.at<float>(ws.L.x),
                                  ws.at<T>(ws.L.xn), xn_lo, ws.err(), st));
  std::vector<Seg> segs(B);
  for (int l = 0; l < c.n_layers; ++l) {
    for (int b = 0; b < B; ++b) segs[b] = Seg{caches[b].k[l], caches[b].vt[l], caches[b].capacity, caches[b].len};
    const bool last = l == c.n_layers - 1;
    dg_status s = layer_batched<T>(m, l, ws, segs, C, prefill ? 1 : 0, last && prefill, last && !prefill, st);
    if (s != DG_OK) return s;
  }
  return DG_OK;
}

// the caches of a batch: each valid, with room for C more positions, none shared
dg_status check_caches(const dg_config& c, const dg_kv_cache* caches, int B, int C) {
  DG_CHECK_ARG(caches && B >= 1, "caches NULL or B < 1");
  for (int b = 0; b < B; ++b) {
    dg_status s = check_cache(c, &caches[b]);
    if (s != DG_OK) return s;
    if ((int64_t)caches[b].len + C > caches[b].capacity)
      return fail(DG_ERR_CAPACITY, "cache %d has no room for the canvas: len %d + C %d > capacity %d", b,
                  caches[b].len, C, caches[b].capacity);
    for (int b2 = 0; b2 < b; ++b2)
      for (int l = 0; l < c.n_layers; ++l)
        DG_CHECK_ARG(caches[b].k[l] != caches[b2].k[l] && caches[b].vt[l] != caches[b2].vt[l],
                     "caches %d and %d share layer %d's buffers", b2, b, l);
  }
  return DG_OK;
}

}  // namespace

extern "C" dg_status dg_prefill_append(dg_model* m, dg_kv_cache* cache, const int32_t* d_tokens, int32_t T,
                                       void* d_ws, size_t ws_bytes, dg_stream stream) {
  DG_CHECK_ARG(m, "model is NULL");
  dg_status s = check_cache(m->cfg, cache);
  if (s != DG_OK) return s;
  DG_CHECK_ARG(d_tokens && T > 0, "tokens NULL or T <= 0");
  if ((int64_t)cache->len + T > cache->capacity)
    return fail(DG_ERR_CAPACITY, "cache overflow: len %d + T %d > capacity %d", cache->len, T, cache->capacity);
  Ws ws;
  if ((s = check_ws(m->cfg, d_ws, ws_bytes, T, &ws)) != DG_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  s = is_bf16(m->cfg) ? run_stack<bf16>(m, cache, d_tokens, T, true, ws, st)
                      : run_stack<float>(m, cache, d_tokens, T, true, ws, st);
  if (s != DG_OK) return s;
  cache->len += T;
  return DG_OK;
}

extern "C" dg_status dg_denoise_pass(dg_model* m, const dg_kv_cache* cache, const int32_t* d_canvas, int32_t C,
                                     float* d_logits, void* d_ws, size_t ws_bytes, dg_stream stream) {
  DG_CHECK_ARG(m, "model is NULL");
  dg_status s = check_cache(m->cfg, cache);
  if (s != DG_OK) return s;
  DG_CHECK_ARG(d_canvas && d_logits && C > 0, "canvas / logits NULL or C <= 0");
  if ((int64_t)cache->len + C > cache->capacity)
    return fail(DG_ERR_CAPACITY, "cache has no room for the canvas: len %d + C %d > capacity %d", cache->len, C,
                cache->capacity);
  Ws ws;
  if ((s = check_ws(m->cfg, d_ws, ws_bytes, C, &ws)) != DG_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const dg_config& c = m->cfg;
  s = is_bf16(c) ? run_stack<bf16>(m, cache, d_canvas, C, false, ws, st)
                 : run_stack<float>(m, cache, d_canvas, C, false, ws, st);
  if (s != DG_OK) return s;
  // vocabulary projection of the final RMSNorm (left in ws.xn by the last layer) to fp32 logits
  if (is_bf16(c)) {
    GemmCall g{DG_K_GEMM_VOCAB, dg::EPI_STORE_F32, &m->out_map, nullptr, ws.at<void>(ws.L.xn), nullptr, C, c.hidden,
               c.vocab, nullptr, nullptr, 0, 256, d_logits, nullptr, c.vocab, 1, 0, kSmemGemm};
    if ((s = gemm_bf16(g, ws.err(), st)) != DG_OK) return s;
  } else {
    LAUNCH(DG_K_GEMM_VOCAB, st,
           dg::launch_simt_gemm_f32(0, (const float*)m->w_out, ws.at<float>(ws.L.xn), nullptr, 1, C, C, c.vocab,
                                    c.hidden, d_logits, c.vocab, st));
  }
  return DG_OK;
}

extern "C" dg_status dg_denoise_update(dg_model* m, const dg_kv_cache* cache, int32_t* d_canvas, int32_t C, int32_t n,
                                       uint64_t seed, uint32_t step, int32_t mask_id, float* d_conf, void* d_ws,
                                       size_t ws_bytes, dg_stream stream) {
  DG_CHECK_ARG(m, "model is NULL");
  if (!is_bf16(m->cfg)) return fail(DG_ERR_UNSUPPORTED, "the fused update runs on the tcgen05 path (bf16 models)");
  dg_status s = check_cache(m->cfg, cache);
  if (s != DG_OK) return s;
  DG_CHECK_ARG(d_canvas, "canvas is NULL");
  DG_CHECK_ARG(C > 0 && C <= 1024, "C must be in [1, 1024]");
  DG_CHECK_ARG(n >= 0 && n <= C, "n must be in [0, C]");
  DG_CHECK_ARG(mask_id < m->cfg.vocab, "mask_id must be < vocab (negative: the re-noising update)");
  if ((int64_t)cache->len + C > cache->capacity)
    return fail(DG_ERR_CAPACITY, "cache has no room for the canvas: len %d + C %d > capacity %d", cache->len, C,
                cache->capacity);
  Ws ws;
  if ((s = check_ws(m->cfg, d_ws, ws_bytes, C, &ws)) != DG_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const dg_config& c = m->cfg;
  if ((s = run_stack<bf16>(m, cache, d_canvas, C, false, ws, st)) != DG_OK) return s;
  CUtensorMap B, Bb;
  if ((s = map_rows(&B, ws.at<void>(ws.L.xn), (uint64_t)C, (uint64_t)c.hidden, 16)) != DG_OK) return s;
  if ((s = map_rows(&Bb, ws.at<void>(ws.L.xn), (uint64_t)C, (uint64_t)c.hidden, 64)) != DG_OK) return s;
  dg::VuParams p{};
  p.K = c.hidden;
  p.V = c.vocab;
  p.m_tiles = ceil_div(c.vocab, 128);
  p.n_max = C < 256 ? ((C + 15) & ~15) : 256;
  p.n_tokens = C;
  p.excl = mask_id < 0 ? -1 : mask_id;
  p.part = ws.at<dg::UpdPart>(ws.L.vtiles);
  p.smem_budget = kSmemGemm;
  p.err = ws.err();
  dg::UpdPart* rows = ws.at<dg::UpdPart>(ws.L.upd);
  LAUNCH(DG_K_GEMM_VOCAB, st, dg::launch_vocab_update(m->out_map, B, Bb, p, st));
  LAUNCH(DG_K_UPDATE_PARTIAL, st, dg::launch_upd_merge_rows(p.part, C, p.m_tiles, rows, st));
  LAUNCH(DG_K_UPDATE_SELECT, st,
         dg::launch_update_select(rows, C, c.vocab, 1, n, seed, step, d_canvas, d_conf, mask_id < 0 ? -1 : mask_id,
                                  st));
  return DG_OK;
}

extern "C" dg_status dg_canvas_update(const float* d_logits, int32_t C, int32_t V, int32_t n_renoise, uint64_t seed,
                                      uint32_t step, int32_t* d_canvas, float* d_conf, void* d_ws, size_t ws_bytes,
                                      dg_stream stream) {
  DG_CHECK_ARG(d_logits && d_canvas && d_ws, "logits / canvas / workspace is NULL");
  DG_CHECK_ARG(C > 0 && C <= 1024, "C must be in [1, 1024]");
  DG_CHECK_ARG(V > 0 && V % 4 == 0, "V must be a positive multiple of 4");
  DG_CHECK_ARG(n_renoise >= 0 && n_renoise <= C, "n_renoise must be in [0, C]");
  DG_CHECK_ARG((reinterpret_cast<uintptr_t>(d_logits) & 15) == 0, "logits must be 16-byte aligned");
  DG_CHECK_ARG((reinterpret_cast<uintptr_t>(d_ws) & 255) == 0, "workspace must be 256-byte aligned");
  if (ws_bytes < dg_update_workspace_bytes(C, V))
    return fail(DG_ERR_CAPACITY, "workspace too small for the update: %zu < %zu", ws_bytes,
                dg_update_workspace_bytes(C, V));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  dg::UpdPart* part = reinterpret_cast<dg::UpdPart*>(static_cast<char*>(d_ws) + 256);
  const int splits = dg::update_splits(C, V);
  LAUNCH(DG_K_UPDATE_PARTIAL, st, dg::launch_update_partial(d_logits, C, V, splits, -1, part, st));
  LAUNCH(DG_K_UPDATE_SELECT, st,
         dg::launch_update_select(part, C, V, splits, n_renoise, seed, step, d_canvas, d_conf, -1, st));
  return DG_OK;
}

extern "C" dg_status dg_canvas_update_masked(const float* d_logits, int32_t C, int32_t V, int32_t n_keep,
                                             int32_t mask_id, int32_t* d_canvas, float* d_conf, void* d_ws,
                                             size_t ws_bytes, dg_stream stream) {
  DG_CHECK_ARG(d_logits && d_canvas && d_ws, "logits / canvas / workspace is NULL");
  DG_CHECK_ARG(C > 0 && C <= 1024, "C must be in [1, 1024]");
  DG_CHECK_ARG(V > 1 && V % 4 == 0, "V must be a multiple of 4 and > 1");
  DG_CHECK_ARG(mask_id >= 0 && mask_id < V, "mask_id must be in [0, V)");
  DG_CHECK_ARG(n_keep >= 0 && n_keep <= C, "n_keep must be in [0, C]");
  DG_CHECK_ARG((reinterpret_cast<uintptr_t>(d_logits) & 15) == 0, "logits must be 16-byte aligned");
  DG_CHECK_ARG((reinterpret_cast<uintptr_t>(d_ws) & 255) == 0, "workspace must be 256-byte aligned");
  if (ws_bytes < dg_update_workspace_bytes(C, V))
    return fail(DG_ERR_CAPACITY, "workspace too small for the update: %zu < %zu", ws_bytes,
                dg_update_workspace_bytes(C, V));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  dg::UpdPart* part = reinterpret_cast<dg::UpdPart*>(static_cast<char*>(d_ws) + 256);
  const int splits = dg::update_splits(C, V);
  LAUNCH(DG_K_UPDATE_PARTIAL, st, dg::launch_update_partial(d_logits, C, V, splits, mask_id, part, st));
  LAUNCH(DG_K_UPDATE_SELECT, st,
         dg::launch_update_select(part, C, V, splits, n_keep, 0, 0, d_canvas, d_conf, mask_id, st));
  return DG_OK;
}

// Everything the passes, updates and the append of a generation call check, checked
// before the first launch so that a rejected call launches nothing.
static dg_status check_generate_args(dg_model* m, const dg_kv_cache* cache, const int32_t* d_canvas, int32_t C,
                                     const float* d_logits, void* d_ws, size_t ws_bytes) {
  DG_CHECK_ARG(d_canvas && d_logits, "canvas / logits is NULL");
  DG_CHECK_ARG(C > 0 && C <= 1024, "C must be in [1, 1024]");
  DG_CHECK_ARG((reinterpret_cast<uintptr_t>(d_logits) & 15) == 0, "logits must be 16-byte aligned");
  dg_status s = check_cache(m->cfg, cache);
  if (s != DG_OK) return s;
  if ((int64_t)cache->len + C > cache->capacity)
    return fail(DG_ERR_CAPACITY, "cache has no room for the canvas: len %d + C %d > capacity %d", cache->len, C,
                cache->capacity);
  Ws ws;
  return check_ws(m->cfg, d_ws, ws_bytes, C, &ws);
}

static int renoise_count(int C, int S, int s, double r0, double r1) {
  const double f = (S == 1) ? r0 : (r0 * (S - 1 - s) + r1 * s) / (double)(S - 1);
  return (int)floor((double)C * f + 1e-9);
}
extern "C" int32_t dg_renoise_count(int32_t C, int32_t S, int32_t step, float r_start, float r_end) {
  if (C < 0 || S < 1 || step < 0 || step >= S) return -1;
  return renoise_count(C, S, step, r_start, r_end);
}

extern "C" dg_status dg_generate_canvas(dg_model* m, dg_kv_cache* cache, int32_t* d_canvas, int32_t C, int32_t S,
                                        float r_start, float r_end, uint64_t seed, int32_t append, float* d_logits,
                                        void* d_ws, size_t ws_bytes, dg_stream stream) {
  DG_CHECK_ARG(m, "model is NULL");
  DG_CHECK_ARG(S >= 1, "S must be >= 1");
  DG_CHECK_ARG(r_start >= 0.f && r_start <= 1.f && r_end >= 0.f && r_end <= 1.f, "re-noise fractions must be in [0,1]");
  dg_status s = check_generate_args(m, cache, d_canvas, C, d_logits, d_ws, ws_bytes);
  if (s != DG_OK) return s;
  for (int step = 0; step < S; ++step) {
    if ((s = dg_denoise_pass(m, cache, d_canvas, C, d_logits, d_ws, ws_bytes, stream)) != DG_OK) return s;
    const int n = renoise_count(C, S, step, r_start, r_end);
    if ((s = dg_canvas_update(d_logits, C, m->cfg.vocab, n, seed, (uint32_t)step, d_canvas, nullptr, d_ws, ws_bytes,
                              stream)) != DG_OK)
      return s;
  }
  if (append) return dg_prefill_append(m, cache, d_canvas, C, d_ws, ws_bytes, stream);
  return DG_OK;
}

extern "C" dg_status dg_generate_canvas_masked(dg_model* m, dg_kv_cache* cache, int32_t* d_canvas, int32_t C,
                                               int32_t S, float keep_start, float keep_end, int32_t mask_id,
                                               int32_t append, float* d_logits, void* d_ws, size_t ws_bytes,
                                               dg_stream stream) {
  DG_CHECK_ARG(m, "model is NULL");
  DG_CHECK_ARG(S >= 1, "S must be >= 1");
  DG_CHECK_ARG(keep_start >= 0.f && keep_start <= 1.f && keep_end >= 0.f && keep_end <= 1.f,
               "keep fractions must be in [0,1]");
  DG_CHECK_ARG(mask_id >= 0 && mask_id < m->cfg.vocab, "mask_id must be in [0, vocab)");
  dg_status s = check_generate_args(m, cache, d_canvas, C, d_logits, d_ws, ws_bytes);
  if (s != DG_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  LAUNCH(DG_K_UPDATE_SELECT, st, dg::launch_fill_i32(d_canvas, C, mask_id, st));
  for (int step = 0; step < S; ++step) {
    if ((s = dg_denoise_pass(m, cache, d_canvas, C, d_logits, d_ws, ws_bytes, stream)) != DG_OK) return s;
    const int n = renoise_count(C, S, step, keep_start, keep_end);
    if ((s = dg_canvas_update_masked(d_logits, C, m->cfg.vocab, n, mask_id, d_canvas, nullptr, d_ws, ws_bytes,
                                     stream)) != DG_OK)
      return s;
  }
  if (append) return dg_prefill_append(m, cache, d_canvas, C, d_ws, ws_bytes, stream);
  return DG_OK;
}

extern "C" dg_status dg_prefill_append_batched(dg_model* m, dg_kv_cache* caches, int32_t B, const int32_t* d_tokens,
                                               int32_t T, void* d_ws, size_t ws_bytes, dg_stream stream) {
  DG_CHECK_ARG(m, "model is NULL");
  DG_CHECK_ARG(d_tokens && T > 0, "tokens NULL or T <= 0");
  DG_CHECK_ARG(B >= 1 && (int64_t)B * T <= (1 << 20), "B must be >= 1 and B * T <= 2^20");
  dg_status s = check_caches(m->cfg, caches, B, T);
  if (s != DG_OK) return s;
  Ws ws;
  if ((s = check_ws(m->cfg, d_ws, ws_bytes, B * T, &ws)) != DG_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  s = is_bf16(m->cfg) ? run_stack_batched<bf16>(m, caches, B, d_tokens, T, true, ws, st)
                      : run_stack_batched<float>(m, caches, B, d_tokens, T, true, ws, st);
  if (s != DG_OK) return s;
  for (int b = 0; b < B; ++b) caches[b].len += T;
  return DG_OK;
}

extern "C" dg_status dg_denoise_pass_batched(dg_model* m, const dg_kv_cache* caches, int32_t B,
                                             const int32_t* d_canvases, int32_t C, float* d_logits, void* d_ws,
                                             size_t ws_bytes, dg_stream stream) {
  DG_CHECK_ARG(m, "model is NULL");
  DG_CHECK_ARG(d_canvases && d_logits && C > 0, "canvases / logits NULL or C <= 0");
  DG_CHECK_ARG(B >= 1 && (int64_t)B * C <= (1 << 20), "B must be >= 1 and B * C <= 2^20");
  dg_status s = check_caches(m->cfg, caches, B, C);
  if (s != DG_OK) return s;
  Ws ws;
  if ((s = check_ws(m->cfg, d_ws, ws_bytes, B * C, &ws)) != DG_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const dg_config& c = m->cfg;
  const int n = B * C;
  s = is_bf16(c) ? run_stack_batched<bf16>(m, caches, B, d_canvases, C, false, ws, st)
                 : run_stack_batched<float>(m, caches, B, d_canvases, C, false, ws, st);
  if (s != DG_OK) return s;
  if (is_bf16(c) && m->vocab_lowp.on) {
    // dense low-precision GEMM: tokens in chunks of up to 128 (each chunk decodes the weight
    // tiles again, so fewer chunks mean less decode work), tiles weight tile major
    const VocabLowp& Vl = m->vocab_lowp;
    const int chunk = n <= 64 ? ((n + 15) & ~15) : 128;
    GemmCall g{DG_K_GEMM_VOCAB, dg::EPI_STORE_F32, &Vl.codes, nullptr, ws.at<void>(ws.L.xn), nullptr, n, c.hidden,
               c.vocab, nullptr, nullptr, ceil_div(n, chunk), chunk, d_logits, nullptr, c.vocab, 1, 0, kSmemGemm};
    if ((s = gemm_lowp(g, Vl.fmt, &Vl.scales, nullptr, Vl.g, 1.0f, ws.err(), st)) != DG_OK) return s;
  } else if (is_bf16(c)) {
    GemmCall g{DG_K_GEMM_VOCAB, dg::EPI_STORE_F32, &m->out_map, nullptr, ws.at<void>(ws.L.xn), nullptr, n, c.hidden,
               c.vocab, nullptr, nullptr, 0, 256, d_logits, nullptr, c.vocab, 1, 0, kSmemGemm};
    if ((s = gemm_bf16(g, ws.err(), st)) != DG_OK) return s;
  } else {
    LAUNCH(DG_K_GEMM_VOCAB, st,
           dg::launch_simt_gemm_f32(0, (const float*)m->w_out, ws.at<float>(ws.L.xn), nullptr, 1, n, n, c.vocab,
                                    c.hidden, d_logits, c.vocab, st));
  }
  return DG_OK;
}

extern "C" dg_status dg_generate_canvases(dg_model* m, dg_kv_cache* caches, int32_t B, int32_t* d_canvases, int32_t C,
                                          int32_t S, float r_start, float r_end, const uint64_t* seeds,
                                          int32_t append, float* d_logits, void* d_ws, size_t ws_bytes,
                                          dg_stream stream) {
  DG_CHECK_ARG(m, "model is NULL");
  DG_CHECK_ARG(S >= 1, "S must be >= 1");
  DG_CHECK_ARG(r_start >= 0.f && r_start <= 1.f && r_end >= 0.f && r_end <= 1.f, "re-noise fractions must be in [0,1]");
  DG_CHECK_ARG(seeds, "seeds is NULL");
  DG_CHECK_ARG(d_canvases && d_logits, "canvases / logits is NULL");
  DG_CHECK_ARG(C > 0 && C <= 1024, "C must be in [1, 1024]");
  DG_CHECK_ARG(B >= 1 && (int64_t)B * C <= (1 << 20), "B must be >= 1 and B * C <= 2^20");
  DG_CHECK_ARG((reinterpret_cast<uintptr_t>(d_logits) & 15) == 0, "logits must be 16-byte aligned");
  dg_status s = check_caches(m->cfg, caches, B, C);
  if (s != DG_OK) return s;
  Ws ws;
  if ((s = check_ws(m->cfg, d_ws, ws_bytes, B * C, &ws)) != DG_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int V = m->cfg.vocab, n = B * C;
  const int splits = dg::update_splits(n, V);
  dg::UpdPart* part = ws.at<dg::UpdPart>(ws.L.upd);
  for (int step = 0; step < S; ++step) {
    if ((s = dg_denoise_pass_batched(m, caches, B, d_canvases, C, d_logits, d_ws, ws_bytes, stream)) != DG_OK)
      return s;
    const int nr = renoise_count(C, S, step, r_start, r_end);
    // row statistics of all B C rows at once, then each canvas's own re-noise set
    LAUNCH(DG_K_UPDATE_PARTIAL, st, dg::launch_update_partial(d_logits, n, V, splits, -1, part, st));
    for (int b = 0; b < B; ++b)
      LAUNCH(DG_K_UPDATE_SELECT, st,
             dg::launch_update_select(part + (size_t)b * C * splits, C, V, splits, nr, seeds[b], (uint32_t)step,
                                      d_canvases + (size_t)b * C, nullptr, -1, st));
  }
  if (append) return dg_prefill_append_batched(m, caches, B, d_canvases, C, d_ws, ws_bytes, stream);
  return DG_OK;
}

static dg_status set_experts_lowp(dg_model* m, int fmt, const dg_expert_weights_mx8* layers, const float* g3) {
  DG_CHECK_ARG(m, "model is NULL");
  if (!layers) {
    m->lowp.clear();
    return DG_OK;
  }
  const dg_config& c = m->cfg;
  DG_CHECK_ARG(is_bf16(c), "low-precision experts need a bf16 model");
  auto a16 = [](const void* q) { return q && (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  for (int l = 0; l < c.n_layers; ++l) {
    const dg_expert_weights_mx8& X = layers[l];
    DG_CHECK_ARG(a16(X.gate) && a16(X.gate_scales) && a16(X.up) && a16(X.up_scales) && a16(X.down) &&
                     a16(X.down_scales),
                 "layer %d: expert pointers must be non-NULL and 16-byte aligned", l);
    if (g3)
      DG_CHECK_ARG(isfinite(g3[3 * l]) && isfinite(g3[3 * l + 1]) && isfinite(g3[3 * l + 2]),
                   "layer %d: tensor scales must be finite", l);
  }
  std::vector<LowpMaps> maps;
  try {
    maps.resize(c.n_layers);
  } catch (...) {
    return fail(DG_ERR_CUDA, "out of host memory");
  }
  const uint64_t E = c.n_experts, F = c.expert_ffn, H = c.hidden;
  auto codes = fmt == dg::FMT_NV4 ? map_codes4 : map_codes;
  auto scales = fmt == dg::FMT_NV4 ? map_scales4 : map_scales;
  for (int l = 0; l < c.n_layers; ++l) {
    const dg_expert_weights_mx8& X = layers[l];
    LowpMaps& M = maps[l];
    dg_status s;
    if ((s = codes(&M.gate, X.gate, E, F, H)) != DG_OK || (s = scales(&M.gate_s, X.gate_scales, E, F, H)) != DG_OK ||
        (s = codes(&M.up, X.up, E, F, H)) != DG_OK || (s = scales(&M.up_s, X.up_scales, E, F, H)) != DG_OK ||
        (s = codes(&M.down, X.down, E, H, F)) != DG_OK || (s = scales(&M.down_s, X.down_scales, E, H, F)) != DG_OK)
      return s;
    M.fmt = fmt;
    M.g_gate = g3 ? g3[3 * l] : 1.0f;
    M.g_up = g3 ? g3[3 * l + 1] : 1.0f;
    M.g_down = g3 ? g3[3 * l + 2] : 1.0f;
  }
  m->lowp.swap(maps);
  return DG_OK;
}

extern "C" dg_status dg_model_set_experts_mx8(dg_model* m, const dg_expert_weights_mx8* layers) {
  return set_experts_lowp(m, dg::FMT_MX8, layers, nullptr);
}

extern "C" dg_status dg_model_set_experts_nv4(dg_model* m, const dg_expert_weights_mx8* layers,
                                              const float* tensor_scales) {
  DG_CHECK_ARG(!layers || tensor_scales, "4-bit experts need their tensor scales");
  return set_experts_lowp(m, dg::FMT_NV4, layers, tensor_scales);
}

static dg_status set_vocab_lowp(dg_model* m, int fmt, const void* codes, const void* scales, float g) {
  DG_CHECK_ARG(m, "model is NULL");
  if (!codes) {
    m->vocab_lowp.on = false;
    return DG_OK;
  }
  const dg_config& c = m->cfg;
  DG_CHECK_ARG(is_bf16(c), "low-precision vocabulary weights need a bf16 model");
  auto a16 = [](const void* q) { return q && (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  DG_CHECK_ARG(a16(codes) && a16(scales), "vocabulary codes and scales must be non-NULL and 16-byte aligned");
  DG_CHECK_ARG(isfinite(g), "the tensor scale must be finite");
  VocabLowp v;
  const uint64_t V = c.vocab, H = c.hidden;
  dg_status s = fmt == dg::FMT_NV4 ? map_codes4(&v.codes, codes, 1, V, H) : map_codes(&v.codes, codes, 1, V, H);
  if (s == DG_OK)
    s = fmt == dg::FMT_NV4 ? map_scales4(&v.scales, scales, 1, V, H) : map_scales(&v.scales, scales, 1, V, H);
  if (s != DG_OK) return s;
  v.fmt = fmt;
  v.g = g;
  v.on = true;
  m->vocab_lowp = v;
  return DG_OK;
}

extern "C" dg_status dg_model_set_vocab_mx8(dg_model* m, const void* codes, const void* scales) {
  return set_vocab_lowp(m, dg::FMT_MX8, codes, scales, 1.0f);
}

extern "C" dg_status dg_model_set_vocab_nv4(dg_model* m, const void* codes, const void* scales, float tensor_scale) {
  return set_vocab_lowp(m, dg::FMT_NV4, codes, scales, tensor_scale);
}

extern "C" dg_status dg_generate_canvases_masked(dg_model* m, dg_kv_cache* caches, int32_t B, int32_t* d_canvases,
                                                 int32_t C, int32_t S, float keep_start, float keep_end,
                                                 int32_t mask_id, int32_t append, float* d_logits, void* d_ws,
                                                 size_t ws_bytes, dg_stream stream) {
  DG_CHECK_ARG(m, "model is NULL");
  DG_CHECK_ARG(S >= 1, "S must be >= 1");
  DG_CHECK_ARG(keep_start >= 0.f && keep_start <= 1.f && keep_end >= 0.f && keep_end <= 1.f,
               "keep fractions must be in [0,1]");
  DG_CHECK_ARG(mask_id >= 0 && mask_id < m->cfg.vocab, "mask_id must be in [0, vocab)");
  DG_CHECK_ARG(d_canvases && d_logits, "canvases / logits is NULL");
  DG_CHECK_ARG(C > 0 && C <= 1024, "C must be in [1, 1024]");
  DG_CHECK_ARG(B >= 1 && (int64_t)B * C <= (1 << 20), "B must be >= 1 and B * C <= 2^20");
  DG_CHECK_ARG((reinterpret_cast<uintptr_t>(d_logits) & 15) == 0, "logits must be 16-byte aligned");
  dg_status s = check_caches(m->cfg, caches, B, C);
  if (s != DG_OK) return s;
  Ws ws;
  if ((s = check_ws(m->cfg, d_ws, ws_bytes, B * C, &ws)) != DG_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int V = m->cfg.vocab, n = B * C;
  const int splits = dg::update_splits(n, V);
  dg::UpdPart* part = ws.at<dg::UpdPart>(ws.L.upd);
  LAUNCH(DG_K_UPDATE_SELECT, st, dg::launch_fill_i32(d_canvases, n, mask_id, st));
  for (int step = 0; step < S; ++step) {
    if ((s = dg_denoise_pass_batched(m, caches, B, d_canvases, C, d_logits, d_ws, ws_bytes, stream)) != DG_OK)
      return s;
    const int nk = renoise_count(C, S, step, keep_start, keep_end);
    LAUNCH(DG_K_UPDATE_PARTIAL, st, dg::launch_update_partial(d_logits, n, V, splits, mask_id, part, st));
    for (int b = 0; b < B; ++b)
      LAUNCH(DG_K_UPDATE_SELECT, st,
             dg::launch_update_select(part + (size_t)b * C * splits, C, V, splits, nk, 0, 0,
                                      d_canvases + (size_t)b * C, nullptr, mask_id, st));
  }
  if (append) return dg_prefill_append_batched(m, caches, B, d_canvases, C, d_ws, ws_bytes, stream);
  return DG_OK;
}

extern "C" dg_status dg_device_status(void* d_ws, dg_stream stream) {
  DG_CHECK_ARG(d_ws, "workspace is NULL");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemcpy(&v, d_ws, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(DG_ERR_CUDA, "device status: %s", cudaGetErrorString(e));
  if (v != 0) {
    const int zero = 0;
    cudaMemcpy(d_ws, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (v == DG_DEVERR_BAD_TOKEN) return fail(DG_ERR_INVALID_ARG, "a token id was outside [0, vocab)");
    if (v == DG_DEVERR_CHECK)
      return fail(DG_ERR_CUDA, "a kernel access failed its bounds or alignment check (checked build); it was skipped");
    return fail(DG_ERR_TIMEOUT, "device error word %d (a bounded wait gave up)", v);
  }
  return DG_OK;
}

extern "C" const char* dg_last_error(void) { return g_err.c_str(); }

// ---------------------------------------------------------------- debug / profiling
extern "C" dg_status dg_set_taps(dg_model* m, const dg_taps* t) {
  DG_CHECK_ARG(m, "model is NULL");
  const int L = m->cfg.n_layers;
  auto grab = [&](auto* const* src, auto& dst) {
    dst.clear();
    if (src) dst.assign(src, src + L);
  };
  if (!t) {
    m->taps_on = false;
    return DG_OK;
  }
  DG_CHECK_ARG(t->rows >= 0, "taps rows must be >= 0");
  grab(t->x_attn, m->tap_x_attn);
  grab(t->x_out, m->tap_x_out);
  grab(t->topk_w, m->tap_topk_w);
  grab(t->topk_idx, m->tap_topk_idx);
  grab(t->counts, m->tap_counts);
  grab(t->perm, m->tap_perm);
  m->tap_unions = t->unions;
  m->tap_rows = t->rows;
  m->taps_on = true;
  return DG_OK;
}

extern "C" dg_status dg_profile_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = on != 0;
  return DG_OK;
}
extern "C" void dg_profile_reset(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  prof_flush_locked();
  for (int i = 0; i < DG_K_COUNT; ++i) g_prof_ms[i] = 0.0, g_prof_n[i] = 0;
}
extern "C" dg_status dg_profile_read(int32_t kind, double* total_ms, int32_t* launches) {
  DG_CHECK_ARG(kind >= 0 && kind < DG_K_COUNT && total_ms && launches, "bad kind / NULL output");
  std::lock_guard<std::mutex> lk(g_prof_mu);
  prof_flush_locked();
  *total_ms = g_prof_ms[kind];
  *launches = g_prof_n[kind];
  return DG_OK;
}
extern "C" const char* dg_kernel_name(int32_t kind) {
  static const char* names[DG_K_COUNT] = {"embed_norm", "rms_norm",   "gemm_qkv",   "rope_kv",        "attention",
                                          "attn_merge", "gemm_o",     "router",     "topk",           "permute",
                                          "gather",     "gemm_gate_up", "swiglu",   "gemm_down",      "combine",
                                          "gemm_vocab", "update_partial", "update_select"};
  return (kind >= 0 && kind < DG_K_COUNT) ? names[kind] : "?";
}
extern "C" int64_t dg_launch_count(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  return g_launches;
}

extern "C" size_t dg_debug_gemm_scratch_bytes(int32_t x_rows, int32_t n_groups) {
  if (x_rows <= 0 || n_groups <= 0) return 0;
  return al(sizeof(dg::TcWorkItem) * ((size_t)x_rows + n_groups + 1) + 16);
}

extern "C" dg_status dg_debug_gemm_bf16(const void* W, const void* W2, int32_t rows, int32_t n_groups,
                                        const void* X, const void* X_lo, int32_t x_rows, int32_t K,
                                        const int32_t* group_off, void* out, void* out_lo, int32_t ld_out,
                                        void* d_scratch, size_t scratch_bytes, int32_t* d_err,
                                        dg_stream stream) {
  DG_CHECK_ARG(W && X && out && d_err && d_scratch, "NULL pointer");
  DG_CHECK_ARG(K > 0 && K % 64 == 0 && rows > 0 && n_groups > 0 && x_rows > 0, "bad GEMM shape");
  DG_CHECK_ARG(group_off || n_groups == 1, "several groups need group_off");
  DG_CHECK_ARG((reinterpret_cast<uintptr_t>(d_scratch) & 255) == 0, "scratch must be 256-byte aligned");
  if (scratch_bytes < dg_debug_gemm_scratch_bytes(x_rows, n_groups))
    return fail(DG_ERR_CAPACITY, "scratch too small: %zu < %zu", scratch_bytes,
                dg_debug_gemm_scratch_bytes(x_rows, n_groups));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  CUtensorMap A, A2;
  dg_status s = map_weights(&A, W, (uint64_t)n_groups, (uint64_t)rows, (uint64_t)K);
  if (s != DG_OK) return s;
  if (W2 && (s = map_weights(&A2, W2, (uint64_t)n_groups, (uint64_t)rows, (uint64_t)K)) != DG_OK) return s;
  dg::TcWorkItem* items = static_cast<dg::TcWorkItem*>(d_scratch);
  int* n_items = reinterpret_cast<int*>(items + x_rows + n_groups);
  int max_items = 0;
  if (group_off) {
    max_items = x_rows / kItemRows + n_groups;
    LAUNCH(DG_K_PERMUTE, st, dg::launch_build_items(group_off, n_groups, kItemRows, x_rows, items, n_items, d_err, st));
  }
  const int n_max = group_off ? kItemRows : (x_rows < 256 ? ((x_rows + 15) & ~15) : 256);
  GemmCall g{DG_K_GEMM_QKV, W2 ? dg::EPI_SWIGLU_BF16 : dg::EPI_STORE_F32, &A, W2 ? &A2 : nullptr, X, X_lo, x_rows,
             K, rows, group_off ? items : nullptr, group_off ? n_items : nullptr, max_items, n_max, out, out_lo,
             ld_out, 1, 0, kSmemGemm};
  return gemm_bf16(g, d_err, st);
}

static dg_status debug_gemm_lowp(int fmt, const void* W, const void* W_scales, float g, const void* W2,
                                 const void* W2_scales, float g2, int32_t rows, int32_t n_groups, const void* X,
                                 const void* X_lo, int32_t x_rows, int32_t K, const int32_t* group_off, void* out,
                                 void* out_lo, int32_t ld_out, void* d_scratch, size_t scratch_bytes, int32_t* d_err,
                                 dg_stream stream);

extern "C" dg_status dg_debug_gemm_mx8(const void* W, const void* W_scales, const void* W2, const void* W2_scales,
                                       int32_t rows, int32_t n_groups, const void* X, const void* X_lo,
                                       int32_t x_rows, int32_t K, const int32_t* group_off, void* out, void* out_lo,
                                       int32_t ld_out, void* d_scratch, size_t scratch_bytes, int32_t* d_err,
                                       dg_stream stream) {
  return debug_gemm_lowp(dg::FMT_MX8, W, W_scales, 1.0f, W2, W2_scales, 1.0f, rows, n_groups, X, X_lo, x_rows, K,
                         group_off, out, out_lo, ld_out, d_scratch, scratch_bytes, d_err, stream);
}

extern "C" dg_status dg_debug_gemm_nv4(const void* W, const void* W_scales, float g, const void* W2,
                                       const void* W2_scales, float g2, int32_t rows, int32_t n_groups, const void* X,
                                       const void* X_lo, int32_t x_rows, int32_t K, const int32_t* group_off,
                                       void* out, void* out_lo, int32_t ld_out, void* d_scratch,
                                       size_t scratch_bytes, int32_t* d_err, dg_stream stream) {
  DG_CHECK_ARG(isfinite(g) && (!W2 || isfinite(g2)), "tensor scales must be finite");
  return debug_gemm_lowp(dg::FMT_NV4, W, W_scales, g, W2, W2_scales, g2, rows, n_groups, X, X_lo, x_rows, K,
                         group_off, out, out_lo, ld_out, d_scratch, scratch_bytes, d_err, stream);
}

static dg_status debug_gemm_lowp(int fmt, const void* W, const void* W_scales, float g, const void* W2,
                                 const void* W2_scales, float g2, int32_t rows, int32_t n_groups, const void* X,
                                 const void* X_lo, int32_t x_rows, int32_t K, const int32_t* group_off, void* out,
                                 void* out_lo, int32_t ld_out, void* d_scratch, size_t scratch_bytes, int32_t* d_err,
                                 dg_stream stream) {
  DG_CHECK_ARG(W && W_scales && X && out && d_err && d_scratch, "NULL pointer");
  DG_CHECK_ARG(!W2 == !W2_scales, "W2 and its scales come together");
  DG_CHECK_ARG(K > 0 && K % 64 == 0 && rows > 0 && rows % 8 == 0 && n_groups > 0 && x_rows > 0, "bad GEMM shape");
  DG_CHECK_ARG(ld_out >= rows, "ld_out < rows");
  DG_CHECK_ARG(group_off || n_groups == 1, "several groups need group_off");
  auto a16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  DG_CHECK_ARG(a16(W) && a16(W_scales) && a16(X) && (!X_lo || a16(X_lo)) && (!W2 || (a16(W2) && a16(W2_scales))),
               "operands must be 16-byte aligned");
  DG_CHECK_ARG((reinterpret_cast<uintptr_t>(d_scratch) & 255) == 0, "scratch must be 256-byte aligned");
  if (scratch_bytes < dg_debug_gemm_scratch_bytes(x_rows, n_groups))
    return fail(DG_ERR_CAPACITY, "scratch too small: %zu < %zu", scratch_bytes,
                dg_debug_gemm_scratch_bytes(x_rows, n_groups));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  constexpr int kRows = 64;  // token rows per tile of the 8-bit GEMM
  CUtensorMap A, A2, S, S2, B, B2, Bb, B2b;
  dg_status s;
  auto codes = fmt == dg::FMT_NV4 ? map_codes4 : map_codes;
  auto scales = fmt == dg::FMT_NV4 ? map_scales4 : map_scales;
  if ((s = codes(&A, W, (uint64_t)n_groups, (uint64_t)rows, (uint64_t)K)) != DG_OK) return s;
  if ((s = scales(&S, W_scales, (uint64_t)n_groups, (uint64_t)rows, (uint64_t)K)) != DG_OK) return s;
  if (W2) {
    if ((s = codes(&A2, W2, (uint64_t)n_groups, (uint64_t)rows, (uint64_t)K)) != DG_OK) return s;
    if ((s = scales(&S2, W2_scales, (uint64_t)n_groups, (uint64_t)rows, (uint64_t)K)) != DG_OK) return s;
  } else {
    A2 = A;
    S2 = S;
  }
  if ((s = map_rows(&B, X, (uint64_t)x_rows, (uint64_t)K, 16)) != DG_OK) return s;
  if ((s = map_rows(&Bb, X, (uint64_t)x_rows, (uint64_t)K, 64)) != DG_OK) return s;
  if (X_lo) {
    if ((s = map_rows(&B2, X_lo, (uint64_t)x_rows, (uint64_t)K, 16)) != DG_OK) return s;
    if ((s = map_rows(&B2b, X_lo, (uint64_t)x_rows, (uint64_t)K, 64)) != DG_OK) return s;
  } else {
    B2 = B;
    B2b = Bb;
  }
  dg::TcWorkItem* items = static_cast<dg::TcWorkItem*>(d_scratch);
  int* n_items = reinterpret_cast<int*>(items + x_rows + n_groups);
  int max_items = 0;
  if (group_off) {
    max_items = x_rows / kRows + n_groups;
    LAUNCH(DG_K_PERMUTE, st, dg::launch_build_items(group_off, n_groups, kRows, x_rows, items, n_items, d_err, st));
  }
  dg::TcGemmParams p{};
  p.K = K;
  p.a_rows_per_group = rows;
  p.m_tiles = ceil_div(rows, 128);
  p.n_max = group_off ? kRows : (x_rows < kRows ? ((x_rows + 15) & ~15) : kRows);
  p.n_tokens = x_rows;
  p.k_splits = 1;
  p.split_stride = 0;
  p.items = group_off ? items : nullptr;
  p.n_items = group_off ? n_items : nullptr;
  p.dual_a = W2 != nullptr;
  p.two_terms = X_lo != nullptr;
  p.out = out;
  p.out_lo = out_lo;
  p.ld_out = ld_out;
  p.smem_budget = kSmemGemm;
  p.err = d_err;
  const int tiles = (group_off ? max_items : ceil_div(x_rows, p.n_max)) * p.m_tiles;
  LAUNCH(DG_K_GEMM_GATE_UP, st,
         dg::launch_tc_gemm_lowp(fmt, W2 ? dg::EPI_SWIGLU_BF16 : dg::EPI_STORE_F32, A, A2, S, S2, B, B2, Bb, B2b,
                                 p, g, g2, tiles, st));
  return DG_OK;
}

static dg_status debug_attention(const void* q, const void* k, const void* vt, int32_t cap, int32_t n_q, int32_t pos0,
                                 int32_t n_keys, int32_t causal, int32_t nq, int32_t nkv, void* out, void* out_lo,
                                 void* d_ws, size_t ws_bytes, dg_stream stream, bool pair) {
  DG_CHECK_ARG(q && k && vt && out && d_ws, "NULL pointer");
  DG_CHECK_ARG(nq > 0 && nkv > 0 && nq % nkv == 0 && n_q > 0 && n_keys > 0 && n_keys <= cap && cap % 8 == 0,
               "bad attention shape");
  DG_CHECK_ARG(!causal || pos0 + n_q <= n_keys, "causal rows need their own keys");
  dg_config c{};
  c.n_layers = 1;
  c.hidden = 128;
  c.n_q_heads = nq;
  c.n_kv_heads = nkv;
  c.head_dim = 128;
  c.n_experts = 1;
  c.top_k = 1;
  c.expert_ffn = 64;
  c.vocab = 128;
  c.rope_theta = 10000.f;
  c.rms_eps = 1e-6f;
  c.dtype = DG_DTYPE_BF16;
  Ws ws;
  dg_status s = check_ws(c, d_ws, ws_bytes, n_q, &ws);
  if (s != DG_OK) return s;
  // the kernels read the low terms of the keys from the 128-aligned start at or below pos0
  // up to n_keys out of the workspace's window (sized for n_q rows): that range must fit it
  DG_CHECK_ARG(pos0 >= 0 && pos0 <= n_keys, "pos0 must lie in [0, n_keys]");
  DG_CHECK_ARG(n_keys - (pos0 / 128) * 128 <= ws.L.lo_rows,
               "keys from the 128-aligned start at or below pos0 exceed the workspace's low-term window");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the pass reads q from the workspace's q buffer and writes o to its o buffer; the low
  // terms of q and of the current K/V are zero here (all inputs are bf16 already)
  cudaError_t e = cudaMemcpyAsync(ws.at<void>(ws.L.q), q, (size_t)nq * n_q * 128 * 2, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws.at<void>(ws.L.q_lo), 0, (size_t)nq * n_q * 128 * 2, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws.at<void>(ws.L.k_lo), 0, (size_t)nkv * ws.L.lo_rows * 128 * 2, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws.at<void>(ws.L.vt_lo), 0, (size_t)nkv * ws.L.lo_rows * 128 * 2, st);
  if (e != cudaSuccess) return fail(DG_ERR_CUDA, "copy q: %s", cudaGetErrorString(e));
  void* kc = const_cast<void*>(k);
  void* vtc = const_cast<void*>(vt);
  if ((s = pair ? attention_pair(c, ws, kc, vtc, cap, n_q, pos0, n_keys, causal, st)
                : attention_single(c, ws, kc, vtc, cap, n_q, pos0, n_keys, causal, st)) != DG_OK)
    return s;
  e = cudaMemcpyAsync(out, ws.at<void>(ws.L.o), (size_t)n_q * nq * 128 * 2, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess && out_lo)
    e = cudaMemcpyAsync(out_lo, ws.at<void>(ws.L.o_lo), (size_t)n_q * nq * 128 * 2, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return fail(DG_ERR_CUDA, "copy o: %s", cudaGetErrorString(e));
  return DG_OK;
}

extern "C" dg_status dg_debug_attention_bf16(const void* q, const void* k, const void* vt, int32_t cap, int32_t n_q,
                                             int32_t pos0, int32_t n_keys, int32_t causal, int32_t nq, int32_t nkv,
                                             void* out, void* out_lo, void* d_ws, size_t ws_bytes, dg_stream stream) {
  return debug_attention(q, k, vt, cap, n_q, pos0, n_keys, causal, nq, nkv, out, out_lo, d_ws, ws_bytes, stream,
                         false);
}

extern "C" dg_status dg_debug_attention_pair_bf16(const void* q, const void* k, const void* vt, int32_t cap,
                                                  int32_t n_q, int32_t pos0, int32_t n_keys, int32_t causal,
                                                  int32_t nq, int32_t nkv, void* out, void* out_lo, void* d_ws,
                                                  size_t ws_bytes, dg_stream stream) {
  return debug_attention(q, k, vt, cap, n_q, pos0, n_keys, causal, nq, nkv, out, out_lo, d_ws, ws_bytes, stream,
                         true);
}

extern "C" dg_status dg_debug_set_wait_limit(uint64_t limit_ns) {
  DG_CHECK_ARG(limit_ns <= DG_WAIT_NS, "limit_ns must be at most %llu", (unsigned long long)DG_WAIT_NS);
  cudaError_t (*const setters[])(uint64_t) = {dg::set_wait_limit_attn, dg::set_wait_limit_attn2,
                                              dg::set_wait_limit_gemm, dg::set_wait_limit_gemm_lowp,
                                              dg::set_wait_limit_vocab_update};
  for (auto f : setters) {
    cudaError_t e = f(limit_ns);
    if (e != cudaSuccess) return fail(DG_ERR_CUDA, "setting the wait limit: %s", cudaGetErrorString(e));
  }
  return DG_OK;
}

extern "C" dg_status dg_debug_mma_rate(int32_t a_tmem, int32_t n, int32_t count, int32_t blocks,
                                       uint64_t* cycles_out, float* ms_out, dg_stream stream) {
  DG_CHECK_ARG(n == 64 || n == 128 || n == 256, "n must be 64, 128 or 256");
  DG_CHECK_ARG(count >= 1 && count <= (1 << 20), "count must be in [1, 1048576]");
  DG_CHECK_ARG(blocks >= 1 && blocks <= 1024, "blocks must be in [1, 1024]");
  DG_CHECK_ARG(cycles_out && ms_out, "NULL output");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned long long* d_cycles = nullptr;
  int* d_err = nullptr;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  cudaError_t e = cudaMalloc(&d_cycles, sizeof(unsigned long long) + sizeof(int));
  if (e == cudaSuccess) {
    d_err = reinterpret_cast<int*>(d_cycles + 1);
    e = cudaMemsetAsync(d_cycles, 0, sizeof(unsigned long long) + sizeof(int), st);
  }
  if (e == cudaSuccess) e = cudaEventCreate(&e0);
  if (e == cudaSuccess) e = cudaEventCreate(&e1);
  if (e == cudaSuccess) e = cudaEventRecord(e0, st);
  if (e == cudaSuccess) e = dg::launch_mma_rate(a_tmem ? 1 : 0, n, count, blocks, d_cycles, d_err, st);
  if (e == cudaSuccess) e = cudaEventRecord(e1, st);
  if (e == cudaSuccess) e = cudaEventSynchronize(e1);
  float ms = 0.f;
  if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, e0, e1);
  unsigned long long cyc = 0;
  int derr = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&cyc, d_cycles, sizeof(cyc), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(&derr, d_err, sizeof(derr), cudaMemcpyDeviceToHost);
  if (e0) cudaEventDestroy(e0);
  if (e1) cudaEventDestroy(e1);
  if (d_cycles) cudaFree(d_cycles);
  if (e != cudaSuccess) return fail(DG_ERR_CUDA, "mma rate probe: %s", cudaGetErrorString(e));
  if (derr) return fail(DG_ERR_TIMEOUT, "mma rate probe: the wait for the MMAs gave up");
  *cycles_out = cyc;
  *ms_out = ms;
  return DG_OK;
}

extern "C" dg_status dg_debug_bounded_wait(void* d_ws, int32_t timeout_ms, dg_stream stream) {
  DG_CHECK_ARG(d_ws, "workspace is NULL");
  DG_CHECK_ARG(timeout_ms >= 1 && timeout_ms <= 10000, "timeout_ms must be in [1, 10000]");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  LAUNCH(DG_K_COUNT - 1, st,
         dg::launch_bounded_wait_selftest(static_cast<int*>(d_ws), (uint64_t)timeout_ms * 1000000ull, st));
  return DG_OK;
}
