// CPU oracle of the block-diffusion denoising pass -- TEST INFRASTRUCTURE ONLY.
//
// Only the tests, the smoke check and the benchmark's CPU baseline load this library
// (through oracle/dg_oracle.py).  Nothing in the product path links, loads or calls
// it; it shares no source, header, table or helper with the CUDA path.
//
// Plain, slow, obviously correct C++ in double precision.  Every matrix product is
// written as its definition: each output element is one dot product summed over the
// shared index in order.  OpenMP only spreads independent output elements (rows, heads,
// experts, vocabulary entries) over the host cores; no sum is split, blocked or fused.
//
// Sources (page title -- section):
//   [DG-explainer]  "DiffusionGemma" video explainer -- "The fix: a 256-token canvas",
//                   "Uniform State Diffusion", "Two modes, one model", "First attempt:
//                   masked diffusion", "Long-form text: chaining canvases"
//   [DLM-exercises] "Module 12. Diffusion Language Models" exercises -- the prefix/block
//                   mask solution (7x7 worked example); the MoE remark in the roofline
//                   solution (FP8 on H100, NVFP4 on Blackwell)
//   [DG-intro]      "Introducing DiffusionGemma: An Attempt to Speed Up Text Generation by
//                   Blocks" -- "What is DiffusionGemma?", "The Meaning of 'Seeing the Whole'"
//
// Readings where the pages are silent: pre-norm RMSNorm without gain (eps from the
// config); RoPE rotate-half with theta from the config at absolute positions; GQA
// query head h -> kv head h / (nq / nkv); attention scale 1/sqrt(d); router on the
// normed residual, top-k by value with ties to the lower expert id, weights = softmax
// over the k chosen logits; SwiGLU experts; untied embedding / output matrices;
// confidence = largest softmax probability (temperature 1); every position takes its
// argmax (ties to the lowest id), then the n lowest-confidence positions (ties to the
// lower position) get a fresh random token.  The masked-diffusion update states its own.
//
// Storage rule.  The pages fix bf16 weights and nothing else.  A bf16 model stores its
// weights and its KV cache in bf16; every value in flight is exact here (double).  So
// the only rounding this oracle performs is where a bf16 model stores a value: the K/V
// a prefill writes to the cache.  Weights arrive as the stored values (bf16 bit
// patterns, fp32 or fp64 arrays) and are widened exactly.
#include <omp.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <numeric>
#include <vector>

extern "C" {

// ---------------------------------------------------------------- storage

enum { OC_BF16 = 0, OC_F32 = 1, OC_F64 = 2 };

// a stored tensor: data pointer and element type (bf16 bit patterns, float or double)
typedef struct {
  const void* p;
  int32_t dtype;
} oc_tensor;

typedef struct {
  int32_t n_layers, hidden, n_q_heads, n_kv_heads, head_dim, n_experts, top_k, expert_ffn, vocab;
  double rope_theta, rms_eps;
  int32_t bf16_storage;  // 1: the KV cache stores bf16 (prefill rounds what it writes)
} oc_config;

// per layer: w_q [nq d][H], w_k, w_v [nkv d][H], w_o [H][nq d], w_router [E][H],
// w_gate, w_up [E][F][H], w_down [E][H][F]; embed, w_out [V][H]
typedef struct {
  oc_tensor embed, w_out;
  const oc_tensor *w_q, *w_k, *w_v, *w_o, *w_router, *w_gate, *w_up, *w_down;
} oc_weights;

// per-layer intermediate values (any pointer may be NULL)
typedef struct {
  double* x_in;           // [T][H] residual entering the layer
  double* attn_o;         // [T][nq d] attention output, heads concatenated
  double* x_attn;         // [T][H] residual after the attention block
  double* x_out;          // [T][H] residual after the MoE block
  double* router_logits;  // [T][E]
  int32_t* topk_idx;      // [T][k]
  double* topk_w;         // [T][k]
  double* router_margin;  // [T] k-th minus (k+1)-th largest router logit
  int64_t* counts;        // [E]
  int64_t* offsets;       // [E+1]
  int64_t* perm;          // [T k]
  int64_t* inv;           // [T k]
  int64_t* union_size;    // [1]
  double* k_new;          // [nkv][T][d] keys of the call's own tokens (after RoPE, in flight)
  double* v_new;          // [nkv][T][d]
} oc_taps;

static inline double bf16_bits_value(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

static inline double load(const oc_tensor& t, size_t i) {
  switch (t.dtype) {
    case OC_BF16: return bf16_bits_value(((const uint16_t*)t.p)[i]);
    case OC_F32: return (double)((const float*)t.p)[i];
    default: return ((const double*)t.p)[i];
  }
}

static void widen_row(const oc_tensor& t, size_t off, int n, double* out) {
  for (int i = 0; i < n; ++i) out[i] = load(t, off + i);
}

// exact value of n stored elements
void oc_widen(oc_tensor t, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = load(t, (size_t)i);
}

// round to the nearest bf16 value (8 significant bits), ties to even; exact in double
double oc_round_bf16_1(double x) {
  if (x == 0.0 || !std::isfinite(x)) return x;
  int e;
  double m = std::frexp(x, &e);            // x = m 2^e, 0.5 <= |m| < 1
  return std::ldexp(std::nearbyint(m * 256.0), e - 8);
}

void oc_round_bf16(const double* x, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oc_round_bf16_1(x[i]);
}

// ---------------------------------------------------------------- primitives

static double dot(const double* a, const double* b, int n) {
  double s = 0.0;
#pragma omp simd reduction(+ : s)
  for (int i = 0; i < n; ++i) s += a[i] * b[i];
  return s;
}

// y[t][n] = sum_k x[t][k] W[n][k] for the N x K matrix stored at W (element offset w0)
static void matmul_xwt(const double* x, int T, int K, const oc_tensor& W, size_t w0, int N, double* y) {
#pragma omp parallel
  {
    std::vector<double> w(K);
#pragma omp for schedule(static)
    for (int n = 0; n < N; ++n) {
      widen_row(W, w0 + (size_t)n * K, K, w.data());
      for (int t = 0; t < T; ++t) y[(size_t)t * N + n] = dot(x + (size_t)t * K, w.data(), K);
    }
  }
}

// y = x / sqrt(mean(x^2) + eps) over each row of H values (unit gain)
void oc_rms_norm(const double* x, int64_t T, int32_t H, double eps, double* y) {
  for (int64_t t = 0; t < T; ++t) {
    const double* r = x + t * H;
    double ss = 0.0;
    for (int i = 0; i < H; ++i) ss += r[i] * r[i];
    const double inv = 1.0 / std::sqrt(ss / H + eps);
    for (int i = 0; i < H; ++i) y[t * H + i] = r[i] * inv;
  }
}

// rotary position embedding on x [n][T][d], rotate-half pairs (i, i + d/2):
// angle(t, i) = pos[t] * theta^(-2i/d)
void oc_rope(double* x, int32_t n, int32_t T, int32_t d, const int64_t* pos, double theta) {
  const int half = d / 2;
  for (int h = 0; h < n; ++h)
    for (int t = 0; t < T; ++t) {
      double* r = x + ((size_t)h * T + t) * d;
      for (int i = 0; i < half; ++i) {
        const double ang = (double)pos[t] * std::pow(theta, -(2.0 * i) / d);
        const double c = std::cos(ang), s = std::sin(ang);
        const double a = r[i], b = r[i + half];
        r[i] = a * c - b * s;
        r[i + half] = b * c + a * s;
      }
    }
}

double oc_silu(double z) { return z / (1.0 + std::exp(-z)); }

void oc_silu_array(const double* z, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oc_silu(z[i]);
}

// [DLM-exercises] prefix/block mask: rows and columns ordered (prefix 0..P-1, block
// 0..C-1); a prefix query sees the prefix keys at or before it, a block query sees the
// whole prefix and the whole block, no prefix query sees a block key
void oc_block_mask(int32_t P, int32_t C, uint8_t* allowed) {
  const int n = P + C;
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < n; ++j) allowed[(size_t)i * n + j] = (i < P) ? (j <= i) : 1;
}

// [DG-explainer] "Two modes, one model": T new tokens at positions P..P+T-1 read keys
// 0..P+T-1 causally (prefill mode)
void oc_causal_rows(int32_t P, int32_t T, uint8_t* allowed) {
  const int n = P + T;
  for (int i = 0; i < T; ++i)
    for (int j = 0; j < n; ++j) allowed[(size_t)i * n + j] = j <= P + i;
}

// masked softmax attention, grouped KV heads: q [nq][Tq][d], k, v [nkv][Tk][d],
// allowed [Tq][Tk] (NULL: every key); query head h reads KV head h / (nq / nkv);
// scores scaled by 1/sqrt(d); out [nq][Tq][d]
void oc_attention(const double* q, const double* k, const double* v, const uint8_t* allowed, int32_t nq, int32_t nkv,
                  int32_t Tq, int32_t Tk, int32_t d, double* out) {
  const int g = nq / nkv;
  const double scale = 1.0 / std::sqrt((double)d);
#pragma omp parallel
  {
    std::vector<double> s(Tk);
#pragma omp for collapse(2) schedule(dynamic, 4)
    for (int h = 0; h < nq; ++h)
      for (int i = 0; i < Tq; ++i) {
        const double* qi = q + ((size_t)h * Tq + i) * d;
        const double* kh = k + (size_t)(h / g) * Tk * d;
        const double* vh = v + (size_t)(h / g) * Tk * d;
        const uint8_t* a = allowed ? allowed + (size_t)i * Tk : nullptr;
        double m = -std::numeric_limits<double>::infinity();
        for (int j = 0; j < Tk; ++j) {
          s[j] = (!a || a[j]) ? dot(qi, kh + (size_t)j * d, d) * scale : -std::numeric_limits<double>::infinity();
          m = std::max(m, s[j]);
        }
        double sum = 0.0;
        for (int j = 0; j < Tk; ++j) {
          s[j] = std::exp(s[j] - m);
          sum += s[j];
        }
        double* o = out + ((size_t)h * Tq + i) * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        for (int j = 0; j < Tk; ++j) {
          if (s[j] == 0.0) continue;
          const double p = s[j] / sum;
          const double* vj = vh + (size_t)j * d;
          for (int c = 0; c < d; ++c) o[c] += p * vj[c];
        }
      }
  }
}

// top-k experts per token by router logit, ties to the lower expert id; idx in
// descending-logit order, w = softmax over the k chosen logits, margin = k-th minus
// (k+1)-th largest logit (+inf when k = E).  [DLM-exercises]: positions route to
// different experts.
void oc_router_topk(const double* logits, int32_t T, int32_t E, int32_t k, int32_t* idx, double* w,
                    double* margin) {
  std::vector<int> order(E);
  for (int t = 0; t < T; ++t) {
    const double* l = logits + (size_t)t * E;
    std::iota(order.begin(), order.end(), 0);
    std::stable_sort(order.begin(), order.end(), [l](int a, int b) { return l[a] > l[b]; });
    double mx = l[order[0]];
    double sum = 0.0;
    for (int j = 0; j < k; ++j) {
      idx[(size_t)t * k + j] = order[j];
      w[(size_t)t * k + j] = std::exp(l[order[j]] - mx);
      sum += w[(size_t)t * k + j];
    }
    for (int j = 0; j < k; ++j) w[(size_t)t * k + j] /= sum;
    if (margin) margin[t] = k < E ? l[order[k - 1]] - l[order[k]] : std::numeric_limits<double>::infinity();
  }
}

// group the T k (token, slot) assignments by expert, stably: perm[p] = flat assignment
// t k + j placed at row p, in (expert, t, j) order; inv = inverse; counts, exclusive
// offsets, and the union size = #experts with a row ([DLM-exercises] MoE remark: a
// pass reads the union of the experts its positions route to)
int64_t oc_expert_permutation(const int32_t* idx, int32_t T, int32_t k, int32_t E, int64_t* counts, int64_t* offsets,
                              int64_t* perm, int64_t* inv) {
  const int64_t n = (int64_t)T * k;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t a = 0; a < n; ++a) counts[idx[a]] += 1;
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  std::vector<int64_t> fill(offsets, offsets + E);
  for (int64_t a = 0; a < n; ++a) perm[fill[idx[a]]++] = a;   // ascending a = ascending (t, j)
  for (int64_t p = 0; p < n; ++p) inv[perm[p]] = p;
  int64_t u = 0;
  for (int e = 0; e < E; ++e) u += counts[e] > 0;
  return u;
}

// ---------------------------------------------------------------- the layer stack

static int64_t rows_of(int64_t T, int64_t cols) { return T * cols; }

// q, k, v of T tokens: RMSNorm, projections, RoPE on q and k at their positions.
// q [nq][T][d], k, v [nkv][T][d]
static void qkv(const oc_config& c, const oc_weights& W, int l, const double* x, int T, const int64_t* pos,
                std::vector<double>& q, std::vector<double>& k, std::vector<double>& v);

void oc_qkv(const oc_config* cp, const oc_weights* Wp, int32_t l, const double* x, int32_t T, const int64_t* pos,
            double* q_out, double* k_out, double* v_out) {
  std::vector<double> q, k, v;
  qkv(*cp, *Wp, l, x, T, pos, q, k, v);
  std::copy(q.begin(), q.end(), q_out);
  std::copy(k.begin(), k.end(), k_out);
  std::copy(v.begin(), v.end(), v_out);
}

// the attention output projection: y [T][H] = o W_o^T with o [nq][T][d], heads
// concatenated per token
void oc_attn_out(const oc_config* cp, const oc_weights* Wp, int32_t l, const double* o, int32_t T, double* y) {
  const int nq = cp->n_q_heads, d = cp->head_dim;
  std::vector<double> oc((size_t)T * nq * d);
  for (int t = 0; t < T; ++t)
    for (int h = 0; h < nq; ++h)
      for (int i = 0; i < d; ++i) oc[(size_t)t * nq * d + h * d + i] = o[((size_t)h * T + t) * d + i];
  matmul_xwt(oc.data(), T, nq * d, Wp->w_o[l], 0, cp->hidden, y);
}

static void qkv(const oc_config& c, const oc_weights& W, int l, const double* x, int T, const int64_t* pos,
                std::vector<double>& q, std::vector<double>& k, std::vector<double>& v) {
  const int H = c.hidden, nq = c.n_q_heads, nkv = c.n_kv_heads, d = c.head_dim;
  std::vector<double> xn(rows_of(T, H)), tq(rows_of(T, nq * d)), tk(rows_of(T, nkv * d)), tv(rows_of(T, nkv * d));
  oc_rms_norm(x, T, H, c.rms_eps, xn.data());
  matmul_xwt(xn.data(), T, H, W.w_q[l], 0, nq * d, tq.data());
  matmul_xwt(xn.data(), T, H, W.w_k[l], 0, nkv * d, tk.data());
  matmul_xwt(xn.data(), T, H, W.w_v[l], 0, nkv * d, tv.data());
  q.assign(rows_of(T, nq * d), 0.0);
  k.assign(rows_of(T, nkv * d), 0.0);
  v.assign(rows_of(T, nkv * d), 0.0);
  for (int t = 0; t < T; ++t) {   // [T][heads d] -> [heads][T][d]
    for (int h = 0; h < nq; ++h)
      for (int i = 0; i < d; ++i) q[((size_t)h * T + t) * d + i] = tq[(size_t)t * nq * d + h * d + i];
    for (int h = 0; h < nkv; ++h)
      for (int i = 0; i < d; ++i) {
        k[((size_t)h * T + t) * d + i] = tk[(size_t)t * nkv * d + h * d + i];
        v[((size_t)h * T + t) * d + i] = tv[(size_t)t * nkv * d + h * d + i];
      }
  }
  oc_rope(q.data(), nq, T, d, pos, c.rope_theta);
  oc_rope(k.data(), nkv, T, d, pos, c.rope_theta);
}

// the attention block of layer l for T tokens at positions pos0..pos0+T-1 over the
// cached keys [0, P) (stored values, [nkv][P][d]) and the tokens' own keys (in flight):
// x_attn = x + attention(...) W_o^T.  causal = 0: denoising mode (every token sees
// every cached and every own key: the block rows of the prefix/block mask);
// causal = 1: prefill mode (token i sees keys up to P + i).
// k_new / v_new (may be NULL) receive the tokens' own K/V, [nkv][T][d].
void oc_attention_block(const oc_config* cp, const oc_weights* Wp, int32_t l, const double* cache_k,
                        const double* cache_v, int32_t P, const double* x, int32_t T, int32_t causal, double* x_attn,
                        double* attn_o, double* k_new, double* v_new) {
  const oc_config& c = *cp;
  const oc_weights& W = *Wp;
  const int H = c.hidden, nq = c.n_q_heads, nkv = c.n_kv_heads, d = c.head_dim;
  std::vector<int64_t> pos(T);
  for (int t = 0; t < T; ++t) pos[t] = (int64_t)P + t;
  std::vector<double> q, k, v;
  qkv(c, W, l, x, T, pos.data(), q, k, v);
  if (k_new) std::copy(k.begin(), k.end(), k_new);
  if (v_new) std::copy(v.begin(), v.end(), v_new);
  const int Tk = P + T;
  std::vector<double> kk((size_t)nkv * Tk * d), vv((size_t)nkv * Tk * d);
  for (int h = 0; h < nkv; ++h) {   // cached prefix (stored) then the tokens' own keys (in flight)
    std::copy(cache_k + (size_t)h * P * d, cache_k + (size_t)(h + 1) * P * d, kk.begin() + (size_t)h * Tk * d);
    std::copy(cache_v + (size_t)h * P * d, cache_v + (size_t)(h + 1) * P * d, vv.begin() + (size_t)h * Tk * d);
    std::copy(k.begin() + (size_t)h * T * d, k.begin() + (size_t)(h + 1) * T * d,
              kk.begin() + ((size_t)h * Tk + P) * d);
    std::copy(v.begin() + (size_t)h * T * d, v.begin() + (size_t)(h + 1) * T * d,
              vv.begin() + ((size_t)h * Tk + P) * d);
  }
  std::vector<uint8_t> mask((size_t)T * Tk);
  if (causal) {
    oc_causal_rows(P, T, mask.data());
  } else {   // the block rows of the prefix/block mask over (prefix, block)
    std::vector<uint8_t> full((size_t)Tk * Tk);
    oc_block_mask(P, T, full.data());
    std::copy(full.begin() + (size_t)P * Tk, full.end(), mask.begin());
  }
  std::vector<double> o((size_t)nq * T * d), y(rows_of(T, H));
  oc_attention(q.data(), kk.data(), vv.data(), mask.data(), nq, nkv, T, Tk, d, o.data());
  if (attn_o)   // heads concatenated per token
    for (int t = 0; t < T; ++t)
      for (int h = 0; h < nq; ++h)
        for (int i = 0; i < d; ++i) attn_o[(size_t)t * nq * d + h * d + i] = o[((size_t)h * T + t) * d + i];
  oc_attn_out(cp, Wp, l, o.data(), T, y.data());
  for (size_t i = 0; i < (size_t)T * H; ++i) x_attn[i] = x[i] + y[i];
}

// the sparse MoE block of layer l on the residual x [T][H]: router on the normed
// residual -> top-k -> stable expert grouping -> per-expert SwiGLU over only the rows
// routed to it (the union of experts) -> combine sum_j w[t][j] y[t][j] in slot order;
// ffn_out = the combine, x_out = x + combine (either may be NULL)
void oc_moe_block(const oc_config* cp, const oc_weights* Wp, int32_t l, const double* x, int32_t T, double* x_out,
                  double* ffn_out, oc_taps* tap) {
  const oc_config& c = *cp;
  const oc_weights& W = *Wp;
  const int H = c.hidden, E = c.n_experts, k = c.top_k, F = c.expert_ffn;
  std::vector<double> xn(rows_of(T, H)), logits(rows_of(T, E)), w(rows_of(T, k)), margin(T);
  std::vector<int32_t> idx(rows_of(T, k));
  oc_rms_norm(x, T, H, c.rms_eps, xn.data());
  matmul_xwt(xn.data(), T, H, W.w_router[l], 0, E, logits.data());
  oc_router_topk(logits.data(), T, E, k, idx.data(), w.data(), margin.data());
  std::vector<int64_t> counts(E), offsets(E + 1), perm((size_t)T * k), inv((size_t)T * k);
  const int64_t u = oc_expert_permutation(idx.data(), T, k, E, counts.data(), offsets.data(), perm.data(), inv.data());
  std::vector<double> ys((size_t)T * k * H, 0.0);
#pragma omp parallel for schedule(dynamic, 1)
  for (int e = 0; e < E; ++e) {
    const int n = (int)counts[e];
    if (n == 0) continue;
    std::vector<double> xe((size_t)n * H), wrow(H), drow(F), g((size_t)n * F), up((size_t)n * F), h((size_t)n * F);
    for (int r = 0; r < n; ++r) {
      const int64_t t = perm[offsets[e] + r] / k;
      std::copy(xn.begin() + t * H, xn.begin() + (t + 1) * H, xe.begin() + (size_t)r * H);
    }
    for (int f = 0; f < F; ++f) {
      widen_row(W.w_gate[l], ((size_t)e * F + f) * H, H, wrow.data());
      for (int r = 0; r < n; ++r) g[(size_t)r * F + f] = dot(xe.data() + (size_t)r * H, wrow.data(), H);
      widen_row(W.w_up[l], ((size_t)e * F + f) * H, H, wrow.data());
      for (int r = 0; r < n; ++r) up[(size_t)r * F + f] = dot(xe.data() + (size_t)r * H, wrow.data(), H);
    }
    for (size_t i = 0; i < (size_t)n * F; ++i) h[i] = oc_silu(g[i]) * up[i];
    for (int o = 0; o < H; ++o) {
      widen_row(W.w_down[l], ((size_t)e * H + o) * F, F, drow.data());
      for (int r = 0; r < n; ++r) ys[(size_t)(offsets[e] + r) * H + o] = dot(h.data() + (size_t)r * F, drow.data(), F);
    }
  }
  std::vector<double> comb(rows_of(T, H), 0.0);
  for (int t = 0; t < T; ++t) {
    double* o = comb.data() + (size_t)t * H;
    for (int j = 0; j < k; ++j) {
      const double wj = w[(size_t)t * k + j];
      const double* y = ys.data() + (size_t)inv[(size_t)t * k + j] * H;
      for (int i = 0; i < H; ++i) o[i] += wj * y[i];
    }
  }
  if (ffn_out) std::copy(comb.begin(), comb.end(), ffn_out);
  if (x_out)
    for (size_t i = 0; i < (size_t)T * H; ++i) x_out[i] = x[i] + comb[i];
  if (tap) {
    if (tap->router_logits) std::copy(logits.begin(), logits.end(), tap->router_logits);
    if (tap->topk_idx) std::copy(idx.begin(), idx.end(), tap->topk_idx);
    if (tap->topk_w) std::copy(w.begin(), w.end(), tap->topk_w);
    if (tap->router_margin) std::copy(margin.begin(), margin.end(), tap->router_margin);
    if (tap->counts) std::copy(counts.begin(), counts.end(), tap->counts);
    if (tap->offsets) std::copy(offsets.begin(), offsets.end(), tap->offsets);
    if (tap->perm) std::copy(perm.begin(), perm.end(), tap->perm);
    if (tap->inv) std::copy(inv.begin(), inv.end(), tap->inv);
    if (tap->union_size) *tap->union_size = u;
  }
}

// residual stream start: the embedding rows of the tokens (untied, unscaled)
void oc_embed(const oc_config* cp, const oc_weights* Wp, const int32_t* tokens, int32_t T, double* x) {
  const int H = cp->hidden;
  for (int t = 0; t < T; ++t) widen_row(Wp->embed, (size_t)tokens[t] * H, H, x + (size_t)t * H);
}

// final RMSNorm, then the projection onto every vocabulary entry: logits [T][V].
// [DG-explainer] "Uniform State Diffusion": every position gets a full distribution.
void oc_vocab_logits(const oc_config* cp, const oc_weights* Wp, const double* x, int32_t T, double* logits) {
  const int H = cp->hidden;
  std::vector<double> xn(rows_of(T, H));
  oc_rms_norm(x, T, H, cp->rms_eps, xn.data());
  matmul_xwt(xn.data(), T, H, Wp->w_out, 0, cp->vocab, logits);
}

// One denoising pass ([DG-explainer] "Two modes, one model": denoising mode): the canvas
// tokens at positions P..P+C-1 attend to the whole cache and the whole canvas; the cache
// (per layer [nkv][P][d], stored values) is read, never written.  logits [C][V]
// (NULL: skip the projection); taps: n_layers records or NULL.
void oc_denoise_pass(const oc_config* cp, const oc_weights* Wp, const double* const* cache_k,
                     const double* const* cache_v, int32_t P, const int32_t* canvas, int32_t C, double* logits,
                     oc_taps* taps) {
  const int H = cp->hidden;
  std::vector<double> x(rows_of(C, H)), xa(rows_of(C, H));
  oc_embed(cp, Wp, canvas, C, x.data());
  for (int l = 0; l < cp->n_layers; ++l) {
    oc_taps* tap = taps ? taps + l : nullptr;
    if (tap && tap->x_in) std::copy(x.begin(), x.end(), tap->x_in);
    oc_attention_block(cp, Wp, l, cache_k[l], cache_v[l], P, x.data(), C, 0, xa.data(), tap ? tap->attn_o : nullptr,
                       tap ? tap->k_new : nullptr, tap ? tap->v_new : nullptr);
    if (tap && tap->x_attn) std::copy(xa.begin(), xa.end(), tap->x_attn);
    oc_moe_block(cp, Wp, l, xa.data(), C, x.data(), nullptr, tap);
    if (tap && tap->x_out) std::copy(x.begin(), x.end(), tap->x_out);
  }
  if (logits) oc_vocab_logits(cp, Wp, x.data(), C, logits);
}

// Causal prefill of T tokens at positions P..P+T-1 ([DG-explainer] "Two modes, one
// model" / "Long-form text: chaining canvases"): k_out, v_out (per layer [nkv][T][d])
// receive the K/V the cache stores for them (rounded to bf16 in a bf16 model).  Only
// K/V matter, so the last layer stops after its K/V.  taps: n_layers - 1 records or NULL.
void oc_prefill(const oc_config* cp, const oc_weights* Wp, const double* const* cache_k, const double* const* cache_v,
                int32_t P, const int32_t* tokens, int32_t T, double* const* k_out, double* const* v_out,
                oc_taps* taps) {
  const int H = cp->hidden, nkv = cp->n_kv_heads, d = cp->head_dim;
  std::vector<double> x(rows_of(T, H)), xa(rows_of(T, H));
  oc_embed(cp, Wp, tokens, T, x.data());
  const size_t nkvd = (size_t)nkv * T * d;
  for (int l = 0; l < cp->n_layers; ++l) {
    oc_taps* tap = (taps && l < cp->n_layers - 1) ? taps + l : nullptr;
    if (tap && tap->x_in) std::copy(x.begin(), x.end(), tap->x_in);
    if (l == cp->n_layers - 1) {   // K/V only
      std::vector<int64_t> pos(T);
      for (int t = 0; t < T; ++t) pos[t] = (int64_t)P + t;
      std::vector<double> q, k, v;
      qkv(*cp, *Wp, l, x.data(), T, pos.data(), q, k, v);
      std::copy(k.begin(), k.end(), k_out[l]);
      std::copy(v.begin(), v.end(), v_out[l]);
    } else {
      oc_attention_block(cp, Wp, l, cache_k[l], cache_v[l], P, x.data(), T, 1, xa.data(),
                         tap ? tap->attn_o : nullptr, k_out[l], v_out[l]);
      if (tap && tap->x_attn) std::copy(xa.begin(), xa.end(), tap->x_attn);
      oc_moe_block(cp, Wp, l, xa.data(), T, x.data(), nullptr, tap);
      if (tap && tap->x_out) std::copy(x.begin(), x.end(), tap->x_out);
    }
    if (cp->bf16_storage) {   // what later calls read: the stored values
      oc_round_bf16(k_out[l], (int64_t)nkvd, k_out[l]);
      oc_round_bf16(v_out[l], (int64_t)nkvd, v_out[l]);
    }
  }
}

// Prefix and canvas recomputed together under the prefix/block mask, without a cache
// ([DLM-exercises] mask solution): per-layer K/V over all P + C positions as a cache
// would store them (k_out, v_out per layer [nkv][P+C][d]) and the canvas logits
// [C][V].  Prefix keys are read as stored values, canvas keys in flight.
void oc_full_sequence_states(const oc_config* cp, const oc_weights* Wp, const int32_t* prefix, int32_t P,
                             const int32_t* canvas, int32_t C, double* const* k_out, double* const* v_out,
                             double* logits) {
  const int H = cp->hidden, nq = cp->n_q_heads, nkv = cp->n_kv_heads, d = cp->head_dim;
  const int n = P + C;
  std::vector<int32_t> toks(n);
  std::copy(prefix, prefix + P, toks.begin());
  std::copy(canvas, canvas + C, toks.begin() + P);
  std::vector<int64_t> pos(n);
  std::iota(pos.begin(), pos.end(), 0);
  std::vector<uint8_t> mask((size_t)n * n);
  oc_block_mask(P, C, mask.data());
  std::vector<double> x(rows_of(n, H)), y(rows_of(n, H)), xm(rows_of(n, H));
  oc_embed(cp, Wp, toks.data(), n, x.data());
  for (int l = 0; l < cp->n_layers; ++l) {
    std::vector<double> q, k, v;
    qkv(*cp, *Wp, l, x.data(), n, pos.data(), q, k, v);
    std::vector<double> ks(k), vs(v);
    if (cp->bf16_storage) {
      oc_round_bf16(ks.data(), (int64_t)ks.size(), ks.data());
      oc_round_bf16(vs.data(), (int64_t)vs.size(), vs.data());
    }
    std::copy(ks.begin(), ks.end(), k_out[l]);
    std::copy(vs.begin(), vs.end(), v_out[l]);
    for (int h = 0; h < nkv; ++h)   // prefix keys as the cache holds them; block keys in flight
      for (int t = 0; t < P; ++t)
        for (int i = 0; i < d; ++i) {
          const size_t a = ((size_t)h * n + t) * d + i;
          k[a] = ks[a];
          v[a] = vs[a];
        }
    std::vector<double> o((size_t)nq * n * d);
    oc_attention(q.data(), k.data(), v.data(), mask.data(), nq, nkv, n, n, d, o.data());
    oc_attn_out(cp, Wp, l, o.data(), n, y.data());
    for (size_t i = 0; i < (size_t)n * H; ++i) xm[i] = x[i] + y[i];
    oc_moe_block(cp, Wp, l, xm.data(), n, x.data(), nullptr, nullptr);
  }
  oc_vocab_logits(cp, Wp, x.data() + (size_t)P * H, C, logits);
}

// ---------------------------------------------------------------- canvas update

static const uint64_t kGamma = 0x9E3779B97F4A7C15ULL;

// SplitMix64 (Steele, Lea & Flood 2014): output number n (0-based) of the stream seeded
// with `seed`
uint64_t oc_splitmix64(uint64_t seed, uint64_t n) {
  uint64_t z = seed + (n + 1) * kGamma;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

// fresh uniform token for re-noising position pos at step `step`: draw number
// (step << 32 | pos) of SplitMix64(seed), reduced to [0, vocab) by multiply-shift on
// its high 32 bits
int64_t oc_renoise_token(uint64_t seed, uint32_t step, uint32_t pos, int64_t vocab) {
  const uint64_t x = oc_splitmix64(seed, ((uint64_t)step << 32) | pos);
  return (int64_t)(((x >> 32) * (uint64_t)vocab) >> 32);
}

// positions re-noised after step s of S: floor(C f_s), the fraction going linearly
// from r_start (first step) to r_end (last step); one step uses r_start
int64_t oc_renoise_count(int64_t C, int64_t S, int64_t s, double r_start, double r_end) {
  if (S == 1) return (int64_t)std::floor(C * r_start + 1e-9);
  const double f = (r_start * (double)(S - 1 - s) + r_end * (double)s) / (double)(S - 1);
  return (int64_t)std::floor(C * f + 1e-9);
}

// [DG-explainer] "Uniform State Diffusion": every position takes its argmax (ties to the
// lowest id); the n_renoise least confident positions (confidence = largest softmax
// probability; ties to the lower position) get a fresh random token.
// Outputs [C]: canvas, argmax, conf, top_margin (top-1 minus top-2 logit), renoised
// (0/1), cut_margin (log-confidence distance to the other side of the cut, +inf when
// n is 0 or C).
void oc_canvas_update(const double* logits, int32_t C, int32_t V, int32_t n_renoise, uint64_t seed, uint32_t step,
                      int32_t* canvas, int32_t* argmax, double* conf, double* top_margin, uint8_t* renoised,
                      double* cut_margin) {
  std::vector<double> lc(C);
  for (int i = 0; i < C; ++i) {
    const double* l = logits + (size_t)i * V;
    int a = 0;
    double m = l[0];
    for (int v = 1; v < V; ++v)
      if (l[v] > m) {
        m = l[v];
        a = v;
      }
    double m2 = -std::numeric_limits<double>::infinity();   // second largest (a duplicate max counts)
    for (int v = 0; v < V; ++v)
      if (v != a) m2 = std::max(m2, l[v]);
    double denom = 0.0;
    for (int v = 0; v < V; ++v) denom += std::exp(l[v] - m);
    argmax[i] = a;
    conf[i] = 1.0 / denom;
    top_margin[i] = V > 1 ? m - m2 : std::numeric_limits<double>::infinity();
    lc[i] = std::log(conf[i]);
  }
  std::vector<int> order(C);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [conf](int a, int b) { return conf[a] < conf[b]; });
  for (int i = 0; i < C; ++i) {
    renoised[i] = 0;
    canvas[i] = argmax[i];
  }
  for (int r = 0; r < n_renoise; ++r) renoised[order[r]] = 1;
  for (int i = 0; i < C; ++i)
    if (renoised[i]) canvas[i] = (int32_t)oc_renoise_token(seed, step, (uint32_t)i, V);
  for (int i = 0; i < C; ++i) cut_margin[i] = std::numeric_limits<double>::infinity();
  if (n_renoise > 0 && n_renoise < C) {
    const double lo_out = lc[order[n_renoise]];      // least confident kept position
    const double hi_in = lc[order[n_renoise - 1]];   // most confident re-noised position
    for (int i = 0; i < C; ++i) cut_margin[i] = renoised[i] ? lo_out - lc[i] : lc[i] - hi_in;
  }
}

// [DG-explainer] "First attempt: masked diffusion": a position holding a token other
// than mask_id is locked; a masked position's candidate is its argmax over every token
// except mask_id (ties to the lowest id), its confidence that token's softmax
// probability over all V logits; of the M masked positions the min(n_keep, M) least
// confident (ties to the lower position) stay masked, the others take their candidates.
// Outputs [C]: canvas_out, cand, conf, top_margin (among candidate logits), kept (0/1),
// cut_margin (masked positions; +inf elsewhere or when nothing is cut).
void oc_canvas_update_masked(const double* logits, int32_t C, int32_t V, const int32_t* canvas_in, int32_t n_keep,
                             int32_t mask_id, int32_t* canvas_out, int32_t* cand, double* conf, double* top_margin,
                             uint8_t* kept, double* cut_margin) {
  const double ninf = -std::numeric_limits<double>::infinity();
  std::vector<double> lc(C);
  for (int i = 0; i < C; ++i) {
    const double* l = logits + (size_t)i * V;
    double m = ninf;
    for (int v = 0; v < V; ++v) m = std::max(m, l[v]);
    double denom = 0.0;
    for (int v = 0; v < V; ++v) denom += std::exp(l[v] - m);
    int a = -1;
    double best = ninf;
    for (int v = 0; v < V; ++v)
      if (v != mask_id && (a < 0 || l[v] > best)) {
        best = l[v];
        a = v;
      }
    double second = ninf;
    for (int v = 0; v < V; ++v)
      if (v != mask_id && v != a) second = std::max(second, l[v]);
    cand[i] = a;
    conf[i] = std::exp(best - m) / denom;
    top_margin[i] = V > 2 ? best - second : std::numeric_limits<double>::infinity();
    lc[i] = std::log(conf[i]);
  }
  std::vector<int> masked;
  for (int i = 0; i < C; ++i)
    if (canvas_in[i] == mask_id) masked.push_back(i);
  const int M = (int)masked.size();
  const int keep = std::min<int>(n_keep, M);
  std::vector<int> order(masked);
  std::stable_sort(order.begin(), order.end(), [conf](int a, int b) { return conf[a] < conf[b]; });
  for (int i = 0; i < C; ++i) {
    kept[i] = 0;
    canvas_out[i] = canvas_in[i];
    cut_margin[i] = std::numeric_limits<double>::infinity();
  }
  for (int i : masked) canvas_out[i] = cand[i];
  for (int r = 0; r < keep; ++r) {
    kept[order[r]] = 1;
    canvas_out[order[r]] = mask_id;
  }
  if (keep > 0 && keep < M) {
    const double lo_out = lc[order[keep]];      // least confident filled position
    const double hi_in = lc[order[keep - 1]];   // most confident position kept masked
    for (int i : masked) cut_margin[i] = kept[i] ? lo_out - lc[i] : lc[i] - hi_in;
  }
}

// ---------------------------------------------------------------- 8- and 4-bit weights
// The OCP "E4M3" element format with MX block scaling (one power-of-two scale per 32
// elements), and E2M1 elements with an E4M3 scale per 16 elements and an fp32 tensor
// scale, written from the published definitions ([DLM-exercises] MoE remark: FP8 and
// NVFP4 deployments).

// E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is subnormal
// (m 2^-9); 0x7F / 0xFF are NaN; no infinities
double oc_e4m3_decode(int32_t code) {
  const double s = (code & 0x80) ? -1.0 : 1.0;
  const int e = (code >> 3) & 0xF, m = code & 0x7;
  if (e == 0xF && m == 0x7) return std::numeric_limits<double>::quiet_NaN();
  if (e == 0) return s * m * std::ldexp(1.0, -9);
  return s * (1.0 + m / 8.0) * std::ldexp(1.0, e - 7);
}

// E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit; exponent 0 is subnormal (m/2)
double oc_e2m1_decode(int32_t code) {
  const double s = (code & 0x8) ? -1.0 : 1.0;
  const int e = (code >> 1) & 0x3, m = code & 0x1;
  if (e == 0) return s * 0.5 * m;
  return s * (1.0 + 0.5 * m) * std::ldexp(1.0, e - 1);
}

// nearest code among the n increasing non-negative values of `pos` (codes 0..n-1),
// ties to the even code; magnitudes beyond the last value saturate; sign_bit on x < 0
static int nearest_code(const double* pos, int n, double x, int sign_bit) {
  const double a = std::min(std::fabs(x), pos[n - 1]);
  int i = 0;
  while (i < n && pos[i] < a) ++i;   // first value >= a
  int c;
  if (pos[i] == a) {
    c = i;
  } else {
    const int lo = i - 1, hi = i;
    const double dlo = a - pos[lo], dhi = pos[hi] - a;
    c = (dlo < dhi || (dlo == dhi && lo % 2 == 0)) ? lo : hi;
  }
  return c | (std::signbit(x) ? sign_bit : 0);
}

static const double* e4m3_positive_values() {   // codes 0x00 .. 0x7E, increasing
  static double v[0x7F];
  static bool init = false;
  if (!init) {
    for (int c = 0; c < 0x7F; ++c) v[c] = oc_e4m3_decode(c);
    init = true;
  }
  return v;
}

int32_t oc_e4m3_encode(double x) { return nearest_code(e4m3_positive_values(), 0x7F, x, 0x80); }

int32_t oc_e2m1_encode(double x) {
  static const double pos[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  return nearest_code(pos, 8, x, 0x8);
}

void oc_e4m3_encode_array(const double* x, int64_t n, uint8_t* codes) {
  for (int64_t i = 0; i < n; ++i) codes[i] = (uint8_t)oc_e4m3_encode(x[i]);
}

void oc_e2m1_encode_array(const double* x, int64_t n, uint8_t* codes) {
  for (int64_t i = 0; i < n; ++i) codes[i] = (uint8_t)oc_e2m1_encode(x[i]);
}

// MX block scaling along rows of length n (rows x n values): each block of 32 shares
// the power-of-two scale X = 2^(floor(log2(max |v|)) - 8) (8 = the largest E4M3
// exponent), each value stored as e4m3_encode(v / X); an all-zero block gets exponent -127
void oc_mx_e4m3_quantize(const double* w, int64_t rows, int32_t n, uint8_t* codes, int32_t* exps) {
  const int nb = n / 32;
  for (int64_t r = 0; r < rows; ++r)
    for (int b = 0; b < nb; ++b) {
      const double* v = w + r * n + b * 32;
      double amax = 0.0;
      for (int i = 0; i < 32; ++i) amax = std::max(amax, std::fabs(v[i]));
      int e = amax > 0 ? (int)std::floor(std::log2(amax)) - 8 : -127;
      e = std::min(127, std::max(-127, e));
      exps[r * nb + b] = e;
      for (int i = 0; i < 32; ++i) codes[r * n + b * 32 + i] = (uint8_t)oc_e4m3_encode(v[i] / std::ldexp(1.0, e));
    }
}

void oc_mx_e4m3_dequantize(const uint8_t* codes, const int32_t* exps, int64_t rows, int32_t n, double* out) {
  const int nb = n / 32;
  for (int64_t r = 0; r < rows; ++r)
    for (int i = 0; i < n; ++i)
      out[r * n + i] = oc_e4m3_decode(codes[r * n + i]) * std::ldexp(1.0, exps[r * nb + i / 32]);
}

// two-level scaling: tensor scale g = max |w| / (448 6); per block of 16 an E4M3 scale
// code for max |v| / (6 g); each value stored as e2m1_encode(v / (s_b g)), s_b the
// decoded block scale.  Returns g.
double oc_nvfp4_quantize(const double* w, int64_t rows, int32_t n, uint8_t* codes, uint8_t* scale_codes) {
  const int nb = n / 16;
  double amax_t = 0.0;
  for (int64_t i = 0; i < rows * n; ++i) amax_t = std::max(amax_t, std::fabs(w[i]));
  const double g = amax_t > 0 ? amax_t / (448.0 * 6.0) : 1.0;
  for (int64_t r = 0; r < rows; ++r)
    for (int b = 0; b < nb; ++b) {
      const double* v = w + r * n + b * 16;
      double amax = 0.0;
      for (int i = 0; i < 16; ++i) amax = std::max(amax, std::fabs(v[i]));
      const int sc = oc_e4m3_encode(amax / (6.0 * g));
      scale_codes[r * nb + b] = (uint8_t)sc;
      const double sb = oc_e4m3_decode(sc);
      const double denom = sb > 0 ? sb * g : 1.0;
      for (int i = 0; i < 16; ++i) codes[r * n + b * 16 + i] = (uint8_t)oc_e2m1_encode(v[i] / denom);
    }
  return g;
}

void oc_nvfp4_dequantize(const uint8_t* codes, const uint8_t* scale_codes, double g, int64_t rows, int32_t n,
                         double* out) {
  const int nb = n / 16;
  for (int64_t r = 0; r < rows; ++r)
    for (int i = 0; i < n; ++i)
      out[r * n + i] = oc_e2m1_decode(codes[r * n + i]) * (oc_e4m3_decode(scale_codes[r * nb + i / 16]) * g);
}

int32_t oc_num_threads(void) { return omp_get_max_threads(); }

}  // extern "C"
