"""CPU oracle of the block-diffusion denoising pass, numpy restatement -- TEST
INFRASTRUCTURE ONLY.  The oracle the tests use is the C++ one (`dg_oracle.cpp`, bound
by `dg_oracle.py`); this independent numpy version of the same definitions is kept as
its cross-check (`tests/test_oracle_cpp.py`).

Nothing in the product path may import, call or execute this module; only the
tests, the smoke check and the benchmark's CPU baseline use it.  It shares no
code with the CUDA path and imports nothing from the package.

Plain, slow, obviously correct numpy in float64.  Matrix products use numpy's
matmul as a library primitive; nothing is blocked, fused or reordered beyond
what each definition states (the vocabulary projection and the expert loop are
evaluated piecewise only to bound memory; every output element is the same
dot product either way).

Sources (page title -- section):
  [DG-explainer]  "DiffusionGemma" video explainer -- "The fix: a 256-token canvas",
                  "Uniform State Diffusion", "Two modes, one model",
                  "Long-form text: chaining canvases"
  [DLM-exercises] "Module 12. Diffusion Language Models" exercises -- the prefix/block
                  mask solution (7x7 worked example) and the MoE remark in the
                  roofline solution
  [DG-intro]      "Introducing DiffusionGemma: An Attempt to Speed Up Text Generation
                  by Blocks" -- "What is DiffusionGemma?", "The Meaning of 'Seeing
                  the Whole'"

Readings where the pages are silent (each one listed in the design notes):
  pre-norm RMSNorm without gain (eps from the config); RoPE rotate-half with
  theta from the config at absolute positions; GQA query head h -> kv head
  h // (nq/nkv); attention scale 1/sqrt(d); router on the fp32-normed residual,
  top-k by value with ties to the lower expert id, weights = softmax over the
  k chosen logits; SwiGLU experts; untied embedding / output matrices;
  confidence = largest softmax probability (temperature 1); every position
  takes its argmax (ties to the lowest id), then the n lowest-confidence
  positions (ties to the lower position) get a fresh random token.  The
  masked-diffusion variant (canvas_update_masked) states its own readings.

Precision model.  The pages fix no precision beyond bf16 weights, so the oracle
follows the kernel's storage precision, because later integer decisions (routing,
argmax, re-noise set) depend on it and both sides must take them at the same
precision.  The fp32 model computes everything in float64 here.  A bf16 model
stores its weights and its KV cache in bf16; everything in flight -- the
activations handed to GEMMs, the query, the K/V of the tokens the call itself
processes (the canvas in a denoising pass, the new tokens in a prefill) and the input
of the vocabulary projection -- is exact here.  So `Precision('bf16')` rounds
(round-to-nearest-even) exactly where a value is stored: K/V written to the cache.
Everything else stays float64.
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------
# storage decoding and rounding


def widen(a: np.ndarray) -> np.ndarray:
    """Exact float64 value of a stored tensor (uint16 = bf16 bit patterns, or a float array)."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (8 significant bits), ties to even."""
    m, e = np.frexp(np.asarray(x, dtype=np.float64))
    return np.ldexp(np.rint(m * 256.0), e - 8)


class Precision:
    def __init__(self, dtype: str):
        assert dtype in ("bf16", "f32")
        self.dtype = dtype

    def store(self, x: np.ndarray) -> np.ndarray:
        """A value stored in the model's storage dtype (KV cache entries)."""
        return round_bf16(x) if self.dtype == "bf16" else x


# ----------------------------------------------------------------------------
# layer primitives


def rms_norm(x: np.ndarray, eps: float) -> np.ndarray:
    """y = x / sqrt(mean(x^2) + eps) over the last axis (unit gain)."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def rope(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotary position embedding, rotate-half pairing (i, i + d/2), on x[..., T, d]."""
    d = x.shape[-1]
    half = d // 2
    inv_freq = theta ** (-(np.arange(half, dtype=np.float64) * 2.0) / d)
    ang = positions.astype(np.float64)[:, None] * inv_freq[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def block_mask(P: int, C: int) -> np.ndarray:
    """Allowed-attention matrix over rows/columns ordered (prefix 0..P-1, block 0..C-1).

    [DLM-exercises], prefix/block mask solution: a prefix query sees only the prefix
    keys at or before it (causal); every block query sees the whole prefix and the
    whole block (bidirectional).  No prefix query sees a block key.
    """
    n = P + C
    allowed = np.zeros((n, n), dtype=bool)
    for i in range(n):
        for j in range(n):
            if i < P:
                allowed[i, j] = j <= i
            else:
                allowed[i, j] = True
    return allowed


def causal_rows(P: int, T: int) -> np.ndarray:
    """Rows for T new tokens at positions P..P+T-1 over keys 0..P+T-1, prefill mode.

    [DG-explainer] "Two modes, one model": prefill attention is causal (left to right).
    """
    allowed = np.zeros((T, P + T), dtype=bool)
    for i in range(T):
        allowed[i, : P + i + 1] = True
    return allowed


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, allowed: np.ndarray) -> np.ndarray:
    """Masked softmax attention with grouped KV heads.

    q [nq][Tq][d]; k, v [nkv][Tk][d]; allowed [Tq][Tk] bool.  Query head h reads
    KV head h // (nq / nkv); scores are scaled by 1/sqrt(d).  Returns [nq][Tq][d].
    """
    nq, Tq, d = q.shape
    nkv = k.shape[0]
    g = nq // nkv
    out = np.empty_like(q)
    for h in range(nq):
        s = (q[h] @ k[h // g].T) / np.sqrt(d)
        s = np.where(allowed, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[h] = p @ v[h // g]
    return out


def router_topk(logits: np.ndarray, k: int):
    """Top-k experts per token by router logit; ties go to the lower expert id.

    Returns (idx [T][k] int32 in descending-logit order, w [T][k] = softmax over the
    k chosen logits, margin [T] = k-th minus (k+1)-th largest logit).
    [DLM-exercises]: "different canvas positions can select different experts".
    """
    T, E = logits.shape
    order = np.argsort(-logits, axis=1, kind="stable")
    idx = order[:, :k].astype(np.int32)
    chosen = np.take_along_axis(logits, order[:, :k], axis=1)
    w = np.exp(chosen - chosen.max(axis=1, keepdims=True))
    w = w / w.sum(axis=1, keepdims=True)
    if k < E:
        nxt = np.take_along_axis(logits, order[:, k:k + 1], axis=1)[:, 0]
        margin = chosen[:, -1] - nxt
    else:
        margin = np.full(T, np.inf)
    return idx, w, margin


def expert_permutation(idx: np.ndarray, n_experts: int):
    """Group the T*k (token, slot) assignments by expert, stably.

    Returns counts [E], offsets [E+1] (exclusive prefix sum), perm [T*k] (perm[p] =
    flattened assignment t*k + j placed at row p, ordered by (expert, t, j)),
    inv [T*k] (inverse of perm) and the expert union size U = #{e : counts[e] > 0},
    the set of experts a pass must read ([DLM-exercises] MoE remark).
    """
    T, k = idx.shape
    flat = idx.reshape(-1)
    keys = sorted(range(T * k), key=lambda a: (int(flat[a]), a // k, a % k))
    perm = np.array(keys, dtype=np.int64)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(T * k)
    counts = np.bincount(flat, minlength=n_experts).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    union = int((counts > 0).sum())
    return counts, offsets, perm, inv, union


# ----------------------------------------------------------------------------
# the transformer stack


def _qkv(model, l: int, x: np.ndarray, positions: np.ndarray, prec: Precision):
    cfg = model.cfg
    nq, nkv, d = cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    L = model.layers[l]
    xn = rms_norm(x, cfg["rms_eps"])
    T = x.shape[0]
    q = (xn @ widen(L["w_q"]).T).reshape(T, nq, d).transpose(1, 0, 2)
    k = (xn @ widen(L["w_k"]).T).reshape(T, nkv, d).transpose(1, 0, 2)
    v = (xn @ widen(L["w_v"]).T).reshape(T, nkv, d).transpose(1, 0, 2)
    q = rope(q, positions, cfg["rope_theta"])
    k = rope(k, positions, cfg["rope_theta"])
    return q, k, v


def _attn_out(model, l: int, o: np.ndarray, prec: Precision) -> np.ndarray:
    T = o.shape[1]
    o = o.transpose(1, 0, 2).reshape(T, -1)
    return o @ widen(model.layers[l]["w_o"]).T


def moe(model, l: int, x: np.ndarray, prec: Precision, tap: dict | None = None) -> np.ndarray:
    """Sparse MoE FFN on the residual x [T][H]; returns the FFN output [T][H].

    Router on the fp32-normed residual -> top-k -> stable expert grouping ->
    per-expert SwiGLU over only the rows routed to it (the union of experts) ->
    combine sum_j w[t,j] * y[t,j] in slot order.
    """
    cfg = model.cfg
    E, k = cfg["n_experts"], cfg["top_k"]
    L = model.layers[l]
    xn = rms_norm(x, cfg["rms_eps"])
    logits = xn @ widen(L["w_router"]).T
    idx, w, margin = router_topk(logits, k)
    counts, offsets, perm, inv, union = expert_permutation(idx, E)
    xs = xn
    T, H = x.shape
    ys = np.zeros((T * k, H))
    for e in range(E):
        rows = perm[offsets[e]:offsets[e + 1]]
        if rows.size == 0:
            continue
        xe = xs[rows // k]
        g = xe @ widen(L["w_gate"][e]).T
        u = xe @ widen(L["w_up"][e]).T
        h = silu(g) * u
        ys[offsets[e]:offsets[e + 1]] = h @ widen(L["w_down"][e]).T
    out = np.zeros((T, H))
    for j in range(k):
        out += w[:, j:j + 1] * ys[inv.reshape(T, k)[:, j]]
    if tap is not None:
        tap.update(router_logits=logits, topk_idx=idx, topk_w=w, router_margin=margin,
                   counts=counts, offsets=offsets, perm=perm, union=union)
    return out


def embed(model, tokens: np.ndarray) -> np.ndarray:
    """Residual stream start: the embedding rows of the canvas tokens (untied, unscaled)."""
    return widen(model.embed[np.asarray(tokens)])


def vocab_logits(model, x: np.ndarray, prec: Precision, rows=None, chunk: int = 16384) -> np.ndarray:
    """Final RMSNorm then projection onto every vocabulary entry (fp64 logits).

    [DG-explainer] "Uniform State Diffusion": every canvas position is updated in
    parallel, so every row gets a full distribution over the vocabulary.
    """
    cfg = model.cfg
    xn = rms_norm(x, cfg["rms_eps"])
    if rows is not None:
        xn = xn[np.asarray(rows)]
    V = cfg["vocab"]
    out = np.empty((xn.shape[0], V))
    for v0 in range(0, V, chunk):
        out[:, v0:v0 + chunk] = xn @ widen(model.w_out[v0:v0 + chunk]).T
    return out


class Cache:
    """Per-layer KV cache in the logical layout K, V [nkv][len][d] (float64 values)."""

    def __init__(self, layers_kv):
        self.k = [widen(k) for k, _ in layers_kv]
        self.v = [widen(v) for _, v in layers_kv]

    @classmethod
    def empty(cls, cfg):
        z = np.zeros((cfg["n_kv_heads"], 0, cfg["head_dim"]))
        c = cls([])
        c.k = [z.copy() for _ in range(cfg["n_layers"])]
        c.v = [z.copy() for _ in range(cfg["n_layers"])]
        return c

    @property
    def len(self) -> int:
        return self.k[0].shape[1]

    def copy(self):
        c = Cache([])
        c.k = [a.copy() for a in self.k]
        c.v = [a.copy() for a in self.v]
        return c


def denoise_pass(model, cache: Cache, canvas: np.ndarray, prec: Precision, logit_rows=None):
    """One denoising pass over the canvas (denoising mode).

    [DG-explainer] "Two modes, one model": every canvas token attends to all other
    canvas tokens and to the KV cache (bidirectional).  [DLM-exercises] mask
    solution: the prefix K/V in the cache is reused as is, only the block's states
    are recomputed, and the cache is not modified.  Canvas positions are
    P..P+C-1 with P = cache length.

    Returns (logits [C or len(logit_rows)][V], per-layer taps).
    """
    cfg = model.cfg
    P = cache.len
    C = len(canvas)
    pos = np.arange(P, P + C)
    x = embed(model, canvas)
    mask = block_mask(P, C)[P:, :]            # the block rows of the prefix/block mask
    taps = []
    for l in range(cfg["n_layers"]):
        tap = {"x_in": x.copy()}
        q, k, v = _qkv(model, l, x, pos, prec)
        kk = np.concatenate([cache.k[l], k], axis=1)   # cached prefix (stored) + canvas (in flight)
        vv = np.concatenate([cache.v[l], v], axis=1)
        o = attention(q, kk, vv, mask)
        tap["attn_o"] = o.transpose(1, 0, 2).reshape(C, -1)
        x = x + _attn_out(model, l, o, prec)
        tap["x_attn"] = x.copy()
        x = x + moe(model, l, x, prec, tap)
        tap["x_out"] = x.copy()
        taps.append(tap)
    return vocab_logits(model, x, prec, rows=logit_rows), taps


def prefill_append(model, cache: Cache, tokens: np.ndarray, prec: Precision, taps: list | None = None) -> Cache:
    """Causal prefill of T tokens at positions P..P+T-1, appending their K/V (prefill mode).

    [DG-explainer] "Two modes, one model" / "Long-form text: chaining canvases": the
    prompt and then each completed canvas are read left to right with causal
    attention and written to the KV cache.  Only K/V matter, so the last layer
    stops after writing its K/V.
    """
    cfg = model.cfg
    P = cache.len
    T = len(tokens)
    pos = np.arange(P, P + T)
    out = cache.copy()
    x = embed(model, tokens)
    mask = causal_rows(P, T)
    for l in range(cfg["n_layers"]):
        q, k, v = _qkv(model, l, x, pos, prec)
        out.k[l] = np.concatenate([cache.k[l], prec.store(k)], axis=1)   # what later calls read
        out.v[l] = np.concatenate([cache.v[l], prec.store(v)], axis=1)
        if l == cfg["n_layers"] - 1:
            break
        o = attention(q, np.concatenate([cache.k[l], k], axis=1), np.concatenate([cache.v[l], v], axis=1), mask)
        x = x + _attn_out(model, l, o, prec)
        tap = {} if taps is not None else None
        x = x + moe(model, l, x, prec, tap)
        if taps is not None:
            taps.append(tap)
    return out


def full_sequence_states(model, prefix_tokens: np.ndarray, canvas: np.ndarray, prec: Precision):
    """Recompute prefix and canvas together under the prefix/block mask, no cache.

    Returns (per-layer K, V over all P+C positions, canvas logits).  Used to check
    that the cached path (prefill the prefix, then denoise against the cache) is
    the same computation ([DLM-exercises] mask solution: prefix K/V reusable).
    """
    cfg = model.cfg
    P, C = len(prefix_tokens), len(canvas)
    toks = np.concatenate([prefix_tokens, canvas])
    pos = np.arange(P + C)
    mask = block_mask(P, C)
    x = embed(model, toks)
    ks, vs = [], []
    for l in range(cfg["n_layers"]):
        q, k, v = _qkv(model, l, x, pos, prec)
        ks.append(prec.store(k))
        vs.append(prec.store(v))
        # prefix keys as the cache holds them; block keys in flight
        kk = np.concatenate([prec.store(k[:, :P]), k[:, P:]], axis=1)
        vv = np.concatenate([prec.store(v[:, :P]), v[:, P:]], axis=1)
        o = attention(q, kk, vv, mask)
        x = x + _attn_out(model, l, o, prec)
        x = x + moe(model, l, x, prec)
    return ks, vs, vocab_logits(model, x[P:], prec)


# ----------------------------------------------------------------------------
# canvas update


_GAMMA = 0x9E3779B97F4A7C15
_MASK64 = (1 << 64) - 1


def splitmix64(seed: int, n: int) -> int:
    """SplitMix64 (Steele, Lea & Flood 2014): output number n (0-based) of the stream seeded with `seed`."""
    z = (seed + (n + 1) * _GAMMA) & _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def renoise_token(seed: int, step: int, pos: int, vocab: int) -> int:
    """Fresh uniform vocabulary token for re-noising position `pos` at denoising step `step`.

    Draw number (step << 32 | pos) of SplitMix64(seed), reduced to [0, vocab) by
    multiply-shift on its high 32 bits.
    """
    x = splitmix64(seed, (step << 32) | pos)
    return ((x >> 32) * vocab) >> 32


def renoise_count(C: int, S: int, s: int, r_start: float, r_end: float) -> int:
    """Positions re-noised after step s of S: floor(C * f_s), with the fraction f_s going
    linearly from r_start (first step) to r_end (last step); one step uses r_start."""
    if S == 1:
        return int(np.floor(C * r_start + 1e-9))
    f = (r_start * (S - 1 - s) + r_end * s) / (S - 1)
    return int(np.floor(C * f + 1e-9))


def canvas_update(logits: np.ndarray, n_renoise: int, seed: int, step: int) -> dict:
    """Update every position, then re-noise the least confident ones.

    [DG-explainer] "Uniform State Diffusion": every position is updated in parallel;
    tokens with low confidence are replaced by a fresh random vocabulary token so
    later passes can correct them.  Confidence = largest softmax probability.

    Returns canvas, argmax, conf, top-1/top-2 logit margin, the re-noised positions
    (as a sorted array) and each position's log-confidence distance to the cut.
    """
    C, V = logits.shape
    m = logits.max(axis=1)
    argmax = np.argmax(logits, axis=1).astype(np.int64)       # first (lowest) id on ties
    denom = np.exp(logits - m[:, None]).sum(axis=1)
    conf = 1.0 / denom
    srt = np.sort(logits, axis=1)
    top_margin = srt[:, -1] - srt[:, -2] if V > 1 else np.full(C, np.inf)
    order = np.argsort(conf, kind="stable")                    # ties: lower position first
    chosen = np.sort(order[:n_renoise])
    canvas = argmax.copy()
    for i in chosen:
        canvas[i] = renoise_token(seed, step, int(i), V)
    # distance (in log-confidence) of each position to the other side of the cut
    lc = np.log(conf)
    cut_margin = np.full(C, np.inf)
    if 0 < n_renoise < C:
        lo_out = lc[order[n_renoise]]       # least confident kept position
        hi_in = lc[order[n_renoise - 1]]    # most confident re-noised position
        sel = np.zeros(C, dtype=bool)
        sel[chosen] = True
        cut_margin = np.where(sel, lo_out - lc, lc - hi_in)
    return dict(canvas=canvas.astype(np.int32), argmax=argmax.astype(np.int32), conf=conf,
                top_margin=top_margin, renoised=chosen, cut_margin=cut_margin)


def canvas_update_masked(logits: np.ndarray, canvas: np.ndarray, n_keep: int, mask_id: int) -> dict:
    """Masked-diffusion update: fill [MASK] positions, which then stay fixed.

    [DG-explainer] "First attempt: masked diffusion": noise is a [MASK] placeholder; the
    model predicts the word and fills it in, and a filled position is locked from then on.
    Readings (the page gives no more): a position holding any token other than
    `mask_id` is locked and keeps it; a masked position's candidate is its argmax over
    every token except `mask_id` (ties to the lowest id), its confidence that token's
    softmax probability over all V logits; of the M masked positions the
    min(n_keep, M) least confident stay masked (ties to the lower position) and the
    others take their candidates.

    Returns the canvas, the candidates, the confidences, each position's top-1/top-2
    margin among the candidate logits, the positions kept masked (sorted) and each masked
    position's log-confidence distance to the cut (inf elsewhere).
    """
    C, V = logits.shape
    canvas = np.asarray(canvas).astype(np.int64)
    m = logits.max(axis=1)
    denom = np.exp(logits - m[:, None]).sum(axis=1)
    cand_logits = logits.copy()
    cand_logits[:, mask_id] = -np.inf
    cand = np.argmax(cand_logits, axis=1).astype(np.int64)      # first (lowest) id on ties
    conf = np.exp(cand_logits[np.arange(C), cand] - m) / denom
    srt = np.sort(cand_logits, axis=1)
    top_margin = srt[:, -1] - srt[:, -2] if V > 2 else np.full(C, np.inf)
    masked = np.nonzero(canvas == mask_id)[0]                    # ascending positions
    keep = min(int(n_keep), len(masked))
    order = masked[np.argsort(conf[masked], kind="stable")]      # ties: lower position first
    kept = np.sort(order[:keep])
    out = canvas.copy()
    out[masked] = cand[masked]
    out[kept] = mask_id
    lc = np.log(conf)
    cut_margin = np.full(C, np.inf)
    if 0 < keep < len(masked):
        lo_out = lc[order[keep]]        # least confident filled position
        hi_in = lc[order[keep - 1]]     # most confident position kept masked
        sel = np.zeros(C, dtype=bool)
        sel[kept] = True
        cut_margin[masked] = np.where(sel[masked], lo_out - lc[masked], lc[masked] - hi_in)
    return dict(canvas=out.astype(np.int32), argmax=cand.astype(np.int32), conf=conf, top_margin=top_margin,
                kept=kept, cut_margin=cut_margin)


def generate_canvas_masked(model, cache: Cache, C: int, S: int, keep_start: float, keep_end: float, mask_id: int,
                           prec: Precision, append: bool, record=None):
    """S passes of masked diffusion from an all-[MASK] canvas, then (optionally) append.

    [DG-explainer] "First attempt: masked diffusion" with the pass loop and the append of
    "Uniform State Diffusion" / "Long-form text: chaining canvases".  After pass s the
    number of positions that stay masked is at most renoise_count(C, S, s, keep_start,
    keep_end).  Returns (canvas, cache).
    """
    cur = np.full(C, mask_id, dtype=np.int32)
    for s in range(S):
        logits, taps = denoise_pass(model, cache, cur, prec)
        n = renoise_count(C, S, s, keep_start, keep_end)
        upd = canvas_update_masked(logits, cur, n, mask_id)
        if record is not None:
            record.append(dict(step=s, canvas_in=cur.copy(), logits=logits, taps=taps, update=upd, n=n))
        cur = upd["canvas"]
    if append:
        cache = prefill_append(model, cache, cur, prec)
    return cur, cache


def generate_canvas(model, cache: Cache, canvas: np.ndarray, S: int, r_start: float, r_end: float,
                    seed: int, prec: Precision, append: bool, record=None):
    """S denoising passes with re-noising, then (optionally) append the canvas by prefill.

    [DG-explainer] "Uniform State Diffusion" (several passes until the canvas
    converges) and "Long-form text: chaining canvases" (a completed canvas is
    appended to the KV cache via a prefill step).  Returns (canvas, cache).
    """
    C = len(canvas)
    cur = np.asarray(canvas, dtype=np.int32).copy()
    for s in range(S):
        logits, taps = denoise_pass(model, cache, cur, prec)
        n = renoise_count(C, S, s, r_start, r_end)
        upd = canvas_update(logits, n, seed, s)
        if record is not None:
            record.append(dict(step=s, canvas_in=cur.copy(), logits=logits, taps=taps, update=upd, n=n))
        cur = upd["canvas"]
    if append:
        cache = prefill_append(model, cache, cur, prec)
    return cur, cache


# ----------------------------------------------------------------------------
# several canvases at once


def denoise_pass_batched(model, caches: list, canvases, prec: Precision):
    """Denoising passes of B independent canvases, canvas b against its own cache.

    Hacker News discussion of DiffusionGemma, the comment on batching: batched requests
    share the reads of common weights -- which is all batching changes.

    Batching shares weight reads, not arithmetic: each canvas attends only to its own
    cache and its own canvas (one request each), and every per-token step (routing,
    experts, vocabulary projection) is row-wise, so canvas b's result is its
    single-canvas pass.  Returns [(logits, taps)] per canvas.
    """
    return [denoise_pass(model, c, np.asarray(x), prec) for c, x in zip(caches, canvases)]


def merge_batch_taps(per_canvas_taps: list, n_experts: int) -> list:
    """Per-layer taps of a batch from the canvases' own taps: row-wise entries stacked in
    canvas order; the expert histogram, stable permutation and union taken over all rows
    together, as one pass over the batch groups them."""
    out = []
    for layer_taps in zip(*per_canvas_taps):
        m = {key: np.concatenate([t[key] for t in layer_taps], axis=0)
             for key in ("x_in", "attn_o", "x_attn", "x_out", "router_logits", "topk_idx", "topk_w", "router_margin")}
        counts, offsets, perm, inv, union = expert_permutation(m["topk_idx"], n_experts)
        m.update(counts=counts, offsets=offsets, perm=perm, union=union)
        out.append(m)
    return out


def generate_canvases(model, caches: list, canvases, S: int, r_start: float, r_end: float, seeds, prec: Precision,
                      append: bool):
    """generate_canvas for each canvas with its own cache and re-noise seed.  Returns
    ([canvas], [cache])."""
    res = [generate_canvas(model, c, x, S, r_start, r_end, sd, prec, append)
           for c, x, sd in zip(caches, canvases, seeds)]
    return [r[0] for r in res], [r[1] for r in res]


# ----------------------------------------------------------------------------
# 8-bit expert weights (groundwork for the FP8 deployment the pages mention): the OCP
# "E4M3" element format and MX block scaling, written from the published definitions.
# Nothing in the pass uses these yet.

E4M3_MAX = 448.0


def e4m3_decode(code: int) -> float:
    """Value of an 8-bit E4M3 code: sign, 4 exponent bits (bias 7), 3 mantissa bits;
    exponent 0 is subnormal (m * 2^-9); 0x7F / 0xFF are NaN; no infinities."""
    code = int(code)  # numpy uint8 arithmetic would wrap in e - 7
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


_E4M3_POS = np.array([e4m3_decode(c) for c in range(0x7F)])  # codes 0x00 .. 0x7E, increasing


def e4m3_encode(x: float) -> int:
    """Nearest E4M3 code (ties to the even code, i.e. even mantissa); magnitudes beyond
    448 saturate to 448."""
    neg = np.signbit(x)
    a = min(abs(float(x)), E4M3_MAX)
    i = int(np.searchsorted(_E4M3_POS, a))  # first value >= a
    if i < len(_E4M3_POS) and _E4M3_POS[i] == a:
        c = i
    else:
        lo, hi = i - 1, i
        dlo, dhi = a - _E4M3_POS[lo], _E4M3_POS[hi] - a
        c = lo if (dlo < dhi or (dlo == dhi and lo % 2 == 0)) else hi
    return c | (0x80 if neg else 0)


def e4m3_encode_array(x) -> np.ndarray:
    """e4m3_encode element by element on an array (the same rule: nearest code, ties to
    the even code, magnitudes beyond 448 saturate), as uint8 codes."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    i = np.searchsorted(_E4M3_POS, a)  # first value >= a (a <= 448, the last value)
    hit = _E4M3_POS[i] == a
    lo = np.maximum(i - 1, 0)
    dlo, dhi = a - _E4M3_POS[lo], _E4M3_POS[i] - a
    pick_lo = (dlo < dhi) | ((dlo == dhi) & (lo % 2 == 0))
    c = np.where(hit, i, np.where(pick_lo, lo, i))
    return (c | np.where(np.signbit(x), 0x80, 0)).astype(np.uint8)


def mx_e4m3_quantize(w: np.ndarray, block: int = 32):
    """MX block scaling along the last axis: each block of `block` consecutive values
    shares the power-of-two scale X = 2^(floor(log2(max |v|)) - 8) (8 = the largest
    E4M3 exponent), and each value is stored as e4m3_encode(v / X).  Returns (codes
    uint8 [..., n], scale exponents int32 [..., n / block]); an all-zero block gets
    exponent -127."""
    w = np.asarray(w, dtype=np.float64)
    assert w.shape[-1] % block == 0
    blocks = w.reshape(*w.shape[:-1], w.shape[-1] // block, block)
    amax = np.abs(blocks).max(axis=-1)
    exp = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 8, -127).astype(np.int32)
    exp = np.clip(exp, -127, 127)
    scaled = blocks / np.ldexp(1.0, exp)[..., None]
    codes = e4m3_encode_array(scaled)
    return codes.reshape(w.shape), exp


_E4M3_ALL = np.array([e4m3_decode(c) for c in range(256)])  # value of every code (NaN at 0x7F, 0xFF)


def mx_e4m3_dequantize(codes: np.ndarray, exp: np.ndarray, block: int = 32) -> np.ndarray:
    """X * e4m3_decode(code) for every element."""
    vals = _E4M3_ALL[np.asarray(codes, dtype=np.int64)]
    blocks = vals.reshape(*vals.shape[:-1], vals.shape[-1] // block, block)
    return (blocks * np.ldexp(1.0, exp)[..., None]).reshape(vals.shape)


# 4-bit elements (E2M1: sign, 2 exponent bits with bias 1, 1 mantissa bit; no inf/NaN)
# scaled per 16-element block by an E4M3 value and per tensor by an fp32 value.


def e2m1_decode(code: int) -> float:
    code = int(code)
    s = -1.0 if code & 0x8 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        return s * 0.5 * m
    return s * (1.0 + 0.5 * m) * 2.0 ** (e - 1)


_E2M1_POS = np.array([e2m1_decode(c) for c in range(8)])  # 0, 0.5, 1, 1.5, 2, 3, 4, 6


def e2m1_encode(x: float) -> int:
    """Nearest E2M1 code (ties to the even code); magnitudes beyond 6 saturate to 6."""
    neg = np.signbit(x)
    a = min(abs(float(x)), 6.0)
    i = int(np.searchsorted(_E2M1_POS, a))
    if i < 8 and _E2M1_POS[i] == a:
        c = i
    else:
        lo, hi = i - 1, i
        dlo, dhi = a - _E2M1_POS[lo], _E2M1_POS[hi] - a
        c = lo if (dlo < dhi or (dlo == dhi and lo % 2 == 0)) else hi
    return c | (0x8 if neg else 0)


def e2m1_encode_array(x) -> np.ndarray:
    """e2m1_encode element by element on an array (nearest code, ties to the even code,
    saturation at 6), as uint8 codes."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), 6.0)
    i = np.searchsorted(_E2M1_POS, a)
    hit = _E2M1_POS[i] == a
    lo = np.maximum(i - 1, 0)
    dlo, dhi = a - _E2M1_POS[lo], _E2M1_POS[i] - a
    c = np.where(hit, i, np.where((dlo < dhi) | ((dlo == dhi) & (lo % 2 == 0)), lo, i))
    return (c | np.where(np.signbit(x), 0x8, 0)).astype(np.uint8)


_E2M1_ALL = np.array([e2m1_decode(c) for c in range(16)])


def nvfp4_quantize(w: np.ndarray, block: int = 16):
    """Two-level scaling along the last axis: a tensor scale g = max |w| / (448 * 6); per
    block of `block` values an E4M3 scale code for max |v| / (6 g); each value stored as
    e2m1_encode(v / (s_b g)) with s_b the decoded block scale.  Returns (codes uint8
    [..., n], block scale codes uint8 [..., n / block], g)."""
    w = np.asarray(w, dtype=np.float64)
    assert w.shape[-1] % block == 0
    amax_t = float(np.abs(w).max())
    g = amax_t / (E4M3_MAX * 6.0) if amax_t > 0 else 1.0
    blocks = w.reshape(*w.shape[:-1], w.shape[-1] // block, block)
    amax = np.abs(blocks).max(axis=-1)
    sc = e4m3_encode_array(amax / (6.0 * g))
    sb = _E4M3_ALL[sc.astype(np.int64)]
    denom = np.where(sb > 0, sb * g, 1.0)[..., None]
    codes = e2m1_encode_array(blocks / denom)
    return codes.reshape(w.shape), sc, g


def nvfp4_dequantize(codes: np.ndarray, scale_codes: np.ndarray, g: float, block: int = 16) -> np.ndarray:
    vals = _E2M1_ALL[np.asarray(codes, dtype=np.int64)]
    sb = _E4M3_ALL[np.asarray(scale_codes, dtype=np.int64)]
    blocks = vals.reshape(*vals.shape[:-1], vals.shape[-1] // block, block)
    return (blocks * (sb * g)[..., None]).reshape(vals.shape)
