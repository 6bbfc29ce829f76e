"""CPU oracle of the block-diffusion denoising pass -- TEST INFRASTRUCTURE ONLY.

Nothing in the product path may import, call or execute this module; only the tests,
the smoke check and the benchmark's CPU baseline use it.  It shares no code with the
CUDA path and imports nothing from the package.

The arithmetic lives in the plain fp64 C++ of `dg_oracle.cpp` (built by
`oracle/build.py` into `libdg_oracle.so`; its header states the sources and the
readings).  This module only marshals numpy arrays into that library and composes its
calls: the multi-step loops (`generate_canvas`, `generate_canvas_masked`) and the
batch helpers run the C++ pass and update once per step or canvas, as the pages'
procedure does.  `dg_oracle_np.py` is an independent numpy restatement of the same
definitions, kept as a cross-check (`tests/test_oracle_cpp.py`).

Sources (page title -- section):
  [DG-explainer]  "DiffusionGemma" video explainer -- "Uniform State Diffusion",
                  "Two modes, one model", "First attempt: masked diffusion",
                  "Long-form text: chaining canvases"
  [DLM-exercises] "Module 12. Diffusion Language Models" exercises -- the prefix/block
                  mask solution, the MoE remark
  Hacker News discussion of DiffusionGemma -- the comment on batching

Storage rule: a bf16 model stores its weights and its KV cache in bf16; every value
in flight is exact (fp64).  `Precision('bf16')` therefore rounds only what a prefill
writes to the cache.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = globals().get("_LIB_OVERRIDE") or os.path.join(_HERE, "libdg_oracle.so")

_P = ctypes.c_void_p
_I32, _I64, _U64, _F64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_double


class OcTensor(ctypes.Structure):
    _fields_ = [("p", _P), ("dtype", _I32)]


class OcConfig(ctypes.Structure):
    _fields_ = [(n, _I32) for n in ("n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "n_experts",
                                    "top_k", "expert_ffn", "vocab")] + \
               [("rope_theta", _F64), ("rms_eps", _F64), ("bf16_storage", _I32)]


class OcWeights(ctypes.Structure):
    _fields_ = [("embed", OcTensor), ("w_out", OcTensor)] + \
               [(n, ctypes.POINTER(OcTensor)) for n in ("w_q", "w_k", "w_v", "w_o", "w_router", "w_gate", "w_up",
                                                        "w_down")]


_TAP_FIELDS = [("x_in", _P), ("attn_o", _P), ("x_attn", _P), ("x_out", _P), ("router_logits", _P),
               ("topk_idx", _P), ("topk_w", _P), ("router_margin", _P), ("counts", _P), ("offsets", _P),
               ("perm", _P), ("inv", _P), ("union_size", _P), ("k_new", _P), ("v_new", _P)]


class OcTaps(ctypes.Structure):
    _fields_ = _TAP_FIELDS


def _declare(lib):
    C, W, T = ctypes.POINTER(OcConfig), ctypes.POINTER(OcWeights), ctypes.POINTER(OcTaps)
    sig = {
        "oc_widen": (None, [OcTensor, _I64, _P]),
        "oc_round_bf16": (None, [_P, _I64, _P]),
        "oc_rms_norm": (None, [_P, _I64, _I32, _F64, _P]),
        "oc_rope": (None, [_P, _I32, _I32, _I32, _P, _F64]),
        "oc_silu_array": (None, [_P, _I64, _P]),
        "oc_block_mask": (None, [_I32, _I32, _P]),
        "oc_causal_rows": (None, [_I32, _I32, _P]),
        "oc_attention": (None, [_P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _P]),
        "oc_router_topk": (None, [_P, _I32, _I32, _I32, _P, _P, _P]),
        "oc_expert_permutation": (_I64, [_P, _I32, _I32, _I32, _P, _P, _P, _P]),
        "oc_qkv": (None, [C, W, _I32, _P, _I32, _P, _P, _P, _P]),
        "oc_attn_out": (None, [C, W, _I32, _P, _I32, _P]),
        "oc_attention_block": (None, [C, W, _I32, _P, _P, _I32, _P, _I32, _I32, _P, _P, _P, _P]),
        "oc_moe_block": (None, [C, W, _I32, _P, _I32, _P, _P, T]),
        "oc_embed": (None, [C, W, _P, _I32, _P]),
        "oc_vocab_logits": (None, [C, W, _P, _I32, _P]),
        "oc_denoise_pass": (None, [C, W, _P, _P, _I32, _P, _I32, _P, T]),
        "oc_prefill": (None, [C, W, _P, _P, _I32, _P, _I32, _P, _P, T]),
        "oc_full_sequence_states": (None, [C, W, _P, _I32, _P, _I32, _P, _P, _P]),
        "oc_splitmix64": (_U64, [_U64, _U64]),
        "oc_renoise_token": (_I64, [_U64, ctypes.c_uint32, ctypes.c_uint32, _I64]),
        "oc_renoise_count": (_I64, [_I64, _I64, _I64, _F64, _F64]),
        "oc_canvas_update": (None, [_P, _I32, _I32, _I32, _U64, ctypes.c_uint32, _P, _P, _P, _P, _P, _P]),
        "oc_canvas_update_masked": (None, [_P, _I32, _I32, _P, _I32, _I32, _P, _P, _P, _P, _P, _P]),
        "oc_e4m3_decode": (_F64, [_I32]),
        "oc_e2m1_decode": (_F64, [_I32]),
        "oc_e4m3_encode": (_I32, [_F64]),
        "oc_e2m1_encode": (_I32, [_F64]),
        "oc_e4m3_encode_array": (None, [_P, _I64, _P]),
        "oc_e2m1_encode_array": (None, [_P, _I64, _P]),
        "oc_mx_e4m3_quantize": (None, [_P, _I64, _I32, _P, _P]),
        "oc_mx_e4m3_dequantize": (None, [_P, _P, _I64, _I32, _P]),
        "oc_nvfp4_quantize": (_F64, [_P, _I64, _I32, _P, _P]),
        "oc_nvfp4_dequantize": (None, [_P, _P, _F64, _I64, _I32, _P]),
        "oc_num_threads": (_I32, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


def _load(path):
    if not os.path.exists(path):
        from oracle import build as _build
        _build.build()
    return _declare(ctypes.CDLL(path))


_lib = _load(LIB_PATH)


def num_threads() -> int:
    """Host threads the oracle's OpenMP loops use."""
    return int(_lib.oc_num_threads())


# ----------------------------------------------------------------------------
# marshalling


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _tensor(a, keep: list) -> OcTensor:
    a = np.asarray(a)
    if a.dtype == np.uint16:
        code = 0
    elif a.dtype == np.float32:
        code = 1
    else:
        a, code = a.astype(np.float64, copy=False), 2
    a = np.ascontiguousarray(a)
    keep.append(a)
    return OcTensor(a.ctypes.data, code)


def _config(model, prec) -> OcConfig:
    c = model.cfg
    return OcConfig(c["n_layers"], c["hidden"], c["n_q_heads"], c["n_kv_heads"], c["head_dim"], c["n_experts"],
                    c["top_k"], c["expert_ffn"], c["vocab"], float(c["rope_theta"]), float(c["rms_eps"]),
                    1 if (prec is not None and prec.dtype == "bf16") else 0)


def _weights(model, keep: list) -> OcWeights:
    w = OcWeights(_tensor(model.embed, keep), _tensor(model.w_out, keep))
    for name in ("w_q", "w_k", "w_v", "w_o", "w_router", "w_gate", "w_up", "w_down"):
        arr = (OcTensor * len(model.layers))(*[_tensor(L[name], keep) for L in model.layers])
        keep.append(arr)
        setattr(w, name, arr)
    return w


def _ptrs(arrays: list, keep: list):
    arr = (ctypes.c_void_p * max(1, len(arrays)))(*[a.ctypes.data for a in arrays])
    keep.append(arr)
    return arr


def _new_taps(cfg, T: int, full: bool = True) -> tuple[dict, OcTaps]:
    H, E, k = cfg["hidden"], cfg["n_experts"], cfg["top_k"]
    nq, nkv, d = cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    t = dict(router_logits=np.empty((T, E)), topk_idx=np.empty((T, k), np.int32), topk_w=np.empty((T, k)),
             router_margin=np.empty(T), counts=np.empty(E, np.int64), offsets=np.empty(E + 1, np.int64),
             perm=np.empty(T * k, np.int64), inv=np.empty(T * k, np.int64), union=np.zeros(1, np.int64))
    if full:
        t.update(x_in=np.empty((T, H)), attn_o=np.empty((T, nq * d)), x_attn=np.empty((T, H)),
                 x_out=np.empty((T, H)), k_new=np.empty((nkv, T, d)), v_new=np.empty((nkv, T, d)))
    s = OcTaps()
    for name, _ in _TAP_FIELDS:
        key = "union" if name == "union_size" else name
        if key in t:
            setattr(s, name, t[key].ctypes.data)
    return t, s


def _finish_taps(t: dict) -> dict:
    t["union"] = int(t["union"][0])
    t.pop("inv", None)
    return t


# ----------------------------------------------------------------------------
# storage decoding and rounding


def widen(a: np.ndarray) -> np.ndarray:
    """Exact float64 value of a stored tensor (uint16 = bf16 bit patterns, or a float array)."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        keep = []
        out = np.empty(a.shape)
        _lib.oc_widen(_tensor(a, keep), a.size, _ptr(out))
        return out
    return np.asarray(a, dtype=np.float64)


def round_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (8 significant bits), ties to even."""
    x = _f64(x)
    out = np.empty_like(x)
    _lib.oc_round_bf16(_ptr(x), x.size, _ptr(out))
    return out


class Precision:
    def __init__(self, dtype: str):
        assert dtype in ("bf16", "f32")
        self.dtype = dtype

    def store(self, x: np.ndarray) -> np.ndarray:
        """A value stored in the model's storage dtype (KV cache entries)."""
        return round_bf16(x) if self.dtype == "bf16" else x


# ----------------------------------------------------------------------------
# layer primitives


def rms_norm(x, eps: float) -> np.ndarray:
    """y = x / sqrt(mean(x^2) + eps) over the last axis (unit gain)."""
    x = _f64(x)
    H = x.shape[-1]
    out = np.empty_like(x)
    _lib.oc_rms_norm(_ptr(x), x.size // H, H, float(eps), _ptr(out))
    return out


def rope(x, positions, theta: float) -> np.ndarray:
    """Rotary position embedding, rotate-half pairing (i, i + d/2), on x[..., T, d]."""
    out = _f64(x).copy()
    T, d = out.shape[-2], out.shape[-1]
    pos = np.ascontiguousarray(positions, dtype=np.int64)
    assert pos.shape == (T,)
    _lib.oc_rope(_ptr(out), out.size // (T * d), T, d, _ptr(pos), float(theta))
    return out


def silu(z) -> np.ndarray:
    z = _f64(z)
    out = np.empty_like(z)
    _lib.oc_silu_array(_ptr(z), z.size, _ptr(out))
    return out if out.ndim else float(out)


def block_mask(P: int, C: int) -> np.ndarray:
    """Allowed-attention matrix over rows/columns ordered (prefix 0..P-1, block 0..C-1).

    [DLM-exercises], prefix/block mask solution: a prefix query sees only the prefix
    keys at or before it (causal); every block query sees the whole prefix and the
    whole block (bidirectional).  No prefix query sees a block key.
    """
    out = np.empty((P + C, P + C), np.uint8)
    _lib.oc_block_mask(P, C, _ptr(out))
    return out.astype(bool)


def causal_rows(P: int, T: int) -> np.ndarray:
    """Rows for T new tokens at positions P..P+T-1 over keys 0..P+T-1, prefill mode."""
    out = np.empty((T, P + T), np.uint8)
    _lib.oc_causal_rows(P, T, _ptr(out))
    return out.astype(bool)


def attention(q, k, v, allowed) -> np.ndarray:
    """Masked softmax attention with grouped KV heads: q [nq][Tq][d]; k, v [nkv][Tk][d];
    allowed [Tq][Tk] bool.  Query head h reads KV head h // (nq / nkv); scale 1/sqrt(d)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    nq, Tq, d = q.shape
    nkv, Tk, _ = k.shape
    a = np.ascontiguousarray(np.broadcast_to(allowed, (Tq, Tk)), dtype=np.uint8)
    out = np.empty_like(q)
    _lib.oc_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(a), nq, nkv, Tq, Tk, d, _ptr(out))
    return out


def router_topk(logits, k: int):
    """Top-k experts per token by router logit; ties go to the lower expert id.

    Returns (idx [T][k] int32 in descending-logit order, w [T][k] = softmax over the k
    chosen logits, margin [T] = k-th minus (k+1)-th largest logit)."""
    logits = _f64(logits)
    T, E = logits.shape
    idx, w, margin = np.empty((T, k), np.int32), np.empty((T, k)), np.empty(T)
    _lib.oc_router_topk(_ptr(logits), T, E, k, _ptr(idx), _ptr(w), _ptr(margin))
    return idx, w, margin


def expert_permutation(idx, n_experts: int):
    """Group the T*k (token, slot) assignments by expert, stably: counts [E], offsets
    [E+1], perm [T*k] (flat assignment t*k + j at row p, in (expert, t, j) order), inv
    [T*k], and the union size U = #{e : counts[e] > 0}."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    counts, offsets = np.empty(n_experts, np.int64), np.empty(n_experts + 1, np.int64)
    perm, inv = np.empty(T * k, np.int64), np.empty(T * k, np.int64)
    u = _lib.oc_expert_permutation(_ptr(idx), T, k, n_experts, _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv))
    return counts, offsets, perm, inv, int(u)


# ----------------------------------------------------------------------------
# the transformer stack


def _qkv(model, l: int, x, positions, prec):
    cfg = model.cfg
    x = _f64(x)
    T = x.shape[0]
    nq, nkv, d = cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    pos = np.ascontiguousarray(positions, dtype=np.int64)
    q, k, v = np.empty((nq, T, d)), np.empty((nkv, T, d)), np.empty((nkv, T, d))
    keep = []
    _lib.oc_qkv(_config(model, prec), _weights(model, keep), l, _ptr(x), T, _ptr(pos), _ptr(q), _ptr(k), _ptr(v))
    return q, k, v


def _attn_out(model, l: int, o, prec) -> np.ndarray:
    o = _f64(o)
    T = o.shape[1]
    y = np.empty((T, model.cfg["hidden"]))
    keep = []
    _lib.oc_attn_out(_config(model, prec), _weights(model, keep), l, _ptr(o), T, _ptr(y))
    return y


def attention_block(model, l: int, cache: "Cache", x, causal: bool, prec) -> dict:
    """The attention block of layer l for the rows x [T][H] at positions len..len+T-1
    over the cache's stored keys and the rows' own keys: denoising mode (causal False)
    or prefill mode.  Returns dict(x_attn, attn_o, k_new, v_new) (own K/V in flight)."""
    cfg = model.cfg
    x = _f64(x)
    T = x.shape[0]
    nq, nkv, d = cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    ck, cv = _f64(cache.k[l]), _f64(cache.v[l])
    out = dict(x_attn=np.empty_like(x), attn_o=np.empty((T, nq * d)), k_new=np.empty((nkv, T, d)),
               v_new=np.empty((nkv, T, d)))
    keep = []
    _lib.oc_attention_block(_config(model, prec), _weights(model, keep), l, _ptr(ck), _ptr(cv), cache.len, _ptr(x),
                            T, 1 if causal else 0, _ptr(out["x_attn"]), _ptr(out["attn_o"]), _ptr(out["k_new"]),
                            _ptr(out["v_new"]))
    return out


def moe_block(model, l: int, x, prec) -> dict:
    """The MoE block of layer l on the residual x [T][H]: dict(x_out, ffn, and the routing
    values: router_logits, topk_idx, topk_w, router_margin, counts, offsets, perm, union)."""
    x = _f64(x)
    T = x.shape[0]
    t, s = _new_taps(model.cfg, T, full=False)
    t["x_out"], t["ffn"] = np.empty_like(x), np.empty_like(x)
    keep = []
    _lib.oc_moe_block(_config(model, prec), _weights(model, keep), l, _ptr(x), T, _ptr(t["x_out"]), _ptr(t["ffn"]),
                      ctypes.byref(s))
    return _finish_taps(t)


def moe(model, l: int, x, prec, tap: dict | None = None) -> np.ndarray:
    """Sparse MoE FFN on the residual x [T][H]; returns the FFN output [T][H] (router ->
    top-k -> stable expert grouping -> SwiGLU over the union of experts -> combine)."""
    r = moe_block(model, l, x, prec)
    if tap is not None:
        tap.update({key: r[key] for key in ("router_logits", "topk_idx", "topk_w", "router_margin", "counts",
                                            "offsets", "perm", "union")})
    return r["ffn"]


def embed(model, tokens) -> np.ndarray:
    """Residual stream start: the embedding rows of the tokens (untied, unscaled)."""
    toks = np.ascontiguousarray(tokens, dtype=np.int32).reshape(-1)
    x = np.empty((len(toks), model.cfg["hidden"]))
    keep = []
    _lib.oc_embed(_config(model, None), _weights(model, keep), _ptr(toks), len(toks), _ptr(x))
    return x.reshape(np.shape(tokens) + (model.cfg["hidden"],))


def vocab_logits(model, x, prec, rows=None, chunk: int = 16384) -> np.ndarray:
    """Final RMSNorm then projection onto every vocabulary entry (fp64 logits).
    [DG-explainer] "Uniform State Diffusion": every canvas position gets a full
    distribution over the vocabulary.  (chunk: accepted for the numpy version's
    signature; the C++ loop needs no chunking.)"""
    x = _f64(x)
    if rows is not None:
        x = np.ascontiguousarray(x[np.asarray(rows)])
    out = np.empty((x.shape[0], model.cfg["vocab"]))
    keep = []
    _lib.oc_vocab_logits(_config(model, prec), _weights(model, keep), _ptr(x), x.shape[0], _ptr(out))
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


def denoise_pass(model, cache: Cache, canvas, prec, logit_rows=None):
    """One denoising pass over the canvas ([DG-explainer] "Two modes, one model",
    denoising mode; [DLM-exercises] mask solution: the cached prefix K/V is read as is,
    only the block is recomputed, the cache is not modified).  Canvas positions are
    P..P+C-1 with P = cache length.  Returns (logits [C or len(logit_rows)][V], per-layer
    taps)."""
    cfg = model.cfg
    toks = np.ascontiguousarray(canvas, dtype=np.int32)
    C = len(toks)
    keep = []
    ks = [_f64(a) for a in cache.k]
    vs = [_f64(a) for a in cache.v]
    taps, structs = [], (OcTaps * cfg["n_layers"])()
    for l in range(cfg["n_layers"]):
        t, s = _new_taps(cfg, C)
        taps.append(t)
        structs[l] = s
    logits = np.empty((C, cfg["vocab"])) if logit_rows is None else None
    _lib.oc_denoise_pass(_config(model, prec), _weights(model, keep), _ptrs(ks, keep), _ptrs(vs, keep), cache.len,
                         _ptr(toks), C, _ptr(logits) if logits is not None else None, structs)
    taps = [_finish_taps(t) for t in taps]
    for t in taps:
        t.pop("k_new"), t.pop("v_new")
    if logit_rows is not None:
        logits = vocab_logits(model, taps[-1]["x_out"], prec, rows=logit_rows)
    return logits, taps


def prefill_append(model, cache: Cache, tokens, prec, taps: list | None = None) -> Cache:
    """Causal prefill of T tokens at positions P..P+T-1, appending their K/V ([DG-explainer]
    "Two modes, one model" / "Long-form text: chaining canvases").  Only K/V matter, so the
    last layer stops after writing its K/V.  taps (a list) receives the routing values of
    every layer but the last."""
    cfg = model.cfg
    toks = np.ascontiguousarray(tokens, dtype=np.int32)
    T, L = len(toks), cfg["n_layers"]
    keep = []
    ks = [_f64(a) for a in cache.k]
    vs = [_f64(a) for a in cache.v]
    k_new = [np.empty((cfg["n_kv_heads"], T, cfg["head_dim"])) for _ in range(L)]
    v_new = [np.empty((cfg["n_kv_heads"], T, cfg["head_dim"])) for _ in range(L)]
    tl, structs = [], (OcTaps * max(1, L - 1))()
    for l in range(L - 1):
        t, s = _new_taps(cfg, T)
        s.k_new = s.v_new = None
        tl.append(t)
        structs[l] = s
    _lib.oc_prefill(_config(model, prec), _weights(model, keep), _ptrs(ks, keep), _ptrs(vs, keep), cache.len,
                    _ptr(toks), T, _ptrs(k_new, keep), _ptrs(v_new, keep), structs if L > 1 else None)
    if taps is not None:
        for t in tl:
            t = _finish_taps(t)
            t.pop("k_new"), t.pop("v_new")
            taps.append(t)
    out = Cache([])
    out.k = [np.concatenate([a, b], axis=1) for a, b in zip(cache.k, k_new)]
    out.v = [np.concatenate([a, b], axis=1) for a, b in zip(cache.v, v_new)]
    return out


def full_sequence_states(model, prefix_tokens, canvas, prec):
    """Recompute prefix and canvas together under the prefix/block mask, no cache.
    Returns (per-layer K, V over all P+C positions as a cache stores them, canvas
    logits) ([DLM-exercises] mask solution: prefix K/V reusable)."""
    cfg = model.cfg
    pre = np.ascontiguousarray(prefix_tokens, dtype=np.int32)
    can = np.ascontiguousarray(canvas, dtype=np.int32)
    P, C, L = len(pre), len(can), cfg["n_layers"]
    ks = [np.empty((cfg["n_kv_heads"], P + C, cfg["head_dim"])) for _ in range(L)]
    vs = [np.empty((cfg["n_kv_heads"], P + C, cfg["head_dim"])) for _ in range(L)]
    logits = np.empty((C, cfg["vocab"]))
    keep = []
    _lib.oc_full_sequence_states(_config(model, prec), _weights(model, keep), _ptr(pre), P, _ptr(can), C,
                                 _ptrs(ks, keep), _ptrs(vs, keep), _ptr(logits))
    return ks, vs, logits


# ----------------------------------------------------------------------------
# canvas update

_GAMMA = 0x9E3779B97F4A7C15


def splitmix64(seed: int, n: int) -> int:
    """SplitMix64 (Steele, Lea & Flood 2014): output number n (0-based) of the stream seeded with `seed`."""
    return int(_lib.oc_splitmix64(seed & 0xFFFFFFFFFFFFFFFF, n & 0xFFFFFFFFFFFFFFFF))


def renoise_token(seed: int, step: int, pos: int, vocab: int) -> int:
    """Fresh uniform vocabulary token for re-noising position `pos` at step `step`: draw
    number (step << 32 | pos) of SplitMix64(seed), multiply-shift on its high 32 bits."""
    return int(_lib.oc_renoise_token(seed & 0xFFFFFFFFFFFFFFFF, step, pos, vocab))


def renoise_count(C: int, S: int, s: int, r_start: float, r_end: float) -> int:
    """Positions re-noised after step s of S: floor(C * f_s), f_s linear from r_start
    (first step) to r_end (last step); one step uses r_start."""
    return int(_lib.oc_renoise_count(C, S, s, float(r_start), float(r_end)))


def canvas_update(logits, n_renoise: int, seed: int, step: int) -> dict:
    """Update every position, then re-noise the least confident ones ([DG-explainer]
    "Uniform State Diffusion"; confidence = largest softmax probability).  Returns canvas,
    argmax, conf, top-1/top-2 logit margin, the re-noised positions (sorted) and each
    position's log-confidence distance to the cut."""
    logits = _f64(logits)
    C, V = logits.shape
    canvas, argmax = np.empty(C, np.int32), np.empty(C, np.int32)
    conf, top, cut = np.empty(C), np.empty(C), np.empty(C)
    ren = np.empty(C, np.uint8)
    _lib.oc_canvas_update(_ptr(logits), C, V, int(n_renoise), seed & 0xFFFFFFFFFFFFFFFF, step, _ptr(canvas),
                          _ptr(argmax), _ptr(conf), _ptr(top), _ptr(ren), _ptr(cut))
    return dict(canvas=canvas, argmax=argmax, conf=conf, top_margin=top, renoised=np.nonzero(ren)[0],
                cut_margin=cut)


def canvas_update_masked(logits, canvas, n_keep: int, mask_id: int) -> dict:
    """Masked-diffusion update ([DG-explainer] "First attempt: masked diffusion"): fill
    [MASK] positions, which then stay fixed.  Returns the canvas, the candidates, the
    confidences, the top-1/top-2 margin among candidate logits, the positions kept masked
    (sorted) and each masked position's log-confidence distance to the cut."""
    logits = _f64(logits)
    C, V = logits.shape
    cin = np.ascontiguousarray(canvas, dtype=np.int32)
    out, cand = np.empty(C, np.int32), np.empty(C, np.int32)
    conf, top, cut = np.empty(C), np.empty(C), np.empty(C)
    kept = np.empty(C, np.uint8)
    _lib.oc_canvas_update_masked(_ptr(logits), C, V, _ptr(cin), int(n_keep), int(mask_id), _ptr(out), _ptr(cand),
                                 _ptr(conf), _ptr(top), _ptr(kept), _ptr(cut))
    return dict(canvas=out, argmax=cand, conf=conf, top_margin=top, kept=np.nonzero(kept)[0], cut_margin=cut)


def generate_canvas_masked(model, cache: Cache, C: int, S: int, keep_start: float, keep_end: float, mask_id: int,
                           prec, append: bool, record=None):
    """S passes of masked diffusion from an all-[MASK] canvas, then (optionally) append
    ([DG-explainer] "First attempt: masked diffusion", "Long-form text").  After pass s at
    most renoise_count(C, S, s, keep_start, keep_end) positions stay masked.  Returns
    (canvas, cache)."""
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


def generate_canvas(model, cache: Cache, canvas, S: int, r_start: float, r_end: float, seed: int, prec,
                    append: bool, record=None):
    """S denoising passes with re-noising, then (optionally) append the canvas by prefill
    ([DG-explainer] "Uniform State Diffusion", "Long-form text: chaining canvases").
    Returns (canvas, cache)."""
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
# several canvases at once (Hacker News discussion, the comment on batching: batched
# requests share the reads of common weights, which is all batching changes)


def denoise_pass_batched(model, caches: list, canvases, prec):
    """Denoising passes of B independent canvases, canvas b against its own cache: each
    request attends only to its own cache and canvas and every per-token step is
    row-wise, so canvas b's result is its single-canvas pass.  [(logits, taps)] per canvas."""
    return [denoise_pass(model, c, np.asarray(x), prec) for c, x in zip(caches, canvases)]


def merge_batch_taps(per_canvas_taps: list, n_experts: int) -> list:
    """Per-layer taps of a batch: row-wise entries stacked in canvas order; the expert
    histogram, stable permutation and union taken over all rows together, as one pass
    over the batch groups them."""
    out = []
    for layer_taps in zip(*per_canvas_taps):
        m = {key: np.concatenate([t[key] for t in layer_taps], axis=0)
             for key in ("x_in", "attn_o", "x_attn", "x_out", "router_logits", "topk_idx", "topk_w", "router_margin")}
        counts, offsets, perm, inv, union = expert_permutation(m["topk_idx"], n_experts)
        m.update(counts=counts, offsets=offsets, perm=perm, union=union)
        out.append(m)
    return out


def generate_canvases(model, caches: list, canvases, S: int, r_start: float, r_end: float, seeds, prec,
                      append: bool):
    """generate_canvas for each canvas with its own cache and re-noise seed.  Returns
    ([canvas], [cache])."""
    res = [generate_canvas(model, c, x, S, r_start, r_end, sd, prec, append)
           for c, x, sd in zip(caches, canvases, seeds)]
    return [r[0] for r in res], [r[1] for r in res]


# ----------------------------------------------------------------------------
# 8- and 4-bit weights: the OCP E4M3 element format with MX block scaling (one
# power-of-two scale per 32 elements), and E2M1 elements with an E4M3 scale per 16 and
# an fp32 tensor scale ([DLM-exercises] MoE remark: FP8 and NVFP4 deployments)

E4M3_MAX = 448.0


def e4m3_decode(code: int) -> float:
    """Value of an E4M3 code: sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0
    is subnormal (m * 2^-9); 0x7F / 0xFF are NaN; no infinities."""
    return float(_lib.oc_e4m3_decode(int(code)))


def e2m1_decode(code: int) -> float:
    """Value of an E2M1 code: sign, 2 exponent bits (bias 1), 1 mantissa bit."""
    return float(_lib.oc_e2m1_decode(int(code)))


_E4M3_POS = np.array([e4m3_decode(c) for c in range(0x7F)])   # codes 0x00 .. 0x7E, increasing
_E4M3_ALL = np.array([e4m3_decode(c) for c in range(256)])
_E2M1_POS = np.array([e2m1_decode(c) for c in range(8)])
_E2M1_ALL = np.array([e2m1_decode(c) for c in range(16)])


def e4m3_encode(x: float) -> int:
    """Nearest E4M3 code (ties to the even code); magnitudes beyond 448 saturate."""
    return int(_lib.oc_e4m3_encode(float(x)))


def e2m1_encode(x: float) -> int:
    """Nearest E2M1 code (ties to the even code); magnitudes beyond 6 saturate."""
    return int(_lib.oc_e2m1_encode(float(x)))


def e4m3_encode_array(x) -> np.ndarray:
    x = _f64(x)
    out = np.empty(x.shape, np.uint8)
    _lib.oc_e4m3_encode_array(_ptr(x), x.size, _ptr(out))
    return out


def e2m1_encode_array(x) -> np.ndarray:
    x = _f64(x)
    out = np.empty(x.shape, np.uint8)
    _lib.oc_e2m1_encode_array(_ptr(x), x.size, _ptr(out))
    return out


def mx_e4m3_quantize(w, block: int = 32):
    """MX block scaling along the last axis (blocks of 32 share X = 2^(floor(log2 max|v|)
    - 8)); returns (codes uint8 [..., n], scale exponents int32 [..., n / 32])."""
    assert block == 32
    w = _f64(w)
    n = w.shape[-1]
    assert n % 32 == 0
    codes = np.empty(w.shape, np.uint8)
    exps = np.empty(w.shape[:-1] + (n // 32,), np.int32)
    _lib.oc_mx_e4m3_quantize(_ptr(w), w.size // n, n, _ptr(codes), _ptr(exps))
    return codes, exps


def mx_e4m3_dequantize(codes, exp, block: int = 32) -> np.ndarray:
    """X * e4m3_decode(code) for every element."""
    assert block == 32
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    exp = np.ascontiguousarray(exp, dtype=np.int32)
    n = codes.shape[-1]
    out = np.empty(codes.shape)
    _lib.oc_mx_e4m3_dequantize(_ptr(codes), _ptr(exp), codes.size // n, n, _ptr(out))
    return out


def nvfp4_quantize(w, block: int = 16):
    """Two-level scaling along the last axis: tensor scale g = max |w| / (448 * 6), an
    E4M3 scale code per block of 16 for max |v| / (6 g), E2M1 codes for v / (s_b g).
    Returns (codes uint8 [..., n], block scale codes uint8 [..., n / 16], g)."""
    assert block == 16
    w = _f64(w)
    n = w.shape[-1]
    assert n % 16 == 0
    codes = np.empty(w.shape, np.uint8)
    sc = np.empty(w.shape[:-1] + (n // 16,), np.uint8)
    g = _lib.oc_nvfp4_quantize(_ptr(w), w.size // n, n, _ptr(codes), _ptr(sc))
    return codes, sc, float(g)


def nvfp4_dequantize(codes, scale_codes, g: float, block: int = 16) -> np.ndarray:
    assert block == 16
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sc = np.ascontiguousarray(scale_codes, dtype=np.uint8)
    n = codes.shape[-1]
    out = np.empty(codes.shape)
    _lib.oc_nvfp4_dequantize(_ptr(codes), _ptr(sc), float(g), codes.size // n, n, _ptr(out))
    return out
