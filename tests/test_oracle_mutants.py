"""Mutation check of the oracle's pins: each plausible mistake below (a dropped term, a
wrong sign, index, operand or tie rule) is planted in the oracle module on the CPU, and
at least one of the named pins must fail under it.  The oracle is only as trustworthy
as its pins; this file shows that they see each of these mistakes.

Nothing here changes the oracle on disk: every mutant replaces one module attribute
for the duration of one test (pytest's monkeypatch), and the functions of the oracle
that call it pick the replacement up through the module's globals.
"""
import math

import numpy as np
import pytest

from oracle import dg_oracle as O
import test_oracle_pins as PINS

_orig = {name: getattr(O, name) for name in dir(O)}


# ---------------------------------------------------------------- the mutants


def _rms_no_eps(x, eps):
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True))


def _rms_sum(x, eps):
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def _rope_sign(x, positions, theta):
    d = x.shape[-1]; half = d // 2
    inv = theta ** (-(np.arange(half) * 2.0) / d)
    a = positions.astype(np.float64)[:, None] * inv[None, :]
    c, s = np.cos(a), np.sin(a)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c + x2 * s, x2 * c - x1 * s], axis=-1)   # rotation by -angle


def _rope_interleaved(x, positions, theta):
    d = x.shape[-1]; half = d // 2
    inv = theta ** (-(np.arange(half) * 2.0) / d)
    a = positions.astype(np.float64)[:, None] * inv[None, :]
    c, s = np.cos(a), np.sin(a)
    x1, x2 = x[..., 0::2], x[..., 1::2]                                  # pairs (2i, 2i+1)
    out = np.empty_like(x)
    out[..., 0::2] = x1 * c - x2 * s
    out[..., 1::2] = x2 * c + x1 * s
    return out


def _rope_freq(x, positions, theta):
    d = x.shape[-1]; half = d // 2
    inv = theta ** (-np.arange(half) / d)                                # factor 2 dropped
    a = positions.astype(np.float64)[:, None] * inv[None, :]
    c, s = np.cos(a), np.sin(a)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def _silu_sign(z):
    return z / (1.0 + np.exp(z))


def _mask_prefix_sees_block(P, C):
    return np.ones((P + C, P + C), dtype=bool)


def _mask_block_causal(P, C):
    return np.tril(np.ones((P + C, P + C), dtype=bool))


def _causal_off_by_one(P, T):
    a = np.zeros((T, P + T), dtype=bool)
    for i in range(T):
        a[i, : P + i] = True                                             # own key missing
    a[0, 0] = True
    return a


def _attention_variant(scale=None, head_map=None, masked=True):
    def att(q, k, v, allowed):
        nq, Tq, d = q.shape
        nkv = k.shape[0]
        g = nq // nkv
        out = np.empty_like(q)
        for h in range(nq):
            kv = head_map(h, nq, nkv) if head_map else h // g
            s = (q[h] @ k[kv].T) * (scale(d) if scale else 1.0 / np.sqrt(d))
            if masked:
                s = np.where(allowed, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            out[h] = (p / p.sum(axis=1, keepdims=True)) @ v[kv]
        return out
    return att


def _router_variant(ties_high=False, full_softmax=False):
    def rt(logits, k):
        T, E = logits.shape
        if ties_high:
            order = (E - 1 - np.argsort(-logits[:, ::-1], axis=1, kind="stable"))
        else:
            order = np.argsort(-logits, axis=1, kind="stable")
        idx = order[:, :k].astype(np.int32)
        chosen = np.take_along_axis(logits, order[:, :k], axis=1)
        if full_softmax:
            p = np.exp(logits - logits.max(axis=1, keepdims=True))
            w = np.take_along_axis(p / p.sum(axis=1, keepdims=True), order[:, :k], axis=1)
        else:
            w = np.exp(chosen - chosen.max(axis=1, keepdims=True))
            w = w / w.sum(axis=1, keepdims=True)
        if k < E:
            margin = chosen[:, -1] - np.take_along_axis(logits, order[:, k:k + 1], axis=1)[:, 0]
        else:
            margin = np.full(T, np.inf)
        return idx, w, margin
    return rt


def _perm_slot_major(idx, n_experts):
    T, k = idx.shape
    flat = idx.reshape(-1)
    perm = np.array(sorted(range(T * k), key=lambda a: (int(flat[a]), a % k, a // k)), dtype=np.int64)
    inv = np.empty_like(perm); inv[perm] = np.arange(T * k)
    counts = np.bincount(flat, minlength=n_experts).astype(np.int64)
    return counts, np.concatenate([[0], np.cumsum(counts)]), perm, inv, int((counts > 0).sum())


def _moe_variant(swap_gate_up=False, reversed_weights=False, raw_input=False):
    def moe(model, l, x, prec, tap=None):
        cfg = model.cfg
        E, k = cfg["n_experts"], cfg["top_k"]
        L = model.layers[l]
        xn = O.rms_norm(x, cfg["rms_eps"])
        idx, w, _ = O.router_topk(xn @ O.widen(L["w_router"]).T, k)
        counts, offsets, perm, inv, _ = O.expert_permutation(idx, E)
        xs = x if raw_input else xn
        T, H = x.shape
        ys = np.zeros((T * k, H))
        for e in range(E):
            rows = perm[offsets[e]:offsets[e + 1]]
            if rows.size == 0:
                continue
            g = xs[rows // k] @ O.widen(L["w_gate"][e]).T
            u = xs[rows // k] @ O.widen(L["w_up"][e]).T
            h = O.silu(u) * g if swap_gate_up else O.silu(g) * u
            ys[offsets[e]:offsets[e + 1]] = h @ O.widen(L["w_down"][e]).T
        out = np.zeros((T, H))
        for j in range(k):
            wj = w[:, k - 1 - j:k - j] if reversed_weights else w[:, j:j + 1]
            out += wj * ys[inv.reshape(T, k)[:, j]]
        return out
    return moe


def _embed_scaled(model, tokens):
    return _orig["widen"](model.embed[np.asarray(tokens)]) * math.sqrt(model.cfg["hidden"])


def _vocab_no_norm(model, x, prec, rows=None, chunk=16384):
    xn = prec.store(x)
    if rows is not None:
        xn = xn[np.asarray(rows)]
    return xn @ O.widen(model.w_out).T


def _round_truncate(x):
    m, e = np.frexp(np.asarray(x, dtype=np.float64))
    return np.ldexp(np.trunc(m * 256.0), e - 8)


def _splitmix_n(seed, n):
    return _orig["splitmix64"](seed, n - 1) if n > 0 else _orig["splitmix64"](seed - O._GAMMA, 0)


def _renoise_low_bits(seed, step, pos, vocab):
    x = O.splitmix64(seed, (step << 32) | pos)
    return ((x & 0xFFFFFFFF) * vocab) >> 32


def _renoise_count_ceil(C, S, s, r0, r1):
    f = r0 if S == 1 else (r0 * (S - 1 - s) + r1 * s) / (S - 1)
    return int(np.ceil(C * f - 1e-9))


def _update_variant(most_confident=False, ties_high_pos=False, argmax_last=False):
    def upd(logits, n_renoise, seed, step):
        r = _orig["canvas_update"](logits, n_renoise, seed, step)
        C, V = logits.shape
        conf = r["conf"]
        if argmax_last:
            r["argmax"] = (V - 1 - np.argmax(logits[:, ::-1], axis=1)).astype(np.int32)
        key = -conf if most_confident else conf
        if ties_high_pos:
            order = (C - 1 - np.argsort(key[::-1], kind="stable"))
        else:
            order = np.argsort(key, kind="stable")
        chosen = np.sort(order[:n_renoise])
        canvas = r["argmax"].astype(np.int64).copy()
        for i in chosen:
            canvas[i] = O.renoise_token(seed, step, int(i), V)
        r["canvas"] = canvas.astype(np.int32)
        r["renoised"] = chosen
        return r
    return upd


def _masked_variant(mask_may_win=False, relock=False, denom_without_mask=False):
    def upd(logits, canvas, n_keep, mask_id):
        C, V = logits.shape
        canvas = np.asarray(canvas).astype(np.int64)
        m = logits.max(axis=1)
        cl = logits.copy()
        if not mask_may_win:
            cl[:, mask_id] = -np.inf
        denom = np.exp((cl if denom_without_mask else logits) - m[:, None]).sum(axis=1)
        cand = np.argmax(cl, axis=1)
        conf = np.exp(cl[np.arange(C), cand] - m) / denom
        masked = np.arange(C) if relock else np.nonzero(canvas == mask_id)[0]
        keep = min(int(n_keep), len(masked))
        order = masked[np.argsort(conf[masked], kind="stable")]
        kept = np.sort(order[:keep])
        out = canvas.copy()
        out[masked] = cand[masked]
        out[kept] = mask_id
        r = _orig["canvas_update_masked"](logits, canvas, n_keep, mask_id)
        r.update(canvas=out.astype(np.int32), argmax=cand.astype(np.int32), conf=conf, kept=kept)
        return r
    return upd


def _e4m3_bias8(code):
    code = int(code)
    s = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 0xF, code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    return s * m * 2.0 ** -9 if e == 0 else s * (1 + m / 8) * 2.0 ** (e - 8)


def _e4m3_subnormal(code):
    code = int(code)
    s = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 0xF, code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    return s * (m / 8) * 2.0 ** -7 if e == 0 else s * (1 + m / 8) * 2.0 ** (e - 7)   # 2^-10 per step


def _e4m3_encode_ties_away(x):
    neg = np.signbit(x)
    a = min(abs(float(x)), O.E4M3_MAX)
    i = int(np.searchsorted(O._E4M3_POS, a))
    if i < len(O._E4M3_POS) and O._E4M3_POS[i] == a:
        c = i
    else:
        c = i - 1 if a - O._E4M3_POS[i - 1] < O._E4M3_POS[i] - a else i
    return c | (0x80 if neg else 0)


def _mx_scale_off_by_one(w, block=32):
    w = np.asarray(w, dtype=np.float64)
    blocks = w.reshape(*w.shape[:-1], w.shape[-1] // block, block)
    amax = np.abs(blocks).max(axis=-1)
    exp = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 7, -127).astype(np.int32)
    scaled = blocks / np.ldexp(1.0, exp)[..., None]
    codes = np.vectorize(O.e4m3_encode, otypes=[np.uint8])(scaled)
    return codes.reshape(w.shape), exp


def _e2m1_subnormal(code):
    code = int(code)
    s = -1.0 if code & 0x8 else 1.0
    e, m = (code >> 1) & 0x3, code & 0x1
    return s * 1.0 * m if e == 0 else s * (1 + 0.5 * m) * 2.0 ** (e - 1)


def _nvfp4_no_six(w, block=16):
    w = np.asarray(w, dtype=np.float64)
    amax_t = float(np.abs(w).max())
    g = amax_t / O.E4M3_MAX if amax_t > 0 else 1.0
    blocks = w.reshape(*w.shape[:-1], w.shape[-1] // block, block)
    amax = np.abs(blocks).max(axis=-1)
    sc = np.vectorize(O.e4m3_encode, otypes=[np.uint8])(amax / g)
    sb = np.vectorize(O.e4m3_decode, otypes=[np.float64])(sc)
    codes = np.vectorize(O.e2m1_encode, otypes=[np.uint8])(blocks / np.where(sb > 0, sb * g, 1.0)[..., None])
    return codes.reshape(w.shape), sc, g


def _denoise_positions_from_zero(model, cache, canvas, prec, logit_rows=None):
    """The pass with canvas positions 0..C-1 instead of P..P+C-1."""
    orig_rope = _orig["rope"]
    O.rope = lambda x, positions, theta: orig_rope(x, positions - positions[0], theta)
    try:
        return _orig["denoise_pass"](model, cache, canvas, prec, logit_rows)
    finally:
        O.rope = orig_rope


def _denoise_writes_cache(model, cache, canvas, prec, logit_rows=None):
    """The pass appending the canvas K/V to the caller's cache."""
    out = _orig["denoise_pass"](model, cache, canvas, prec, logit_rows)
    grown = _orig["prefill_append"](model, cache, canvas, prec)
    cache.k, cache.v = grown.k, grown.v
    return out


def _prefill_bidirectional(P, T):
    return np.ones((T, P + T), dtype=bool)


def _attention_wrong_axis(q, k, v, allowed):
    nq, Tq, d = q.shape
    g = nq // k.shape[0]
    out = np.empty_like(q)
    for h in range(nq):
        s = np.where(allowed, (q[h] @ k[h // g].T) / np.sqrt(d), -np.inf)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p = p / np.maximum(p.sum(axis=0, keepdims=True), 1e-300)       # normalised over queries
        out[h] = p @ v[h // g]
    return out


def _update_conf_is_max_logit(logits, n_renoise, seed, step):
    r = _orig["canvas_update"](logits, n_renoise, seed, step)
    C, V = logits.shape
    key = logits.max(axis=1)
    chosen = np.sort(np.argsort(key, kind="stable")[:n_renoise])
    canvas = r["argmax"].astype(np.int64).copy()
    for i in chosen:
        canvas[i] = O.renoise_token(seed, step, int(i), V)
    r.update(canvas=canvas.astype(np.int32), renoised=chosen, conf=np.exp(key))
    return r


def _e2m1_encode_ties_up(x):
    neg = np.signbit(x)
    a = min(abs(float(x)), 6.0)
    i = int(np.searchsorted(O._E2M1_POS, a))
    if i < 8 and O._E2M1_POS[i] == a:
        c = i
    else:
        c = i - 1 if a - O._E2M1_POS[i - 1] < O._E2M1_POS[i] - a else i
    return c | (0x8 if neg else 0)


def _array_ties_away(table, top, sign_bit):
    def enc(x):
        x = np.asarray(x, dtype=np.float64)
        a = np.minimum(np.abs(x), top)
        i = np.searchsorted(table, a)
        lo = np.maximum(i - 1, 0)
        c = np.where(table[i] == a, i, np.where(a - table[lo] < table[i] - a, lo, i))
        return (c | np.where(np.signbit(x), sign_bit, 0)).astype(np.uint8)
    return enc


def _merge_taps_per_canvas(per_canvas_taps, n_experts):
    """Rows stacked, but the permutation kept per canvas (offset) instead of grouped over the batch."""
    out = []
    for layer_taps in zip(*per_canvas_taps):
        m = {key: np.concatenate([t[key] for t in layer_taps], axis=0)
             for key in ("x_in", "attn_o", "x_attn", "x_out", "router_logits", "topk_idx", "topk_w", "router_margin")}
        perms, base = [], 0
        for t in layer_taps:
            perms.append(np.asarray(t["perm"]) + base)
            base += t["topk_idx"].size
        counts = sum(t["counts"] for t in layer_taps)
        m.update(counts=counts, offsets=np.concatenate([[0], np.cumsum(counts)]), perm=np.concatenate(perms),
                 union=int((counts > 0).sum()))
        out.append(m)
    return out


def _batched_shared_cache(model, caches, canvases, prec):
    """Every canvas attends to the first canvas's cache."""
    return [_orig["denoise_pass"](model, caches[0], np.asarray(x), prec) for x in canvases]


def _generate_first_seed(model, caches, canvases, S, r_start, r_end, seeds, prec, append):
    res = [_orig["generate_canvas"](model, c, x, S, r_start, r_end, seeds[0], prec, append)
           for c, x in zip(caches, canvases)]
    return [r[0] for r in res], [r[1] for r in res]


def _generate_no_append(model, caches, canvases, S, r_start, r_end, seeds, prec, append):
    res = [_orig["generate_canvas"](model, c, x, S, r_start, r_end, sd, prec, False)
           for c, x, sd in zip(caches, canvases, seeds)]
    return [r[0] for r in res], [r[1] for r in res]


def _generate_step_plus_one(model, cache, canvas, S, r_start, r_end, seed, prec, append, record=None):
    C = len(canvas)
    cur = np.asarray(canvas, dtype=np.int32).copy()
    for s in range(S):
        logits, taps = O.denoise_pass(model, cache, cur, prec)
        n = O.renoise_count(C, S, s, r_start, r_end)
        upd = O.canvas_update(logits, n, seed, s + 1)
        if record is not None:
            record.append(dict(step=s, canvas_in=cur.copy(), logits=logits, taps=taps, update=upd, n=n))
        cur = upd["canvas"]
    if append:
        cache = O.prefill_append(model, cache, cur, prec)
    return cur, cache


def _masked_generation_from_noise(model, cache, C, S, keep_start, keep_end, mask_id, prec, append, record=None):
    cur = np.arange(C, dtype=np.int32) % mask_id            # not an all-[MASK] canvas
    for s in range(S):
        logits, taps = O.denoise_pass(model, cache, cur, prec)
        n = O.renoise_count(C, S, s, keep_start, keep_end)
        upd = O.canvas_update_masked(logits, cur, n, mask_id)
        if record is not None:
            record.append(dict(step=s, canvas_in=cur.copy(), logits=logits, taps=taps, update=upd, n=n))
        cur = upd["canvas"]
    if append:
        cache = O.prefill_append(model, cache, cur, prec)
    return cur, cache


def _widen_shift8(a):
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(8)).view(np.float32).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


def _prefill_unrounded(model, cache, tokens, prec, taps=None):
    return _orig["prefill_append"](model, cache, tokens, O.Precision("f32"), taps)


def _denoise_cache_stored_again(model, cache, canvas, prec, logit_rows=None):
    """The pass with the canvas's own K/V rounded to storage precision too."""
    orig_qkv = _orig["_qkv"]

    def qkv(model_, l, x, positions, prec_):
        q, k, v = orig_qkv(model_, l, x, positions, prec_)
        return q, prec_.store(k), prec_.store(v)
    O._qkv = qkv
    try:
        return _orig["denoise_pass"](model, cache, canvas, prec, logit_rows)
    finally:
        O._qkv = orig_qkv


# name -> (attribute, replacement, pins that must see it)
MUTANTS = {
    "widen shifts bf16 bits by 8": ("widen", _widen_shift8, ["test_widen_bf16_bits"]),
    "bf16 rounding truncates": ("round_bf16", _round_truncate, ["test_round_bf16_ties_and_library"]),
    "rms_norm drops eps": ("rms_norm", _rms_no_eps, ["test_rms_norm_closed_forms"]),
    "rms_norm sum instead of mean": ("rms_norm", _rms_sum, ["test_rms_norm_closed_forms"]),
    "rope rotates the wrong way": ("rope", _rope_sign, ["test_rope_closed_form_and_relative_position"]),
    "rope interleaved pairs": ("rope", _rope_interleaved, ["test_rope_closed_form_and_relative_position"]),
    "rope frequency exponent halved": ("rope", _rope_freq, ["test_rope_closed_form_and_relative_position"]),
    "silu sign": ("silu", _silu_sign, ["test_silu_closed_forms"]),
    "prefix rows see block keys": ("block_mask", _mask_prefix_sees_block,
                                   ["test_block_mask_matches_worked_example"]),
    "block rows causal": ("block_mask", _mask_block_causal, ["test_block_mask_matches_worked_example"]),
    "prefill row misses its own key": ("causal_rows", _causal_off_by_one,
                                       ["test_causal_rows_are_prefix_rows_of_mask"]),
    "prefill bidirectional": ("causal_rows", _prefill_bidirectional,
                              ["test_causal_rows_are_prefix_rows_of_mask",
                               "test_chunked_prefill_equals_single_prefill"]),
    "attention scale 1/d": ("attention", _attention_variant(scale=lambda d: 1.0 / d),
                            ["test_attention_two_keys_logistic_scale"]),
    "attention unscaled": ("attention", _attention_variant(scale=lambda d: 1.0),
                           ["test_attention_two_keys_logistic_scale"]),
    "gqa interleaved head map": ("attention", _attention_variant(head_map=lambda h, nq, nkv: h % nkv),
                                 ["test_attention_gqa_head_mapping"]),
    "attention ignores the mask": ("attention", _attention_variant(masked=False),
                                   ["test_attention_closed_forms"]),
    "softmax normalised over queries": ("attention", _attention_wrong_axis, ["test_attention_closed_forms"]),
    "router ties to the higher id": ("router_topk", _router_variant(ties_high=True),
                                     ["test_router_topk_special_cases"]),
    "router weights not renormalised": ("router_topk", _router_variant(full_softmax=True),
                                        ["test_router_topk_brute_force_subsets"]),
    "permutation (expert, slot, token)": ("expert_permutation", _perm_slot_major,
                                          ["test_expert_permutation_invariants"]),
    "moe gate and up swapped": ("moe", _moe_variant(swap_gate_up=True),
                                ["test_moe_identical_experts_equals_dense_swiglu"]),
    "moe combine weights reversed": ("moe", _moe_variant(reversed_weights=True),
                                     ["test_moe_combine_pairs_each_weight_with_its_expert"]),
    "moe experts read the un-normed residual": ("moe", _moe_variant(raw_input=True),
                                                ["test_moe_identical_experts_equals_dense_swiglu"]),
    "embedding scaled by sqrt(H)": ("embed", _embed_scaled, ["test_single_token_pass_closed_form"]),
    "no final norm": ("vocab_logits", _vocab_no_norm, ["test_single_token_pass_closed_form"]),
    "pass positions start at 0": ("denoise_pass", _denoise_positions_from_zero,
                                  ["test_prefix_kv_reuse_equals_full_recompute"]),
    "pass writes the cache": ("denoise_pass", _denoise_writes_cache,
                              ["test_denoise_pass_leaves_cache_untouched"]),
    "canvas K/V rounded in flight": ("denoise_pass", _denoise_cache_stored_again,
                                     ["test_bf16_storage_rounds_what_prefill_writes_and_nothing_in_flight"]),
    "prefill stores unrounded K/V": ("prefill_append", _prefill_unrounded,
                                     ["test_bf16_storage_rounds_what_prefill_writes_and_nothing_in_flight"]),
    "splitmix64 counter off by one": ("splitmix64", _splitmix_n, ["test_splitmix64_known_answers"]),
    "re-noise token from the low bits": ("renoise_token", _renoise_low_bits,
                                         ["test_renoise_token_is_the_top_bits_of_the_published_draw"]),
    "re-noise count rounds up": ("renoise_count", _renoise_count_ceil, ["test_renoise_schedule_golden"]),
    "re-noise the most confident": ("canvas_update", _update_variant(most_confident=True),
                                    ["test_canvas_update_renoise_set_brute_force"]),
    "re-noise ties to the higher position": ("canvas_update", _update_variant(ties_high_pos=True),
                                             ["test_canvas_update_special_cases"]),
    "argmax ties to the last id": ("canvas_update", _update_variant(argmax_last=True),
                                   ["test_canvas_update_special_cases"]),
    "confidence is the max logit": ("canvas_update", _update_conf_is_max_logit,
                                    ["test_canvas_update_renoise_set_brute_force"]),
    "masked: the mask id may win": ("canvas_update_masked", _masked_variant(mask_may_win=True),
                                    ["test_masked_update_worked_example"]),
    "masked: locked positions re-decided": ("canvas_update_masked", _masked_variant(relock=True),
                                            ["test_masked_update_worked_example"]),
    "masked: confidence normalised without the mask id": (
        "canvas_update_masked", _masked_variant(denom_without_mask=True), ["test_masked_update_worked_example"]),
    "e4m3 bias 8": ("e4m3_decode", _e4m3_bias8, ["test_e4m3_decode_closed_forms"]),
    "e4m3 subnormal scale": ("e4m3_decode", _e4m3_subnormal, ["test_e4m3_decode_closed_forms"]),
    "e4m3 ties away from even": ("e4m3_encode", _e4m3_encode_ties_away,
                                 ["test_e4m3_encode_round_trip_rounding_saturation"]),
    "mx scale exponent off by one": ("mx_e4m3_quantize", _mx_scale_off_by_one, ["test_mx_e4m3_block_scaling"]),
    "e2m1 subnormal value": ("e2m1_decode", _e2m1_subnormal, ["test_e2m1_codes_rounding_saturation"]),
    "e2m1 ties away from even": ("e2m1_encode", _e2m1_encode_ties_up, ["test_e2m1_codes_rounding_saturation"]),
    "nvfp4 tensor scale without the 6": ("nvfp4_quantize", _nvfp4_no_six, ["test_nvfp4_block_scaling"]),
    "batch permutation kept per canvas": ("merge_batch_taps", _merge_taps_per_canvas,
                                          ["test_batch_reads_the_union_of_the_canvases_experts"]),
    "batched canvases share a cache": ("denoise_pass_batched", _batched_shared_cache,
                                       ["test_batched_canvases_do_not_see_each_other"]),
    "batched generation with one seed": ("generate_canvases", _generate_first_seed,
                                         ["test_batched_canvases_do_not_see_each_other"]),
    "batched generation skips the append": ("generate_canvases", _generate_no_append,
                                            ["test_batched_canvases_do_not_see_each_other"]),
    "generation re-noises with the next step's draws": ("generate_canvas", _generate_step_plus_one,
                                                        ["test_resume_from_a_middle_pass_reproduces_the_run"]),
    "masked generation starts from noise": ("generate_canvas_masked", _masked_generation_from_noise,
                                            ["test_generate_masked_loop_properties"]),
    "array e4m3 encoder ties away from even": ("e4m3_encode_array", _array_ties_away(O._E4M3_POS, 448.0, 0x80),
                                               ["test_e4m3_array_encoder_is_the_scalar_rule"]),
    "array e2m1 encoder ties away from even": ("e2m1_encode_array", _array_ties_away(O._E2M1_POS, 6.0, 0x8),
                                               ["test_e2m1_array_encoder_is_the_scalar_rule"]),
}


def _qkv_rope_on_v(model, l, x, positions, prec):
    q, k, v = _orig["_qkv"](model, l, x, positions, prec)
    return q, k, O.rope(v, positions, model.cfg["rope_theta"])


def _qkv_no_rope_on_k(model, l, x, positions, prec):
    q, _, v = _orig["_qkv"](model, l, x, positions, prec)
    _, k, _ = _orig["_qkv"](model, l, x, np.zeros_like(positions), prec)   # position 0: no rotation
    return q, k, v


def _qkv_no_rope(model, l, x, positions, prec):
    return _orig["_qkv"](model, l, x, np.zeros_like(positions), prec)


def _attn_out_heads_not_gathered(model, l, o, prec):
    return o.reshape(o.shape[1], -1) @ O.widen(model.layers[l]["w_o"]).T


def _mx_deq_neighbour_scale(codes, exp, block=32):
    return _orig["mx_e4m3_dequantize"](codes, np.roll(exp, 1, axis=-1), block)


def _mx_deq_row_scale(codes, exp, block=32):
    return _orig["mx_e4m3_dequantize"](codes, np.broadcast_to(exp.max(axis=-1, keepdims=True), exp.shape), block)


def _nv_deq_neighbour_scale(codes, sc, g, block=16):
    return _orig["nvfp4_dequantize"](codes, np.roll(sc, 1, axis=-1), g, block)


def _full_states_causal(model, prefix_tokens, canvas, prec):
    saved = O.block_mask
    O.block_mask = lambda P, C: O.causal_rows(0, P + C)
    try:
        return _orig["full_sequence_states"](model, prefix_tokens, canvas, prec)
    finally:
        O.block_mask = saved


MUTANTS.update({
    "RoPE applied to v": ("_qkv", _qkv_rope_on_v, ["test_attention_sees_relative_positions_only"]),
    "no RoPE on k": ("_qkv", _qkv_no_rope_on_k, ["test_attention_sees_relative_positions_only"]),
    "no RoPE at all": ("_qkv", _qkv_no_rope, ["test_attention_sees_relative_positions_only"]),
    "heads not gathered before the output projection": (
        "_attn_out", _attn_out_heads_not_gathered, ["test_prefix_kv_reuse_equals_full_recompute"]),
    "mx dequantised with the neighbouring block's scale": (
        "mx_e4m3_dequantize", _mx_deq_neighbour_scale, ["test_block_scales_stay_with_their_blocks"]),
    "mx dequantised with one scale per row": (
        "mx_e4m3_dequantize", _mx_deq_row_scale, ["test_block_scales_stay_with_their_blocks"]),
    "nvfp4 dequantised with the neighbouring block's scale": (
        "nvfp4_dequantize", _nv_deq_neighbour_scale, ["test_block_scales_stay_with_their_blocks"]),
    "full recompute with a causal mask over the canvas": (
        "full_sequence_states", _full_states_causal, ["test_prefix_kv_reuse_equals_full_recompute"]),
})


def _run_pins(names):
    failed = []
    for n in names:
        try:
            getattr(PINS, n)()
        except AssertionError:
            failed.append(n)
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_see_the_mutant(name, monkeypatch):
    attr, fn, pins = MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    assert _run_pins(pins), f"no pin sees the mutant '{name}' (ran {pins})"
