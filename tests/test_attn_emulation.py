"""Both attention kernels replayed at the address level on the CPU (tests/tc_emu.py): every
TMA box, shared-memory offset, descriptor start, TMEM column, packed-P layout and output
index as the kernel source computes it, in an order the kernel's barriers allow, against
the oracle's attention at the GPU test's tolerance.

The head-pair kernel (tc_attn2_kernel, validated on a B200) is the control for the
model; tc_attn_kernel, restructured (query tile in TMEM, three-slot ring, separate load
and MMA warps), is replayed the same way before its first run.  The head-pair kernel (tc_attn2_kernel, not yet run) is replayed
with its load warp running as far ahead as its slot plan lets it, so a slot reused too
early, an S/P buffer overwritten before its PV, or a wrong column or offset changes the
result.  Planted mistakes in the transcription are caught, which shows the replay is
sharp enough to see them.
"""
from __future__ import annotations

import math

import numpy as np
import pytest

import tc_emu as T
from oracle import dg_oracle as O
from test_attn_geometry import choose_pair, lo_rows, splits_single

D = 128
NEG = np.float32(-np.inf)


# ---------------------------------------------------------------- inputs
def build(seed, nq, nkv, n_q, pos0, n_keys, causal, lo_scale=2.0 ** -9):
    """The attention of one pass: query (fp32 as bf16 hi + lo), the cache's bf16 K and V^T,
    and the low terms of the call's own K/V (positions pos0 .. n_keys - 1) in a window of
    rows counted from base = the multiple of 128 at or below pos0, zero before pos0."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((nq, n_q, D)).astype(np.float32)
    q_hi = T.bf16_bits(q)
    q_lo = T.bf16_bits(q - T.bf16_value(q_hi))
    cap = -(-n_keys // 8) * 8 + 8
    Kc = T.bf16_bits(rng.standard_normal((nkv, cap, D)).astype(np.float32))
    Vc = T.bf16_bits(rng.standard_normal((nkv, cap, D)).astype(np.float32))
    base = (pos0 // 128) * 128
    Lc = lo_rows(n_q)
    K_lo = np.zeros((nkv, Lc, D), np.uint16)
    V_lo = np.zeros((nkv, Lc, D), np.uint16)
    own = n_keys - pos0
    K_lo[:, pos0 - base:n_keys - base] = T.bf16_bits(rng.standard_normal((nkv, own, D)).astype(np.float32) * lo_scale)
    V_lo[:, pos0 - base:n_keys - base] = T.bf16_bits(rng.standard_normal((nkv, own, D)).astype(np.float32) * lo_scale)
    pos = pos0 + np.arange(n_q)
    key_lim = np.minimum(pos + 1, n_keys) if causal else np.full(n_q, n_keys)
    return dict(nq=nq, nkv=nkv, n_q=n_q, pos0=pos0, n_keys=n_keys, causal=causal, base=base,
                q_hi=q_hi, q_lo=q_lo, Kc=Kc, Vt=np.ascontiguousarray(Vc.transpose(0, 2, 1)), K_lo=K_lo,
                Vt_lo=np.ascontiguousarray(V_lo.transpose(0, 2, 1)), key_lim=key_lim)


def maps(c):
    """The tensors the kernels' tensor maps cover (extents as the host encodes them)."""
    nk, b = c["n_keys"], c["base"]
    return dict(Q=c["q_hi"], Ql=c["q_lo"], K=c["Kc"][:, :nk, :], Vt=c["Vt"][:, :, :nk],
                Kl=c["K_lo"][:, :nk - b, :], Vtl=c["Vt_lo"][:, :, :nk - b])


def oracle(c):
    nk, b = c["n_keys"], c["base"]
    q = T.bf16_value(c["q_hi"]).astype(np.float64) + T.bf16_value(c["q_lo"])
    K = T.bf16_value(c["Kc"][:, :nk]).astype(np.float64)
    V = T.bf16_value(c["Vt"][:, :, :nk]).transpose(0, 2, 1).astype(np.float64)
    K[:, b:] += T.bf16_value(c["K_lo"][:, :nk - b])
    V[:, b:] += T.bf16_value(c["Vt_lo"][:, :, :nk - b]).transpose(0, 2, 1)
    allowed = np.arange(nk)[None, :] < c["key_lim"][:, None]
    out = O.attention(q, K, V, allowed)                       # [nq][n_q][d]
    return out.transpose(1, 0, 2).reshape(c["n_q"], -1)


def within(got, ref):
    rms = math.sqrt(float(np.mean(ref * ref)))
    return bool((np.abs(got - ref) <= 1e-4 * np.abs(ref) + 1e-4 * rms).all())


# ---------------------------------------------------------------- shared pieces
def softmax_chunk(s_raw, key0, key_lim, scale_log2, m_used, l):
    """One chunk of a thread's row: scale, mask, lazy max; returns (s, rmax-applied state)."""
    s = (s_raw.view(np.float32) * scale_log2).astype(np.float32)
    keys = key0 + np.arange(s.shape[1])
    s = np.where(keys[None, :] >= key_lim[:, None], NEG, s).astype(np.float32)
    return s


def p_words(s, m_used, l):
    """P = exp2(s - m) for 2 x 16 keys at a time, packed hi / lo (as the kernels), and the
    row sums accumulated pair by pair in fp32."""
    n = s.shape[1]
    with np.errstate(invalid="ignore", over="ignore"):
        p = np.where(np.isneginf(s), np.float32(0), np.exp2((s - m_used[:, None]).astype(np.float32)))
    p = p.astype(np.float32)
    for e in range(0, n, 2):
        l = (l + (p[:, e] + p[:, e + 1]).astype(np.float32)).astype(np.float32)
    hi = T.bf16_value(T.bf16_bits(p))
    lo = (p - hi).astype(np.float32)
    wh = T.pack_bf16x2(p[:, 0::2], p[:, 1::2])
    wl = T.pack_bf16x2(lo[:, 0::2], lo[:, 1::2])
    return wh, wl, l


def lazy_update(rmax, m_used, l, warp_rescale):
    upd = rmax > m_used + np.float32(8.0)
    with np.errstate(invalid="ignore"):
        alpha = np.where(upd, np.exp2((m_used - rmax).astype(np.float32)), np.float32(1.0)).astype(np.float32)
    any_w = np.repeat(np.array([upd[w * 32:(w + 1) * 32].any() for w in range(4)]), 32)
    warp_rescale(any_w, alpha)
    l = np.where(upd, (l * alpha).astype(np.float32), l).astype(np.float32)
    m_used = np.where(upd, rmax, m_used).astype(np.float32)
    return m_used, l


def softmax_chunk_raw(raw, key0, key_lim):
    """The head-pair kernel's chunk: raw scores (fp32), -inf at or past each row's key
    limit; the row maximum is taken on the raw scores and scaled afterwards."""
    s = raw.view(np.float32).copy()
    keys = key0 + np.arange(s.shape[1])
    return np.where(keys[None, :] >= key_lim[:, None], NEG, s).astype(np.float32)


def p_words_one_term(s_raw, scale, m_used, l_pair):
    """The head-pair kernel's P: 2^(fma(s, scale, -m)) rounded to bf16 and packed in pairs;
    the row sum adds the rounded values, as two fp32 partial sums (even and odd keys)."""
    neg_m = np.where(np.isneginf(m_used), np.float32(0), -m_used).astype(np.float64)
    with np.errstate(invalid="ignore", over="ignore"):
        t = (s_raw.astype(np.float64) * np.float64(scale) + neg_m[:, None]).astype(np.float32)
        p = np.exp2(t.astype(np.float64)).astype(np.float32)
    hi = T.bf16_value(T.bf16_bits(p)).astype(np.float32)
    le, lo_ = l_pair
    for e in range(0, p.shape[1], 2):
        le = (le + hi[:, e]).astype(np.float32)
        lo_ = (lo_ + hi[:, e + 1]).astype(np.float32)
    return T.pack_bf16x2(p[:, 0::2], p[:, 1::2]), (le, lo_)


def p_rounding_bounds(c):
    """The exact attention (fp64) and, per element, the effect of rounding each probability
    once to bf16 (relative error at most u = 2^-8; the row sum adds the rounded values, so
    the output is an exact weighted mean): worst case u / (1 - u) * sum_j p_j |v_j - o| /
    sum_j p_j, bounded above by u / (1 - u) * (p @ |V| / l + |o|); and the variance
    (u^2 / 3) * sum_j p_j^2 (v_j - o)^2 / l^2 of independent roundings."""
    nk, b = c["n_keys"], c["base"]
    q = T.bf16_value(c["q_hi"]).astype(np.float64) + T.bf16_value(c["q_lo"])
    K = T.bf16_value(c["Kc"][:, :nk]).astype(np.float64)
    V = T.bf16_value(c["Vt"][:, :, :nk]).transpose(0, 2, 1).astype(np.float64)
    K[:, b:] += T.bf16_value(c["K_lo"][:, :nk - b])
    V[:, b:] += T.bf16_value(c["Vt_lo"][:, :, :nk - b]).transpose(0, 2, 1)
    allowed = np.arange(nk)[None, :] < c["key_lim"][:, None]
    nq, n_q = q.shape[0], q.shape[1]
    g = nq // K.shape[0]
    u = 2.0 ** -8
    o_all, worst_all, var_all = [], [], []
    for h in range(nq):
        s = q[h] @ K[h // g].T / math.sqrt(D)
        s = np.where(allowed, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        p = np.where(allowed, np.exp(s - np.where(np.isfinite(m), m, 0)), 0.0)
        l = p.sum(axis=1, keepdims=True)
        lsafe = np.where(l > 0, l, 1.0)
        Vh = V[h // g]
        o = p @ Vh / lsafe
        worst = u / (1 - u) * (p @ np.abs(Vh) / lsafe + np.abs(o))
        p2 = p * p
        var = (u * u / 3.0) * (p2 @ (Vh * Vh) - 2 * o * (p2 @ Vh) + o * o * p2.sum(axis=1, keepdims=True)) / lsafe ** 2
        o_all.append(o)
        worst_all.append(worst)
        var_all.append(np.maximum(var, 0))
    cat = lambda xs: np.stack(xs).transpose(1, 0, 2).reshape(n_q, -1)
    return cat(o_all), cat(worst_all), cat(var_all)


def within_one_term_p(got, c):
    """The head-pair kernel's output against the exact attention: every element within the
    worst case of its probabilities' one-term rounding plus the fp32 allowance of the rest
    (1e-4 of the element and of the RMS), and the RMS error within 1.5 times the RMS the
    independent roundings predict (plus 1e-5 of the RMS)."""
    o, worst, var = p_rounding_bounds(c)
    rms = math.sqrt(float(np.mean(o * o)))
    err = np.abs(got - o)
    ok_each = bool((err <= worst + 1e-4 * np.abs(o) + 1e-4 * rms).all())
    ok_rms = math.sqrt(float(np.mean(err * err))) <= 1.5 * math.sqrt(float(np.mean(var))) + 1e-5 * rms
    return ok_each and ok_rms


def p_words_fma(s_raw, scale, m_used, l_pair):
    """P = 2^(fma(s, scale, -m)) (one rounding; offset 0 where the row has seen no key),
    packed hi / lo, and the row sum as two fp32 partial sums (even and odd keys)."""
    neg_m = np.where(np.isneginf(m_used), np.float32(0), -m_used).astype(np.float64)
    with np.errstate(invalid="ignore", over="ignore"):
        t = (s_raw.astype(np.float64) * np.float64(scale) + neg_m[:, None]).astype(np.float32)
        p = np.exp2(t.astype(np.float64)).astype(np.float32)
    le, lo_ = l_pair
    for e in range(0, p.shape[1], 2):
        le = (le + p[:, e]).astype(np.float32)
        lo_ = (lo_ + p[:, e + 1]).astype(np.float32)
    hi = T.bf16_value(T.bf16_bits(p))
    lo = (p - hi).astype(np.float32)
    wh = T.pack_bf16x2(p[:, 0::2], p[:, 1::2])
    wl = T.pack_bf16x2(lo[:, 0::2], lo[:, 1::2])
    return wh, wl, (le, lo_)


def epilogue(tm, o_cols, l, m_used, rows, out, out_lo, part_o, part_lse, sp, h, n_splits, nq, n_q, col0=0, ncols=128):
    inv = np.where(l > 0, (np.float32(1.0) / np.where(l > 0, l, 1)).astype(np.float32), np.float32(0)).astype(np.float32)
    o = (tm.f32(o_cols, ncols) * inv[:, None]).astype(np.float32)
    valid = rows < n_q
    if n_splits == 1:
        hi = T.bf16_value(T.bf16_bits(o))
        lo = T.bf16_value(T.bf16_bits((o - hi).astype(np.float32)))
        out[rows[valid], h * D + col0:h * D + col0 + ncols] = hi[valid]
        out_lo[rows[valid], h * D + col0:h * D + col0 + ncols] = lo[valid]
    else:
        part_o[sp, h, rows[valid], col0:col0 + ncols] = o[valid]
        if part_lse is not None:
            with np.errstate(divide="ignore"):
                lse = np.where(l > 0, m_used + np.log2(np.where(l > 0, l, 1)).astype(np.float32), NEG)
            part_lse[sp, h, rows[valid]] = lse[valid]


def merge(part_o, part_lse, n_splits):
    mx = part_lse[:n_splits].max(axis=0)                        # [nq][n_q]
    num = np.zeros(part_o.shape[1:], np.float32)
    den = np.zeros(part_lse.shape[1:], np.float32)
    for s in range(n_splits):
        lse = part_lse[s]
        with np.errstate(invalid="ignore"):
            w = np.where(np.isneginf(lse), np.float32(0), np.exp2((lse - mx).astype(np.float32))).astype(np.float32)
        num = (num + w[..., None] * part_o[s]).astype(np.float32)
        den = (den + w).astype(np.float32)
    v = np.where(den[..., None] > 0, num / np.where(den > 0, den, 1)[..., None], 0).astype(np.float32)
    hi = T.bf16_value(T.bf16_bits(v))
    lo = T.bf16_value(T.bf16_bits((v - hi).astype(np.float32)))
    nq, n_q = v.shape[0], v.shape[1]
    return (hi + lo).transpose(1, 0, 2).reshape(n_q, nq * D)


def merge2(part_o, part_lse, n_splits):
    """attn_merge2_kernel: per (row, head) warp, lane s holds split s's lse; maximum and the
    weight sum by butterflies, the columns accumulated over the splits in order, times the
    reciprocal of the sum."""
    nq, n_q = part_lse.shape[1], part_lse.shape[2]
    lanes = np.full((32, nq, n_q), NEG, np.float32)
    lanes[:n_splits] = part_lse[:n_splits]
    mx = lanes.copy()
    o = 16
    while o:
        mx = np.maximum(mx, mx[np.arange(32) ^ o])
        o >>= 1
    with np.errstate(invalid="ignore"):
        wt = np.where(np.isneginf(lanes), np.float32(0), np.exp2((lanes - mx).astype(np.float32))).astype(np.float32)
    den = wt.copy()
    o = 16
    while o:
        den = (den + den[np.arange(32) ^ o]).astype(np.float32)
        o >>= 1
    acc = np.zeros(part_o.shape[1:], np.float32)
    for sp in range(n_splits):
        acc = (acc + wt[sp][..., None] * part_o[sp]).astype(np.float32)
    inv = np.where(den[0] > 0, (np.float32(1) / np.where(den[0] > 0, den[0], 1)).astype(np.float32), np.float32(0))
    v = (acc * inv[..., None]).astype(np.float32)
    hi = T.bf16_value(T.bf16_bits(v))
    lo = T.bf16_value(T.bf16_bits((v - hi).astype(np.float32)))
    return (hi + lo).transpose(1, 0, 2).reshape(n_q, nq * D)


# ---------------------------------------------------------------- tc_attn_kernel
def run_single(c, bug=None):
    """tc_attn_kernel: one head x 128 rows x 128-key chunks; the query tile in TMEM (hi at
    column 0, lo at 64, packed bf16 pairs along d, stored by the softmax warps), S at 128,
    O at 256, one P buffer (hi at 384, lo at 448); three 64 KB K/V slots in the slot plan
    (a current chunk takes two), the load warp running as far ahead as freed slots allow.

    bug: "no_p_wait" -- the softmax writes P(j) without waiting for PV(j - 1);
    "q_lo_cols" -- the lo query terms stored over the hi ones' columns; "no_pv_first" --
    the plain issue order where two own-key chunks follow each other."""
    nq, nkv, n_q, pos0, n_keys, causal = (c[k] for k in ("nq", "nkv", "n_q", "pos0", "n_keys", "causal"))
    m = maps(c)
    group = nq // nkv
    n_splits, cps = splits_single(n_q, nq, n_keys)
    HALF, SLOT, SLOTS = 128 * 128, 4 * 128 * 128, 3
    sSlot = 0
    TM_QHI, TM_QLO, TM_S, TM_O, TM_PHI, TM_PLO = 0, 64, 128, 256, 384, 448
    if bug == "q_lo_cols":
        TM_QLO = 32
    scale = np.float32(1.4426950408889634 / math.sqrt(D))
    out = np.zeros((n_q, nq * D), np.float32)
    out_lo = np.zeros_like(out)
    part_o = np.zeros((n_splits, nq, n_q, D), np.float32)
    part_lse = np.full((n_splits, nq, n_q), NEG, np.float32)

    def q_words(bits, h, q_row0):
        """The query rows of one head as the softmax warps store them: word c of a row holds
        elements 2c (low half) and 2c + 1 (high half); rows past n_q are zero."""
        rows = np.zeros((128, D), np.uint16)
        n = min(128, n_q - q_row0)
        rows[:n] = bits[h, q_row0:q_row0 + n]
        r32 = rows.astype(np.uint32)
        return (r32[:, 0::2] | (r32[:, 1::2] << 16)).astype(np.uint32)

    for qt in range(-(-n_q // 128)):
        for h in range(nq):
            for sp in range(n_splits):
                kvh = h // group
                q_row0 = qt * 128
                rows_here = min(128, n_q - q_row0)
                kv_end = min(n_keys, pos0 + q_row0 + rows_here) if causal else n_keys
                nch_total = -(-kv_end // 128)
                c_begin = sp * cps
                nck = min(nch_total, c_begin + cps) - c_begin
                rows = q_row0 + np.arange(128)
                if nck <= 0:
                    continue                                  # empty partial: zeros, lse -inf
                sm, tm = T.Smem(SLOTS * SLOT), T.Tmem()
                is_cur = lambda j: (c_begin + j) * 128 >= c["base"]
                tm.t[:, TM_QHI:TM_QHI + 64] = q_words(c["q_hi"], h, q_row0)
                tm.t[:, TM_QLO:TM_QLO + 64] = q_words(c["q_lo"], h, q_row0)
                # the slot plan (AtSlotPlan::take), and which chunk's PV frees each slot use
                plan, nxt, uses = [], 0, [0] * SLOTS
                for j in range(nck):
                    parts = []
                    for _ in range(2 if is_cur(j) else 1):
                        parts.append((nxt, uses[nxt]))
                        uses[nxt] += 1
                        nxt = (nxt + 1) % SLOTS
                    plan.append(parts)
                holder = {}
                loaded = [0]

                def pump():
                    """The load warp: the next chunk's slots, each once its previous use was freed."""
                    while loaded[0] < nck:
                        j = loaded[0]
                        if any(s in holder for s, _ in plan[j]):
                            return
                        key0 = (c_begin + j) * 128
                        for i, (s, _) in enumerate(plan[j]):
                            k = sSlot + s * SLOT
                            v = k + 2 * HALF
                            mk, mv = ("K", "Vt") if i == 0 else ("Kl", "Vtl")
                            krow = key0 if i == 0 else key0 - c["base"]
                            sm.tma_load_3d(k, m[mk], 0, krow, kvh, 64, 128)
                            sm.tma_load_3d(k + HALF, m[mk], 64, krow, kvh, 64, 128)
                            sm.tma_load_3d(v, m[mv], krow, 0, kvh, 64, 128)
                            sm.tma_load_3d(v + HALF, m[mv], krow + 64, 0, kvh, 64, 128)
                            holder[s] = j
                        loaded[0] += 1

                def issue_s(j):
                    cur = len(plan[j]) == 2
                    k = sSlot + plan[j][0][0] * SLOT
                    kl = sSlot + plan[j][1][0] * SLOT if cur else 0
                    for kb in range(2):
                        for kk in range(4):
                            qc, off = kb * 32 + kk * 8, kb * HALF + kk * 32
                            T.mma_ts(tm, sm, TM_S, TM_QHI + qc, k + off, 128, 128, (kb | kk) != 0)
                            T.mma_ts(tm, sm, TM_S, TM_QLO + qc, k + off, 128, 128, True)
                            if cur:
                                T.mma_ts(tm, sm, TM_S, TM_QHI + qc, kl + off, 128, 128, True)

                def issue_pv(k_):
                    cur = len(plan[k_]) == 2
                    v = sSlot + plan[k_][0][0] * SLOT + 2 * HALF
                    vl = sSlot + plan[k_][1][0] * SLOT + 2 * HALF if cur else 0
                    for kb in range(2):
                        for kk in range(4):
                            pcol, vd = kb * 32 + kk * 8, v + kb * HALF + kk * 32
                            T.mma_ts(tm, sm, TM_O, TM_PHI + pcol, vd, 128, D, k_ > 0 or (kb | kk) != 0)
                            T.mma_ts(tm, sm, TM_O, TM_PLO + pcol, vd, 128, D, True)
                            if cur:
                                T.mma_ts(tm, sm, TM_O, TM_PHI + pcol, vl + kb * HALF + kk * 32, 128, D, True)
                    for s, _ in plan[k_]:                    # the commits free chunk k_'s slots
                        if holder.get(s) == k_:
                            del holder[s]
                    pump()

                # issued PVs run on the tensor pipe later: deferred until the next MMA issue
                # (in-order pipe), the softmax's wait for the previous PV, a wait for a slot,
                # or the end
                pending = []

                def flush():
                    while pending:
                        issue_pv(pending.pop(0))

                m_used = np.full(128, NEG, np.float32)
                lsum = [np.zeros(128, np.float32), np.zeros(128, np.float32)]
                key_lim = np.array([c["key_lim"][r] if r < n_q else n_keys for r in rows])

                def softmax(j):
                    nonlocal m_used
                    s_h, hmax = [], []
                    for hf in range(2):
                        raw = np.concatenate([tm.t[:, TM_S + hf * 64 + cc * 16:TM_S + hf * 64 + cc * 16 + 16]
                                              for cc in range(4)], axis=1)
                        s = softmax_chunk(raw, (c_begin + j) * 128 + hf * 64, key_lim, scale, None, None)
                        s_h.append(s)
                        hmax.append(s.max(axis=1))
                    rmax = np.maximum(hmax[0], hmax[1])
                    if j > 0 and bug != "no_p_wait":
                        flush()                               # PV(j - 1) has read P and added into O
                    for hf in range(2):
                        def rescale(any_w, alpha, hf=hf):
                            if j > 0 and any_w.any():
                                blk = tm.f32(TM_O + hf * 64, 64)
                                blk[any_w] = (blk[any_w] * alpha[any_w, None]).astype(np.float32)
                        mu, lsum[hf] = lazy_update(rmax, m_used, lsum[hf], rescale)
                    m_used = mu
                    for hf in range(2):
                        wh, wl, lsum[hf] = p_words(s_h[hf], m_used, lsum[hf])
                        tm.t[:, TM_PHI + hf * 32:TM_PHI + hf * 32 + 32] = wh
                        tm.t[:, TM_PLO + hf * 32:TM_PLO + hf * 32 + 32] = wl

                pump()
                for j in range(nck):
                    pv_first = j >= 1 and len(plan[j - 1]) + len(plan[j]) > SLOTS
                    if bug == "no_pv_first":
                        pv_first = False
                    if pv_first:
                        pending.append(j - 1)
                    if loaded[0] <= j:
                        flush()                               # the slots come free as pending PVs complete
                    assert loaded[0] > j, "the MMA warp would wait for a chunk the load warp cannot load"
                    flush()
                    issue_s(j)
                    if j >= 1 and not pv_first:
                        pending.append(j - 1)
                    softmax(j)
                pending.append(nck - 1)
                flush()
                l = (lsum[0] + lsum[1]).astype(np.float32)
                for hf in range(2):
                    epilogue(tm, TM_O + hf * 64, l, m_used, rows, out, out_lo, part_o,
                             part_lse if hf == 0 else None, sp, h, n_splits, nq, n_q, col0=hf * 64, ncols=64)
    return (out + out_lo) if n_splits == 1 else merge(part_o, part_lse, n_splits)


# ---------------------------------------------------------------- tc_attn2_kernel
def run_pair(c, bug=None, force_pair=None):
    """tc_attn2_kernel: a head pair (one head for odd groups) x 128 rows x 128-key chunks,
    a ring of three 32 KB half-slots (a chunk's K, then its V^T, each with its low term
    for own keys), per head one S/P region at 256 hl (P one bf16 term) and O at 256 hl +
    128."""
    nq, nkv, n_q, pos0, n_keys, causal = (c[k] for k in ("nq", "nkv", "n_q", "pos0", "n_keys", "causal"))
    m = maps(c)
    group = nq // nkv
    pair, n_splits, cps = choose_pair(n_q, nq, group, n_keys)
    if force_pair is not None:                       # either mode, whatever the host would choose
        from test_attn_geometry import splits_pair
        pair = force_pair and group % 2 == 0
        n_splits, cps = splits_pair(n_q, nq, group, n_keys, pair)
    W, BLK = 128, 128 * 128
    QHEAD, HSLOT = 4 * BLK, 2 * BLK
    HSLOTS = 3
    phys = (lambda s_: s_ % 2) if bug == "two_slots" else (lambda s_: s_)   # a ring one half-slot short
    sQ, sHalf = 0, 2 * QHEAD
    a2_sp = lambda hl: hl * 256
    a2_o = lambda hl: hl * 256 + 128
    p_step = 4 if bug == "p_col_step" else 8     # packed P columns per 16 keys
    scale = np.float32(1.4426950408889634 / math.sqrt(D))
    nh = 2 if pair else 1
    out = np.zeros((n_q, nq * D), np.float32)
    out_lo = np.zeros_like(out)
    part_o = np.zeros((n_splits, nq, n_q, D), np.float32)
    part_lse = np.full((n_splits, nq, n_q), NEG, np.float32)
    for qt in range(-(-n_q // 128)):
        for y in range(nq // nh):
            h0 = y * nh
            kvh = h0 // group
            for sp in range(n_splits):
                q_row0 = qt * 128
                rows_here = min(128, n_q - q_row0)
                kv_end = min(n_keys, pos0 + q_row0 + rows_here) if causal else n_keys
                nch_total = -(-kv_end // W)
                c_begin = sp * cps
                nck = min(nch_total, c_begin + cps) - c_begin
                rows = q_row0 + np.arange(128)
                if nck <= 0:
                    continue
                sm, tm = T.Smem(2 * QHEAD + 3 * HSLOT), T.Tmem()
                is_cur = lambda j: (c_begin + j) * W >= c["base"]
                for hl in range(nh):
                    q = sQ + hl * QHEAD
                    for off, mp, x in ((0, "Q", 0), (BLK, "Q", 64), (2 * BLK, "Ql", 0), (3 * BLK, "Ql", 64)):
                        sm.tma_load_3d(q + off, m[mp], x, q_row0, h0 + hl, 64, 128)
                # the half-slot plan (HalfSlotPlan::take): per chunk its K parts, then its V parts
                plan, items, nxt = [], [], 0
                for j in range(nck):
                    n = 2 if is_cur(j) else 1
                    ks, vs = [], []
                    for lst in (ks, vs):
                        for i in range(n):
                            lst.append(nxt)
                            items.append((j, "K" if lst is ks else "V", i, nxt))
                            nxt = (nxt + 1) % HSLOTS
                    plan.append((ks, vs))
                holder = {}                                   # half-slot -> (chunk, operand) held until freed
                loaded = [0]                                  # items loaded so far (in order)

                def pump():
                    """The load warp: the next items, each once its half-slot's previous use was freed."""
                    while loaded[0] < len(items):
                        j, op, i, s = items[loaded[0]]
                        if s in holder:
                            return
                        key0 = (c_begin + j) * W
                        krow = key0 if i == 0 else key0 - c["base"]
                        dst = sHalf + phys(s) * HSLOT
                        if op == "K":
                            mk = "K" if i == 0 else "Kl"
                            sm.tma_load_3d(dst, m[mk], 0, krow, kvh, 64, 128)
                            sm.tma_load_3d(dst + BLK, m[mk], 64, krow, kvh, 64, 128)
                        else:
                            mv = "Vt" if i == 0 else "Vtl"
                            sm.tma_load_3d(dst, m[mv], krow, 0, kvh, 64, 128)
                            sm.tma_load_3d(dst + BLK, m[mv], krow + 64, 0, kvh, 64, 128)
                        holder[s] = (j, op)
                        loaded[0] += 1

                def ready(j, op):
                    pump()
                    need = [it for it in items if it[0] == j and it[1] == op]
                    assert all(items.index(it) < loaded[0] for it in need), \
                        "the MMA warp would wait for a half-slot the load warp cannot fill"

                def free(j, op):
                    for s in (plan[j][0] if op == "K" else plan[j][1]):
                        if holder.get(s) == (j, op):
                            del holder[s]
                    pump()

                def issue_s(hl, j):
                    ks = plan[j][0]
                    d = a2_sp(hl)
                    q, ql = sQ + hl * QHEAD, sQ + hl * QHEAD + 2 * BLK
                    k = sHalf + phys(ks[0]) * HSLOT
                    kl = sHalf + phys(ks[1]) * HSLOT if len(ks) == 2 else 0
                    for kb in range(2):
                        for kk in range(4):
                            o = kb * BLK + kk * 32
                            T.mma_ss(tm, sm, d, q + o, k + o, 128, W, (kb | kk) != 0)
                            T.mma_ss(tm, sm, d, ql + o, k + o, 128, W, True)
                            if len(ks) == 2:
                                T.mma_ss(tm, sm, d, q + o, kl + o, 128, W, True)

                def issue_pv(hl, j):
                    vs = plan[j][1]
                    o, pp = a2_o(hl), a2_sp(hl)
                    v = sHalf + phys(vs[0]) * HSLOT
                    vl = sHalf + phys(vs[1]) * HSLOT if len(vs) == 2 else 0
                    for kk in range(8):
                        vo = (kk >> 2) * BLK + (kk & 3) * 32
                        T.mma_ts(tm, sm, o, pp + kk * p_step, v + vo, 128, D, j > 0 or kk != 0)
                        if len(vs) == 2:
                            T.mma_ts(tm, sm, o, pp + kk * 8, vl + vo, 128, D, True)

                m_used = [np.full(128, NEG, np.float32) for _ in range(nh)]
                lpair = [(np.zeros(128, np.float32), np.zeros(128, np.float32)) for _ in range(nh)]
                key_lim = np.array([c["key_lim"][r] if r < n_q else n_keys for r in rows])

                def softmax(hl, j):
                    spa = a2_sp(hl)
                    raw = np.concatenate([tm.t[:, spa + cc * 16:spa + cc * 16 + 16] for cc in range(8)], axis=1)
                    s = softmax_chunk_raw(raw, (c_begin + j) * W, key_lim)

                    def rescale(any_w, alpha):
                        if j > 0 and any_w.any():                 # PV(j - 1) has completed
                            blk = tm.f32(a2_o(hl), D)
                            blk[any_w] = (blk[any_w] * alpha[any_w, None]).astype(np.float32)
                    le, lo_ = lpair[hl]
                    m_old = m_used[hl]
                    rmax = (s.max(axis=1) * scale).astype(np.float32)
                    m_used[hl], le = lazy_update(rmax, m_old, le, rescale)
                    _, lo_ = lazy_update(rmax, m_old, lo_, lambda a, b: None)
                    wh, lpair[hl] = p_words_one_term(s, scale, m_used[hl], (le, lo_))
                    tm.t[:, spa:spa + 64] = wh                # P (one bf16 term) over this row's S

                pump()
                for j in range(nck):
                    ready(j, "K")
                    for hl in range(nh):
                        issue_s(hl, j)
                        if bug == "k_free_after_first_head" and hl == 0:
                            free(j, "K")                      # the commit placed before the second head's S
                    free(j, "K")
                    for hl in range(nh):
                        softmax(hl, j)
                    ready(j, "V")
                    for hl in range(nh):
                        issue_pv(hl, j)
                    free(j, "V")
                for hl in range(nh):
                    lsum = (lpair[hl][0] + lpair[hl][1]).astype(np.float32)
                    epilogue(tm, a2_o(hl), lsum, m_used[hl], rows, out, out_lo, part_o, part_lse, sp, h0 + hl,
                             n_splits, nq, n_q)
    return (out + out_lo) if n_splits == 1 else merge2(part_o, part_lse, n_splits)


CASES = [
    # seed, nq, nkv, n_q, pos0, n_keys, causal
    (1, 4, 2, 100, 200, 300, False),       # canvas over a ragged prefix, head pairs, own-key chunks
    (2, 4, 1, 200, 50, 250, True),         # causal prefill rows, ragged tiles
    (3, 2, 2, 64, 600, 664, False),        # group 1: one head per CTA
    (4, 2, 1, 128, 1536, 1664, False),     # long prefix: several splits and a merge
    (5, 2, 1, 300, 0, 300, True),          # causal from an empty cache: own keys throughout
    (21, 4, 2, 128, 3584, 3712, False),    # long prefix: 12 splits of 5 chunks, slots reused many times
    (22, 2, 2, 256, 2048, 2304, True),     # causal, two query tiles: the first tile's later splits are empty
]


@pytest.mark.parametrize("case", CASES)
def test_validated_kernel_replay_matches_the_oracle(case):
    """The control: the kernel that passes on a B200 passes in the model too."""
    c = build(*case)
    assert within(run_single(c), oracle(c))


@pytest.mark.parametrize("force_pair", [None, True, False])
@pytest.mark.parametrize("case", CASES)
def test_head_pair_kernel_replay_matches_the_oracle(case, force_pair):
    """As the host chooses, and in both modes (two heads per CTA, one head per CTA)."""
    c = build(*case)
    assert within_one_term_p(run_pair(c, force_pair=force_pair), c)


@pytest.mark.parametrize("case", CASES)
def test_head_pair_kernel_replay_with_large_low_terms(case):
    """Every case again with the own keys' low terms at 2^-3 of the values, so that their
    slots, rows and MMAs are checked above the probabilities' rounding."""
    c = build(*case, lo_scale=2.0 ** -3)
    assert within_one_term_p(run_pair(c), c)


@pytest.mark.parametrize("bug", ["p_col_step", "k_free_after_first_head"])
def test_planted_mistakes_in_the_head_pair_replay_are_caught(bug):
    """P's packed columns stepped wrongly (4 per 16 keys instead of 8), or the K half-slots
    freed after the first head's S MMAs (the load warp then fills them before the second
    head reads K): either gives a wrong result or cannot proceed."""
    c = build(6, 4, 2, 100, 200, 300, False)
    assert within_one_term_p(run_pair(c, force_pair=True), c)
    try:
        ok = within_one_term_p(run_pair(c, bug=bug, force_pair=True), c)
    except AssertionError:
        ok = False
    assert not ok


def test_the_one_term_check_sees_a_dropped_low_term():
    """The kernel adds the own keys' low terms whatever their size, so a case with large
    low terms (2^-3 of the values, where a real rounding leaves at most 2^-9) makes their
    path visible above the probabilities' rounding: the replay passes, and the replay with
    the low terms of the own K and V dropped fails."""
    c = build(1, 4, 2, 100, 200, 300, False, lo_scale=2.0 ** -3)
    c2 = dict(c)
    c2["K_lo"] = np.zeros_like(c["K_lo"])
    c2["Vt_lo"] = np.zeros_like(c["Vt_lo"])
    assert within_one_term_p(run_pair(c), c)
    assert not within_one_term_p(run_pair(c2), c)


def test_a_ring_one_slot_short_is_caught():
    """Two slots for the three-slot plan: chunks overwrite K/V still to be read."""
    c = build(1, 4, 2, 100, 200, 300, False)
    try:
        ok = within_one_term_p(run_pair(c, bug="two_slots"), c)
    except AssertionError:
        ok = False
    assert not ok
