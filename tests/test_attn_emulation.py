"""Both attention kernels replayed at the address level on the CPU (tests/tc_emu.py): every
TMA box, shared-memory offset, descriptor start, TMEM column, packed-P layout and output
index as the kernel source computes it, in an order the kernel's barriers allow, against
the oracle's attention at the GPU test's tolerance.

The head-pair kernel (tc_attn2_kernel, validated on a B200) is the control for the
model; the single-head kernel (tc_attn_kernel: two S buffers, one P buffer, a ring of
five half-slots) is replayed the same way before its first run.  Both are replayed with
their load warp running as far ahead as the half-slot plan lets it, and the single-head
kernel with S(j) computed before the softmax of chunk j - 1 reads its own S, so a
half-slot reused too early, an S or P buffer overwritten before it is read, or a wrong
column or offset changes the result.  Planted mistakes in the transcription are caught,
which shows the replay is sharp enough to see them.
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
def build(seed, nq, nkv, n_q, pos0, n_keys, causal):
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
    K_lo[:, pos0 - base:n_keys - base] = T.bf16_bits(rng.standard_normal((nkv, own, D)).astype(np.float32) * 2 ** -9)
    V_lo[:, pos0 - base:n_keys - base] = T.bf16_bits(rng.standard_normal((nkv, own, D)).astype(np.float32) * 2 ** -9)
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


# ---------------------------------------------------------------- tc_attn2_kernel
def run_pair(c, bug=None, force_pair=None):
    """tc_attn2_kernel: a head pair (one head for odd groups) x 128 rows x 128-key chunks,
    a ring of three 32 KB half-slots (a chunk's K, then its V^T, each with its low term
    for own keys), per head one S/P region at 256 hl and O at 256 hl + 128."""
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
    p_lo = 32 if bug == "p_lo_offset" else 64
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
                # the half-slot ring (entry e in half-slot e % 3): per chunk its K parts, then its V parts
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
                        T.mma_ts(tm, sm, o, pp + kk * 8, v + vo, 128, D, j > 0 or kk != 0)
                        T.mma_ts(tm, sm, o, pp + p_lo + kk * 8, v + vo, 128, D, True)
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
                    wh, wl, lpair[hl] = p_words_fma(s, scale, m_used[hl], (le, lo_))
                    tm.t[:, spa:spa + 64] = wh                # P over this row's S: hi, then lo
                    tm.t[:, spa + p_lo:spa + p_lo + 64] = wl

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


# ---------------------------------------------------------------- tc_attn_kernel
def run_single(c, bug=None):
    """tc_attn_kernel: one head x 128 rows x 128-key chunks; the query tile (hi + lo) in
    shared memory by TMA, then a ring of three 32 KB half-slots for K and one of two for V^T
    (with their low terms for own keys); TMEM: S buffers at columns 0 and 128, O at 256,
    P hi at 384 and lo at 448.  The replay runs S as far ahead as the barriers let it: S(j + 2)
    lands in S buffer j & 1 as soon as the softmax has read S(j) -- before it writes P(j)
    where chunk j + 2's K could be loaded by then, else after PV(j) frees half-slots; the
    two load threads fill their rings' half-slots as soon as they are freed.

    bug: "one_s_buffer" -- both S buffers at column 0; "p_lo_offset" -- P lo at 416, half
    over P hi; "q_lo_block" -- the query's lo MMAs read its hi blocks; "v_free_early" -- a
    chunk's V^T half-slots freed before its PV."""
    nq, nkv, n_q, pos0, n_keys, causal = (c[k] for k in ("nq", "nkv", "n_q", "pos0", "n_keys", "causal"))
    m = maps(c)
    group = nq // nkv
    n_splits, cps = splits_single(n_q, nq, n_keys)
    W, BLK = 128, 128 * 128
    QTILE, HSLOT, KSLOTS, VSLOTS = 4 * BLK, 2 * BLK, 3, 2
    HSLOTS = KSLOTS + VSLOTS
    sQ, sHalf = 0, QTILE
    at_s = (lambda b: 0) if bug == "one_s_buffer" else (lambda b: b * 128)
    AT_O, AT_PHI = 256, 384
    AT_PLO = 416 if bug == "p_lo_offset" else 448
    ql_off = 0 if bug == "q_lo_block" else 2 * BLK
    scale = np.float32(1.4426950408889634 / math.sqrt(D))
    out = np.zeros((n_q, nq * D), np.float32)
    out_lo = np.zeros_like(out)
    part_o = np.zeros((n_splits, nq, n_q, D), np.float32)
    part_lse = np.full((n_splits, nq, n_q), NEG, np.float32)
    for qt in range(-(-n_q // 128)):
        for h in range(nq):
            kvh = h // group
            for sp in range(n_splits):
                q_row0 = qt * 128
                rows_here = min(128, n_q - q_row0)
                kv_end = min(n_keys, pos0 + q_row0 + rows_here) if causal else n_keys
                nch_total = -(-kv_end // W)
                c_begin = sp * cps
                nck = min(nch_total, c_begin + cps) - c_begin
                rows = q_row0 + np.arange(128)
                if nck <= 0:
                    continue                                  # empty partial: zeros, lse -inf
                sm, tm = T.Smem(QTILE + HSLOTS * HSLOT), T.Tmem()
                is_cur = lambda j: (c_begin + j) * W >= c["base"]
                for off, mp, x in ((0, "Q", 0), (BLK, "Q", 64), (2 * BLK, "Ql", 0), (3 * BLK, "Ql", 64)):
                    sm.tma_load_3d(sQ + off, m[mp], x, q_row0, h, 64, 128)
                # the rings (K entry e in half-slot e % 3, V^T entry e in 3 + e % 2): per chunk
                # its K parts, then its V^T parts, in the load warp's order
                plan, items, ek, ev = [], [], 0, 0
                for j in range(nck):
                    n = 2 if is_cur(j) else 1
                    ks = [(ek + i) % KSLOTS for i in range(n)]
                    vs = [KSLOTS + (ev + i) % VSLOTS for i in range(n)]
                    items += [(j, "K", i, ks[i]) for i in range(n)] + [(j, "V", i, vs[i]) for i in range(n)]
                    plan.append((ks, vs))
                    ek += n
                    ev += n
                holder = {}                                   # half-slot -> (chunk, operand) held until freed
                queues = {op: [it for it in items if it[1] == op] for op in ("K", "V")}
                loaded = {"K": 0, "V": 0}                     # entries each load thread issued, in order

                def pump():
                    """The two load threads: the next entries of their rings, each once its
                    half-slot's previous use was freed."""
                    for op in ("K", "V"):
                        qq = queues[op]
                        while loaded[op] < len(qq):
                            j, _, i, s_ = qq[loaded[op]]
                            if s_ in holder:
                                break
                            key0 = (c_begin + j) * W
                            krow = key0 if i == 0 else key0 - c["base"]
                            dst = sHalf + s_ * HSLOT
                            if op == "K":
                                mk = "K" if i == 0 else "Kl"
                                sm.tma_load_3d(dst, m[mk], 0, krow, kvh, 64, 128)
                                sm.tma_load_3d(dst + BLK, m[mk], 64, krow, kvh, 64, 128)
                            else:
                                mv = "Vt" if i == 0 else "Vtl"
                                sm.tma_load_3d(dst, m[mv], krow, 0, kvh, 64, 128)
                                sm.tma_load_3d(dst + BLK, m[mv], krow + 64, 0, kvh, 64, 128)
                            holder[s_] = (j, op)
                            loaded[op] += 1

                def ready(j, op):
                    pump()
                    need = [it for it in queues[op] if it[0] == j]
                    assert all(queues[op].index(it) < loaded[op] for it in need), \
                        "the MMA thread would wait for a half-slot the load thread cannot fill"

                def free(j, op):
                    for s_ in (plan[j][0] if op == "K" else plan[j][1]):
                        if holder.get(s_) == (j, op):
                            del holder[s_]
                    pump()

                def issue_s(j):
                    ks = plan[j][0]
                    d = at_s(j & 1)
                    k = sHalf + ks[0] * HSLOT
                    kl = sHalf + ks[1] * HSLOT if len(ks) == 2 else 0
                    for kb in range(2):
                        for kk in range(4):
                            o = kb * BLK + kk * 32
                            T.mma_ss(tm, sm, d, sQ + o, k + o, 128, W, (kb | kk) != 0)
                            T.mma_ss(tm, sm, d, sQ + ql_off + o, k + o, 128, W, True)
                            if len(ks) == 2:
                                T.mma_ss(tm, sm, d, sQ + o, kl + o, 128, W, True)

                def issue_pv(j):
                    vs = plan[j][1]
                    v = sHalf + vs[0] * HSLOT
                    vl = sHalf + vs[1] * HSLOT if len(vs) == 2 else 0
                    for kk in range(8):
                        vo = (kk >> 2) * BLK + (kk & 3) * 32
                        T.mma_ts(tm, sm, AT_O, AT_PHI + kk * 8, v + vo, 128, D, j > 0 or kk != 0)
                        T.mma_ts(tm, sm, AT_O, AT_PLO + kk * 8, v + vo, 128, D, True)
                        if len(vs) == 2:
                            T.mma_ts(tm, sm, AT_O, AT_PHI + kk * 8, vl + vo, 128, D, True)

                m_used = np.full(128, NEG, np.float32)
                lpair = (np.zeros(128, np.float32), np.zeros(128, np.float32))
                key_lim = np.array([c["key_lim"][r] if r < n_q else n_keys for r in rows])

                def read_s(j):
                    sb = at_s(j & 1)
                    return np.concatenate([tm.t[:, sb + cc * 16:sb + cc * 16 + 16] for cc in range(8)], axis=1)

                def softmax(j, raw):
                    nonlocal m_used, lpair
                    s = softmax_chunk_raw(raw, (c_begin + j) * W, key_lim)

                    def rescale(any_w, alpha):
                        if j > 0 and any_w.any():                 # PV(j - 1) has completed
                            blk = tm.f32(AT_O, D)
                            blk[any_w] = (blk[any_w] * alpha[any_w, None]).astype(np.float32)
                    le, lo_ = lpair
                    rmax = (s.max(axis=1) * scale).astype(np.float32)
                    m_new, le = lazy_update(rmax, m_used, le, rescale)
                    _, lo_ = lazy_update(rmax, m_used, lo_, lambda a, b: None)
                    m_used = m_new
                    wh, wl, lpair = p_words_fma(s, scale, m_used, (le, lo_))
                    tm.t[:, AT_PHI:AT_PHI + 64] = wh
                    tm.t[:, AT_PLO:AT_PLO + 64] = wl

                def pv(j):
                    if bug == "v_free_early":
                        free(j, "V")
                    ready(j, "V")
                    issue_pv(j)
                    free(j, "V")

                def s_mmas(j):
                    ready(j, "K")
                    issue_s(j)
                    free(j, "K")

                def k_loaded(j):
                    pump()
                    return all(queues["K"].index(it) < loaded["K"] for it in queues["K"] if it[0] == j)

                pump()
                for j in range(min(nck, 2)):
                    s_mmas(j)
                for j in range(nck):
                    raw = read_s(j)                           # S buffer j & 1 is free again
                    early = j + 2 < nck and k_loaded(j + 2)
                    if early:
                        s_mmas(j + 2)
                    softmax(j, raw)                           # after PV(j - 1): rescale O, write P(j)
                    pv(j)
                    if j + 2 < nck and not early:
                        s_mmas(j + 2)
                lsum = (lpair[0] + lpair[1]).astype(np.float32)
                epilogue(tm, AT_O, lsum, m_used, rows, out, out_lo, part_o, part_lse, sp, h, n_splits, nq, n_q)
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


@pytest.mark.parametrize("force_pair", [None, True, False])
@pytest.mark.parametrize("case", CASES)
def test_validated_kernel_replay_matches_the_oracle(case, force_pair):
    """The control: the head-pair kernel, which passes on a B200, passes in the model too --
    as the host chooses, and in both modes (two heads per CTA, one head per CTA)."""
    c = build(*case)
    assert within(run_pair(c, force_pair=force_pair), oracle(c))


@pytest.mark.parametrize("case", CASES)
def test_single_head_kernel_replay_matches_the_oracle(case):
    c = build(*case)
    assert within(run_single(c), oracle(c))


def test_a_dropped_low_term_is_caught():
    c = build(1, 4, 2, 100, 200, 300, False)
    c2 = dict(c, K_lo=np.zeros_like(c["K_lo"]), Vt_lo=np.zeros_like(c["Vt_lo"]))
    assert within(run_single(c), oracle(c))
    assert not within(run_single(c2), oracle(c))
    assert not within(run_pair(c2), oracle(c))


@pytest.mark.parametrize("bug", ["p_lo_offset", "k_free_after_first_head"])
def test_planted_mistakes_in_the_head_pair_replay_are_caught(bug):
    """A P lo block written half-way into the hi block, or the K half-slots freed after the
    first head's S MMAs (the load warp then fills them before the second head reads K):
    either gives a wrong result or cannot proceed."""
    c = build(6, 4, 2, 100, 200, 300, False)
    assert within(run_pair(c, force_pair=True), oracle(c))
    try:
        ok = within(run_pair(c, bug=bug, force_pair=True), oracle(c))
    except AssertionError:
        ok = False
    assert not ok


@pytest.mark.parametrize("bug,case", [("one_s_buffer", (4, 2, 1, 128, 1536, 1664, False)),
                                      ("p_lo_offset", (5, 2, 1, 300, 0, 300, True)),
                                      ("q_lo_block", (1, 4, 2, 100, 200, 300, False)),
                                      ("v_free_early", (23, 16, 8, 256, 1792, 2048, False))])
def test_planted_mistakes_in_the_single_head_replay_are_caught(bug, case):
    """Both S buffers at the same columns (S(j) lands over S(j - 1) before its softmax reads
    it), P lo half-way into P hi, the query's lo tile read from its hi blocks, or a chunk's
    V^T half-slots freed before its PV: a wrong result or no progress."""
    c = build(*case)
    assert within(run_single(c), oracle(c))
    try:
        ok = within(run_single(c, bug=bug), oracle(c))
    except AssertionError:
        ok = False
    assert not ok


def test_a_ring_one_slot_short_is_caught():
    """Two slots for the three-slot plan: chunks overwrite K/V still to be read."""
    c = build(1, 4, 2, 100, 200, 300, False)
    try:
        ok = within(run_pair(c, bug="two_slots"), oracle(c))
    except AssertionError:
        ok = False
    assert not ok
