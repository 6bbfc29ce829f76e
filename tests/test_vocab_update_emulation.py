"""The fused vocabulary/update kernel (tc_vocab_update_kernel, then upd_merge_rows_kernel)
replayed at the address level on the CPU (tests/tc_emu.py), against the oracle's update.

Transcribed from the kernel source: the persistent walk over (128-id tile, token chunk)
tiles, id tile first, with its k-block rotation, the stage layout (weight tile, then token boxes of 64
and 16 rows), the MMAs into one of two accumulator buffers, and the statistics epilogue:
warp lg's lane holds id m 128 + 32 lg + lane, each group of 32 token columns is reduced
by transposed shuffles (max with the first argmax, the sum of exp(l - column max), and
where the excluded id is one of the warp's, the candidate skipping it), lane L ends with
column L's record, and warp 0 merges the four warps' records in id order into
part[token][tile].  The row merge then reduces a token's tile
records in lane order and a butterfly.  The records must give the oracle's argmax /
candidate exactly and its confidence to rounding; each epilogue runs as late as its
accumulator buffer allows.  The butterflies use float64 exp (the device exponential is
not the object here).
"""
from __future__ import annotations

import math

import numpy as np
import pytest

import tc_emu as T
from oracle import dg_oracle as O

BM, BK = 128, 64
BIG = 0x7FFFFFFF
NEG = -math.inf


def ms_merge(m, s, om, os):
    if om == NEG:
        return m, s
    if m == NEG:
        return om, os
    if om > m:
        return om, s * math.exp(m - om) + os
    if om < m:
        return m, s + os * math.exp(om - m)
    return m, s + os


def cand_merge(m2, a, om2, oa):
    return (om2, oa) if (om2 > m2 or (om2 == m2 and oa < a)) else (m2, a)


def tr_argmax(m, a, bug=None):
    """vu_tr_argmax over the warp: m, a [lane][32 columns] -> (max, first argmax) of column L
    in lane L.  At the stage with offset o a lane keeps the upper half of its columns when
    bit o of its lane is set, and merges the partner's values for that half into it."""
    m, a = m.astype(np.float64), a.astype(np.int64)
    o = 16
    while o:
        lanes = np.arange(32)
        up = (lanes & o) != 0
        if bug == "kept_half":
            up = ~up
        km = np.where(up[:, None], m[:, o:2 * o], m[:, :o])
        ka = np.where(up[:, None], a[:, o:2 * o], a[:, :o])
        sm = np.where(up[:, None], m[:, :o], m[:, o:2 * o])
        sa = np.where(up[:, None], a[:, :o], a[:, o:2 * o])
        rm, ra = sm[lanes ^ o], sa[lanes ^ o]
        take = (rm > km) | ((rm == km) & (ra < ka))
        m = np.where(take, rm, km)
        a = np.where(take, ra, ka)
        o >>= 1
    return m[:, 0], a[:, 0]


def tr_sum(e):
    """vu_tr_sum: e [lane][32 columns] -> column L's sum in lane L (same exchange pattern)."""
    o = 16
    while o:
        lanes = np.arange(32)
        up = (lanes & o) != 0
        ke = np.where(up[:, None], e[:, o:2 * o], e[:, :o])
        se = np.where(up[:, None], e[:, :o], e[:, o:2 * o])
        e = ke + se[lanes ^ o]
        o >>= 1
    return e[:, 0]


def warp_argmax(v, ids):
    v, ids = list(v), list(ids)
    o = 16
    while o:
        nv, ni = v[:], ids[:]
        for ln in range(32):
            if v[ln ^ o] > v[ln] or (v[ln ^ o] == v[ln] and ids[ln ^ o] < ids[ln]):
                nv[ln], ni[ln] = v[ln ^ o], ids[ln ^ o]
        v, ids = nv, ni
        o >>= 1
    return v[0], ids[0]


def run_vocab_update(Wout, X, V, excl, n_max, smem_budget=200 * 1024, grid=5, bug=None):
    """Wout bf16 bits [V][K]; X bf16 bits [C][K] (the normed state, one term).  Returns the
    merged record (m, s, a, m2) per token."""
    C, K = X.shape
    a_bytes, b_bytes = BM * BK * 2, n_max * 128
    stage_bytes = a_bytes + b_bytes
    stages = min(smem_budget // stage_bytes, 8)
    acc_cols = n_max
    nkb = K // BK
    m_tiles = -(-V // BM)
    chunks = -(-C // n_max)
    n_tiles = chunks * m_tiles
    part = [[None] * m_tiles for _ in range(C)]
    for cta in range(min(grid, n_tiles)):
        sm = T.Smem(stages * stage_bytes)
        tm = T.Tmem(max(32, 1 << (2 * acc_cols - 1).bit_length()))
        tiles = list(range(cta, n_tiles, grid))
        its = [(t, kb) for t in tiles for kb in range(nkb)]
        loaded = mma_done = 0
        pending = []

        def geom(t):
            m, row0 = t // chunks, (t % chunks) * n_max            # id tile first, then token chunk
            rows = min(n_max, C - row0)
            return m, row0, rows, (rows + 15) & ~15

        def load(it):
            t, kb = its[it]
            m, row0, rows, n_pad = geom(t)
            sa = (it % stages) * stage_bytes
            sb = sa + a_bytes
            kx = ((kb + t) % nkb) * BK
            sm.tma_load(sa, Wout, (kx, m * BM), (64, 128), 128)
            r = 0
            while r + 64 <= n_pad:
                sm.tma_load(sb + r * 128, X, (kx, row0 + r), (64, 64), 128)
                r += 64
            while r < n_pad:
                sm.tma_load(sb + r * 128, X, (kx, row0 + r), (64, 16), 128)
                r += 16

        def epilogue(j, t):
            m, row0, rows, n_pad = geom(t)
            d0 = (j & 1) * acc_cols
            for c0 in range(0, n_pad, 32):
                width = 32 if c0 + 16 < n_pad else 16      # the last group may hold 16 columns
                red = [[None] * 32 for _ in range(4)]
                for lg in range(4):
                    ids = np.array([m * BM + lg * 32 + ln for ln in range(32)])
                    valid = ids < V
                    vals = np.full((32, 32), NEG)              # [lane][column]
                    vals[:, :width] = tm.f32(d0 + c0, width)[lg * 32:lg * 32 + 32].astype(np.float64)
                    vals[~valid] = NEG
                    aid = np.where(valid, ids, BIG)[:, None].repeat(32, axis=1)
                    col_m, col_a = tr_argmax(vals.copy(), aid.copy(), bug)
                    with np.errstate(invalid="ignore"):             # -inf - -inf where a column is empty
                        e = np.where(vals == NEG, 0.0, np.exp(vals - col_m[None, :]))  # column q's max from lane q
                    col_s = tr_sum(e)
                    cand_m, cand_a = col_m, col_a
                    if excl >= 0 and excl in ids:
                        ev = np.where((ids == excl)[:, None], NEG, vals)
                        ea = np.where(((ids == excl) | ~valid)[:, None], BIG, aid)
                        cand_m, cand_a = tr_argmax(ev, ea, bug)
                    for ln in range(32):
                        red[lg][ln] = (col_m[ln], col_s[ln], cand_a[ln], cand_m[ln])
                for ln in range(32):
                    if c0 + ln < rows:
                        mm, ss, aa, m2 = red[0][ln]
                        for w2 in range(1, 4):
                            xm, xs, xa, xm2 = red[w2][ln]
                            mm, ss = ms_merge(mm, ss, xm, xs)
                            m2, aa = cand_merge(m2, aa, xm2, xa)
                        tile = m if bug != "record_tile" else 0
                        part[row0 + c0 + ln][tile] = (mm, ss, aa, m2)

        for it in range(len(its)):
            while loaded < len(its) and loaded < mma_done + stages:
                load(loaded)
                loaded += 1
            t, kb = its[it]
            j = tiles.index(t)
            if kb == 0:
                while pending and pending[0][0] <= j - 2:
                    epilogue(*pending.pop(0))
            m, row0, rows, n_pad = geom(t)
            d0 = (j & 1) * acc_cols if bug != "one_acc" else 0
            sa = (it % stages) * stage_bytes
            for kk in range(BK // 16):
                T.mma_ss(tm, sm, d0, sa + kk * 32, sa + a_bytes + kk * 32, BM, n_pad, kb != 0 or kk != 0)
            mma_done += 1
            if kb == nkb - 1:
                pending.append((j, t))
        while pending:
            epilogue(*pending.pop(0))
    # the row merge: thread t of 128 takes tiles t, t + 128, ...; a butterfly within each
    # warp; then the four warps' records in warp order
    out = []
    for row in range(C):
        thr = []
        for t_ in range(128):
            mm, ss, m2, aa = NEG, 0.0, NEG, BIG
            for t in range(t_, m_tiles, 128):
                xm, xs, xa, xm2 = part[row][t]
                mm, ss = ms_merge(mm, ss, xm, xs)
                m2, aa = cand_merge(m2, aa, xm2, xa)
            thr.append((mm, ss, m2, aa))
        warps = []
        for w in range(4):
            lanes = thr[32 * w:32 * w + 32]
            o = 16
            while o:
                new = []
                for ln in range(32):
                    mm, ss, m2, aa = lanes[ln]
                    om, os, om2, oa = lanes[ln ^ o]
                    mm, ss = ms_merge(mm, ss, om, os)
                    m2, aa = cand_merge(m2, aa, om2, oa)
                    new.append((mm, ss, m2, aa))
                lanes = new
                o >>= 1
            warps.append(lanes[0])
        mm, ss, m2, aa = warps[0]
        for w in range(1, 4):
            om, os, om2, oa = warps[w]
            mm, ss = ms_merge(mm, ss, om, os)
            m2, aa = cand_merge(m2, aa, om2, oa)
        out.append((mm, ss, aa, m2))
    return out


def inputs(seed, C, V, K):
    rng = np.random.default_rng(seed)
    W = T.bf16_bits((rng.standard_normal((V, K)) * 0.05).astype(np.float32))
    X = T.bf16_bits(rng.standard_normal((C, K)).astype(np.float32))
    lg = T.bf16_value(X).astype(np.float64) @ T.bf16_value(W).astype(np.float64).T
    return W, X, lg


@pytest.mark.parametrize("C,V,K", [(20, 384, 128), (70, 300, 192), (33, 1024, 64)])
def test_fused_records_replay_gives_the_oracle_update(C, V, K):
    W, X, lg = inputs(C + V, C, V, K)
    n_max = ((C + 15) & ~15) if C < 256 else 256
    if C == 70:
        n_max = 32                                     # several token chunks per id tile
    rec = run_vocab_update(W, X, V, -1, n_max)
    want = O.canvas_update(lg, 0, 1, 0)
    for i, (m, s, a, m2) in enumerate(rec):
        assert a == want["argmax"][i] and m2 == m
        assert abs(1.0 / s - want["conf"][i]) <= 1e-5 * want["conf"][i]


def test_fused_masked_records_replay_gives_the_oracle_update():
    C, V, K = 24, 256, 128
    W, X, _ = inputs(5, C, V, K)
    mask_id = V - 3
    # the mask id's row points along token 0: its logit there is the row maximum, so the
    # candidate must skip it
    W[mask_id] = T.bf16_bits((0.2 * T.bf16_value(X[0])).astype(np.float32))
    lg = T.bf16_value(X).astype(np.float64) @ T.bf16_value(W).astype(np.float64).T
    assert lg[0].argmax() == mask_id
    rec = run_vocab_update(W, X, V, mask_id, 32)
    want = O.canvas_update_masked(lg, np.full(C, mask_id), 0, mask_id)
    for i, (m, s, a, m2) in enumerate(rec):
        assert a == want["argmax"][i] and a != mask_id
        assert abs(math.exp(m2 - m) / s - want["conf"][i]) <= 1e-5 * want["conf"][i]
    assert rec[0][0] > rec[0][3]                      # token 0: its maximum is the excluded id


@pytest.mark.parametrize("bug", ["record_tile", "one_acc", "kept_half"])
def test_planted_mistakes_in_the_fused_replay_are_caught(bug):
    """Every tile's record written to tile 0, one accumulator buffer for two tiles in
    flight, or the transposed reduction keeping the wrong half (column L's record lands in
    another lane): the update differs from the oracle's (or records are missing)."""
    C, V, K = 40, 512, 128
    W, X, lg = inputs(3, C, V, K)
    want = O.canvas_update(lg, 0, 1, 0)
    try:
        rec = run_vocab_update(W, X, V, -1, 16, grid=2, bug=bug)
        ok = all(a == want["argmax"][i] and abs(1.0 / s - want["conf"][i]) <= 1e-5 * want["conf"][i]
                 for i, (m, s, a, m2) in enumerate(rec))
    except (TypeError, AssertionError):
        ok = False
    assert not ok
