"""The fused vocabulary/update path's reductions, replayed on the CPU against the oracle's
canvas update.

The kernel's epilogue reduces, per token, each 128-id tile in four warps of 32 ids:
a butterfly (max, first argmax) with ties to the lower id, the same for the candidate
that skips an excluded id, and a butterfly sum of exp(l - warp max); the four warp
records are merged in id order, and a row kernel merges a token's tile records (lane l
takes tiles l, l + 32, ..., then a butterfly across lanes).  The selection then reads
one record per token: confidence 1 / s (re-noising update) or exp(m2 - m) / s (masked).
Replaying these steps (exp in float64: the replay checks the reduction's logic, not the
device exponential) must give the oracle's argmax / candidate ids exactly and its
confidences to rounding, ties and an excluded maximum included.
"""
import math

import numpy as np
import pytest

from oracle import dg_oracle as O

NEG = -math.inf
BIG = 0x7FFFFFFF


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


def butterfly_argmax(vals, ids):
    vals, ids = list(vals), list(ids)
    o = 16
    while o:
        nv, ni = vals[:], ids[:]
        for ln in range(32):
            om, oa = vals[ln ^ o], ids[ln ^ o]
            if om > vals[ln] or (om == vals[ln] and oa < ids[ln]):
                nv[ln], ni[ln] = om, oa
        vals, ids = nv, ni
        o >>= 1
    assert len(set(zip(vals, ids))) == 1   # every lane holds the same result
    return vals[0], ids[0]


def butterfly_sum(e):
    e = list(e)
    o = 16
    while o:
        e = [e[ln] + e[ln ^ o] for ln in range(32)]
        o >>= 1
    return e[0]


def tile_record(lg_row, t, excl):
    """One token's record over tile t (128 ids) as the epilogue forms it."""
    recs = []
    for w in range(4):
        ids = [t * 128 + w * 32 + ln for ln in range(32)]
        v = [float(lg_row[i]) for i in ids]
        wm, wa = butterfly_argmax(v, ids)
        if excl >= 0:
            cm, ca = butterfly_argmax([NEG if i == excl else x for i, x in zip(ids, v)],
                                      [BIG if i == excl else i for i in ids])
        else:
            cm, ca = wm, wa
        s = butterfly_sum([0.0 if x == NEG else math.exp(x - wm) for x in v])
        recs.append((wm, s, ca, cm))
    m, s, a, m2 = recs[0]
    for (xm, xs, xa, xm2) in recs[1:]:
        m, s = ms_merge(m, s, xm, xs)
        m2, a = cand_merge(m2, a, xm2, xa)
    return m, s, a, m2


def row_record(lg_row, excl):
    tiles = len(lg_row) // 128
    recs = [tile_record(lg_row, t, excl) for t in range(tiles)]
    lanes = []
    for ln in range(32):
        m, s, m2, a = NEG, 0.0, NEG, BIG
        for t in range(ln, tiles, 32):
            xm, xs, xa, xm2 = recs[t]
            m, s = ms_merge(m, s, xm, xs)
            m2, a = cand_merge(m2, a, xm2, xa)
        lanes.append((m, s, m2, a))
    o = 16
    while o:
        new = []
        for ln in range(32):
            m, s, m2, a = lanes[ln]
            om, os, om2, oa = lanes[ln ^ o]
            m, s = ms_merge(m, s, om, os)
            m2, a = cand_merge(m2, a, om2, oa)
            new.append((m, s, m2, a))
        lanes = new
        o >>= 1
    return lanes[0]


def _logits(rng, C, V):
    lg = (rng.standard_normal((C, V)) * 2.0).astype(np.float32).astype(np.float64)
    # ties across lanes, warps and tiles, and dominant entries
    lg[0, 5] = lg[0, V // 2 + 44] = lg[0, V - 24] = 9.0  # three-way tie for the maximum: id 5 wins
    lg[1, V // 2 + 2] = lg[1, V // 2 + 3] = 7.5          # tie inside one warp
    lg[2, 40] = lg[2, 80] = 8.25                         # tie across warps of a tile
    lg[3, 17] = 30.0                                     # one dominant logit: confidence 1
    return lg


@pytest.mark.parametrize("V", [128, 1024, 4096 + 128])
def test_fused_records_give_the_oracle_update(V):
    rng = np.random.default_rng(V)
    C = 6
    lg = _logits(rng, C, V)
    want = O.canvas_update(lg, 0, 1, 0)
    for i in range(C):
        m, s, m2, a = row_record(lg[i], -1)
        assert a == want["argmax"][i]
        assert m2 == m
        assert abs(1.0 / s - want["conf"][i]) <= 1e-12 * want["conf"][i] + 1e-15
    assert row_record(lg[0], -1)[3] == 5


@pytest.mark.parametrize("V", [256, 2048])
def test_fused_records_give_the_oracle_masked_update(V):
    rng = np.random.default_rng(V + 1)
    C = 6
    lg = _logits(rng, C, V)
    mask_id = V - 3
    lg[4, mask_id] = 50.0                                # the excluded id holds the maximum
    canvas = np.full(C, mask_id)
    want = O.canvas_update_masked(lg, canvas, 0, mask_id)
    for i in range(C):
        m, s, m2, a = row_record(lg[i], mask_id)
        assert a == want["argmax"][i] and a != mask_id
        conf = math.exp(m2 - m) / s
        assert abs(conf - want["conf"][i]) <= 1e-12 * want["conf"][i] + 1e-300
    m, s, m2, a = row_record(lg[4], mask_id)
    assert m == 50.0 and m2 < 50.0 and a == want["argmax"][4]
