"""The attention kernels' tile procedure, replayed on the CPU against the oracle's attention.

Per query row and chunk of keys, the kernels: form S from two (three on the call's own
keys) bf16 products in fp32, scaled to log2 units; raise the row's running maximum only
when the chunk's maximum exceeds it by more than 8 (then rescale O and the row sum);
write P = exp2(S - m) as bf16 hi + lo; add P_hi V + P_lo V (+ P_hi V_lo on own keys) into
O in fp32; and at the end divide by the row sum, or, with the keys split over CTAs, emit
O / l and log2-sum-exp for a merge that weights each split by exp2(lse - max lse).

The replay runs that procedure in float32 (bf16 rounding to nearest even, exp2 in
float64 rounded to float32: the replay checks the procedure, not the device exponential)
at the chunk width of today's kernel (128 keys) and of the redesign (64 keys, a head pair
per CTA), and must meet the GPU attention test's tolerance against the oracle's fp64
attention.  Dropping any one term or step fails it (the mutants below).
"""
import math

import numpy as np
import pytest

from oracle import dg_oracle as O

LAZY = 8.0


def bf16(x):
    """Round float32 values to the nearest bf16 (ties to even), returned as float32."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def f32_mm(a, b):
    return (a.astype(np.float64) @ b.astype(np.float64)).astype(np.float32)


def tile_replay(q_hi, q_lo, K, V, K_lo, V_lo, cur0, key_lim, k_begin, k_end, W, skip=()):
    """One CTA's rows of one head over keys [k_begin, k_end) in chunks of W keys.

    q_hi/q_lo [R][d]; K, V [n][d] bf16 values (cached, and the hi part of own keys);
    K_lo/V_lo [n][d], zero before `cur0`; key_lim [R]: keys >= key_lim[r] are masked.
    Returns (O / l [R][d], lse [R] in log2 units)."""
    R, d = q_hi.shape
    scale_log2 = np.float32(1.0 / math.sqrt(d) / math.log(2.0))
    m_used = np.full(R, -np.inf, np.float32)
    l = np.zeros(R, np.float32)
    o = np.zeros((R, d), np.float32)
    base = (cur0 // W) * W
    for key0 in range(k_begin, k_end, W):
        ks = slice(key0, min(key0 + W, K.shape[0]))
        cur = key0 >= base and K_lo is not None
        s = f32_mm(q_hi, K[ks].T)
        if "q_lo" not in skip:
            s = s + f32_mm(q_lo, K[ks].T)
        if cur and "k_lo" not in skip:
            s = s + f32_mm(q_hi, K_lo[ks].T)
        s = (s * scale_log2).astype(np.float32)
        keys = np.arange(ks.start, ks.stop)
        s = np.where(keys[None, :] < key_lim[:, None], s, -np.inf).astype(np.float32)
        rmax = s.max(axis=1)
        upd = rmax > m_used + LAZY if "lazy" not in skip else rmax > m_used
        with np.errstate(invalid="ignore"):               # -inf - -inf in rows not updated
            alpha = np.where(upd, np.exp2((m_used - rmax).astype(np.float64)).astype(np.float32), np.float32(1.0))
        if "rescale_o" not in skip:
            o = (o * alpha[:, None]).astype(np.float32)
        if "rescale_l" not in skip:
            l = (l * alpha).astype(np.float32)
        m_used = np.where(upd, rmax, m_used).astype(np.float32)
        with np.errstate(invalid="ignore"):
            p = np.where(np.isneginf(s), 0.0, np.exp2((s - m_used[:, None]).astype(np.float64))).astype(np.float32)
        l = (l + p.sum(axis=1, dtype=np.float32)).astype(np.float32)
        p_hi = bf16(p)
        p_lo = bf16(p - p_hi)
        acc = f32_mm(p_hi, V[ks])
        if "p_lo" not in skip:
            acc = acc + f32_mm(p_lo, V[ks])
        if cur and "v_lo" not in skip:
            acc = acc + f32_mm(p_hi, V_lo[ks])
        o = (o + acc).astype(np.float32)
    inv = np.where(l > 0, 1.0 / np.where(l > 0, l, 1.0), 0.0).astype(np.float32)
    with np.errstate(divide="ignore"):
        lse = np.where(l > 0, m_used + np.log2(np.where(l > 0, l, 1.0)), -np.inf).astype(np.float32)
    return (o * inv[:, None]).astype(np.float32), lse


def merge(parts, skip=()):
    """Weight each split's O / l by exp2(lse - max lse); empty splits (lse = -inf) drop out."""
    los = np.stack([lse for _, lse in parts])             # [S][R]
    mx = los.max(axis=0)
    num = np.zeros_like(parts[0][0], dtype=np.float32)
    den = np.zeros(los.shape[1], np.float32)
    for o, lse in parts:
        with np.errstate(invalid="ignore"):
            w = np.where(np.isneginf(lse), 0.0, np.exp2((lse - mx).astype(np.float64))).astype(np.float32)
        if "merge_weight" in skip:
            w = np.where(np.isneginf(lse), 0.0, 1.0).astype(np.float32)
        num = (num + w[:, None] * o).astype(np.float32)
        den = (den + w).astype(np.float32)
    return np.where(den[:, None] > 0, num / np.where(den > 0, den, 1.0)[:, None], 0.0).astype(np.float32)


def case(seed, nq, nkv, n_q, pos0, n_keys, causal, d=128):
    """Seeded query (fp32 as hi + lo), cache K/V in bf16, the call's own K/V (positions
    pos0 .. pos0 + n_q - 1 at or before n_keys) with low parts; same recipe as the GPU
    attention test (unit normal values)."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((nq, n_q, d)).astype(np.float32)
    q_hi = bf16(q)
    q_lo = bf16(q - q_hi)
    K = bf16(rng.standard_normal((nkv, n_keys, d)).astype(np.float32))
    V = bf16(rng.standard_normal((nkv, n_keys, d)).astype(np.float32))
    cur0 = min(pos0, n_keys)
    K_lo = np.zeros_like(K)
    V_lo = np.zeros_like(V)
    K_lo[:, cur0:] = bf16(rng.standard_normal((nkv, n_keys - cur0, d)).astype(np.float32) * 2.0 ** -9)
    V_lo[:, cur0:] = bf16(rng.standard_normal((nkv, n_keys - cur0, d)).astype(np.float32) * 2.0 ** -9)
    pos = pos0 + np.arange(n_q)
    key_lim = np.minimum(pos + 1, n_keys) if causal else np.full(n_q, n_keys)
    return q_hi, q_lo, K, V, K_lo, V_lo, cur0, key_lim


def replay_attention(c, W, n_splits, pair_heads, skip=()):
    """All heads, query tiles of 128 rows, the keys split into n_splits ranges of whole
    chunks; with pair_heads a CTA runs heads 2i and 2i+1 of one KV head over the same
    K/V chunks (the redesign) — the arithmetic per head is unchanged, so the pair only
    fixes which chunks the two heads see together."""
    q_hi, q_lo, K, V, K_lo, V_lo, cur0, key_lim = c
    nq, n_q, d = q_hi.shape
    nkv, n_keys = K.shape[0], K.shape[1]
    g = nq // nkv
    out = np.zeros((nq, n_q, d), np.float32)
    heads = [(h, h + 1) for h in range(0, nq, 2)] if pair_heads and g % 2 == 0 else [(h,) for h in range(nq)]
    for hs in heads:
        kvh = hs[0] // g
        assert all(h // g == kvh for h in hs)
        for r0 in range(0, n_q, 128):
            rs = slice(r0, min(r0 + 128, n_q))
            lim = key_lim[rs]
            kv_end = int(lim.max())
            nch = -(-kv_end // W)
            per = -(-nch // n_splits)
            for h in hs:
                parts = []
                for sp in range(n_splits):
                    c0, c1 = sp * per, min(nch, (sp + 1) * per)
                    if c1 <= c0:
                        parts.append((np.zeros((rs.stop - rs.start, d), np.float32),
                                      np.full(rs.stop - rs.start, -np.inf, np.float32)))
                        continue
                    parts.append(tile_replay(q_hi[h, rs], q_lo[h, rs], K[kvh], V[kvh], K_lo[kvh], V_lo[kvh], cur0,
                                             lim, c0 * W, min(c1 * W, kv_end), W, skip))
                out[h, rs] = parts[0][0] if n_splits == 1 else merge(parts, skip)
    return out


def oracle_attention(c):
    q_hi, q_lo, K, V, K_lo, V_lo, cur0, key_lim = c
    n_q, n_keys = q_hi.shape[1], K.shape[1]
    allowed = np.arange(n_keys)[None, :] < key_lim[:, None]
    q = q_hi.astype(np.float64) + q_lo
    return O.attention(q, K.astype(np.float64) + K_lo, V.astype(np.float64) + V_lo, allowed)


def within_gpu_tolerance(got, ref):
    rms = math.sqrt(float(np.mean(ref * ref)))
    return bool((np.abs(got - ref) <= 1e-4 * np.abs(ref) + 1e-4 * rms).all())


CASES = [
    # seed, nq, nkv, n_q, pos0, n_keys, causal
    (1, 4, 2, 100, 200, 300, False),     # canvas rows over a ragged prefix + canvas
    (2, 4, 1, 200, 50, 250, True),       # prefill rows, causal, ragged
    (3, 2, 2, 64, 1200, 1264, False),    # long keys, GQA group 1 (no head pair)
    (4, 8, 2, 256, 640, 896, False),     # group 4: two head pairs per KV head
    (5, 2, 1, 300, 0, 300, True),        # prefill from an empty cache
]


@pytest.mark.parametrize("W", [128, 64])
@pytest.mark.parametrize("n_splits", [1, 3])
@pytest.mark.parametrize("cs", CASES)
def test_tile_procedure_meets_the_gpu_tolerance(cs, W, n_splits):
    c = case(*cs)
    ref = oracle_attention(c)
    got = replay_attention(c, W, n_splits, pair_heads=(W == 64))
    assert within_gpu_tolerance(got, ref), np.abs(got - ref).max()


def test_scores_far_apart_exercise_the_lazy_rescale():
    """Rows whose later chunks hold much larger scores: the maximum is raised mid-row (so O
    and l are rescaled) and the result still meets the tolerance."""
    c = list(case(7, 2, 1, 128, 512, 640, False))
    K = c[2].copy()
    K[0, 400:460] *= 4.0                                   # keys in the 7th chunk of 64 stand out
    c[2] = bf16(K)
    ref = oracle_attention(tuple(c))
    for W in (64, 128):
        assert within_gpu_tolerance(replay_attention(tuple(c), W, 1, False), ref)
        for step in ("rescale_o", "rescale_l"):
            assert not within_gpu_tolerance(replay_attention(tuple(c), W, 1, False, skip=(step,)), ref)


@pytest.mark.parametrize("step", ["q_lo", "k_lo", "p_lo", "v_lo", "merge_weight"])
def test_each_term_is_needed(step):
    """Every term and step of the procedure is visible at this tolerance: leaving one out
    fails it (the canvas case with splits, so the merge and the own-key terms are live;
    the rescales are checked where the maximum is raised mid-row, above)."""
    c = case(11, 4, 2, 100, 200, 300, False)
    ref = oracle_attention(c)
    assert within_gpu_tolerance(replay_attention(c, 64, 3, True), ref)
    assert not within_gpu_tolerance(replay_attention(c, 64, 3, True, skip=(step,)), ref)


def test_bf16_rounding_helper():
    """Ties to even and the round-trip of representable values."""
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 3.0e38], np.float32)
    want = np.array([1.0, 1.0, 1.0 + 4 * 2 ** -8, 1.0, -2.5, np.float32(3.0e38)], np.float64)
    got = bf16(x).astype(np.float64)
    assert got[:5].tolist() == want[:5].tolist()
    assert abs(got[5] - 3.0e38) / 3.0e38 < 2 ** -8
