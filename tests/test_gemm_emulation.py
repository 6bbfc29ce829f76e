"""The bf16 GEMM (tc_gemm_kernel, validated on a B200) replayed at the address level on the
CPU (tests/tc_emu.py): the control for the GEMM half of the hardware model, and a CPU
check for later changes to the kernel.

Transcribed from the kernel source: the persistent tile walk (grouped: item-major;
dense: token chunk, then split, then weight tile; dealt in serpentine rounds with the
partial weight tiles last), the k-block rotation within a split,
the k-block ring (each k-block's buffer: one or two weight tiles, then one or two token
terms of the tile's padded rows, at the next offset of the ring or at 0 when it would run
past the end; a buffer is loaded only once no k-block in flight overlaps it),
the MMAs into one of two accumulator buffers (a second weight matrix n_max columns on),
and the epilogue's indices: fp32 stores into the split's slab, or SwiGLU with bf16 hi /
lo.  The producer runs as far ahead as the ring allows and each epilogue as late as
its accumulator buffer allows.  Results are compared with fp64 products of the same bf16
values.
"""
from __future__ import annotations

import numpy as np
import pytest

import tc_emu as T
from oracle import dg_oracle as O

BM, BK = 128, 64


def tile_walk(cta, grid, n_tiles, m_tiles, rows_a, tile_rows=BM):
    """TileWalk: rounds of `grid` tiles, every other round in reverse CTA order, over a list
    with the whole weight tiles first and each work item's partial last weight tile (when
    rows_a is not a multiple of the tile's weight rows) at the end."""
    partial = m_tiles > 1 and rows_a % tile_rows != 0
    full = n_tiles - n_tiles // m_tiles if partial else n_tiles

    def order(k):
        if full == n_tiles:
            return k
        if k < full:
            return (k // (m_tiles - 1)) * m_tiles + k % (m_tiles - 1)
        return (k - full) * m_tiles + (m_tiles - 1)
    out, r = [], 0
    while r * grid < n_tiles:
        c = grid - 1 - cta if r & 1 else cta
        k = r * grid + c
        r += 1
        if k < n_tiles:
            out.append(order(k))
    return out


def run_gemm(W, X_hi, X_lo, rows_a, K, ld_out, items=None, n_max=64, k_splits=1, W2=None, split_stride=0,
             smem_budget=200 * 1024, grid=5, bug=None, m_pair=None):
    """W / W2: bf16 bits [G][rows][K]; X_hi / X_lo: bf16 bits [n][K]; items: (group, row0,
    rows) or None (dense).  m_pair: tiles of two consecutive 128-row weight tiles (default:
    as the host chooses, fp32-store GEMMs of at least 256 weight rows, dense or grouped).  Returns the
    output array as the kernel writes it."""
    terms = 2 if X_lo is not None else 1
    if m_pair is None:
        m_pair = W2 is None and rows_a >= 256
    n_a = 2 if (W2 is not None or m_pair) else 1
    tile_rows = 2 * BM if m_pair else BM
    a_bytes = BM * BK * 2
    acc_cols = n_max * n_a
    nbuf = 2 if 2 * acc_cols <= 512 else 1
    tmem_cols = 32
    while tmem_cols < nbuf * acc_cols:
        tmem_cols <<= 1
    assert tmem_cols <= 512
    nkb = K // BK // k_splits
    m_tiles = -(-rows_a // tile_rows)
    n_tokens = X_hi.shape[0]
    dense = items is None
    chunks = -(-n_tokens // n_max)
    n_items = chunks * k_splits if dense else len(items)
    n_tiles = n_items * m_tiles
    swiglu = W2 is not None
    if swiglu:
        out = np.full((n_tokens, ld_out), np.nan)
        out_lo = np.zeros((n_tokens, ld_out))
    else:
        out = np.full(k_splits * split_stride if k_splits > 1 else n_tokens * ld_out, np.nan)
        out_lo = None

    def tile_of(t):
        item, m = t // m_tiles, t % m_tiles
        if dense:
            chunk, split = item // k_splits, item % k_splits
            row0 = chunk * n_max
            return 0, row0, min(n_max, n_tokens - row0), split, m
        g, row0, rows = items[item]
        return g, row0, rows, 0, m

    def kb_bytes(t):
        n_pad = (tile_of(t)[2] + 15) & ~15
        return n_a * a_bytes + terms * n_pad * 128

    for cta in range(min(grid, n_tiles)):
        sm, tm = T.Smem(smem_budget), T.Tmem(tmem_cols)
        sm.b[:] = 0xFF      # shared memory starts as NaN bf16 pairs: rows no load wrote must stay unused
        tiles = tile_walk(cta, grid, n_tiles, m_tiles, rows_a, tile_rows)
        its = [(t, kb) for t in tiles for kb in range(nkb)]
        offs, foots, head = [], [], 0         # KbRing: each k-block's offset, size and footprint
        for t, _ in its:
            n = kb_bytes(t)
            if head + n > smem_budget:
                foots.append(smem_budget - head + n)
                off, head = 0, n
            else:
                foots.append(n)
                off, head = head, head + n
            offs.append((off, n))
        loaded = mma_done = 0
        pending = []

        def can_load(it):
            """The buffer's footprint fits beside those of the k-blocks in flight (loaded, not
            yet consumed), and fewer than 16 are in flight."""
            if it == mma_done:                 # nothing in flight: the producer waits for nothing
                return True
            if it - mma_done >= 16:
                return False
            return sum(foots[mma_done:it + 1]) <= smem_budget

        def load(it):
            t, kb = its[it]
            g, row0, rows, split, m = tile_of(t)
            n_pad = (rows + 15) & ~15
            sa = offs[it][0]
            sb = sa + n_a * a_bytes
            kx = (split * nkb + (kb + t) % nkb) * BK
            sm.tma_load(sa, W, (kx, m * tile_rows, g), (64, 128, 1), 128)
            if W2 is not None:
                sm.tma_load(sa + a_bytes, W2, (kx, m * tile_rows, g), (64, 128, 1), 128)
            if m_pair:
                sm.tma_load(sa + a_bytes, W, (kx, m * tile_rows + BM, g), (64, 128, 1), 128)
            r = 0
            lo_off = n_pad * 128 if bug != "lo_offset" else n_pad * 64
            while r + 64 <= n_pad:
                sm.tma_load(sb + r * 128, X_hi, (kx, row0 + r), (64, 64), 128)
                if terms == 2:
                    sm.tma_load(sb + lo_off + r * 128, X_lo, (kx, row0 + r), (64, 64), 128)
                r += 64
            while r < n_pad:
                sm.tma_load(sb + r * 128, X_hi, (kx, row0 + r), (64, 16), 128)
                if terms == 2:
                    sm.tma_load(sb + lo_off + r * 128, X_lo, (kx, row0 + r), (64, 16), 128)
                r += 16

        def epilogue(j, t):
            g, row0, rows, split, m = tile_of(t)
            for half in range(2 if m_pair else 1):
                epilogue_half(j, t, half)

        def epilogue_half(j, t, half):
            g, row0, rows, split, m = tile_of(t)
            n_pad = (rows + 15) & ~15
            fuse = terms == 2 and 2 * n_pad <= n_max and bug != "no_fuse_add"
            d0 = (j % nbuf) * acc_cols + half * n_max
            f = m * tile_rows + half * BM + np.arange(BM)
            ok = f < rows_a

            def col_sum(c):
                v = tm.f32(c, 1)[:, 0]
                if fuse:                                # the lo term's column, n_pad further on
                    v = (v + tm.f32(c + n_pad, 1)[:, 0]).astype(np.float32)
                return v.astype(np.float64)
            for col in range(rows):
                a = col_sum(d0 + col)
                if swiglu:
                    b = col_sum(d0 + n_max + col)
                    hv = (a / (1.0 + np.exp(-a)) * b).astype(np.float32)
                    hi = T.bf16_value(T.bf16_bits(hv)).astype(np.float64)
                    out[row0 + col, f[ok]] = hi[ok]
                    out_lo[row0 + col, f[ok]] = T.bf16_value(T.bf16_bits((hv - hi).astype(np.float32)))[ok]
                else:
                    slab = split * split_stride if bug != "no_slab" else 0
                    out[slab + (row0 + col) * ld_out + f[ok]] = a[ok]

        for it in range(len(its)):
            while loaded < len(its) and can_load(loaded):
                load(loaded)
                loaded += 1
            assert loaded > it, "the MMA warp would wait for a k-block the producer cannot load"
            t, kb = its[it]
            j = tiles.index(t)
            if kb == 0:
                while pending and pending[0][0] <= j - nbuf:
                    epilogue(*pending.pop(0))
            g, row0, rows, split, m = tile_of(t)
            n_pad = (rows + 15) & ~15
            d0 = (j % nbuf) * acc_cols
            d1 = d0 + (n_max if bug != "d1" else acc_cols // 4)
            sa = offs[it][0]
            sb = sa + n_a * a_bytes
            # both token terms in one MMA of N = 2 n_pad where they fit the accumulator twice
            fuse = terms == 2 and 2 * n_pad <= n_max
            nn = 2 * n_pad if fuse else n_pad
            for kk in range(BK // 16):
                acc = kb != 0 or kk != 0
                T.mma_ss(tm, sm, d0, sa + kk * 32, sb + kk * 32, BM, nn, acc)
                if terms == 2 and not fuse:
                    T.mma_ss(tm, sm, d0, sa + kk * 32, sb + n_pad * 128 + kk * 32, BM, n_pad, True)
                if n_a == 2:
                    T.mma_ss(tm, sm, d1, sa + a_bytes + kk * 32, sb + kk * 32, BM, nn, acc)
                    if terms == 2 and not fuse:
                        T.mma_ss(tm, sm, d1, sa + a_bytes + kk * 32, sb + n_pad * 128 + kk * 32, BM, n_pad, True)
            mma_done += 1
            if kb == nkb - 1:
                pending.append((j, t))
        while pending:
            epilogue(*pending.pop(0))
    return out, out_lo


def bf16_pair(rng, n, K):
    x = rng.standard_normal((n, K)).astype(np.float32)
    hi = T.bf16_bits(x)
    lo = T.bf16_bits((x - T.bf16_value(hi)).astype(np.float32))
    return T.bf16_value(hi).astype(np.float64) + T.bf16_value(lo), hi, lo


def weights(rng, G, rows, K):
    w = T.bf16_bits((rng.standard_normal((G, rows, K)) * 0.05).astype(np.float32))
    return w, T.bf16_value(w).astype(np.float64)


def test_dense_two_term_split_k_gemm_replay():
    """The QKV / output projection shape: dense tokens in chunks, two terms, split-K slabs
    (their sum is the product)."""
    rng = np.random.default_rng(1)
    n, rows, K, ks = 150, 320, 512, 2
    x, hi, lo = bf16_pair(rng, n, K)
    W, w = weights(rng, 1, rows, K)
    out, _ = run_gemm(W, hi, lo, rows, K, rows, n_max=128, k_splits=ks, split_stride=n * rows)
    got = out.reshape(ks, n, rows).sum(axis=0)
    ref = x @ w[0].T
    assert np.abs(got - ref).max() / np.abs(ref).max() < 2e-6


def test_grouped_gate_up_swiglu_replay():
    rng = np.random.default_rng(2)
    counts, F, K = [20, 0, 150, 7], 192, 256
    off = np.concatenate([[0], np.cumsum(counts)]).astype(int)
    items = [(e, r0, min(128, off[e + 1] - r0)) for e in range(4) for r0 in range(off[e], off[e + 1], 128)]
    x, hi, lo = bf16_pair(rng, int(off[-1]), K)
    Wg, wg = weights(rng, 4, F, K)
    Wu, wu = weights(rng, 4, F, K)
    out, out_lo = run_gemm(Wg, hi, lo, F, K, F, items=items, n_max=128, W2=Wu)
    got = out + out_lo
    for e in range(4):
        xe = x[off[e]:off[e + 1]]
        if len(xe):
            ref = O.silu(xe @ wg[e].T) * (xe @ wu[e].T)
            assert np.abs(got[off[e]:off[e + 1]] - ref).max() / np.abs(ref).max() < 1e-4, e


@pytest.mark.parametrize("smem_budget", [200 * 1024, 96 * 1024, 64 * 1024])
def test_grouped_ring_of_mixed_tiles_replay(smem_budget):
    """Expert tiles of 16 to 128 token rows in one launch: k-block buffers of 36 to 64 KB
    wrap around a ring that holds five, two or one of them, and a buffer is loaded only
    once the k-blocks it overlaps are consumed."""
    rng = np.random.default_rng(12)
    counts, F, K = [16, 3, 128, 40, 0, 77, 16, 9], 256, 384
    E = len(counts)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(int)
    items = [(e, r0, min(128, off[e + 1] - r0)) for e in range(E) for r0 in range(off[e], off[e + 1], 128)]
    x, hi, lo = bf16_pair(rng, int(off[-1]), K)
    Wg, wg = weights(rng, E, F, K)
    Wu, wu = weights(rng, E, F, K)
    out, out_lo = run_gemm(Wg, hi, lo, F, K, F, items=items, n_max=128, W2=Wu, smem_budget=smem_budget, grid=3)
    got = out + out_lo
    for e in range(E):
        xe = x[off[e]:off[e + 1]]
        if len(xe):
            ref = O.silu(xe @ wg[e].T) * (xe @ wu[e].T)
            assert np.abs(got[off[e]:off[e + 1]] - ref).max() / np.abs(ref).max() < 1e-4, e


def test_vocab_single_term_replay():
    """The vocabulary projection shape: one term, all tokens in one chunk of up to 256."""
    rng = np.random.default_rng(3)
    n, V, K = 200, 384, 128
    _, hi, _ = bf16_pair(rng, n, K)
    x = T.bf16_value(hi).astype(np.float64)
    W, w = weights(rng, 1, V, K)
    out, _ = run_gemm(W, hi, None, V, K, V, n_max=208)
    ref = x @ w[0].T
    assert np.abs(out.reshape(n, V) - ref).max() / np.abs(ref).max() < 2e-6


@pytest.mark.parametrize("bug", ["d1", "no_slab", "lo_offset", "no_fuse_add"])
def test_planted_mistakes_in_the_gemm_replay_are_caught(bug):
    """An accumulator at the wrong column, split-K slabs over each other, the lo token term
    half-way into the hi rows, or an epilogue that leaves out the lo term's columns of a
    tile whose two terms share one MMA: each moves the result well past the fp32 level."""
    rng = np.random.default_rng(4)
    if bug == "no_fuse_add":
        counts, F, K = [20, 7], 128, 128      # tiles of 32 and 16 rows: both terms in one MMA
        off = np.concatenate([[0], np.cumsum(counts)]).astype(int)
        items = [(e, int(off[e]), counts[e]) for e in range(2)]
        x, hi, lo = bf16_pair(rng, int(off[-1]), K)
        Wg, wg = weights(rng, 2, F, K)
        Wu, wu = weights(rng, 2, F, K)
        out, out_lo = run_gemm(Wg, hi, lo, F, K, F, items=items, n_max=128, W2=Wu, bug=bug)
        ref = O.silu(x[:20] @ wg[0].T) * (x[:20] @ wu[0].T)
        got = (out + out_lo)[:20]
    elif bug == "d1":
        counts, F, K = [40, 90], 128, 128
        off = np.concatenate([[0], np.cumsum(counts)]).astype(int)
        items = [(e, r0, min(64, off[e + 1] - r0)) for e in range(2) for r0 in range(off[e], off[e + 1], 64)]
        x, hi, lo = bf16_pair(rng, int(off[-1]), K)
        Wg, wg = weights(rng, 2, F, K)
        Wu, wu = weights(rng, 2, F, K)
        out, out_lo = run_gemm(Wg, hi, lo, F, K, F, items=items, n_max=64, W2=Wu, bug=bug)
        ref = O.silu(x[:40] @ wg[0].T) * (x[:40] @ wu[0].T)
        got = (out + out_lo)[:40]
    else:
        n, rows, K, ks = 60, 128, 256, 2
        x, hi, lo = bf16_pair(rng, n, K)
        W, w = weights(rng, 1, rows, K)
        out, _ = run_gemm(W, hi, lo, rows, K, rows, n_max=64, k_splits=ks, split_stride=n * rows, bug=bug)
        got = np.nan_to_num(out.reshape(ks, n, rows)).sum(axis=0)
        ref = x @ w[0].T
    assert not (np.abs(got - ref).max() / np.abs(ref).max() <= 1e-3)   # off by more, or NaN


@pytest.mark.parametrize("n_items,m_tiles,rows_a,grid", [(128, 6, 704, 148), (54, 8, 1024, 148), (7, 6, 704, 5),
                                                        (1, 22, 2816, 148), (3, 1, 100, 148)])
def test_tile_walk_covers_every_tile_once_and_balances_the_weight_bytes(n_items, m_tiles, rows_a, grid):
    """Every tile is walked by exactly one CTA, and no CTA streams more weight rows than the
    ceiling of the average plus one partial tile (the large model's gate/up GEMM: 5 whole
    tiles' worth at most, where the plain strided walk gives some CTA 6)."""
    n_tiles = n_items * m_tiles
    walks = [tile_walk(c, grid, n_tiles, m_tiles, rows_a) for c in range(grid)]
    seen = sorted(t for w in walks for t in w)
    assert seen == list(range(n_tiles))
    rows = lambda t: min(BM, rows_a - (t % m_tiles) * BM)
    load = [sum(rows(t) for t in w) for w in walks]
    avg = sum(load) / grid
    assert max(load) <= -(-avg // BM) * BM + BM // 2
    if (n_items, m_tiles, grid) == (128, 6, 148):
        assert max(load) == 5 * BM
        strided = [sum(rows(t) for t in range(c, n_tiles, grid)) for c in range(grid)]
        assert max(strided) == 6 * BM


@pytest.mark.parametrize("rows,n,terms,n_max", [(320, 150, 2, 128), (704, 37, 2, 128), (384, 200, 1, 256),
                                               (256, 16, 1, 256)])
def test_paired_weight_tiles_replay(rows, n, terms, n_max):
    """Dense projections with paired weight tiles (two 128-row tiles sharing each token
    load; a partial pair where the rows end mid-pair); with 256 tokens per tile the two
    accumulators fill TMEM and the kernel keeps one buffer.  The unpaired replay agrees to
    fp32 summation order (a tile's k-blocks start at a rotation that depends on its index)."""
    rng = np.random.default_rng(rows + n)
    K = 256
    x, hi, lo = bf16_pair(rng, n, K)
    if terms == 1:
        lo = None
        x = T.bf16_value(hi).astype(np.float64)
    W, w = weights(rng, 1, rows, K)
    out, _ = run_gemm(W, hi, lo, rows, K, rows, n_max=n_max, m_pair=True)
    ref = x @ w[0].T
    assert np.abs(out.reshape(n, rows) - ref).max() / np.abs(ref).max() < 2e-6
    plain, _ = run_gemm(W, hi, lo, rows, K, rows, n_max=n_max, m_pair=False)
    assert np.abs(out - plain).max() / np.abs(ref).max() < 2e-6


@pytest.mark.parametrize("m_pair", [True, False])
def test_grouped_down_projection_in_weight_tile_pairs_replay(m_pair):
    """The expert down projection's shape (fp32 store, grouped, 16-ish token rows per
    expert) with its weight tiles paired, as the host runs it, and unpaired: both match
    fp64 products; weight rows (384) not a multiple of the pair (256) leave a partial pair."""
    rng = np.random.default_rng(13)
    counts, H, F = [16, 0, 40, 9, 130], 384, 192
    E = len(counts)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(int)
    items = [(e, r0, min(128, off[e + 1] - r0)) for e in range(E) for r0 in range(off[e], off[e + 1], 128)]
    x, hi, lo = bf16_pair(rng, int(off[-1]), F)
    W, w = weights(rng, E, H, F)
    out, _ = run_gemm(W, hi, lo, H, F, H, items=items, n_max=128, m_pair=m_pair, grid=3)
    got = out.reshape(int(off[-1]), H)
    for e in range(E):
        xe = x[off[e]:off[e + 1]]
        if len(xe):
            ref = xe @ w[e].T
            assert np.abs(got[off[e]:off[e + 1]] - ref).max() / np.abs(ref).max() < 1e-5, e
