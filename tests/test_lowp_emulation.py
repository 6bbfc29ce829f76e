"""The 8/4-bit expert GEMM (tc_gemm_lowp_kernel) replayed at the address level on the CPU
(tests/tc_emu.py), against the oracle's dequantised weights.

Transcribed from the kernel source: the persistent tile walk with its k-block rotation,
the stage layout (token tiles, then code tiles, then scale tiles), the code tiles' 64- or
32-byte swizzle and the decoders' swizzled reads, the scale bytes each decoder half
takes, the TMEM columns of decoded weights (four stages, a second weight matrix 32
columns on) and of the two accumulator buffers, the MMAs with A from TMEM, and the
epilogue's indices, SwiGLU pairing and 4-bit tensor scales.  Each code is decoded by
value (the bit-level decode is checked against the oracle for every code and scale in
the decode design tests).  The roles run as far ahead as the kernel's barriers allow
(loads up to the stage ring, decoding up to the TMEM stages), and each epilogue runs as
late as it may, just before its accumulator buffer is reused.
"""
from __future__ import annotations

import numpy as np
import pytest

import tc_emu as T
from oracle import dg_oracle as O

BM, BK, T_STAGES = 128, 64, 4


def decode_mx8(codes, e8):
    return np.vectorize(O.e4m3_decode, otypes=[float])(codes) * np.ldexp(1.0, e8.astype(np.int64) - 127)


def decode_nv4(codes, sc):
    return np.vectorize(O.e2m1_decode, otypes=[float])(codes) * np.vectorize(O.e4m3_decode, otypes=[float])(sc)


def run_lowp(fmt, W, S, X_hi, X_lo, items, rows_a, K, ld_out, W2=None, S2=None, g=1.0, g2=1.0, n_max=64,
             smem_budget=200 * 1024, grid=3, bug=None):
    """W / W2: codes as the library stores them (8-bit [G][rows][K]; 4-bit packed
    [G][rows][K / 2]); S / S2: the library's scale bytes; items: (group, row0, rows), or
    None for the dense mode (one weight matrix, tokens in chunks of n_max, tiles ordered
    weight tile major)."""
    nv4 = fmt == "nv4"
    A_BYTES = BM * BK // 2 if nv4 else BM * BK
    S_BYTES = BM * 4 if nv4 else BM * 2
    terms = 2 if X_lo is not None else 1
    n_a = 2 if W2 is not None else 1
    b_bytes = n_max * 128
    a_off = terms * b_bytes
    s_off = a_off + n_a * A_BYTES
    stage_bytes = (s_off + n_a * S_BYTES + 1023) & ~1023
    stages = min(smem_budget // stage_bytes, 8)
    acc_cols = n_max * n_a
    a_col0 = 2 * acc_cols
    a_stage_cols = 32 * n_a
    tmem_cols = 32
    while tmem_cols < a_col0 + T_STAGES * a_stage_cols:
        tmem_cols <<= 1
    assert tmem_cols <= 512
    nkb = K // BK
    m_tiles = -(-rows_a // BM)
    G = W.shape[0]
    n_tokens = X_hi.shape[0]
    # the tensors the maps cover: codes (G, rows, K or K / 2) with a 64- or 32-byte swizzle;
    # scales 8-bit (G, K / 64, rows * 2), 4-bit (G * K / 64, rows / 4, 16); tokens (n, K) bf16
    if nv4:
        S_map = S.reshape(G * nkb, rows_a // 4, 16)
        S2_map = S2.reshape(G * nkb, rows_a // 4, 16) if S2 is not None else None
    else:
        S_map = S.reshape(G, nkb, rows_a * 2)
        S2_map = S2.reshape(G, nkb, rows_a * 2) if S2 is not None else None
    swz_span = 32 if nv4 else 64
    out = np.full((n_tokens, ld_out), np.nan)
    out_lo = np.zeros((n_tokens, ld_out))
    dense = items is None
    chunks = -(-n_tokens // n_max)
    n_tiles = chunks * m_tiles if dense else len(items) * m_tiles
    for cta in range(min(grid, n_tiles)):
        sm, tm = T.Smem(stages * stage_bytes), T.Tmem(tmem_cols)
        tiles = list(range(cta, n_tiles, grid))
        its = [(t, kb) for t in tiles for kb in range(nkb)]       # iteration -> (tile, k-block)
        loaded = decoded = mma_done = 0
        pending_epi = []                                         # (tile index j, tile) awaiting their epilogue

        def tile_of(t):
            if dense:
                row0 = (t % chunks) * n_max
                return 0, row0, min(n_max, n_tokens - row0), t // chunks
            g_, row0, rows = items[t // m_tiles]
            return g_, row0, rows, t % m_tiles

        def load(it):
            t, kb = its[it]
            g_, row0, rows, m = tile_of(t)
            n_pad = (rows + 15) & ~15
            st = (it % stages) * stage_bytes
            kbx = (kb + t) % nkb
            kx = kbx * BK
            ax = kx // 2 if nv4 else kx
            s0 = 0 if nv4 else m * BM * 2
            s1 = m * (BM // 4) if nv4 else kbx
            s2 = g_ * nkb + kbx if nv4 else g_
            sbox = (16, 32, 1) if nv4 else (256, 1, 1)
            cbox = (32, 128, 1) if nv4 else (64, 128, 1)
            sm.tma_load(st + a_off, W, (ax, m * BM, g_), cbox, swz_span)
            sm.tma_load(st + s_off, S_map, (s0, s1, s2), sbox, 0)
            if n_a == 2:
                sm.tma_load(st + a_off + A_BYTES, W2, (ax, m * BM, g_), cbox, swz_span)
                sm.tma_load(st + s_off + S_BYTES, S2_map, (s0, s1, s2), sbox, 0)
            r = 0
            while r + 64 <= n_pad:
                sm.tma_load(st + r * 128, X_hi, (kx, row0 + r), (64, 64), 128)
                if terms == 2:
                    sm.tma_load(st + b_bytes + r * 128, X_lo, (kx, row0 + r), (64, 64), 128)
                r += 64
            while r < n_pad:
                sm.tma_load(st + r * 128, X_hi, (kx, row0 + r), (64, 16), 128)
                if terms == 2:
                    sm.tma_load(st + b_bytes + r * 128, X_lo, (kx, row0 + r), (64, 16), 128)
                r += 16

        def decode(it):
            st = (it % stages) * stage_bytes
            ts = it % T_STAGES
            rows_ = np.arange(BM)
            for half in range(2):
                for a in range(n_a):
                    if nv4:
                        swz = (rows_ >> 2) & 1
                        base = st + a_off + a * A_BYTES + rows_ * 32 + ((half ^ swz) << 4)
                        byts = sm.b[base[:, None] + np.arange(16)[None, :]]            # [128][16]
                        codes = np.empty((BM, 32), np.uint8)
                        codes[:, 0::2], codes[:, 1::2] = byts & 0xF, byts >> 4
                        sc = st + s_off + a * S_BYTES + rows_ * 4 + 2 * half
                        scl = np.stack([sm.b[sc], sm.b[sc + 1]], axis=1)                  # [128][2]
                        vals = decode_nv4(codes, np.repeat(scl, 16, axis=1))
                    else:
                        swz = (rows_ >> 1) & 3
                        chunks = []
                        for c2 in range(2):
                            c = 2 * half + c2
                            base = st + a_off + a * A_BYTES + rows_ * 64 + ((c ^ swz) << 4)
                            chunks.append(sm.b[base[:, None] + np.arange(16)[None, :]])
                        codes = np.concatenate(chunks, axis=1)                              # [128][32]
                        e8 = sm.b[st + s_off + a * S_BYTES + rows_ * 2 + half].astype(np.int64)
                        vals = decode_mx8(codes, np.repeat(e8[:, None], 32, axis=1))
                    bits = T.bf16_bits(vals.astype(np.float32))
                    assert np.array_equal(T.bf16_value(bits).astype(np.float64), vals), "decode not exact in bf16"
                    words = bits[:, 0::2].astype(np.uint32) | (bits[:, 1::2].astype(np.uint32) << 16)
                    col = a_col0 + ts * a_stage_cols + a * 32 + half * 16
                    if bug == "dec_col":
                        col = a_col0 + ts * a_stage_cols + half * 16
                    tm.t[:, col:col + 16] = words

        def epilogue(j, t):
            g_, row0, rows, m = tile_of(t)
            buf = j & 1
            d0 = buf * acc_cols
            f = m * BM + np.arange(BM)
            for col in range(rows):
                a = tm.f32(d0 + col, 1)[:, 0].astype(np.float64) * (g if nv4 else 1.0)
                a = a.astype(np.float32).astype(np.float64)
                ok = f < rows_a
                if n_a == 2:
                    b = tm.f32(d0 + n_max + col, 1)[:, 0].astype(np.float64) * (g2 if nv4 else 1.0)
                    hv = (a / (1.0 + np.exp(-a)) * b).astype(np.float32)
                    hi = T.bf16_value(T.bf16_bits(hv)).astype(np.float64)
                    out[row0 + col, f[ok]] = hi[ok]
                    out_lo[row0 + col, f[ok]] = T.bf16_value(T.bf16_bits((hv - hi).astype(np.float32)))[ok]
                else:
                    out[row0 + col, f[ok]] = a[ok]

        for it in range(len(its)):
            # the producer runs up to the stage ring ahead of the slowest consumer
            while loaded < len(its) and loaded < mma_done + stages:
                load(loaded)
                loaded += 1
            # the decoders run up to the TMEM stages ahead of the MMAs
            while decoded < loaded and decoded < mma_done + T_STAGES:
                decode(decoded)
                decoded += 1
            t, kb = its[it]
            j = tiles.index(t)
            if kb == 0:
                # this tile's accumulator buffer was last used by tile j - 2: its epilogue now
                while pending_epi and pending_epi[0][0] <= j - 2:
                    epilogue(*pending_epi.pop(0))
            g_, row0, rows, m = tile_of(t)
            n_pad = (rows + 15) & ~15
            buf = j & 1
            d0 = buf * acc_cols
            d1 = d0 + n_max
            sb = (it % stages) * stage_bytes
            a0 = a_col0 + (it % T_STAGES) * a_stage_cols
            for kk in range(BK // 16):
                acc = kb != 0 or kk != 0
                ak = a0 + kk * 8
                T.mma_ts(tm, sm, d0, ak, sb + kk * 32, BM, n_pad, acc)
                if terms == 2:
                    T.mma_ts(tm, sm, d0, ak, sb + b_bytes + kk * 32, BM, n_pad, True)
                if n_a == 2:
                    T.mma_ts(tm, sm, d1, ak + 32, sb + kk * 32, BM, n_pad, acc)
                    if terms == 2:
                        T.mma_ts(tm, sm, d1, ak + 32, sb + b_bytes + kk * 32, BM, n_pad, True)
            mma_done += 1
            if kb == nkb - 1:
                pending_epi.append((j, t))
        while pending_epi:
            epilogue(*pending_epi.pop(0))
    return out, out_lo


# ---------------------------------------------------------------- inputs
def items_of(counts, item_rows=64):
    off = np.concatenate([[0], np.cumsum(counts)]).astype(int)
    return [(e, r0, min(item_rows, off[e + 1] - r0)) for e in range(len(counts))
            for r0 in range(off[e], off[e + 1], item_rows)], off


def tokens(rng, n, K):
    x = rng.standard_normal((n, K))
    hi = T.bf16_bits(x.astype(np.float32))
    lo = T.bf16_bits((x.astype(np.float32) - T.bf16_value(hi)).astype(np.float32))
    return T.bf16_value(hi).astype(np.float64) + T.bf16_value(lo), hi, lo


def mx8_weights(rng, G, rows, K):
    from block_diffusion_lm_masked_b200 import dg as dg_pack
    codes, exps = O.mx_e4m3_quantize(rng.standard_normal((G, rows, K)) * 0.02)
    return codes, dg_pack.pack_mx8_scales(exps), O.mx_e4m3_dequantize(codes, exps)


def nv4_weights(rng, G, rows, K):
    from block_diffusion_lm_masked_b200 import dg as dg_pack
    codes, sc, g = O.nvfp4_quantize(rng.standard_normal((G, rows, K)) * 0.02)
    return dg_pack.pack_nv4_codes(codes), dg_pack.pack_nv4_scales(sc), g, O.nvfp4_dequantize(codes, sc, g)


CASES = [([0, 3, 17, 70, 1], 192, 256), ([64, 65], 128, 128), ([5], 320, 192)]


@pytest.mark.parametrize("counts,rows,K", CASES)
def test_mx8_grouped_two_term_gemm_replay(counts, rows, K):
    rng = np.random.default_rng(sum(counts) + rows)
    items, off = items_of(counts)
    codes, S, wq = mx8_weights(rng, len(counts), rows, K)
    x, hi, lo = tokens(rng, int(off[-1]), K)
    out, _ = run_lowp("mx8", codes, S, hi, lo, items, rows, K, rows)
    for e in range(len(counts)):
        ref = x[off[e]:off[e + 1]] @ wq[e].T
        if ref.size:
            assert np.abs(out[off[e]:off[e + 1]] - ref).max() / np.abs(ref).max() < 2e-5, e


@pytest.mark.parametrize("fmt", ["mx8", "nv4"])
def test_gate_up_swiglu_replay(fmt):
    rng = np.random.default_rng(7)
    counts, F, K = [20, 0, 64, 7], 192, 256
    items, off = items_of(counts)
    x, hi, lo = tokens(rng, int(off[-1]), K)
    if fmt == "mx8":
        cg, sg, wg = mx8_weights(rng, 4, F, K)
        cu, su, wu = mx8_weights(rng, 4, F, K)
        out, out_lo = run_lowp(fmt, cg, sg, hi, lo, items, F, K, F, W2=cu, S2=su)
    else:
        cg, sg, gg, wg = nv4_weights(rng, 4, F, K)
        cu, su, gu, wu = nv4_weights(rng, 4, F, K)
        out, out_lo = run_lowp(fmt, cg, sg, hi, lo, items, F, K, F, W2=cu, S2=su, g=gg, g2=gu)
    got = out + out_lo
    for e in range(4):
        xe = x[off[e]:off[e + 1]]
        if len(xe):
            ref = O.silu(xe @ wg[e].T) * (xe @ wu[e].T)
            assert np.abs(got[off[e]:off[e + 1]] - ref).max() / np.abs(ref).max() < 1e-4, e


def test_nv4_down_replay():
    rng = np.random.default_rng(9)
    counts, H, F = [9, 70, 0, 2], 256, 192
    items, off = items_of(counts)
    codes, S, g, wq = nv4_weights(rng, 4, H, F)
    x, hi, lo = tokens(rng, int(off[-1]), F)
    out, _ = run_lowp("nv4", codes, S, hi, lo, items, H, F, H, g=g)
    for e in range(4):
        ref = x[off[e]:off[e + 1]] @ wq[e].T
        if ref.size:
            assert np.abs(out[off[e]:off[e + 1]] - ref).max() / np.abs(ref).max() < 2e-5, e


def test_a_planted_decode_column_mistake_is_caught():
    """The second weight matrix's decoded tile written over the first's: the gate/up
    product is wrong."""
    rng = np.random.default_rng(7)
    counts, F, K = [20, 64], 128, 128
    items, off = items_of(counts)
    x, hi, lo = tokens(rng, int(off[-1]), K)
    cg, sg, wg = mx8_weights(rng, 2, F, K)
    cu, su, wu = mx8_weights(rng, 2, F, K)
    out, out_lo = run_lowp("mx8", cg, sg, hi, lo, items, F, K, F, W2=cu, S2=su, bug="dec_col")
    ref = O.silu(x[:20] @ wg[0].T) * (x[:20] @ wu[0].T)
    assert np.abs((out + out_lo)[:20] - ref).max() / np.abs(ref).max() > 1e-2


@pytest.mark.parametrize("fmt,n_max", [("mx8", 64), ("mx8", 128), ("nv4", 128)])
def test_dense_vocab_gemm_replay(fmt, n_max):
    """The dense mode as the vocabulary projection uses it: one weight matrix of V rows,
    the canvas rows in chunks of up to 128 tokens (one term), tiles weight tile major."""
    rng = np.random.default_rng(11)
    n, V, H = 150, 640, 128
    x, hi, _ = tokens(rng, n, H)
    x = T.bf16_value(hi).astype(np.float64)
    if fmt == "mx8":
        codes, S, wq = mx8_weights(rng, 1, V, H)
        out, _ = run_lowp(fmt, codes, S, hi, None, None, V, H, V, grid=7, n_max=n_max)
    else:
        codes, S, g, wq = nv4_weights(rng, 1, V, H)
        out, _ = run_lowp(fmt, codes, S, hi, None, None, V, H, V, g=g, grid=7, n_max=n_max)
    ref = x @ wq[0].T
    assert np.abs(out - ref).max() / np.abs(ref).max() < 2e-5
