"""The 4-bit decode that the low-precision GEMM kernel applies (format NV4), replayed on
the CPU with the kernel's own tables and byte-permute selectors, for every code in every
position and every block-scale code, against the oracle's decoding.  The byte permute
picks result byte i by nibble i of the selector from the bytes of (x, y) -- its documented
meaning -- and only the low 16 bits of the selector are read.
"""
import struct

import numpy as np
import pytest

from oracle import dg_oracle as O

NV4_HI_A, NV4_HI_B = 0x3F3F3F00, 0x40404040
NV4_LO_A, NV4_LO_B = 0xC0800000, 0xC0804000


def byte_perm(x, y, sel):
    src = [(x >> (8 * i)) & 0xFF for i in range(4)] + [(y >> (8 * i)) & 0xFF for i in range(4)]
    assert not sel & 0x8888                      # no sign-replicating selectors in use
    return sum(src[(sel >> (4 * i)) & 0x7] << (8 * i) for i in range(4))


def bf16_value(b):
    s = -1.0 if b & 0x8000 else 1.0
    e, m = (b >> 7) & 0xFF, b & 0x7F
    assert e != 0xFF
    return s * m * 2.0 ** -133 if e == 0 else s * (1 + m / 128) * 2.0 ** (e - 127)


def bf16_bits(v):
    b = struct.unpack("<I", struct.pack("<f", v))[0]
    assert b & 0xFFFF == 0
    return b >> 16


def decode8(x, mm):
    """The kernel's nv4_decode8, step by step: eight decoded values (times the multiplier)."""
    mags = x & 0x77777777
    h0, h1 = byte_perm(NV4_HI_A, NV4_HI_B, mags & 0xFFFF), byte_perm(NV4_HI_A, NV4_HI_B, mags >> 16)
    l0, l1 = byte_perm(NV4_LO_A, NV4_LO_B, mags & 0xFFFF), byte_perm(NV4_LO_A, NV4_LO_B, mags >> 16)
    xs = (x << 4) & 0xFFFFFFFF
    m = [byte_perm(l0, h0, 0x5140), byte_perm(l0, h0, 0x7362), byte_perm(l1, h1, 0x5140), byte_perm(l1, h1, 0x7362)]
    out = []
    for j, sel in enumerate((0x4000, 0x5010, 0x6020, 0x7030)):
        w = m[j] | (byte_perm(xs, x, sel) & 0x80008000)
        for h in (0, 1):
            out.append(bf16_value((w >> (16 * h)) & 0xFFFF) * bf16_value((mm >> (16 * h)) & 0xFFFF))
    return out


def scale_pair(sc):
    """The kernel's e4m3_scale_pair: the E4M3 value as a bf16 pair (exact)."""
    f = struct.unpack("<f", struct.pack("<I", (sc & 0x7F) << 20))[0] * 2.0 ** 120
    h = bf16_bits(f)
    return h | (h << 16)


def test_tables_hold_the_e2m1_magnitudes():
    for i in range(8):
        tbl_hi = (NV4_HI_A, NV4_HI_B)[i // 4] >> (8 * (i % 4)) & 0xFF
        tbl_lo = (NV4_LO_A, NV4_LO_B)[i // 4] >> (8 * (i % 4)) & 0xFF
        assert bf16_value(tbl_hi << 8 | tbl_lo) == O.e2m1_decode(i)


def test_scale_pair_is_the_e4m3_value_for_every_scale_code():
    for sc in range(0x7F):                       # non-negative, not NaN
        mm = scale_pair(sc)
        assert bf16_value(mm & 0xFFFF) == bf16_value(mm >> 16) == O.e4m3_decode(sc)


@pytest.mark.parametrize("sc", [0x01, 0x08, 0x38, 0x40, 0x66, 0x7E])
def test_decode8_matches_the_oracle_for_every_code_in_every_position(sc):
    mm = scale_pair(sc)
    s = O.e4m3_decode(sc)
    rng = np.random.default_rng(sc)
    for pos in range(8):
        for c in range(16):
            codes = [int(v) for v in rng.integers(0, 16, 8)]
            codes[pos] = c
            x = sum(v << (4 * i) for i, v in enumerate(codes))
            got = decode8(x, mm)
            assert got == [O.e2m1_decode(v) * s for v in codes], (codes, sc)


def test_decoding_quantised_weights_gives_the_oracle_dequantisation():
    """Weights quantised by the oracle's NVFP4 quantiser, packed the library's way and
    decoded the kernel's way (code x block scale, then the tensor scale g as the epilogue
    applies it): the oracle's dequantised weights."""
    from block_diffusion_lm_masked_b200 import dg
    rng = np.random.default_rng(9)
    w = rng.standard_normal((1, 2, 64)) * 0.02
    codes, sc, g = O.nvfp4_quantize(w)
    want = O.nvfp4_dequantize(codes, sc, g)
    packed, scales = dg.pack_nv4_codes(codes), dg.pack_nv4_scales(sc)
    for r in range(2):
        row = packed[0, r]
        for q in range(8):                       # eight 32-bit words of eight codes
            x = int.from_bytes(bytes(row[4 * q:4 * q + 4]), "little")
            blk = (8 * q) // 16
            got = decode8(x, scale_pair(int(scales[0, 0, r, blk])))
            # code x block scale is exact; times g the two sides round once each, in fp64
            np.testing.assert_allclose(np.array(got) * g, want[0, r, 8 * q:8 * q + 8], rtol=4e-16, atol=0)


def test_nv4_packing_layouts():
    from block_diffusion_lm_masked_b200 import dg
    rng = np.random.default_rng(2)
    c = rng.integers(0, 16, (2, 8, 128)).astype(np.uint8)
    p = dg.pack_nv4_codes(c)
    assert p.shape == (2, 8, 64)
    assert ((p & 0xF) == c[..., 0::2]).all() and ((p >> 4) == c[..., 1::2]).all()
    sc = rng.integers(0, 0x7F, (2, 8, 8)).astype(np.uint8)
    ps = dg.pack_nv4_scales(sc)
    assert ps.shape == (2, 2, 8, 4)
    for g_, j, f, b in np.ndindex(*ps.shape):
        assert ps[g_, j, f, b] == sc[g_, f, 4 * j + b]
    with pytest.raises(ValueError):
        dg.pack_nv4_codes(np.full((1, 1, 2), 16))
