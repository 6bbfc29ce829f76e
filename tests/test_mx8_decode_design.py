"""The integer decode that the 8-bit-weight GEMM kernel applies, replayed on the CPU for
every E4M3 code and every allowed block scale, against the oracle's decoding.

The kernel turns four codes (one 32-bit word) into two bf16x2 words with two byte
permutes, a mask, a shift and a select per pair, then one bf16x2 multiply by the
pair (2^(s - 7), 2^(s - 7)).  Those steps are integer operations with a documented
meaning (the byte-permute selector picks result byte i by nibble i from the bytes of
(x, y)), so replaying them here checks the design of the decode -- bit placement, the
2^-120 offset, the multiplier's bits, subnormal codes -- independently of the GPU.
The bf16 multiply is replayed as a correctly rounded bf16 product: one operand is a power
of two, so the product is exact whenever it is representable, which holds for every code
once the block scale is at least 2^-118 (E8M0 >= 9).
"""
import numpy as np
import pytest

from oracle import dg_oracle as O


def byte_perm(x: int, y: int, sel: int) -> int:
    src = [(x >> (8 * i)) & 0xFF for i in range(4)] + [(y >> (8 * i)) & 0xFF for i in range(4)]
    return sum(src[(sel >> (4 * i)) & 0x7] << (8 * i) for i in range(4))


def bf16_value(bits16: int) -> float:
    s = -1.0 if bits16 & 0x8000 else 1.0
    e = (bits16 >> 7) & 0xFF
    m = bits16 & 0x7F
    assert e != 0xFF
    if e == 0:
        return s * m * 2.0 ** -133          # subnormal: (m / 128) 2^-126
    return s * (1.0 + m / 128.0) * 2.0 ** (e - 127)


def round_bf16(v: float) -> float:
    """Nearest bf16 value (ties to even), subnormals included (quantum 2^-133 below 2^-126)."""
    if v == 0.0:
        return v
    e = int(np.floor(np.log2(abs(v))))
    q = 2.0 ** -133 if e < -126 else 2.0 ** (e - 7)
    return round(v / q) * q


def decode4(x: int, mm: int):
    """The kernel's mx8_decode4, step by step; returns the four decoded values."""
    mag = x & 0x7F7F7F7F
    s01, s23 = byte_perm(x, 0, 0x1404), byte_perm(x, 0, 0x3424)
    m01, m23 = byte_perm(mag, 0, 0x1404) >> 4, byte_perm(mag, 0, 0x3424) >> 4
    out = []
    for pair in ((s01 & 0x80008000) | m01, (s23 & 0x80008000) | m23):
        for h in (0, 1):
            a = bf16_value((pair >> (16 * h)) & 0xFFFF)
            b = bf16_value((mm >> (16 * h)) & 0xFFFF)
            out.append(round_bf16(a * b))  # the bf16 multiply: exact unless the product is below 2^-126
    return out


def multiplier(e8: int) -> int:
    mh = (e8 + 120) << 7
    return mh | (mh << 16)


def test_multiplier_bits_are_two_to_the_s_minus_7():
    for e8 in range(0, 135):
        mm = multiplier(e8)
        assert bf16_value(mm & 0xFFFF) == bf16_value(mm >> 16) == 2.0 ** (e8 - 7)
    assert ((135 + 120) << 7) >> 7 == 0xFF            # s = 135 would give an infinite multiplier


def test_bit_placement_gives_value_times_two_to_minus_120():
    """Before the multiply, each half is the code's value times 2^-120, normal and
    subnormal codes alike, with the sign in place."""
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        x = c | (c ^ 0x80) << 8           # the code and its negation as codes 0 and 1
        pair = (byte_perm(x, 0, 0x1404) & 0x80008000) | (byte_perm(x & 0x7F7F7F7F, 0, 0x1404) >> 4)
        assert bf16_value(pair & 0xFFFF) == O.e4m3_decode(c) * 2.0 ** -120
        assert bf16_value(pair >> 16) == O.e4m3_decode(c ^ 0x80) * 2.0 ** -120


@pytest.mark.parametrize("e8", [0, 1, 9, 100, 119, 120, 127, 134])
def test_decode4_matches_the_oracle_for_every_code(e8):
    """Every valid code in every byte position, for block scales from 2^-127 to 2^7.  At
    the smallest scales the exact value of a subnormal code can fall below bf16's
    smallest subnormal (2^-133); there the product rounds, which the test accounts
    for by comparing with the value rounded to bf16."""
    valid = [c for c in range(256) if c not in (0x7F, 0xFF)]
    mm = multiplier(e8)
    rng = np.random.default_rng(e8)
    for start in range(0, len(valid), 4):
        codes = valid[start:start + 4]
        while len(codes) < 4:
            codes.append(int(rng.choice(valid)))
        for perm in (codes, codes[::-1]):
            x = sum(c << (8 * i) for i, c in enumerate(perm))
            got = decode4(x, mm)
            for c, g in zip(perm, got):
                want = O.e4m3_decode(c) * 2.0 ** (e8 - 127)
                assert g == round_bf16(want), (hex(c), e8, g, want)
                if abs(want) >= 2.0 ** -126 or e8 >= 9:
                    assert g == want, (hex(c), e8, g, want)   # exact for every scale >= 2^-118


def test_decode_of_quantised_weights_is_the_oracle_dequantisation():
    """Realistic weights (N(0, 0.02)) quantised by the oracle: decoding their codes the
    kernel's way with their block scales reproduces mx_e4m3_dequantize exactly."""
    rng = np.random.default_rng(7)
    w = rng.standard_normal((4, 64)) * 0.02
    codes, exps = O.mx_e4m3_quantize(w)
    want = O.mx_e4m3_dequantize(codes, exps)
    for r in range(4):
        for b in range(2):
            mm = multiplier(int(exps[r, b]) + 127)
            blk = [int(c) for c in codes[r, 32 * b:32 * b + 32]]
            got = []
            for q in range(8):
                got += decode4(sum(c << (8 * i) for i, c in enumerate(blk[4 * q:4 * q + 4])), mm)
            np.testing.assert_array_equal(got, want[r, 32 * b:32 * b + 32])
