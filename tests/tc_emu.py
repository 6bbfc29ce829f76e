"""An address-level model of the pieces of the Blackwell SM the attention kernels use, for
replaying a kernel's exact offsets, columns and issue order on the CPU (test helper).

- Shared memory is a flat byte array whose offsets count from a 1024-byte aligned base.
  The 128-byte swizzle maps a logical byte address L to L ^ (((L >> 7) & 7) << 4): the
  16-byte chunk index (bits 4-6) is XORed with the 128-byte row index within an 8-row,
  1024-byte atom (bits 7-9).  A TMA tile load with that swizzle writes box row r, chunk c
  at chunk c ^ (r & 7) of row r, which is the same map applied to dst + 128 r + 16 c.
- A K-major operand descriptor with the 128-byte swizzle and an 8-row stride of 1024 bytes
  reads row i of a K = 16 step (32 bytes) at logical bytes start + 1024 (i // 8) +
  128 (i % 8) + 0..31, through the same map; moving along K adds 32 bytes to the start.
- Tensor memory is 128 lanes x 512 columns of 32 bits.  An MMA with an M = 128 tile
  writes row i to lane i, column n to column d + n (fp32).  With A in tensor memory
  (kind::f16), row i's K elements 2c and 2c + 1 are the low and high bf16 halves of
  column a + c.
- A tile load reads zero outside the tensor.
Accumulation is modelled in float64 and rounded to float32 once per MMA; exp2 in float32
through numpy.  The model checks addressing and data flow, not rounding order.
"""
from __future__ import annotations

import numpy as np


def bf16_bits(x) -> np.ndarray:
    """float32 values -> bf16 bit patterns (round to nearest, ties to even)."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return (((b + 0x7FFF + ((b >> 16) & 1)) >> 16) & 0xFFFF).astype(np.uint16)


def bf16_value(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def sw128(addr: np.ndarray) -> np.ndarray:
    return addr ^ (((addr >> 7) & 7) << 4)


def swizzle(addr: np.ndarray, span: int) -> np.ndarray:
    """TMA swizzle modes: 16-byte chunk bits XORed with the bits above 128 bytes, three
    (128-byte span), two (64) or one (32); span 0 is no swizzle."""
    mask = {128: 7, 64: 3, 32: 1, 0: 0}[span]
    return addr ^ (((addr >> 7) & mask) << 4)


class Smem:
    def __init__(self, nbytes: int):
        self.b = np.zeros(nbytes, dtype=np.uint8)
        self.bytes_loaded = 0

    def tma_load_3d(self, dst: int, tensor: np.ndarray, x: int, y: int, z: int, bx: int, by: int, swizzle=True):
        """tensor: bf16 bits [dim2][dim1][dim0]; box (bx, by, 1) at (x, y, z); rows of the box
        are 2 bx bytes, 128 with the swizzle."""
        assert (x * 2) % 16 == 0, "TMA x coordinate not on a 16-byte boundary"
        assert dst % 1024 == 0 or not swizzle
        d2, d1, d0 = tensor.shape
        box = np.zeros((by, bx), dtype=np.uint16)
        ys = np.arange(y, y + by)
        xs = np.arange(x, x + bx)
        okr = (ys >= 0) & (ys < d1)
        okc = (xs >= 0) & (xs < d0)
        if 0 <= z < d2:
            box[np.ix_(okr, okc)] = tensor[z][np.ix_(ys[okr], xs[okc])]
        row_bytes = 2 * bx
        assert not swizzle or row_bytes == 128
        raw = box.view(np.uint8).reshape(by, row_bytes)
        L = dst + np.arange(by)[:, None] * row_bytes + np.arange(row_bytes)[None, :]
        phys = sw128(L) if swizzle else L
        assert phys.max() < self.b.size
        self.b[phys.ravel()] = raw.ravel()
        self.bytes_loaded += by * row_bytes

    def tma_load(self, dst: int, tensor: np.ndarray, coords, box, span: int):
        """Tile load of a 2-D or 3-D tensor (numpy, innermost axis last) at coords (x, y[, z])
        with box (bx, by[, 1]); rows of the box are bx elements, written one after another
        from dst through the given swizzle; elements outside the tensor read as zero."""
        es = tensor.dtype.itemsize
        x, y = coords[0], coords[1]
        z = coords[2] if len(coords) > 2 else 0
        bx, by = box[0], box[1]
        assert (x * es) % 16 == 0, "TMA x coordinate not on a 16-byte boundary"
        assert span == 0 or (bx * es == span and dst % (8 * span if span else 1) == 0 and dst % 128 == 0)
        t3 = tensor if tensor.ndim == 3 else tensor[None]
        d2, d1, d0 = t3.shape
        blk = np.zeros((by, bx), dtype=tensor.dtype)
        ys, xs = np.arange(y, y + by), np.arange(x, x + bx)
        okr, okc = (ys >= 0) & (ys < d1), (xs >= 0) & (xs < d0)
        if 0 <= z < d2:
            blk[np.ix_(okr, okc)] = t3[z][np.ix_(ys[okr], xs[okc])]
        row_bytes = bx * es
        raw = blk.view(np.uint8).reshape(by, row_bytes)
        L = dst + np.arange(by)[:, None] * row_bytes + np.arange(row_bytes)[None, :]
        phys = swizzle(L, span)
        assert phys.max() < self.b.size
        self.b[phys.ravel()] = raw.ravel()
        self.bytes_loaded += by * row_bytes

    def kmajor_sw128(self, start: int, rows: int) -> np.ndarray:
        """Rows x 16 bf16 (bits) of one K = 16 step through a K-major 128-byte-swizzle descriptor."""
        i = np.arange(rows)[:, None]
        L = start + 1024 * (i // 8) + 128 * (i % 8) + np.arange(32)[None, :]
        phys = sw128(L)
        assert phys.max() < self.b.size
        return self.b[phys].reshape(rows, 32).copy().view(np.uint16).reshape(rows, 16)


class Tmem:
    def __init__(self, cols=512):
        self.t = np.zeros((128, cols), dtype=np.uint32)

    def f32(self, c0, n):
        return self.t[:, c0:c0 + n].view(np.float32)

    def ld(self, lane0, col, n=16):
        """tcgen05.ld 32x32b: 32 lanes from lane0, n columns from col."""
        assert col + n <= self.t.shape[1]
        return self.t[lane0:lane0 + 32, col:col + n].copy()

    def st(self, lane0, col, vals):
        assert col + vals.shape[1] <= self.t.shape[1]
        self.t[lane0:lane0 + 32, col:col + vals.shape[1]] = vals

    def a_operand(self, col, M=128):
        """A from tensor memory for one K = 16 step: M x 16 bf16 bits."""
        w = self.t[:M, col:col + 8]
        out = np.empty((M, 16), dtype=np.uint16)
        out[:, 0::2] = (w & 0xFFFF).astype(np.uint16)
        out[:, 1::2] = (w >> 16).astype(np.uint16)
        return out


def _accumulate(tm: Tmem, d_col: int, prod: np.ndarray, acc: bool):
    M, N = prod.shape
    assert d_col + N <= tm.t.shape[1]
    cur = tm.f32(d_col, N)[:M].astype(np.float64) if acc else 0.0
    tm.t[:M, d_col:d_col + N] = (cur + prod).astype(np.float32).view(np.uint32)


def mma_ss(tm: Tmem, sm: Smem, d_col: int, a_start: int, b_start: int, M: int, N: int, acc: bool):
    """D[M x N] (+)= A[M x 16] B[N x 16]^T, both operands K-major in shared memory."""
    A = bf16_value(sm.kmajor_sw128(a_start, M)).astype(np.float64)
    B = bf16_value(sm.kmajor_sw128(b_start, N)).astype(np.float64)
    _accumulate(tm, d_col, A @ B.T, acc)


def mma_ts(tm: Tmem, sm: Smem, d_col: int, a_col: int, b_start: int, M: int, N: int, acc: bool):
    """D[M x N] (+)= A[M x 16] B[N x 16]^T, A from tensor memory."""
    A = bf16_value(tm.a_operand(a_col, M)).astype(np.float64)
    B = bf16_value(sm.kmajor_sw128(b_start, N)).astype(np.float64)
    _accumulate(tm, d_col, A @ B.T, acc)


def pack_bf16x2(p0: np.ndarray, p1: np.ndarray) -> np.ndarray:
    """__floats2bfloat162_rn(p0, p1) as a 32-bit word: p0 in the low half."""
    return bf16_bits(p0).astype(np.uint32) | (bf16_bits(p1).astype(np.uint32) << 16)


def unpack_lo_hi(w: np.ndarray):
    return bf16_value(w & 0xFFFF), bf16_value(w >> 16)
