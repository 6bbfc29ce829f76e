"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This module draws random numbers and nothing else: it holds none of the
denoising pass's arithmetic.  Every value is a pure function of
(seed, tensor id, element index), so the same tensor can be regenerated
bit-for-bit on any machine, in any chunking, with any number of threads.

Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) used in counter mode: draw number `c` of a
stream seeded with `s` is the SplitMix64 output for state s + (c+1)*gamma.
Normals come from the Box-Muller transform (Box & Muller 1958) on two such
draws; integers in [0, n) from the multiply-shift reduction of the high 32
bits (Lemire 2019).

Workload recipe (block-diffusion pages: the canvas of random vocabulary
tokens on "Uniform State Diffusion"; the configs' N(0, 0.02) weights):
  * weights       ~ N(0, 0.02), rounded once to bf16 (fp32 for the fp32 model)
  * cached K / V  ~ N(0, 1) in the activation dtype, treated as post-RoPE
  * token ids     ~ uniform over the vocabulary
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22

SEED_WEIGHTS = 1234
SEED_TOKENS = 1235
SEED_RENOISE = 1236


def splitmix64(seed: int, counters: np.ndarray) -> np.ndarray:
    """SplitMix64 output number `counters` (0-based) of the stream seeded with `seed`."""
    with np.errstate(over="ignore"):
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + (counters.astype(np.uint64) + np.uint64(1)) * GAMMA
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def _tensor_base(tensor_id: int) -> np.uint64:
    return np.uint64(tensor_id) << np.uint64(42)


def _normal_chunk(seed, tensor_id, lo, hi, std):
    idx = np.arange(lo, hi, dtype=np.uint64)
    base = _tensor_base(tensor_id)
    x1 = splitmix64(seed, base | (idx << np.uint64(1)))
    x2 = splitmix64(seed, base | (idx << np.uint64(1)) | np.uint64(1))
    u1 = ((x1 >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
    u2 = (x2 >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    return std * np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def _bf16_bits_from_f64(v: np.ndarray) -> np.ndarray:
    # round-to-nearest-even onto 8 significant bits, done exactly in float64
    m, e = np.frexp(v)
    r = np.ldexp(np.rint(m * 256.0), e - 8)
    return (r.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def _parallel(n, fn):
    chunks = [(lo, min(n, lo + _CHUNK)) for lo in range(0, n, _CHUNK)]
    if len(chunks) <= 1:
        for lo, hi in chunks:
            fn(lo, hi)
        return
    with ThreadPoolExecutor(max_workers=min(len(chunks), os.cpu_count() or 1)) as ex:
        list(ex.map(lambda c: fn(*c), chunks))


def normal(seed: int, tensor_id: int, shape, std: float, dtype: str) -> np.ndarray:
    """N(0, std^2) tensor. dtype 'bf16' -> uint16 bf16 bit patterns; 'f32' -> float32."""
    n = int(np.prod(shape))
    if dtype == "bf16":
        out = np.empty(n, dtype=np.uint16)

        def fill(lo, hi):
            out[lo:hi] = _bf16_bits_from_f64(_normal_chunk(seed, tensor_id, lo, hi, std))
    elif dtype == "f32":
        out = np.empty(n, dtype=np.float32)

        def fill(lo, hi):
            out[lo:hi] = _normal_chunk(seed, tensor_id, lo, hi, std).astype(np.float32)
    else:
        raise ValueError(dtype)
    _parallel(n, fill)
    return out.reshape(shape)


def tokens(seed: int, tensor_id: int, n: int, vocab: int) -> np.ndarray:
    """n token ids uniform over [0, vocab)."""
    idx = np.arange(n, dtype=np.uint64)
    x = splitmix64(seed, _tensor_base(tensor_id) | idx)
    with np.errstate(over="ignore"):
        return (((x >> np.uint64(32)) * np.uint64(vocab)) >> np.uint64(32)).astype(np.int32)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---- tensor ids (fixed enumeration so any tensor can be regenerated alone) ----
TID_EMBED = 1
TID_W_OUT = 2
TID_PREFIX_TOKENS = 3
TID_W_OUT_MX8 = 4
TID_W_OUT_NV4 = 5


def tid_canvas_noise(canvas_index: int) -> int:
    return 64 + canvas_index


def tid_layer(layer: int, j: int) -> int:
    """j: 0 w_q, 1 w_k, 2 w_v, 3 w_o, 4 w_router, 5 w_gate, 6 w_up, 7 w_down, 8 cache K, 9 cache V,
    10-12 8-bit gate / up / down codes, 13-15 4-bit gate / up / down codes"""
    return 1024 + 16 * layer + j


class Model:
    """Synthetic random-init weights of one config, in the logical layouts the oracle reads.

    All matrices are [out_features][in_features] (y = x @ W^T).
      embed [V][H], w_out [V][H]
      per layer: w_q [nq*d][H], w_k [nkv*d][H], w_v [nkv*d][H], w_o [H][nq*d],
                 w_router [E][H] (float32, bf16-representable in bf16 models),
                 w_gate [E][F][H], w_up [E][F][H], w_down [E][H][F]
    Storage: 'bf16' -> uint16 bit patterns, 'f32' -> float32.
    """

    def __init__(self, cfg: dict, seed: int = SEED_WEIGHTS):
        self.cfg = cfg
        dt = cfg["dtype"]
        H, nq, nkv, d = cfg["hidden"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
        E, F, V = cfg["n_experts"], cfg["expert_ffn"], cfg["vocab"]
        std = 0.02
        self.embed = normal(seed, TID_EMBED, (V, H), std, dt)
        self.w_out = normal(seed, TID_W_OUT, (V, H), std, dt)
        self.layers = []
        for l in range(cfg["n_layers"]):
            wr = normal(seed, tid_layer(l, 4), (E, H), std, dt)
            self.layers.append(dict(
                w_q=normal(seed, tid_layer(l, 0), (nq * d, H), std, dt),
                w_k=normal(seed, tid_layer(l, 1), (nkv * d, H), std, dt),
                w_v=normal(seed, tid_layer(l, 2), (nkv * d, H), std, dt),
                w_o=normal(seed, tid_layer(l, 3), (H, nq * d), std, dt),
                w_router=bf16_bits_to_f32(wr) if dt == "bf16" else wr,
                w_gate=normal(seed, tid_layer(l, 5), (E, F, H), std, dt),
                w_up=normal(seed, tid_layer(l, 6), (E, F, H), std, dt),
                w_down=normal(seed, tid_layer(l, 7), (E, H, F), std, dt),
            ))


def _codes8(seed, tensor_id, shape, n_mag):
    """Bytes: a random sign (bit 7) over a magnitude uniform over [0, n_mag)."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint8)

    def fill(lo, hi):
        x = splitmix64(seed, _tensor_base(tensor_id) | np.arange(lo, hi, dtype=np.uint64))
        with np.errstate(over="ignore"):
            mag = ((x >> np.uint64(32)) * np.uint64(n_mag)) >> np.uint64(32)
        out[lo:hi] = (mag | (((x >> np.uint64(31)) & np.uint64(1)) << np.uint64(7))).astype(np.uint8)

    _parallel(n, fill)
    return out.reshape(shape)


def mx8_experts(cfg: dict, seed: int = SEED_WEIGHTS):
    """Synthetic 8-bit expert weights drawn directly as MX-FP8 data (random bytes, no
    quantiser): per layer dict(gate=(codes, exps), up=..., down=...) with codes uint8
    [E][F][H] (down [E][H][F]) -- a random sign over an E4M3 magnitude code uniform over
    0x00..0x6F -- and every block exponent -12 (one per 32 elements), so weights are
    E4M3 values up to 120 times 2^-12 (magnitudes up to about 0.03)."""
    E, F, H = cfg["n_experts"], cfg["expert_ffn"], cfg["hidden"]
    out = []
    for l in range(cfg["n_layers"]):
        d = {}
        for j, (name, shape) in enumerate((("gate", (E, F, H)), ("up", (E, F, H)), ("down", (E, H, F)))):
            codes = _codes8(seed, tid_layer(l, 10 + j), shape, 0x70)
            d[name] = (codes, np.full(shape[:-1] + (shape[-1] // 32,), -12, dtype=np.int32))
        out.append(d)
    return out


def nv4_experts(cfg: dict, seed: int = SEED_WEIGHTS):
    """Synthetic 4-bit expert weights drawn directly as NVFP4-style data (random nibbles, no
    quantiser): per layer dict(gate=(codes, scale_codes, g), up=..., down=...) with one
    uniformly random E2M1 code per byte [E][F][H] (down [E][H][F]), every E4M3 block
    scale 0.25 (code 0x28, one per 16 elements) and tensor scale 2^-6, so weights are
    E2M1 values times 2^-8 (magnitudes up to about 0.023)."""
    E, F, H = cfg["n_experts"], cfg["expert_ffn"], cfg["hidden"]
    out = []
    for l in range(cfg["n_layers"]):
        d = {}
        for j, (name, shape) in enumerate((("gate", (E, F, H)), ("up", (E, F, H)), ("down", (E, H, F)))):
            b = _codes8(seed, tid_layer(l, 13 + j), shape, 8)  # sign in bit 7 over a magnitude in [0, 8)
            codes = ((b >> 4) & 0x8) | (b & 0x7)
            d[name] = (codes.astype(np.uint8), np.full(shape[:-1] + (shape[-1] // 16,), 0x28, dtype=np.uint8),
                       2.0 ** -6)
        out.append(d)
    return out


def mx8_vocab(cfg: dict, seed: int = SEED_WEIGHTS):
    """Synthetic 8-bit output matrix drawn directly as MX-FP8 data, as mx8_experts: codes
    uint8 [V][H] and every block exponent -12 (one per 32 elements)."""
    V, H = cfg["vocab"], cfg["hidden"]
    return _codes8(seed, TID_W_OUT_MX8, (V, H), 0x70), np.full((V, H // 32), -12, dtype=np.int32)


def nv4_vocab(cfg: dict, seed: int = SEED_WEIGHTS):
    """Synthetic 4-bit output matrix drawn directly as NVFP4-style data, as nv4_experts:
    one E2M1 code per byte [V][H], every block scale code 0x28 (0.25), tensor scale 2^-6."""
    V, H = cfg["vocab"], cfg["hidden"]
    b = _codes8(seed, TID_W_OUT_NV4, (V, H), 8)
    return (((b >> 4) & 0x8) | (b & 0x7)).astype(np.uint8), np.full((V, H // 16), 0x28, dtype=np.uint8), 2.0 ** -6


def prefix_cache(cfg: dict, P: int, seed: int = SEED_WEIGHTS):
    """Cached prefix K/V ~ N(0,1) per layer, logical layout [nkv][P][d] each."""
    nkv, d, dt = cfg["n_kv_heads"], cfg["head_dim"], cfg["dtype"]
    out = []
    for l in range(cfg["n_layers"]):
        k = normal(seed, tid_layer(l, 8), (nkv, P, d), 1.0, dt)
        v = normal(seed, tid_layer(l, 9), (nkv, P, d), 1.0, dt)
        out.append((k, v))
    return out


def to_f64(a: np.ndarray) -> np.ndarray:
    """Exact widening of stored weights (bf16 bit patterns or float32) to float64."""
    if a.dtype == np.uint16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)
