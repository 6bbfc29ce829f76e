"""Roofline arithmetic for one denoising pass.

A pass can finish no sooner than the slower of its two lower bounds, algorithmic
FLOPs at the tensor peak and algorithmic bytes at HBM bandwidth; the bounds do
not add ("Module 12. Diffusion Language Models" exercises, roofline solution:
lower bounds, not their sum under perfect overlap).

Algorithmic bytes count what a pass must move at least once: every weight it
touches (attention projections, router, the union of routed experts, the output
matrix), the cached K/V it attends over, the canvas K/V it writes, and the fp32
logits it writes and the update reads back.  FLOPs count 2 per multiply-add of
the dense contractions, with only the k routed experts per token.
"""
from __future__ import annotations


def time_bound(flops: float, nbytes: float, peak_flops: float, bw_bytes: float) -> float:
    return max(flops / peak_flops, nbytes / bw_bytes)


def wbytes(cfg: dict) -> int:
    return 2 if cfg["dtype"] == "bf16" else 4


def layer_attn_weight_bytes(cfg: dict) -> int:
    H, nq, nkv, d = cfg["hidden"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    return wbytes(cfg) * H * (nq * d + 2 * nkv * d) + wbytes(cfg) * nq * d * H


# bytes per expert weight of the 8-bit format: one E4M3 code plus one E8M0 scale per 32
MX8_WBYTES = 1.0 + 1.0 / 32.0
# and of the 4-bit format: half a byte per E2M1 code plus one E4M3 scale per 16
NV4_WBYTES = 0.5 + 1.0 / 16.0


def expert_bytes(cfg: dict, union: int, ew: float | None = None) -> float:
    """Weights of `union` experts (gate, up and down matrices); `ew` bytes per expert
    weight (default: the model dtype's)."""
    return (wbytes(cfg) if ew is None else ew) * 3 * cfg["hidden"] * cfg["expert_ffn"] * union


def gate_up_bytes(cfg: dict, union: int, rows: int, ew: float | None = None) -> float:
    """Gate/up grouped GEMM: its weights for the touched experts, its gathered input rows, its output."""
    H, F, b = cfg["hidden"], cfg["expert_ffn"], wbytes(cfg)
    return (b if ew is None else ew) * 2 * H * F * union + b * rows * H + b * rows * F


def down_bytes(cfg: dict, union: int, rows: int, ew: float | None = None) -> float:
    H, F, b = cfg["hidden"], cfg["expert_ffn"], wbytes(cfg)
    return (b if ew is None else ew) * H * F * union + b * rows * F + 4 * rows * H


def vocab_bytes(cfg: dict, C: int) -> int:
    return wbytes(cfg) * cfg["vocab"] * cfg["hidden"] + wbytes(cfg) * C * cfg["hidden"] + 4 * C * cfg["vocab"]


def update_bytes(cfg: dict, C: int) -> int:
    """Canvas update: reads the fp32 logits once (plus the canvas in/out)."""
    return 4 * C * cfg["vocab"] + 8 * C


def update_record_bytes(cfg: dict, C: int) -> int:
    """The fused update's tile records: one 16-byte record per token and 128 vocabulary ids."""
    return 16 * C * ((cfg["vocab"] + 127) // 128)


def attention_flops(cfg: dict, P: int, C: int) -> float:
    """Canvas queries over P + C keys: QK^T and PV, per layer."""
    return 4.0 * C * cfg["n_q_heads"] * cfg["head_dim"] * (P + C)


def pass_flops(cfg: dict, P: int, C: int) -> float:
    H, nq, nkv, d = cfg["hidden"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    E, k, F, V = cfg["n_experts"], cfg["top_k"], cfg["expert_ffn"], cfg["vocab"]
    per_layer = (2.0 * C * H * (nq + 2 * nkv) * d + attention_flops(cfg, P, C) + 2.0 * C * nq * d * H
                 + 2.0 * C * H * E + 6.0 * H * F * C * k)
    return cfg["n_layers"] * per_layer + 2.0 * C * H * V


def prefill_flops(cfg: dict, P: int, T: int) -> float:
    """Causal prefill of T tokens after P cached ones: every layer's projections; below
    the last layer (which stops after its K/V) causal attention (token i reads P + i + 1
    keys), the output projection, the router and the k routed experts per token."""
    H, nq, nkv, d = cfg["hidden"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    E, k, F, L = cfg["n_experts"], cfg["top_k"], cfg["expert_ffn"], cfg["n_layers"]
    keys = T * P + T * (T + 1) / 2.0
    return (L * 2.0 * T * H * (nq + 2 * nkv) * d
            + (L - 1) * (4.0 * nq * d * keys + 2.0 * T * nq * d * H + 2.0 * T * H * E + 6.0 * H * F * T * k))


def prefill_bytes(cfg: dict, P: int, T: int, unions) -> float:
    """Causal prefill's bytes: every layer's QKV weights and the K/V it writes; below the
    last layer the output projection, the router, the union of experts and the cached K/V."""
    H, nq, nkv, d, E, L = (cfg["hidden"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"], cfg["n_experts"],
                           cfg["n_layers"])
    b = wbytes(cfg)
    total = 0.0
    for l in range(L):
        total += b * H * (nq + 2 * nkv) * d + b * 2 * nkv * d * T
        if l < L - 1:
            total += b * nq * d * H + 4 * H * E + expert_bytes(cfg, unions[l]) + b * 2 * nkv * d * (P + T)
    return total


def pass_bytes(cfg: dict, P: int, C: int, unions, ew: float | None = None) -> float:
    """`unions`: the expert union size of each layer (one int per layer)."""
    return pass_bytes_batched(cfg, [P], C, unions, ew)


def pass_bytes_batched(cfg: dict, prefixes, C: int, unions, ew: float | None = None,
                       vw: float | None = None) -> float:
    """A pass over one canvas of C positions per cache prefix in `prefixes`: every weight
    once (the experts of the batch's union), each canvas's K/V and logits traffic.  `ew`
    and `vw`: bytes per expert and per output-matrix weight (default: the model dtype's)."""
    H, nkv, d, E, V = cfg["hidden"], cfg["n_kv_heads"], cfg["head_dim"], cfg["n_experts"], cfg["vocab"]
    b = wbytes(cfg)
    B = len(prefixes)
    total = 0.0
    for l in range(cfg["n_layers"]):
        total += layer_attn_weight_bytes(cfg) + 4 * H * E + expert_bytes(cfg, unions[l], ew)
        for P in prefixes:
            total += b * 2 * nkv * d * (P + C)    # K/V read (cached prefix + canvas)
            total += b * 2 * nkv * d * C          # canvas K/V written
    total += (b if vw is None else vw) * V * H + B * (4 * C * V + 4 * C * V)   # output matrix, logits write + read
    return total


# ---- the exercises' dense-8B H100 arithmetic model, used to check this calculator ----

def dense_weight_read_s(params: float, bytes_per_param: float, bw_bytes: float) -> float:
    return params * bytes_per_param / bw_bytes


def dense_pass_s(params: float, positions: int, bytes_per_param: float, bw_bytes: float, peak_flops: float) -> float:
    return time_bound(2.0 * params * positions, params * bytes_per_param, peak_flops, bw_bytes)


def breakeven_steps(canvas: int, diffusion_pass_s: float, ar_rate: float) -> float:
    """Largest real S with canvas / (S * t_pass) > ar_rate."""
    return canvas / (diffusion_pass_s * ar_rate)
