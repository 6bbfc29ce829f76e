"""Time the block-masked attention launch alone on synthetic bf16 data.

    python -m block_diffusion_lm_masked_b200.attention_probe [--queries 256] [--keys 8192]
        [--heads 16] [--kv-heads 8] [--launches 6] [--pair]

The queries sit at the last positions of the key range (a canvas over a cached prefix,
bidirectional).  Prints the median CUDA-event time of the debug attention entry (which
also launches the split-KV merge) and the algorithmic FLOP rate 4 * queries * heads *
128 * keys / time.  --pair times the head-pair kernel instead.
"""
from __future__ import annotations

import argparse

import torch

from block_diffusion_lm_masked_b200 import configs as CF
from block_diffusion_lm_masked_b200 import dg


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--queries", type=int, default=256)
    ap.add_argument("--keys", type=int, default=8192)
    ap.add_argument("--heads", type=int, default=16)
    ap.add_argument("--kv-heads", type=int, default=8)
    ap.add_argument("--launches", type=int, default=6)
    ap.add_argument("--pair", action="store_true", help="the head-pair kernel (dg_debug_attention_pair_bf16)")
    a = ap.parse_args()
    g = torch.Generator(device="cuda").manual_seed(7)
    d, n_q, n_keys, nq, nkv = 128, a.queries, a.keys, a.heads, a.kv_heads
    cap = n_keys + 8
    q = torch.randn(nq, n_q, d, generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn(nkv, cap, d, generator=g, device="cuda").to(torch.bfloat16)
    vt = torch.randn(nkv, d, cap, generator=g, device="cuda").to(torch.bfloat16)
    cfg = dict(CF.CONFIGS["layer1_bf16"], n_q_heads=nq, n_kv_heads=nkv, hidden=128, expert_ffn=64, n_experts=1,
               top_k=1, vocab=128, n_layers=1)
    ws = dg.Workspace(cfg, n_q)
    out = torch.zeros(n_q, nq * d, dtype=torch.bfloat16, device="cuda")
    lo = torch.zeros_like(out)
    fn = dg.debug_attention_pair_bf16 if a.pair else dg.debug_attention_bf16
    ts = []
    for it in range(a.launches):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn(q, k, vt, n_keys, n_keys - n_q, False, out, ws, out_lo=lo)
        e1.record()
        e1.synchronize()
        if it:
            ts.append(e0.elapsed_time(e1) * 1e3)
    dg.device_status(ws)
    us = sorted(ts)[len(ts) // 2]
    fl = 4.0 * n_q * nq * d * n_keys
    kind = "attention (head pairs)" if a.pair else "attention"
    print(f"{kind}: {n_q} queries x {nq} heads ({nkv} kv heads) over {n_keys} keys: {us:.1f} us per call "
          f"(attention + merge), {fl / us / 1e6:.0f} TFLOP/s algorithmic")
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
