"""The five workload shapes of the block-diffusion denoising pass (shapes only, no arithmetic).

Model fields mirror the C-ABI's dg_config; workload fields say how a run drives
the pass: cached prefix length P, canvas length C, denoising steps S with the
re-noise fraction going linearly from renoise_start to renoise_end, and for the
chained workload a random prompt and a number of canvases appended by prefill.
"""

_BASE_BF16 = dict(hidden=2048, n_q_heads=16, n_kv_heads=4, head_dim=128, n_experts=64, top_k=4,
                  expert_ffn=1024, vocab=32768, rope_theta=10000.0, rms_eps=1e-6, dtype="bf16")

CONFIGS = {
    # tiny fp32 correctness model: 2 layers, H256, 4q/2kv heads d64, E8 top-2, F512, V1024; P64, C32, 1 pass, 25% re-noise
    "tiny_fp32": dict(n_layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, n_experts=8, top_k=2,
                      expert_ffn=512, vocab=1024, rope_theta=10000.0, rms_eps=1e-6, dtype="f32",
                      prefix=64, canvas=32, steps=1, renoise_start=0.25, renoise_end=0.25),
    # single-layer bf16 pass: H2048, 16q/4kv d128, E64 top-4, F1024, V32768; P1024 cached N(0,1) K/V, C256, 1 pass
    "layer1_bf16": dict(_BASE_BF16, n_layers=1, prefix=1024, canvas=256, steps=1,
                        renoise_start=0.25, renoise_end=0.25),
    # full canvas denoise: 8 layers of the single-layer shape, P2048, C256, 16 steps, re-noise 50% -> 0%
    "denoise8_bf16": dict(_BASE_BF16, n_layers=8, prefix=2048, canvas=256, steps=16,
                          renoise_start=0.5, renoise_end=0.0),
    # chained canvases: 8 layers, 512-token random prompt prefilled, 4 canvases x 16 steps, each appended by causal prefill
    "chained8_bf16": dict(_BASE_BF16, n_layers=8, prefix=0, prompt=512, canvas=256, steps=16, n_canvases=4,
                          renoise_start=0.5, renoise_end=0.0),
    # large pass: 4 layers, H2816, 16q/8kv d128, E128 top-8, F704, V262144; P32768, C256, 8 steps
    "large4_bf16": dict(n_layers=4, hidden=2816, n_q_heads=16, n_kv_heads=8, head_dim=128, n_experts=128, top_k=8,
                        expert_ffn=704, vocab=262144, rope_theta=10000.0, rms_eps=1e-6, dtype="bf16",
                        prefix=32768, canvas=256, steps=8, renoise_start=0.5, renoise_end=0.0),
}

ORDER = ["tiny_fp32", "layer1_bf16", "denoise8_bf16", "chained8_bf16", "large4_bf16"]


def model_fields(cfg: dict) -> dict:
    keys = ("n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "n_experts", "top_k",
            "expert_ffn", "vocab", "rope_theta", "rms_eps", "dtype")
    return {k: cfg[k] for k in keys}


def scaled(cfg: dict, **over) -> dict:
    """A copy of `cfg` with some fields replaced (used for reduced-size parity cases)."""
    out = dict(cfg)
    out.update(over)
    return out
