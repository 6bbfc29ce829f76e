"""The C++ oracle against its independent numpy restatement (oracle/dg_oracle_np.py) on
the same seeded inputs: two programs written separately from the same definitions must
agree to fp64 rounding on every intermediate value, and exactly on every integer
decision (routing, permutation, argmax, re-noise set)."""
import numpy as np
import pytest

from oracle import dg_oracle as O
from oracle import dg_oracle_np as N
from block_diffusion_lm_masked_b200 import configs as CF
from block_diffusion_lm_masked_b200 import synth

SMALL_BF16 = dict(n_layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=128, n_experts=8, top_k=2,
                  expert_ffn=192, vocab=2048, rope_theta=10000.0, rms_eps=1e-6, dtype="bf16")
CONT = ("x_in", "attn_o", "x_attn", "x_out", "router_logits", "topk_w", "router_margin")
DISC = ("topk_idx", "counts", "offsets", "perm")


def _rel(a, b):
    return np.abs(np.asarray(a) - np.asarray(b)).max() / max(np.sqrt(np.mean(np.asarray(b) ** 2)), 1e-300)


def _same_taps(ta, tb):
    for a, b in zip(ta, tb):
        for k in CONT:
            assert _rel(a[k], b[k]) < 1e-12, k
        for k in DISC:
            np.testing.assert_array_equal(a[k], b[k])
        assert a["union"] == b["union"]


@pytest.mark.parametrize("cfg,P,C", [(CF.CONFIGS["tiny_fp32"], 64, 32), (SMALL_BF16, 200, 100), (SMALL_BF16, 0, 37)])
def test_denoise_pass_agrees(cfg, P, C):
    m = synth.Model(cfg)
    kv = synth.prefix_cache(cfg, P)
    canvas = synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(3), C, cfg["vocab"])
    prec_o, prec_n = O.Precision(cfg["dtype"]), N.Precision(cfg["dtype"])
    lo, to = O.denoise_pass(m, O.Cache(kv), canvas, prec_o)
    ln, tn = N.denoise_pass(m, N.Cache(kv), canvas, prec_n)
    assert _rel(lo, ln) < 1e-12
    _same_taps(to, tn)
    n = C // 4
    uo, un = O.canvas_update(lo, n, synth.SEED_RENOISE, 2), N.canvas_update(ln, n, synth.SEED_RENOISE, 2)
    for k in ("canvas", "argmax", "renoised"):
        np.testing.assert_array_equal(uo[k], un[k])
    for k in ("conf", "top_margin", "cut_margin"):
        fin = np.isfinite(un[k])
        np.testing.assert_array_equal(np.isfinite(uo[k]), fin)
        assert np.abs(uo[k][fin] - un[k][fin]).max(initial=0) < 1e-12
    mo = O.canvas_update_masked(lo, canvas, n, 5)
    mn = N.canvas_update_masked(ln, canvas, n, 5)
    for k in ("canvas", "argmax", "kept"):
        np.testing.assert_array_equal(mo[k], mn[k])


def test_prefill_and_full_recompute_agree():
    cfg = SMALL_BF16
    m = synth.Model(cfg)
    kv = synth.prefix_cache(cfg, 61)
    toks = synth.tokens(synth.SEED_TOKENS, 77, 90, cfg["vocab"])
    to, tn = [], []
    a = O.prefill_append(m, O.Cache(kv), toks, O.Precision("bf16"), to)
    b = N.prefill_append(m, N.Cache(kv), toks, N.Precision("bf16"), tn)
    for l in range(cfg["n_layers"]):
        # stored bf16 values: identical except where the fp64 value sits on a rounding tie
        assert np.mean(a.k[l] != b.k[l]) < 1e-4 and np.mean(a.v[l] != b.v[l]) < 1e-4
    for x, y in zip(to, tn):
        np.testing.assert_array_equal(x["topk_idx"], y["topk_idx"])
        np.testing.assert_array_equal(x["perm"], y["perm"])
    ko, vo, lo = O.full_sequence_states(m, toks[:50], toks[50:], O.Precision("bf16"))
    kn, vn, ln = N.full_sequence_states(m, toks[:50], toks[50:], N.Precision("bf16"))
    assert _rel(lo, ln) < 1e-12
    for l in range(cfg["n_layers"]):
        assert np.mean(ko[l] != kn[l]) < 1e-4


def test_primitives_agree():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((7, 48)) * 3
    assert _rel(O.rms_norm(x, 1e-6), N.rms_norm(x, 1e-6)) < 1e-14
    q = rng.standard_normal((4, 9, 16))
    pos = np.arange(100, 109)
    assert _rel(O.rope(q, pos, 1e4), N.rope(q, pos, 1e4)) < 1e-13
    k, v = rng.standard_normal((2, 13, 16)), rng.standard_normal((2, 13, 16))
    mask = N.block_mask(4, 9)[4:]
    np.testing.assert_array_equal(O.block_mask(4, 9), N.block_mask(4, 9))
    np.testing.assert_array_equal(O.causal_rows(5, 6), N.causal_rows(5, 6))
    assert _rel(O.attention(q, k, v, mask), N.attention(q, k, v, mask)) < 1e-13
    lg = rng.standard_normal((20, 10))
    lg[3, 4] = lg[3, 7]   # an exact tie
    for a, b in zip(O.router_topk(lg, 3), N.router_topk(lg, 3)):
        np.testing.assert_allclose(a, b, rtol=1e-14, atol=0)
    idx = O.router_topk(lg, 3)[0]
    for a, b in zip(O.expert_permutation(idx, 10), N.expert_permutation(idx, 10)):
        np.testing.assert_array_equal(a, b)
    z = np.linspace(-30, 30, 101)
    assert _rel(O.silu(z), N.silu(z)) < 1e-15
    vals = rng.standard_normal(5000) * 10.0 ** rng.integers(-30, 30, 5000)
    np.testing.assert_array_equal(O.round_bf16(vals), N.round_bf16(vals))
    for seed, n in ((0, 0), (1234, 17), (2 ** 63 + 5, 2 ** 40)):
        assert O.splitmix64(seed, n) == N.splitmix64(seed, n)
    for args in ((256, 16, 3, 0.5, 0.0), (32, 1, 0, 0.25, 0.25), (256, 8, 7, 0.5, 0.0)):
        assert O.renoise_count(*args) == N.renoise_count(*args)


def test_low_precision_formats_agree():
    rng = np.random.default_rng(6)
    for c in range(256):
        a, b = O.e4m3_decode(c), N.e4m3_decode(c)
        assert (np.isnan(a) and np.isnan(b)) or a == b
    for c in range(16):
        assert O.e2m1_decode(c) == N.e2m1_decode(c)
    x = np.concatenate([rng.standard_normal(3000) * 50, O._E4M3_POS, -O._E4M3_POS,
                        (O._E4M3_POS[1:] + O._E4M3_POS[:-1]) / 2, [1000.0, -1000.0, 0.0, -0.0]])
    np.testing.assert_array_equal(O.e4m3_encode_array(x), N.e4m3_encode_array(x))
    y = np.concatenate([rng.standard_normal(3000) * 3, (O._E2M1_POS[1:] + O._E2M1_POS[:-1]) / 2, [7.0, -9.0]])
    np.testing.assert_array_equal(O.e2m1_encode_array(y), N.e2m1_encode_array(y))
    w = rng.standard_normal((3, 5, 64)) * 0.02
    w[0, 0, :32] = 0.0
    for a, b in zip(O.mx_e4m3_quantize(w), N.mx_e4m3_quantize(w)):
        np.testing.assert_array_equal(a, b)
    co, eo = O.mx_e4m3_quantize(w)
    np.testing.assert_array_equal(O.mx_e4m3_dequantize(co, eo), N.mx_e4m3_dequantize(co, eo))
    qo, qn = O.nvfp4_quantize(w), N.nvfp4_quantize(w)
    np.testing.assert_array_equal(qo[0], qn[0])
    np.testing.assert_array_equal(qo[1], qn[1])
    assert qo[2] == qn[2]
    np.testing.assert_array_equal(O.nvfp4_dequantize(*qo), N.nvfp4_dequantize(*qn))
