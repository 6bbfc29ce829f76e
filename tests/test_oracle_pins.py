"""Pins of the CPU oracle to facts fixed outside it: the pages' worked example and
printed numbers, closed forms, invariants, brute force on tiny inputs and library
routines.  Each test is chosen so that a plausible mistake (dropped term, wrong
sign or index, transposed operand) in the oracle fails it.
"""
import itertools
import math

import numpy as np
import pytest
import torch

from conftest import golden_path
from oracle import dg_oracle as O
from block_diffusion_lm_masked_b200 import roofline as R
from block_diffusion_lm_masked_b200 import synth


def _read_golden(name):
    rows = []
    with open(golden_path(name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ---------------------------------------------------------------- mask

def test_block_mask_matches_worked_example():
    """The printed 7x7 prefix/block mask (P=3 prefix rows, 4 block rows)."""
    want = np.array([[int(v) for v in r] for r in _read_golden("block_mask_p3_c4.txt")], dtype=bool)
    assert want.shape == (7, 7)
    np.testing.assert_array_equal(O.block_mask(3, 4), want)


def test_causal_rows_are_prefix_rows_of_mask():
    # prefill of T tokens after P cached ones = the causal rows P..P+T-1 of a mask with no block
    full = O.block_mask(9, 0)
    np.testing.assert_array_equal(O.causal_rows(4, 5), full[4:9, :9])


# ---------------------------------------------------------------- RNG

def test_splitmix64_known_answers():
    want = [int(r[0], 16) for r in _read_golden("splitmix64_seed0.txt")]
    assert [O.splitmix64(0, i) for i in range(3)] == want
    # the input generator's own implementation agrees with the published values too
    got = synth.splitmix64(0, np.arange(3, dtype=np.uint64))
    assert [int(v) for v in got] == want


def test_renoise_token_is_the_top_bits_of_the_published_draw():
    """At step 0, position p uses draw number p of SplitMix64(seed); the token is the
    multiply-shift of that draw's top 32 bits, so for V = 2^b it is the top b bits."""
    pub = [int(r[0], 16) for r in _read_golden("splitmix64_seed0.txt")]
    for p, x in enumerate(pub):
        assert O.renoise_token(0, 0, p, 1 << 32) == x >> 32
        assert O.renoise_token(0, 0, p, 2) == x >> 63
        assert O.renoise_token(0, 0, p, 1 << 10) == x >> 54
        assert O.renoise_token(0, 0, p, 1000) == (x >> 32) * 1000 // (1 << 32)


def test_renoise_tokens_uniform_chi2():
    V, n = 64, 64 * 400
    draws = [O.renoise_token(1236, s, p, V) for s in range(4) for p in range(n // 4)]
    counts = np.bincount(draws, minlength=V)
    exp = n / V
    chi2 = ((counts - exp) ** 2 / exp).sum()
    # 63 degrees of freedom: mean 63, sd ~11.2; 130 is > 6 sd out
    assert chi2 < 130
    assert min(draws) >= 0 and max(draws) < V


def test_renoise_tokens_in_range_for_non_power_of_two():
    V = 1000
    toks = [O.renoise_token(7, 3, p, V) for p in range(5000)]
    assert 0 <= min(toks) and max(toks) < V
    assert len(set(toks)) > 900


# ---------------------------------------------------------------- rounding

def test_round_bf16_ties_and_library():
    assert O.round_bf16(np.array([1.0]))[0] == 1.0
    assert O.round_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 1.0                    # tie -> even
    assert O.round_bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6    # tie -> even (up)
    assert O.round_bf16(np.array([-1.0 - 2.0 ** -8 - 2.0 ** -20]))[0] == -1.0 - 2.0 ** -7
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))).astype(np.float32)
    lib = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_bf16(x.astype(np.float64)), lib)


def test_widen_bf16_bits():
    bits = np.array([0x3F80, 0xBF80, 0x4049, 0x0000], dtype=np.uint16)
    np.testing.assert_array_equal(O.widen(bits), [1.0, -1.0, 3.140625, 0.0])


# ---------------------------------------------------------------- norms, rope, silu

def test_rms_norm_closed_forms():
    x = np.full((1, 8), 3.0)
    np.testing.assert_allclose(O.rms_norm(x, 1e-6), 3.0 / np.sqrt(9.0 + 1e-6), rtol=1e-15)
    rng = np.random.default_rng(1)
    y = O.rms_norm(rng.standard_normal((5, 64)) * 7.0, 0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=1), 1.0, rtol=1e-12)


def test_rope_closed_form_and_relative_position():
    # d = 2: the single pair rotates by the position itself
    x = np.array([[[1.0, 0.0]]] * 1)
    for pos in (0, 1, 5):
        r = O.rope(x, np.array([pos]), 10000.0)
        np.testing.assert_allclose(r[0, 0], [math.cos(pos), math.sin(pos)], atol=1e-15)
    # pair i rotates at theta^(-2i/d); rotate-half pairs (i, i + d/2)
    d, theta = 8, 100.0
    e = np.zeros((1, 1, d))
    e[0, 0, 1] = 1.0
    r = O.rope(e, np.array([3]), theta)[0, 0]
    ang = 3 * theta ** (-2.0 / d)
    np.testing.assert_allclose(r[[1, 1 + d // 2]], [math.cos(ang), math.sin(ang)], atol=1e-14)
    assert np.abs(np.delete(r, [1, 1 + d // 2])).max() == 0.0
    # dot products depend on the position difference only, norms are preserved
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 1, 16))
    k = rng.standard_normal((1, 1, 16))
    dots = [float(O.rope(q, np.array([m]), 1e4)[0, 0] @ O.rope(k, np.array([m - 3]), 1e4)[0, 0])
            for m in (3, 10, 77, 1000)]
    np.testing.assert_allclose(dots, dots[0], rtol=1e-9)
    np.testing.assert_allclose(np.linalg.norm(O.rope(q, np.array([12345]), 1e4)), np.linalg.norm(q), rtol=1e-12)


def test_rope_composes_as_a_rotation_and_norm_is_scale_free():
    """RoPE at p1 then at p2 is RoPE at p1 + p2 (each pair turns by an angle linear in the
    position); RMSNorm without eps ignores the scale of its input."""
    rng = np.random.default_rng(12)
    x = rng.standard_normal((2, 3, 16))
    for p1, p2 in ((0, 5), (7, 11), (1000, 24)):
        a = O.rope(O.rope(x, np.array([p1] * 3), 1e4), np.array([p2] * 3), 1e4)
        np.testing.assert_allclose(a, O.rope(x, np.array([p1 + p2] * 3), 1e4), rtol=1e-9, atol=1e-12)
    y = rng.standard_normal((4, 32))
    np.testing.assert_allclose(O.rms_norm(7.5 * y, 0.0), O.rms_norm(y, 0.0), rtol=1e-13)


def test_attention_ignores_an_equal_shift_of_a_rows_scores():
    """Adding c q / |q|^2 to every key raises each of that query's scores by the same
    c / sqrt(d): the softmax, hence the output row, does not change."""
    rng = np.random.default_rng(13)
    d = 16
    q = rng.standard_normal((1, 1, d))
    k = rng.standard_normal((1, 7, d))
    v = rng.standard_normal((1, 7, d))
    allowed = np.ones((1, 7), dtype=bool)
    shifted = k + 3.0 * q[0, 0] / np.dot(q[0, 0], q[0, 0])
    np.testing.assert_allclose(O.attention(q, shifted, v, allowed), O.attention(q, k, v, allowed), rtol=1e-12)


def test_silu_closed_forms():
    np.testing.assert_allclose(O.silu(np.array([0.0, 50.0, -50.0, 1.0])),
                               [0.0, 50.0, -50.0 * math.exp(-50.0) / (1 + math.exp(-50.0)), 1 / (1 + math.exp(-1))],
                               rtol=1e-12, atol=1e-300)


# ---------------------------------------------------------------- attention

def test_attention_closed_forms():
    rng = np.random.default_rng(3)
    d = 16
    # all keys equal -> uniform weights -> mean of the allowed values
    q = rng.standard_normal((1, 2, d))
    k = np.tile(rng.standard_normal((1, 1, d)), (1, 5, 1))
    v = rng.standard_normal((1, 5, d))
    allowed = np.array([[1, 1, 1, 0, 0], [1, 1, 1, 1, 1]], dtype=bool)
    o = O.attention(q, k, v, allowed)
    np.testing.assert_allclose(o[0, 0], v[0, :3].mean(axis=0), rtol=1e-12)
    np.testing.assert_allclose(o[0, 1], v[0].mean(axis=0), rtol=1e-12)
    # one allowed key -> that value
    o1 = O.attention(q, rng.standard_normal((1, 5, d)), v, np.eye(2, 5, 2, dtype=bool))
    np.testing.assert_allclose(o1[0, 0], v[0, 2], rtol=1e-12)
    np.testing.assert_allclose(o1[0, 1], v[0, 3], rtol=1e-12)


def test_attention_two_keys_logistic_scale():
    d = 4
    q = np.zeros((1, 1, d)); q[0, 0, 0] = 1.0
    k = np.zeros((1, 2, d)); k[0, 0, 0] = 3.0; k[0, 1, 0] = -1.0
    v = np.zeros((1, 2, d)); v[0, 0, 1] = 1.0; v[0, 1, 2] = 1.0
    o = O.attention(q, k, v, np.ones((1, 2), dtype=bool))
    p0 = 1.0 / (1.0 + math.exp((-1.0 - 3.0) / math.sqrt(d)))
    np.testing.assert_allclose(o[0, 0], [0.0, p0, 1 - p0, 0.0], rtol=1e-12)


def test_attention_gqa_head_mapping():
    # 4 query heads, 2 kv heads: heads 0,1 read kv 0; heads 2,3 read kv 1 (contiguous groups)
    rng = np.random.default_rng(4)
    q = rng.standard_normal((4, 3, 8))
    k = rng.standard_normal((2, 6, 8))
    v = np.zeros((2, 6, 8)); v[0] += 1.5; v[1] -= 2.5
    o = O.attention(q, k, v, np.ones((3, 6), dtype=bool))
    np.testing.assert_allclose(o[:2], 1.5, rtol=1e-12)
    np.testing.assert_allclose(o[2:], -2.5, rtol=1e-12)


def test_attention_block_rows_bidirectional_prefix_rows_causal():
    rng = np.random.default_rng(5)
    P, C, d = 3, 4, 8
    q = rng.standard_normal((1, P + C, d)); k = rng.standard_normal((1, P + C, d)); v = rng.standard_normal((1, P + C, d))
    m = O.block_mask(P, C)
    base = O.attention(q, k, v, m)
    # perturbing the last block key changes every block row but no prefix row
    k2 = k.copy(); k2[0, -1] += 1.0
    pert = O.attention(q, k2, v, m)
    np.testing.assert_array_equal(pert[0, :P], base[0, :P])
    assert np.all(np.abs(pert[0, P:] - base[0, P:]).max(axis=1) > 0)
    # permuting block keys/values together leaves block rows unchanged (bidirectional, no order)
    perm = np.concatenate([np.arange(P), P + rng.permutation(C)])
    np.testing.assert_allclose(O.attention(q, k[:, perm], v[:, perm], m)[0, P:], base[0, P:], rtol=1e-12)


# ---------------------------------------------------------------- router / permutation

def test_router_topk_brute_force_subsets():
    rng = np.random.default_rng(6)
    for E, k in ((6, 2), (7, 3), (5, 1)):
        logits = rng.standard_normal((20, E))
        idx, w, margin = O.router_topk(logits, k)
        for t in range(20):
            best = max(itertools.combinations(range(E), k), key=lambda s: sum(logits[t, list(s)]))
            assert set(idx[t]) == set(best)
            srt = sorted(logits[t], reverse=True)
            assert margin[t] == pytest.approx(srt[k - 1] - srt[k])
            ch = logits[t, idx[t]]
            assert list(ch) == sorted(ch, reverse=True)
            np.testing.assert_allclose(w[t], np.exp(ch) / np.exp(ch).sum(), rtol=1e-12)


def test_router_topk_special_cases():
    lg = np.array([[0.3, -1.0, 2.0, 0.5]])
    idx, w, _ = O.router_topk(lg, 4)           # k = E: dense mixture = full softmax
    np.testing.assert_allclose(w[0], np.exp(lg[0, idx[0]]) / np.exp(lg[0]).sum(), rtol=1e-12)
    idx1, w1, _ = O.router_topk(lg, 1)         # k = 1: single expert, weight 1
    assert idx1[0, 0] == 2 and w1[0, 0] == 1.0
    idxt, _, mt = O.router_topk(np.zeros((1, 5)), 2)   # all tied: lowest ids
    assert list(idxt[0]) == [0, 1] and mt[0] == 0.0


def test_expert_permutation_invariants():
    rng = np.random.default_rng(7)
    T, k, E = 37, 3, 9
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    counts, offsets, perm, inv, union = O.expert_permutation(idx, E)
    assert counts.sum() == T * k
    assert sorted(perm.tolist()) == list(range(T * k))
    assert union == len({int(e) for e in idx.reshape(-1)})
    assert k <= union <= min(E, T * k)
    flat = idx.reshape(-1)
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert all(flat[a] == e for a in seg)
        assert list(seg) == sorted(seg)        # (token, slot) ascending within an expert
    np.testing.assert_array_equal(perm[inv], np.arange(T * k))


# ---------------------------------------------------------------- MoE

def _tiny_cfg(**over):
    cfg = dict(n_layers=1, hidden=16, n_q_heads=2, n_kv_heads=1, head_dim=8, n_experts=4, top_k=2,
               expert_ffn=12, vocab=40, rope_theta=10000.0, rms_eps=1e-6, dtype="f32")
    cfg.update(over)
    return cfg


class _M:
    def __init__(self, cfg, seed=11):
        rng = np.random.default_rng(seed)
        H, nq, nkv, d, E, F, V = (cfg[x] for x in ("hidden", "n_q_heads", "n_kv_heads", "head_dim",
                                                   "n_experts", "expert_ffn", "vocab"))
        self.cfg = cfg
        self.embed = rng.standard_normal((V, H)) * 0.5
        self.w_out = rng.standard_normal((V, H)) * 0.3
        self.layers = [dict(w_q=rng.standard_normal((nq * d, H)) * 0.3, w_k=rng.standard_normal((nkv * d, H)) * 0.3,
                            w_v=rng.standard_normal((nkv * d, H)) * 0.3, w_o=rng.standard_normal((H, nq * d)) * 0.3,
                            w_router=rng.standard_normal((E, H)), w_gate=rng.standard_normal((E, F, H)) * 0.3,
                            w_up=rng.standard_normal((E, F, H)) * 0.3, w_down=rng.standard_normal((E, H, F)) * 0.3)
                       for _ in range(cfg["n_layers"])]


def _swiglu(x, wg, wu, wd):
    g = x @ wg.T
    return ((g / (1 + np.exp(-g))) * (x @ wu.T)) @ wd.T


def test_moe_identical_experts_equals_dense_swiglu():
    cfg = _tiny_cfg()
    m = _M(cfg)
    L = m.layers[0]
    for e in range(1, cfg["n_experts"]):
        L["w_gate"][e] = L["w_gate"][0]; L["w_up"][e] = L["w_up"][0]; L["w_down"][e] = L["w_down"][0]
    x = np.random.default_rng(8).standard_normal((9, cfg["hidden"]))
    xn = x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + cfg["rms_eps"])
    got = O.moe(m, 0, x, O.Precision("f32"))
    np.testing.assert_allclose(got, _swiglu(xn, L["w_gate"][0], L["w_up"][0], L["w_down"][0]), rtol=1e-12, atol=1e-13)


def test_moe_router_reads_the_normed_residual():
    """Pre-norm MoE (reading #1): the block sees the residual only through its RMSNorm, so
    with eps = 0 scaling a token's residual by any c > 0 changes neither its routing (the
    router logits, hence the top-k and their softmax weights) nor its FFN output."""
    cfg = _tiny_cfg(rms_eps=0.0, n_experts=6, top_k=3)
    m = _M(cfg)
    x = np.random.default_rng(21).standard_normal((8, cfg["hidden"]))
    c = np.array([0.25, 0.5, 1.0, 3.0, 7.0, 0.1, 2.0, 40.0])[:, None]
    a = O.moe_block(m, 0, x, O.Precision("f32"))
    b = O.moe_block(m, 0, c * x, O.Precision("f32"))
    np.testing.assert_allclose(b["router_logits"], a["router_logits"], rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(b["topk_idx"], a["topk_idx"])
    np.testing.assert_allclose(b["topk_w"], a["topk_w"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(b["ffn"], a["ffn"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(b["x_out"], c * x + a["ffn"], rtol=1e-11, atol=1e-11)


def test_moe_k1_routes_each_token_to_its_argmax_expert():
    cfg = _tiny_cfg(top_k=1)
    m = _M(cfg)
    L = m.layers[0]
    x = np.random.default_rng(9).standard_normal((7, cfg["hidden"]))
    xn = x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + cfg["rms_eps"])
    got = O.moe(m, 0, x, O.Precision("f32"))
    for t in range(7):
        e = int(np.argmax(xn[t] @ L["w_router"].T))
        want = _swiglu(xn[t:t + 1], L["w_gate"][e], L["w_up"][e], L["w_down"][e])[0]
        np.testing.assert_allclose(got[t], want, rtol=1e-12, atol=1e-13)


def test_moe_combine_pairs_each_weight_with_its_expert():
    """Experts that differ only by a scale c_e of their down projection: the MoE output of
    token t is (sum_j w[t,j] c_{e_j}) times one SwiGLU, with the top-k and the weights
    found here by brute force over each token's router logits."""
    cfg = _tiny_cfg(n_experts=5, top_k=3)
    m = _M(cfg)
    L = m.layers[0]
    c = np.array([1.0, 2.0, 4.0, 8.0, 16.0])
    for e in range(5):
        L["w_gate"][e] = L["w_gate"][0]; L["w_up"][e] = L["w_up"][0]; L["w_down"][e] = c[e] * L["w_down"][0]
    x = np.random.default_rng(12).standard_normal((11, cfg["hidden"]))
    xn = x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + cfg["rms_eps"])
    got = O.moe(m, 0, x, O.Precision("f32"))
    base = _swiglu(xn, L["w_gate"][0], L["w_up"][0], L["w_down"][0])
    for t in range(11):
        r = (xn[t] @ L["w_router"].T).tolist()
        top = sorted(range(5), key=lambda e: (-r[e], e))[:3]
        z = [math.exp(r[e] - r[top[0]]) for e in top]
        scale = sum(zi / sum(z) * c[e] for zi, e in zip(z, top))
        np.testing.assert_allclose(got[t], scale * base[t], rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- whole pass

def test_single_token_pass_closed_form():
    """C=1, empty cache, one expert: attention over one key returns its value, so the
    pass reduces to plain matrix products written out here."""
    cfg = _tiny_cfg(n_experts=1, top_k=1, n_q_heads=2, n_kv_heads=1)
    m = _M(cfg)
    L = m.layers[0]
    tok = np.array([17])
    logits, _ = O.denoise_pass(m, O.Cache.empty(cfg), tok, O.Precision("f32"))
    eps = cfg["rms_eps"]
    nrm = lambda z: z / np.sqrt(np.mean(z * z) + eps)
    x = m.embed[17].copy()
    v = nrm(x) @ L["w_v"].T                     # one kv head, position 0 (no rotation of v)
    x = x + np.concatenate([v, v]) @ L["w_o"].T   # both query heads read that kv head
    x = x + _swiglu(nrm(x)[None], L["w_gate"][0], L["w_up"][0], L["w_down"][0])[0]
    np.testing.assert_allclose(logits[0], nrm(x) @ m.w_out.T, rtol=1e-11, atol=1e-12)


def test_attention_sees_relative_positions_only():
    """RoPE rotates q and k by their absolute positions, so q.k depends on the positions'
    difference only: shifting every position by the same amount leaves the attention
    output unchanged, while changing the spacing changes it.  (Rotating v as well, or
    leaving k unrotated, breaks the first; no rotation at all breaks the second.)"""
    cfg = _tiny_cfg(n_q_heads=2, n_kv_heads=1)
    m = _M(cfg)
    x = np.random.default_rng(5).standard_normal((6, cfg["hidden"]))
    prec = O.Precision("f32")
    allowed = np.ones((6, 6), dtype=bool)

    def out(pos):
        q, k, v = O._qkv(m, 0, x, np.asarray(pos), prec)
        return O._attn_out(m, 0, O.attention(q, k, v, allowed), prec)
    base = out(np.arange(6) + 3)
    np.testing.assert_allclose(out(np.arange(6) + 1000), base, rtol=1e-9, atol=1e-12)
    assert np.abs(out(2 * np.arange(6) + 3) - base).max() > 1e-3 * np.abs(base).max()


def test_block_scales_stay_with_their_blocks():
    """Rows whose 32- (MX) or 16-element (NVFP4) blocks differ in magnitude by powers of two:
    every dequantised element is within its own block's rounding bound, which a scale
    taken from the neighbouring block, or one scale per row, violates."""
    rng = np.random.default_rng(47)
    kx = rng.integers(-12, 13, size=(5, 8))                                # per-block magnitudes
    w = rng.standard_normal((5, 8, 32)) * np.ldexp(1.0, kx)[..., None]
    w = w.reshape(5, 256)
    codes, exp = O.mx_e4m3_quantize(w)
    dq = O.mx_e4m3_dequantize(codes, exp)
    amax = np.repeat(np.abs(w).reshape(5, 8, 32).max(axis=-1), 32, axis=-1).reshape(w.shape)
    X = np.repeat(np.ldexp(1.0, exp), 32, axis=-1).reshape(w.shape)
    # E4M3 keeps 3 mantissa bits down to 2^-6 of the scale: each error within 2^-4 |w| or the
    # subnormal step 2^-9 X (X <= amax / 2^8), plus what saturation at 448 X cuts off
    sat = np.maximum(np.abs(w) - 448.0 * X, 0.0)
    assert np.all(np.abs(dq - w) <= 2.0 ** -4 * np.abs(w) + 2.0 ** -17 * amax + sat)
    kn = rng.integers(-6, 7, size=(4, 8))
    w4 = (rng.standard_normal((4, 8, 16)) * np.ldexp(1.0, kn)[..., None]).reshape(4, 128)
    c4, sc4, g4 = O.nvfp4_quantize(w4)
    dq4 = O.nvfp4_dequantize(c4, sc4, g4)
    amax4 = np.repeat(np.abs(w4).reshape(4, 8, 16).max(axis=-1), 16, axis=-1).reshape(w4.shape)
    # E2M1: half a step, at most a sixth of the block's largest magnitude, plus the block
    # scale's own E4M3 rounding
    assert np.all(np.abs(dq4 - w4) <= (1 / 6 + 2.0 ** -4) * amax4 + 1e-12)


def test_zero_mixing_weights_pass_is_embedding_readout():
    cfg = _tiny_cfg(n_layers=2)
    m = _M(cfg)
    for L in m.layers:
        L["w_o"][:] = 0.0
        L["w_down"][:] = 0.0
    toks = np.array([3, 9, 3, 27, 0])
    cache = O.Cache([(np.random.default_rng(1).standard_normal((1, 6, 8)),) * 2] * 2)
    logits, _ = O.denoise_pass(m, cache, toks, O.Precision("f32"))
    e = m.embed[toks]
    np.testing.assert_allclose(logits, (e / np.sqrt(np.mean(e * e, axis=1, keepdims=True) + 1e-6)) @ m.w_out.T,
                               rtol=1e-12)


def test_prefix_kv_reuse_equals_full_recompute():
    """The cached path (causal prefill of the prefix, then a denoising pass against the
    cache) equals recomputing prefix and block together under the prefix/block mask."""
    cfg = _tiny_cfg(n_layers=2)
    m = _M(cfg)
    pre = np.array([5, 1, 33, 8, 20, 2])
    can = np.array([11, 39, 0, 7])
    prec = O.Precision("f32")
    cache = O.prefill_append(m, O.Cache.empty(cfg), pre, prec)
    logits, _ = O.denoise_pass(m, cache, can, prec)
    ks, vs, full_logits = O.full_sequence_states(m, pre, can, prec)
    P = len(pre)
    for l in range(cfg["n_layers"]):
        np.testing.assert_allclose(cache.k[l], ks[l][:, :P], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(cache.v[l], vs[l][:, :P], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(logits, full_logits, rtol=1e-10, atol=1e-11)


def test_chunked_prefill_equals_single_prefill():
    """Causality: prefilling 3 then 5 tokens gives the K/V of prefilling all 8 at once
    (exactly when nothing is rounded; with bf16 storage the second chunk reads the first
    chunk's K/V as stored, so the two agree to bf16 rounding)."""
    cfg = _tiny_cfg(n_layers=2)
    m = _M(cfg)
    toks = np.array([4, 8, 15, 16, 23, 42 % 40, 1, 2])
    for dt, tol in (("f32", 1e-12), ("bf16", 2e-2)):
        prec = O.Precision(dt)
        one = O.prefill_append(m, O.Cache.empty(cfg), toks, prec)
        two = O.prefill_append(m, O.prefill_append(m, O.Cache.empty(cfg), toks[:3], prec), toks[3:], prec)
        for l in range(2):
            np.testing.assert_allclose(two.k[l], one.k[l], rtol=tol, atol=tol)
            np.testing.assert_allclose(two.v[l], one.v[l], rtol=tol, atol=tol)


def _is_nearest_bf16(stored, exact):
    """Each stored value has 8 significant bits and lies within half a bf16 step of the exact one."""
    st = np.asarray(stored, dtype=np.float64)
    bits = st.astype(np.float32).view(np.uint32)
    representable = np.all(st.astype(np.float32).astype(np.float64) == st) and np.all((bits & 0xFFFF) == 0)
    _, e = np.frexp(exact)
    half_step = np.ldexp(1.0, e - 9)
    return representable and bool(np.all(np.abs(st - exact) <= half_step))


def test_bf16_storage_rounds_what_prefill_writes_and_nothing_in_flight():
    """The storage rule in a bf16 model: prefill rounds the K/V it writes to the nearest
    bf16 value and nothing else, so its residual stream matches the f32 model's; a
    denoising pass rounds nothing at all (canvas K/V, vocabulary input in flight), so
    against a given cache the two precisions give the same logits, the plain product of
    the normed final state and the output matrix."""
    cfg = _tiny_cfg(n_layers=2)
    m = _M(cfg)
    toks = np.array([4, 8, 15, 16, 23, 2])
    f32, b16 = O.Precision("f32"), O.Precision("bf16")
    exact = O.prefill_append(m, O.Cache.empty(cfg), toks, f32)
    stored = O.prefill_append(m, O.Cache.empty(cfg), toks, b16)
    for l in range(2):
        for a, b in ((stored.k[l], exact.k[l]), (stored.v[l], exact.v[l])):
            assert _is_nearest_bf16(a, b)
            assert np.abs(a - b).max() > 0
    can = np.array([7, 30, 1])
    lf, tf = O.denoise_pass(m, stored, can, f32)
    lb, tb = O.denoise_pass(m, stored, can, b16)
    for a, b in zip(tf, tb):
        for key in ("attn_o", "x_attn", "x_out"):
            np.testing.assert_array_equal(a[key], b[key])
    xn = O.rms_norm(tf[-1]["x_out"], cfg["rms_eps"])
    np.testing.assert_allclose(lb, xn @ m.w_out.T, rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(lb, lf)


def test_denoise_pass_leaves_cache_untouched():
    cfg = _tiny_cfg()
    m = _M(cfg)
    cache = O.prefill_append(m, O.Cache.empty(cfg), np.array([1, 2, 3]), O.Precision("f32"))
    before = cache.copy()
    O.denoise_pass(m, cache, np.array([4, 5]), O.Precision("f32"))
    for l in range(cfg["n_layers"]):
        np.testing.assert_array_equal(cache.k[l], before.k[l])
        np.testing.assert_array_equal(cache.v[l], before.v[l])


# ---------------------------------------------------------------- several canvases

def test_batch_reads_the_union_of_the_canvases_experts():
    """A batch of canvases groups all rows by expert at once: its histogram is the sum of
    the canvases' histograms and the experts it reads are the set union of theirs, never
    more than the sum of the per-canvas unions (the bytes a batch saves)."""
    cfg = _tiny_cfg(n_layers=2, n_experts=8, top_k=2)
    m = _M(cfg)
    prec = O.Precision("f32")
    rng = np.random.default_rng(21)
    caches = [O.prefill_append(m, O.Cache.empty(cfg), rng.integers(0, 40, P), prec) if P else O.Cache.empty(cfg)
              for P in (3, 0, 7)]
    canvases = [rng.integers(0, 40, 5) for _ in range(3)]
    res = O.denoise_pass_batched(m, caches, canvases, prec)
    merged = O.merge_batch_taps([t for _, t in res], cfg["n_experts"])
    for l in range(2):
        sets = [set(t[l]["topk_idx"].reshape(-1).tolist()) for _, t in res]
        assert merged[l]["union"] == len(set().union(*sets)) <= sum(len(x) for x in sets)
        np.testing.assert_array_equal(merged[l]["counts"], sum(t[l]["counts"] for _, t in res))
        assert merged[l]["counts"].sum() == 3 * 5 * 2
        # the batch permutation is the stable grouping of the stacked routing
        flat = merged[l]["topk_idx"].reshape(-1)
        assert list(merged[l]["perm"]) == sorted(range(flat.size), key=lambda a: (int(flat[a]), a))


def test_batched_canvases_do_not_see_each_other():
    """Each canvas of a batch is its own request: replacing another canvas's tokens or
    cache leaves its logits exactly unchanged, and a batch of one is the single pass."""
    cfg = _tiny_cfg(n_layers=2)
    m = _M(cfg)
    prec = O.Precision("f32")
    rng = np.random.default_rng(22)
    c0 = O.prefill_append(m, O.Cache.empty(cfg), rng.integers(0, 40, 4), prec)
    c1 = O.prefill_append(m, O.Cache.empty(cfg), rng.integers(0, 40, 6), prec)
    x0, x1 = rng.integers(0, 40, 5), rng.integers(0, 40, 5)
    a = O.denoise_pass_batched(m, [c0, c1], [x0, x1], prec)
    b = O.denoise_pass_batched(m, [c0, O.Cache.empty(cfg)], [x0, rng.integers(0, 40, 5)], prec)
    np.testing.assert_array_equal(a[0][0], b[0][0])
    for (lg, _), c, x in zip(a, (c0, c1), (x0, x1)):     # every canvas is its own single pass
        single, _ = O.denoise_pass(m, c, x, prec)
        np.testing.assert_array_equal(lg, single)
    outs, caches = O.generate_canvases(m, [c0, c1], [x0, x1], 3, 0.5, 0.0, [5, 6], prec, True)
    one, cache_one = O.generate_canvas(m, c1, x1, 3, 0.5, 0.0, 6, prec, True)
    np.testing.assert_array_equal(outs[1], one)
    assert caches[0].len == c0.len + 5 and caches[1].len == cache_one.len


# ---------------------------------------------------------------- canvas update
# ---------------------------------------------------------------- canvas update

def test_canvas_update_special_cases():
    rng = np.random.default_rng(10)
    C, V = 12, 50
    lg = rng.standard_normal((C, V))
    u0 = O.canvas_update(lg, 0, 99, 0)
    np.testing.assert_array_equal(u0["canvas"], np.argmax(lg, axis=1))
    uc = O.canvas_update(lg, C, 99, 5)
    np.testing.assert_array_equal(uc["canvas"], [O.renoise_token(99, 5, i, V) for i in range(C)])
    # confidence closed form: one logit a, the rest 0
    lg2 = np.zeros((2, V)); lg2[0, 3] = 2.0; lg2[1, 7] = 40.0
    u2 = O.canvas_update(lg2, 0, 1, 0)
    np.testing.assert_allclose(u2["conf"][0], math.exp(2.0) / (math.exp(2.0) + V - 1), rtol=1e-14)
    assert u2["conf"][1] == pytest.approx(1.0, abs=1e-15)
    assert list(u2["argmax"]) == [3, 7]
    # ties: argmax takes the lowest id; equal confidences re-noise lower positions first
    u3 = O.canvas_update(np.zeros((4, 6)), 2, 1, 0)
    assert list(u3["argmax"]) == [0, 0, 0, 0] and list(u3["renoised"]) == [0, 1]


def test_canvas_update_ignores_a_constant_added_to_a_row():
    rng = np.random.default_rng(14)
    lg = rng.standard_normal((9, 33)) * 3
    shift = rng.standard_normal((9, 1)) * 100
    a, b = O.canvas_update(lg, 4, 3, 1), O.canvas_update(lg + shift, 4, 3, 1)
    np.testing.assert_array_equal(a["canvas"], b["canvas"])
    np.testing.assert_allclose(a["conf"], b["conf"], rtol=1e-10)


def test_canvas_update_renoise_set_brute_force():
    rng = np.random.default_rng(11)
    C, V, n = 30, 20, 11
    lg = rng.standard_normal((C, V)) * 2
    u = O.canvas_update(lg, n, 5, 3)
    conf = [math.exp(max(r)) / sum(math.exp(x) for x in r) for r in lg.tolist()]
    want = sorted(sorted(range(C), key=lambda i: (conf[i], i))[:n])
    assert list(u["renoised"]) == want
    keep = [i for i in range(C) if i not in want]
    assert all(u["canvas"][i] == int(np.argmax(lg[i])) for i in keep)
    assert all(u["cut_margin"] >= 0)


def _masked_example():
    rec = {}
    with open(golden_path("masked_update_example.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, _, rest = line.partition(" ")
            rec[key] = rest.strip()
    logits = np.array([[float(v) for v in row.split()] for row in rec["logits"].split("|")])
    return (logits, np.array(rec["canvas_in"].split(), dtype=np.int64), int(rec["mask_id"]), int(rec["n_keep"]),
            np.array(rec["canvas_out"].split(), dtype=np.int64), rec["conf"].split())


def test_masked_update_worked_example():
    logits, cin, mask_id, n_keep, cout, conf = _masked_example()
    got = O.canvas_update_masked(logits, cin, n_keep, mask_id)
    np.testing.assert_array_equal(got["canvas"], cout)
    for i, c in enumerate(conf):
        if c != "-":
            assert abs(got["conf"][i] - float(c)) < 5e-7
    np.testing.assert_array_equal(got["kept"], [0])


def test_masked_update_special_cases():
    rng = np.random.default_rng(31)
    C, V, mask_id = 40, 97, 96
    logits = rng.standard_normal((C, V)) * 3.0
    canvas = np.where(rng.random(C) < 0.6, mask_id, rng.integers(0, mask_id, C))
    masked = canvas == mask_id
    # n_keep = 0: every masked position takes its best non-mask token; locked ones keep theirs
    got = O.canvas_update_masked(logits, canvas, 0, mask_id)
    want = np.where(masked, np.argmax(logits[:, :mask_id], axis=1), canvas)
    np.testing.assert_array_equal(got["canvas"], want)
    # n_keep >= M: nothing changes
    np.testing.assert_array_equal(O.canvas_update_masked(logits, canvas, C, mask_id)["canvas"], canvas)
    # the mask id is never a fill value, even where it has the largest logit
    big = logits.copy()
    big[:, mask_id] = 50.0
    g2 = O.canvas_update_masked(big, canvas, 0, mask_id)
    np.testing.assert_array_equal(g2["canvas"], want)
    assert np.all(g2["conf"] < 1e-15)
    # a single dominant logit: confidence 1
    one = np.full((C, V), -1e4)
    one[np.arange(C), np.arange(C) % mask_id] = 0.0
    assert np.allclose(O.canvas_update_masked(one, canvas, 0, mask_id)["conf"], 1.0)


def test_masked_schedule_unmasks_to_zero_and_locks():
    """From an all-[MASK] canvas, the keep counts renoise_count(C, S, s, (S-1)/S, 0) leave
    exactly that many positions masked after pass s (C/S fewer per pass), none at the
    end, and a filled position never changes again."""
    rng = np.random.default_rng(32)
    C, V, S, mask_id = 64, 50, 8, 49
    cur = np.full(C, mask_id)
    for s in range(S):
        n = O.renoise_count(C, S, s, (S - 1) / S, 0.0)
        nxt = O.canvas_update_masked(rng.standard_normal((C, V)), cur, n, mask_id)["canvas"]
        filled = cur != mask_id
        np.testing.assert_array_equal(nxt[filled], cur[filled])
        assert int((nxt == mask_id).sum()) == n == C * (S - 1 - s) // S
        cur = nxt
    assert not np.any(cur == mask_id)


def test_generate_masked_loop_properties():
    """The masked generation loop on a tiny model: it starts from an all-[MASK] canvas,
    leaves exactly the scheduled number masked after each pass, never changes a filled
    position, ends with none masked, and appends the final canvas."""
    cfg = _tiny_cfg(n_layers=1)
    m = _M(cfg)
    C, S, mask_id = 12, 4, cfg["vocab"] - 1
    rec = []
    cache0 = O.Cache.empty(cfg)
    out, cache = O.generate_canvas_masked(m, cache0, C, S, (S - 1) / S, 0.0, mask_id, O.Precision("f32"), True, rec)
    assert len(rec) == S and np.all(rec[0]["canvas_in"] == mask_id)
    for r in rec:
        cin, cout = r["canvas_in"], r["update"]["canvas"]
        assert int((cout == mask_id).sum()) == r["n"] == C * (S - 1 - r["step"]) // S
        filled = cin != mask_id
        np.testing.assert_array_equal(cout[filled], cin[filled])
    assert not np.any(out == mask_id)
    assert cache.len == C


def test_resume_from_a_middle_pass_reproduces_the_run():
    """The generation state is (cache, canvas, pass index, seed): the re-noise draws are
    counter-based on (seed, pass, position), so restarting at pass s from the canvas the
    run had there gives the same final canvas."""
    cfg = _tiny_cfg(n_layers=1)
    m = _M(cfg)
    S, prec, seed = 5, O.Precision("f32"), 99
    cache = O.Cache.empty(cfg)
    start = np.random.default_rng(3).integers(0, cfg["vocab"], 10).astype(np.int32)
    rec = []
    full, _ = O.generate_canvas(m, cache, start, S, 0.5, 0.0, seed, prec, False, rec)
    for s0 in (1, 3):
        cur = rec[s0]["canvas_in"].copy()
        for s in range(s0, S):
            logits, _ = O.denoise_pass(m, cache, cur, prec)
            cur = O.canvas_update(logits, O.renoise_count(len(cur), S, s, 0.5, 0.0), seed, s)["canvas"]
        np.testing.assert_array_equal(cur, full)


def test_e4m3_decode_closed_forms():
    d = O.e4m3_decode
    assert d(0x00) == 0.0 and np.signbit(d(0x80)) and d(0x80) == 0.0
    assert d(0x01) == 2.0 ** -9 and d(0x07) == 7 * 2.0 ** -9       # subnormals
    assert d(0x08) == 2.0 ** -6 and d(0x0F) == 1.875 * 2.0 ** -6   # smallest binade of normals
    assert d(0x38) == 1.0 and d(0x39) == 1.125 and d(0x7E) == 448.0
    assert np.isnan(d(0x7F)) and np.isnan(d(0xFF))
    assert d(np.uint8(0x30)) == 0.5                                # numpy integer codes decode the same
    pos = [d(c) for c in range(0x7F)]
    assert all(a < b for a, b in zip(pos, pos[1:]))
    for c in range(0x7F):
        assert d(c | 0x80) == -d(c)
    # within a binade the spacing is 2^(e-7) / 8
    for e in range(1, 15):
        vals = [d((e << 3) | m) for m in range(8)]
        assert np.allclose(np.diff(vals), 2.0 ** (e - 7) / 8, rtol=0, atol=0)


def test_e4m3_encode_round_trip_rounding_saturation():
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert O.e4m3_encode(O.e4m3_decode(c)) == c
    enc = O.e4m3_encode
    assert enc(1.0625) == 0x38 and enc(1.1875) == 0x3A              # ties go to the even mantissa
    assert enc(1.07) == 0x39 and enc(-1.07) == 0xB9
    assert enc(2.0 ** -10) == 0x00 and enc(1.5 * 2.0 ** -10) == 0x01  # around the smallest subnormal
    assert enc(464.0) == 0x7E and enc(1000.0) == 0x7E and enc(-1e6) == 0xFE   # saturation


def test_e4m3_array_encoder_is_the_scalar_rule():
    """The array form of the encoder agrees with e4m3_encode on every code value, every
    midpoint between neighbours (the ties), values just beside them, saturation, signed
    zeros and random values across the whole range."""
    pos = np.array([O.e4m3_decode(c) for c in range(0x7F)])
    mids = (pos[1:] + pos[:-1]) / 2
    rng = np.random.default_rng(41)
    xs = np.concatenate([pos, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9), [448.0, 449.0, 464.0, 1e6],
                         [0.0, -0.0], rng.standard_normal(4000) * np.exp(rng.uniform(-12, 7, 4000))])
    xs = np.concatenate([xs, -xs])
    got = O.e4m3_encode_array(xs)
    assert got.dtype == np.uint8
    assert list(got) == [O.e4m3_encode(v) for v in xs]


def test_mx_e4m3_block_scaling():
    rng = np.random.default_rng(41)
    w = rng.standard_normal((6, 128)) * np.array([1e-3, 0.02, 1.0, 7.0, 300.0, 1e4])[:, None]
    w[2, 32:64] = 0.0                                                   # one all-zero block
    codes, exp = O.mx_e4m3_quantize(w)
    dq = O.mx_e4m3_dequantize(codes, exp)
    blocks = w.reshape(6, 4, 32)
    amax = np.abs(blocks).max(axis=-1)
    nz = amax > 0
    # the block's largest magnitude lands in [256, 512) after scaling
    r = amax[nz] / np.ldexp(1.0, exp[nz])
    assert np.all((r >= 256) & (r < 512))
    assert np.all(dq.reshape(6, 4, 32)[~nz] == 0)
    # relative error of a 3-bit mantissa (half a unit in the last place) for values in the
    # normal range that did not saturate
    X = np.repeat(np.ldexp(1.0, exp), 32, axis=-1).reshape(w.shape)
    sc = np.abs(w) / X
    ok = (sc >= 2.0 ** -6) & (sc <= 448.0)
    assert np.all(np.abs(dq - w)[ok] <= 2.0 ** -4 * np.abs(w)[ok] + 1e-300)
    sat = sc > 464.0
    assert np.all(np.abs(dq[sat]) == 448.0 * X[sat])
    # a hand example: [3, 0, ...]: X = 2^(1 - 8), 3 / X = 384 = 1.5 * 2^8, exact
    c1, e1 = O.mx_e4m3_quantize(np.array([3.0] + [0.0] * 31))
    assert e1[0] == -7 and c1[0] == 0x7C and O.mx_e4m3_dequantize(c1, e1)[0] == 3.0


def test_e2m1_codes_rounding_saturation():
    assert [O.e2m1_decode(c) for c in range(8)] == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in range(8):
        assert O.e2m1_decode(c | 0x8) == -O.e2m1_decode(c)
        assert O.e2m1_encode(O.e2m1_decode(c)) == c
    enc = O.e2m1_encode
    assert enc(0.25) == 0 and enc(0.75) == 2 and enc(1.25) == 2 and enc(1.75) == 4   # ties to even
    assert enc(2.5) == 4 and enc(3.5) == 6 and enc(5.0) == 6                          # ties to even
    assert enc(2.4) == 4 and enc(5.1) == 7 and enc(100.0) == 7 and enc(-100.0) == 0xF


def test_e2m1_array_encoder_is_the_scalar_rule():
    pos = np.array([O.e2m1_decode(c) for c in range(8)])
    mids = (pos[1:] + pos[:-1]) / 2
    rng = np.random.default_rng(43)
    xs = np.concatenate([pos, mids, np.nextafter(mids, 0), np.nextafter(mids, 9), [6.0, 6.5, 7.0, 100.0], [0.0, -0.0],
                         rng.standard_normal(3000) * 3])
    xs = np.concatenate([xs, -xs])
    got = O.e2m1_encode_array(xs)
    assert got.dtype == np.uint8
    assert list(got) == [O.e2m1_encode(v) for v in xs]


def test_nvfp4_block_scaling():
    rng = np.random.default_rng(43)
    w = rng.standard_normal((4, 64)) * np.array([0.01, 0.2, 1.0, 5.0])[:, None]
    codes, sc, g = O.nvfp4_quantize(w)
    dq = O.nvfp4_dequantize(codes, sc, g)
    assert g == np.abs(w).max() / (448.0 * 6.0)
    # the tensor's largest value: block scale 448 exactly, element code 6, reproduced
    i = np.unravel_index(np.argmax(np.abs(w)), w.shape)
    assert O.e4m3_decode(int(sc[i[0], i[1] // 16])) == 448.0 and abs(dq[i]) == pytest.approx(abs(w[i]))
    # every element within half an E2M1 step of its scaled value (the step is at most 2 at
    # the top of the range) after the block scale's own rounding
    sb = np.vectorize(O.e4m3_decode)(sc)
    X = np.repeat(sb * g, 16, axis=-1).reshape(w.shape)
    sc_v = np.abs(w) / X
    assert np.all(np.abs(dq - w) <= np.where(sc_v <= 2, 0.25, np.where(sc_v <= 4, 0.5, 1.0)) * X + 1e-15)
    # values that are E2M1 grid points of an exactly representable scale come back exactly
    exact = np.array([[6.0, -4.0, 3.0, 0.5] * 4]) * 2.0
    c2, s2, g2 = O.nvfp4_quantize(exact)
    np.testing.assert_array_equal(O.nvfp4_dequantize(c2, s2, g2), exact)


def test_renoise_schedule_golden():
    g = {r[0]: [int(v) for v in r[1:]] for r in _read_golden("renoise_schedule.txt")}
    assert [O.renoise_count(256, 16, s, 0.5, 0.0) for s in range(16)] == g["S16"]
    assert [O.renoise_count(256, 8, s, 0.5, 0.0) for s in range(8)] == g["S8"]
    assert O.renoise_count(256, 1, 0, 0.25, 0.25) == g["S1_C256_q25"][0]
    assert O.renoise_count(32, 1, 0, 0.25, 0.25) == g["S1_C32_q25"][0]


# ---------------------------------------------------------------- roofline calculator

def test_roofline_batch_and_8bit_accounting():
    """A batch of one is the single pass; a batch of B counts the weights once and each
    canvas's K/V and logits B times; 8-bit experts count 1 + 1/32 bytes per weight."""
    from block_diffusion_lm_masked_b200 import configs as CF
    cfg = CF.CONFIGS["layer1_bf16"]
    P, C, U = 1024, 256, [52]
    one = R.pass_bytes(cfg, P, C, U)
    assert R.pass_bytes_batched(cfg, [P], C, U) == one
    H, nkv, d, V, F = cfg["hidden"], cfg["n_kv_heads"], cfg["head_dim"], cfg["vocab"], cfg["expert_ffn"]
    per_canvas = 2 * 2 * nkv * d * (P + C) + 2 * 2 * nkv * d * C + 8 * C * V
    assert R.pass_bytes_batched(cfg, [P] * 4, C, U) == one + 3 * per_canvas
    assert one - R.pass_bytes(cfg, P, C, U, ew=R.MX8_WBYTES) == (2 - 1 - 1 / 32) * 3 * H * F * 52
    assert R.gate_up_bytes(cfg, 52, 1024, ew=1.0) == 2 * H * F * 52 + 2 * 1024 * (H + F)
    # a 4-bit output matrix: 1/2 + 1/16 bytes per weight instead of 2, counted once per batch
    saved = (2 - 0.5 - 1 / 16) * V * H
    assert R.pass_bytes_batched(cfg, [P] * 4, C, U) - R.pass_bytes_batched(cfg, [P] * 4, C, U, vw=R.NV4_WBYTES) == saved


def test_roofline_reproduces_exercise_arithmetic():
    g = {r[0]: float(r[1]) for r in _read_golden("roofline_h100_model.txt")}
    bw, peak = 3.35e12, 990e12
    assert R.dense_weight_read_s(8e9, 2, bw) * 1e3 == pytest.approx(g["weight_read_bf16_ms"], abs=5e-4)
    assert R.dense_weight_read_s(8e9, 0.5, bw) * 1e3 == pytest.approx(g["weight_read_4bit_ms"], abs=5e-4)
    assert 2 * 8e9 * 256 / peak * 1e3 == pytest.approx(g["compute_floor_256_ms"], abs=5e-4)
    ar = R.dense_pass_s(8e9, 1, 2, bw, peak)
    assert ar == pytest.approx(g["ar_pass_s"], rel=1e-6)
    assert 1.0 / ar == pytest.approx(g["ar_ceiling_tok_s"], rel=1e-6)
    t1024 = R.dense_pass_s(8e9, 1024, 2, bw, peak)     # compute-bound: the larger bound wins
    assert t1024 == pytest.approx(g["diffusion_pass_1024_s"], rel=1e-6)
    s = R.breakeven_steps(1024, t1024, 1.0 / ar)
    assert s == pytest.approx(g["breakeven_steps"], abs=5e-3)
    assert math.floor(s) == int(g["max_steps"])
