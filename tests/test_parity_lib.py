"""The comparison rules of the GPU parity tests, checked on planted CPU data (no GPU):
in the free-running comparison an allowed routing difference switches the rest of a pass
to structure-only checks, a routing difference at a clear margin fails, and the causal
reach of a prefill starts at the first position whose routing actually differs; the
teacher-forced stage checks accept the oracle's own pass dressed as GPU taps and reject
a wrong layer, a wrong route and a wrong token."""
import numpy as np
import pytest
import torch

import parity_lib as PL

CFG = dict(top_k=2, n_experts=4, dtype="bf16")


def _taps(topk, x_attn, x_out, counts=None, device="cpu"):
    L = len(topk)
    t = dict(topk_idx=[torch.tensor(a, dtype=torch.int32) for a in topk],
             topk_w=[torch.full(np.asarray(a).shape, 0.5) for a in topk],
             x_attn=[torch.tensor(a, dtype=torch.float32) for a in x_attn],
             x_out=[torch.tensor(a, dtype=torch.float32) for a in x_out])
    cnt, perm, uni = [], [], []
    for a in topk:
        a = np.asarray(a)
        c = np.bincount(a.reshape(-1), minlength=CFG["n_experts"])
        cnt.append(torch.tensor(c, dtype=torch.int32))
        flat = a.reshape(-1)
        perm.append(torch.tensor(sorted(range(flat.size), key=lambda i: (int(flat[i]), i)), dtype=torch.int32))
        uni.append(int((c > 0).sum()))
    t.update(counts=cnt, perm=perm, unions=torch.tensor(uni, dtype=torch.int32))
    return t


def _oracle_taps(topk, margins, x_attn, x_out):
    out = []
    for a, m, xa, xo in zip(topk, margins, x_attn, x_out):
        a = np.asarray(a)
        flat = a.reshape(-1)
        out.append(dict(topk_idx=a, topk_w=np.full(a.shape, 0.5), router_margin=np.asarray(m, dtype=float),
                        counts=np.bincount(flat, minlength=CFG["n_experts"]),
                        perm=sorted(range(flat.size), key=lambda i: (int(flat[i]), i)),
                        x_attn=np.asarray(xa, dtype=float), x_out=np.asarray(xo, dtype=float)))
    return out


def _pass(rows=3, layers=3, seed=0):
    rng = np.random.default_rng(seed)
    topk = [np.array([[0, 1], [2, 3], [1, 2]])[:rows] for _ in range(layers)]
    xa = [rng.standard_normal((rows, 4)) for _ in range(layers)]
    xo = [rng.standard_normal((rows, 4)) for _ in range(layers)]
    return topk, xa, xo


def test_identical_pass_compares_in_full():
    topk, xa, xo = _pass()
    logits = np.random.default_rng(1).standard_normal((3, 5))
    report = []
    ex = PL.compare_pass(CFG, _taps(topk, xa, xo), logits, _oracle_taps(topk, [[1, 1, 1]] * 3, xa, xo), logits, report)
    assert ex == set() and report[-1]["logits"] == 0.0


def test_near_tie_flip_turns_rest_of_pass_structure_only():
    topk, xa, xo = _pass()
    g_topk = [t.copy() for t in topk]
    g_topk[0][1] = [2, 0]                           # row 1 routes differently at layer 0 ...
    margins = [[1, 5e-4, 1], [1, 1, 1], [1, 1, 1]]   # ... where the oracle's margin is a near tie
    g_xa = [a.copy() for a in xa]
    g_xa[1] = g_xa[1] + 10.0                         # later layers may then differ arbitrarily
    logits = np.zeros((3, 5))
    report = []
    ex = PL.compare_pass(CFG, _taps(g_topk, g_xa, xo), logits + 7.0, _oracle_taps(topk, margins, xa, xo), logits,
                         report)
    assert ex == {0, 1, 2}
    assert report[-1] == dict(logits=None, diverged_after_layer=0)


def test_flip_at_clear_margin_fails():
    topk, xa, xo = _pass()
    g_topk = [t.copy() for t in topk]
    g_topk[1][2] = [0, 2]
    with pytest.raises(AssertionError, match="routing"):
        PL.compare_pass(CFG, _taps(g_topk, xa, xo), np.zeros((3, 5)),
                        _oracle_taps(topk, [[1, 1, 1]] * 3, xa, xo), np.zeros((3, 5)))


def test_hidden_state_outside_tolerance_fails():
    topk, xa, xo = _pass()
    g_xo = [a.copy() for a in xo]
    g_xo[2][0, 0] += 0.5                             # ~0.5 RMS at the last layer
    with pytest.raises(AssertionError, match="MoE residual"):
        PL.compare_pass(CFG, _taps(topk, xa, g_xo), np.zeros((3, 5)),
                        _oracle_taps(topk, [[1, 1, 1]] * 3, xa, xo), np.zeros((3, 5)))


def test_causal_reach_from_actual_flips():
    # two layers' taps of a 6-token prefill at offset 10; the GPU differs at position 3 of layer 0
    o_topk = [np.tile([[0, 1]], (6, 1)), np.tile([[2, 3]], (6, 1))]
    g_topk = [t.copy() for t in o_topk]
    g_topk[0][3] = [1, 2]
    taps = [dict(topk_idx=o_topk[0], router_margin=np.array([1, 1, 1, 5e-4, 1, 1])),
            dict(topk_idx=o_topk[1], router_margin=np.ones(6))]
    reach = PL.causal_reach([(10, g_topk, taps)], 3)
    assert reach == [None, 13, 13]
    # near ties that did not flip reach nothing
    assert PL.causal_reach([(10, o_topk, taps)], 3) == [None, None, None]
    # a flip at a clear margin before any reach is an error
    taps[0]["router_margin"][3] = 1.0
    with pytest.raises(AssertionError, match="prefill layer 0 position 13"):
        PL.causal_reach([(10, g_topk, taps)], 3)


# ---------------------------------------------------------------- teacher-forced checks

from oracle import dg_oracle as O  # noqa: E402
from block_diffusion_lm_masked_b200 import synth  # noqa: E402

SMALL = dict(n_layers=2, hidden=64, n_q_heads=4, n_kv_heads=2, head_dim=16, n_experts=6, top_k=2,
             expert_ffn=48, vocab=256, rope_theta=10000.0, rms_eps=1e-6, dtype="bf16")


def _oracle_as_gpu(cfg, P, C, seed=3):
    """A pass computed by the oracle and dressed as the GPU's taps (fp32 tensors), so the
    forced checks see 'GPU' stages that are exact up to fp32 storage."""
    host = synth.Model(cfg)
    kv = synth.prefix_cache(cfg, P)
    oc = O.Cache(kv)
    canvas = synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(seed), C, cfg["vocab"])
    prec = O.Precision(cfg["dtype"])
    logits, taps = O.denoise_pass(host, oc, canvas, prec)
    t = dict(x_attn=[torch.tensor(x["x_attn"], dtype=torch.float32) for x in taps],
             x_out=[torch.tensor(x["x_out"], dtype=torch.float32) for x in taps],
             topk_idx=[torch.tensor(x["topk_idx"], dtype=torch.int32) for x in taps],
             topk_w=[torch.tensor(x["topk_w"], dtype=torch.float32) for x in taps],
             counts=[torch.tensor(x["counts"], dtype=torch.int32) for x in taps],
             perm=[torch.tensor(x["perm"], dtype=torch.int32) for x in taps],
             unions=torch.tensor([x["union"] for x in taps], dtype=torch.int32))
    return host, oc, canvas, prec, logits.astype(np.float32), t


def test_forced_check_accepts_the_oracle_itself():
    host, oc, canvas, prec, logits, t = _oracle_as_gpu(SMALL, 40, 24)
    n = 6
    upd = O.canvas_update(logits.astype(np.float64), n, 77, 1)
    stats = PL.forced_pass_check(SMALL, host, prec, oc, canvas, t, logits, upd["canvas"], upd["conf"], n, 77, 1)
    assert max(stats["attn"]) < 1e-6 and max(stats["moe"]) < 1e-6 and stats["logits"] < 1e-6


def test_forced_check_sees_a_wrong_layer_a_wrong_route_and_a_wrong_token():
    host, oc, canvas, prec, logits, t = _oracle_as_gpu(SMALL, 40, 24)
    n = 6
    upd = O.canvas_update(logits.astype(np.float64), n, 77, 1)
    # a residual off by 5% in the second layer's attention stage
    bad = dict(t, x_attn=list(t["x_attn"]))
    bad["x_attn"][1] = bad["x_attn"][1] * 1.05
    with pytest.raises(AssertionError, match="layer 1"):
        PL.forced_pass_check(SMALL, host, prec, oc, canvas, bad, logits)
    # a row routed to another expert at a clear margin (its counts / permutation follow it)
    bad = dict(t, topk_idx=[x.clone() for x in t["topk_idx"]], counts=list(t["counts"]), perm=list(t["perm"]),
               unions=t["unions"].clone())
    m = O.moe_block(host, 0, t["x_attn"][0].double().numpy(), prec)
    row = int(np.argmax(m["router_margin"]))
    gi = bad["topk_idx"][0].numpy()
    gi[row, 0] = [e for e in range(SMALL["n_experts"]) if e not in gi[row]][0]
    c = np.bincount(gi.reshape(-1), minlength=SMALL["n_experts"])
    bad["counts"][0] = torch.tensor(c, dtype=torch.int32)
    flat = gi.reshape(-1)
    bad["perm"][0] = torch.tensor(sorted(range(flat.size), key=lambda a: (int(flat[a]), a)), dtype=torch.int32)
    bad["unions"][0] = int((c > 0).sum())
    with pytest.raises(AssertionError, match="routing"):
        PL.forced_pass_check(SMALL, host, prec, oc, canvas, bad, logits)
    # a token that is not the argmax of the same logits, away from the re-noise cut
    out = upd["canvas"].copy()
    i = int(np.argmax(np.where(np.isin(np.arange(24), upd["renoised"]), -np.inf, upd["cut_margin"])))
    out[i] = (out[i] + 1) % SMALL["vocab"]
    with pytest.raises(AssertionError, match="tokens differ"):
        PL.forced_pass_check(SMALL, host, prec, oc, canvas, t, logits, out, upd["conf"], n, 77, 1)


def test_stored_kv_rule():
    """A stored bf16 value is the rounding of an fp32 value within the fp32 tolerance of
    the exact one: a tiny element whose exact value sits just short of a rounding boundary
    may round to the neighbour (half a step plus 1e-4 of the rms away); an element a
    whole step off at a large magnitude, or too many neighbour roundings, fail."""
    from oracle import dg_oracle as O
    prec = O.Precision("bf16")
    rng = np.random.default_rng(3)
    exact = rng.standard_normal((2, 64, 16)) * 0.3
    stored = O.round_bf16(exact)
    assert PL.kv_stored_close(stored, exact, prec)[0]
    # a tiny element just below a rounding boundary, stored one step up
    e2, s2 = exact.copy(), stored.copy()
    sp = PL.bf16_spacing(2.8e-4)
    e2[0, 0, 0] = -(2.44140625e-4 + 18.977 * sp)
    s2[0, 0, 0] = -(2.44140625e-4 + 20 * sp)
    ok, frac, _ = PL.kv_stored_close(s2, e2, prec)
    assert ok and frac > 0
    # a large element one whole step off
    s3 = stored.copy()
    i = np.unravel_index(np.argmax(np.abs(exact)), exact.shape)
    s3[i] = stored[i] + np.sign(stored[i]) * PL.bf16_spacing(stored[i])
    assert not PL.kv_stored_close(s3, exact, prec)[0]
    # neighbour roundings on more than 1% of the elements
    s4 = stored.copy()
    flat = s4.reshape(-1)
    idx = np.argsort(np.abs(exact).reshape(-1))[:40]   # the smallest: inside the rms floor
    flat[idx] += PL.bf16_spacing(flat[idx])
    ok, frac, _ = PL.kv_stored_close(s4, exact, prec)
    assert not ok and frac > 0.01


def _update(logits, n):
    from oracle import dg_oracle as O
    return O.canvas_update(logits, n, 11, 0)


def test_free_running_update_margins_follow_the_logit_shift():
    """The free-running update check widens its margins to the measured logit difference:
    the oracle's update of logits shifted by delta passes against the unshifted update
    when delta is passed, and a token changed at a clear margin still fails."""
    rng = np.random.default_rng(5)
    C, V, n = 48, 64, 12
    lo = rng.standard_normal((C, V))
    delta = 2e-2
    lg = lo + rng.uniform(-delta, delta, size=lo.shape)
    up_o, up_g = _update(lo, n), _update(lg, n)
    PL.compare_update(up_g["canvas"], up_g["conf"], up_o, set(), n, PL.logit_shift(lg, lo))
    # a kept position given another token although its top margin is large
    kept = [i for i in range(C) if i not in set(up_o["renoised"].tolist())
            and up_o["top_margin"][i] > 10 * delta and up_o["cut_margin"][i] > 10 * delta]
    assert kept
    bad = up_g["canvas"].copy()
    bad[kept[0]] = (bad[kept[0]] + 1) % V
    with pytest.raises(AssertionError):
        PL.compare_update(bad, up_g["conf"], up_o, set(), n, PL.logit_shift(lg, lo))
    # a confidence off by more than exp(2 delta)
    conf = np.asarray(up_g["conf"], dtype=np.float64).copy()
    conf[kept[0]] *= 1.2
    with pytest.raises(AssertionError):
        PL.compare_update(up_g["canvas"], conf, up_o, set(), n, PL.logit_shift(lg, lo))
