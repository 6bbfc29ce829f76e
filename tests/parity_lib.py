"""Shared pieces of the GPU parity tests: build the same seeded inputs for the CUDA
path and the oracle, run both, and compare under the stated tolerances.

Two kinds of comparison (the workload's tolerance statement, read as described in the
design notes):

Teacher-forced stage checks (`forced_pass_check`, `forced_prefill_check`) -- the parity
bar.  Each stage of the GPU pass is compared with the oracle's same stage applied to
the GPU's own stage input, upcast to fp64: the attention block of layer l on the GPU's
residual entering layer l, the MoE block on the GPU's residual after attention, the
vocabulary projection on the GPU's final residual, the update on the GPU's logits, a
prefill layer's stored K/V on the GPU's residual entering it.  A near-tie difference
at one stage therefore never hides a later stage, and every layer of every pass is
compared numerically:
  * routing indices, expert permutations and re-noise sets exactly, except positions
    whose oracle margin is below 1e-3 (router: k-th minus (k+1)-th logit; re-noise:
    log-confidence distance to the cut), which are exempt for that stage only;
  * routing weights within 2e-2 relative; hidden states and logits within
    max |gpu - oracle| / rms(oracle) <= 2e-2 (bf16) or 1e-4 (fp32);
  * canvas tokens exactly (the argmax of identical logits), confidences within 1e-5;
  * stored K/V: each element within half a bf16 step (its rounding) plus the fp32
    tolerance (1e-4 of the rms) of the exact value, and at most 1% of the elements
    different from the exact value's own rounding (values computed in fp32 from the same
    input round alike except near a rounding boundary).

Free-running comparison (`compare_pass`, `compare_update`) -- reported beside it: the
oracle's whole pass from the same canvas and cache against the GPU's.  Routing
differences at near ties are allowed; after one at a layer before the last, the two
sides compute different problems, so the rest of that free-running pass is checked
for structure only (the forced checks above still cover every stage).  The update is
compared with margins widened to the measured logit difference of the two passes
(`logit_shift`): each side updates its own logits.
"""
from __future__ import annotations

import numpy as np
import torch

from block_diffusion_lm_masked_b200 import dg, synth
from oracle import dg_oracle as O

ROUTE_MARGIN = 1e-3
CUT_MARGIN = 1e-3
TOKEN_MARGIN = 1e-2
WEIGHT_RTOL = 2e-2      # routing weights of rows routed alike, relative
CONF_RTOL = 1e-5        # confidences from identical logits (fp32 against fp64)


def tol(cfg):
    return 2e-2 if cfg["dtype"] == "bf16" else 1e-4


def rel_err(gpu, ref, rows=None):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if rows is not None:
        keep = np.ones(ref.shape[0], dtype=bool)
        keep[list(rows)] = False
        gpu, ref = gpu[keep], ref[keep]
    rms = np.sqrt(np.mean(ref * ref))
    return float(np.abs(gpu - ref).max() / rms)


def round_up(x, m):
    return (x + m - 1) // m * m


class Setup:
    """One config's seeded inputs on both sides."""

    def __init__(self, cfg, P, capacity=None, with_prefix=True, device="cuda"):
        self.cfg = cfg
        self.host = synth.Model(cfg)
        self.model = dg.Model(self.host, device)
        self.prec = O.Precision(cfg["dtype"])
        cap = capacity or round_up(P + 1024, 8)
        self.cache = dg.KVCache(cfg, cap, device)
        if with_prefix and P > 0:
            kv = synth.prefix_cache(cfg, P)
            self.cache.load_prefix(kv)
            self.ocache = O.Cache(kv)
        else:
            self.ocache = O.Cache.empty(cfg)
        self.device = device

    def workspace(self, max_tokens):
        return dg.Workspace(self.cfg, max_tokens, self.device)

    def taps(self, C):
        return make_taps(self.model, self.cfg, C, self.device)


def make_taps(model, cfg, C, device="cuda"):
    """Per-layer tap buffers for calls of up to C rows, installed on the model."""
    L, H, k, E = cfg["n_layers"], cfg["hidden"], cfg["top_k"], cfg["n_experts"]
    t = dict(x_attn=[torch.zeros(C, H, device=device) for _ in range(L)],
             x_out=[torch.zeros(C, H, device=device) for _ in range(L)],
             topk_idx=[torch.zeros(C, k, dtype=torch.int32, device=device) for _ in range(L)],
             topk_w=[torch.zeros(C, k, device=device) for _ in range(L)],
             counts=[torch.zeros(E, dtype=torch.int32, device=device) for _ in range(L)],
             perm=[torch.zeros(C * k, dtype=torch.int32, device=device) for _ in range(L)],
             unions=torch.zeros(L, dtype=torch.int32, device=device), rows=C)
    model.set_taps(t)
    return t


def compare_pass(cfg, taps_gpu, logits_gpu, taps_o, logits_o, report=None, exempt=None):
    """Layer-by-layer comparison of one pass; returns the set of exempt rows.

    `exempt`: rows already exempt on entry (positions whose input token differs).

    A routing difference allowed at layer l (a near tie) gives that row a different MoE
    output, and from layer l + 1 on its K/V reach every other row through block
    attention: the two sides then solve different problems.  The layers after the first
    such difference are checked for structure only (the GPU's permutation, counts and
    union consistent with its own routing), and every row of the pass is returned
    exempt, so that the update is checked for structure only as well."""
    t = tol(cfg)
    k, E = cfg["top_k"], cfg["n_experts"]
    exempt = set() if exempt is None else set(exempt)
    C = logits_gpu.shape[0]
    diverged = None   # layer of the first allowed routing difference
    for l, to in enumerate(taps_o):
        gi = taps_gpu["topk_idx"][l].cpu().numpy()
        counts = taps_gpu["counts"][l].cpu().numpy()
        assert counts.sum() == gi.shape[0] * k
        np.testing.assert_array_equal(counts, np.bincount(gi.reshape(-1), minlength=E))
        # the GPU permutation must be the stable grouping of the GPU's own routing
        perm = taps_gpu["perm"][l].cpu().numpy()
        flat = gi.reshape(-1)
        want = sorted(range(flat.size), key=lambda a: (int(flat[a]), a))
        np.testing.assert_array_equal(perm, want)
        assert int(taps_gpu["unions"][l].item()) == int((counts > 0).sum())
        for row in range(gi.shape[0]):
            assert len(set(gi[row].tolist())) == k and gi[row].min() >= 0 and gi[row].max() < E
        if diverged is not None:
            continue
        xa = taps_gpu["x_attn"][l].cpu().numpy()
        e_attn = rel_err(xa, to["x_attn"], exempt)
        assert e_attn <= t, f"layer {l} attention residual: rel err {e_attn:.3e} > {t}"
        gw = taps_gpu["topk_w"][l].cpu().numpy()
        oi, ow, om = to["topk_idx"], to["topk_w"], to["router_margin"]
        flipped = False
        for row in range(gi.shape[0]):
            if row in exempt:
                continue
            if set(gi[row].tolist()) != set(oi[row].tolist()):
                assert om[row] < ROUTE_MARGIN, (
                    f"layer {l} row {row}: routing {sorted(gi[row])} vs oracle {sorted(oi[row])}, margin {om[row]:.3e}")
                exempt.add(row)
                flipped = True
                continue
            # weights per expert
            gmap = dict(zip(gi[row].tolist(), gw[row].tolist()))
            for e, w in zip(oi[row].tolist(), ow[row].tolist()):
                assert abs(gmap[e] - w) <= WEIGHT_RTOL * w, (l, row, e, gmap[e], w)
        if not exempt:
            np.testing.assert_array_equal(counts, to["counts"])
            # tokens of each expert segment, in order (independent of the slot order)
            np.testing.assert_array_equal(perm // k, np.asarray(to["perm"]) // k)
        xo = taps_gpu["x_out"][l].cpu().numpy()
        e_out = rel_err(xo, to["x_out"], exempt)
        assert e_out <= t, f"layer {l} MoE residual: rel err {e_out:.3e} > {t}"
        if report is not None:
            report.append(dict(layer=l, attn=e_attn, out=e_out, exempt=len(exempt)))
        if flipped and l + 1 < len(taps_o):
            diverged = l
    if diverged is not None:
        if report is not None:
            report.append(dict(logits=None, diverged_after_layer=diverged))
        return set(range(C))
    e_log = rel_err(logits_gpu, logits_o, exempt)
    assert e_log <= t, f"logits rel err {e_log:.3e} > {t}"
    if report is not None:
        report.append(dict(logits=e_log))
    return exempt


def causal_reach(runs, n_layers):
    """For each layer l, the first cache position whose K/V may legitimately differ.

    `runs`: (position offset, GPU top-k per layer [T][k], oracle taps per layer) for each
    prefill call, in order.  A row routed differently at layer l (allowed only at a near
    tie, which is asserted for every row not already reached) has a different hidden
    state from layer l + 1 on, and through causal attention so has every later position
    in the layers above."""
    reach = [None] * n_layers
    for off, gpu_topk, taps in runs:
        for l, t in enumerate(taps):
            gi = np.asarray(gpu_topk[l])
            oi, om = t["topk_idx"], np.asarray(t["router_margin"])
            for r in range(gi.shape[0]):
                if reach[l] is not None and off + r >= reach[l]:
                    break
                if set(gi[r].tolist()) != set(np.asarray(oi[r]).tolist()):
                    assert om[r] < ROUTE_MARGIN, (
                        f"prefill layer {l} position {off + r}: routing {sorted(gi[r])} vs oracle "
                        f"{sorted(oi[r])}, margin {om[r]:.3e}")
                    for l2 in range(l + 1, n_layers):
                        reach[l2] = off + r if reach[l2] is None else min(reach[l2], off + r)
                    break
    return reach


def prefill_topk(st, T):
    """Taps sized for a T-token prefill; returns the per-layer top-k device tensors."""
    return st.taps(T)["topk_idx"]


def stored_kv(oc, cfg):
    """The oracle cache's (already stored-precision) K/V as arrays dg.KVCache.load_prefix
    takes: bf16 bit patterns (exact: every value is a bf16 value) or float32."""
    out = []
    for k, v in zip(oc.k, oc.v):
        pair = []
        for a in (k, v):
            f = np.ascontiguousarray(a.astype(np.float32))
            assert np.array_equal(f.astype(np.float64), a)
            if cfg["dtype"] == "bf16":
                bits = f.view(np.uint32)
                assert not (bits & 0xFFFF).any()
                pair.append((bits >> 16).astype(np.uint16))
            else:
                pair.append(f)
        out.append(tuple(pair))
    return out


def kv_close_causal(cache, oc, reach, label):
    """Every layer's K and V against the oracle's, up to that layer's causal reach of a
    near-tie routing row; returns the fraction of positions compared."""
    total, seen = 0, 0
    for l in range(len(reach)):
        k, v = cache.logical(l)
        n = oc.k[l].shape[1]
        stop = n if reach[l] is None else reach[l]
        for name, a, b in (("K", k, oc.k[l]), ("V", v, oc.v[l])):
            ok, frac, worst = kv_close(np.asarray(a)[:, :stop], np.asarray(b)[:, :stop])
            assert ok, f"{label} layer {l} {name}: {frac:.2%} differ; {worst}"
        total += n
        seen += stop
    return seen / max(total, 1)


def bf16_spacing(x):
    """Distance between consecutive bf16 values around |x| (8 significant bits)."""
    _, e = np.frexp(np.abs(np.asarray(x, np.float64)))
    return np.ldexp(1.0, e - 8)


def kv_close(gpu, ref, skip_positions=(), tol_rms=2e-2):
    """bf16-stored K/V against the oracle's rounded values.  The two sides round values
    that differ by the hidden-state error of the layer that produced them, so an element
    may differ by one rounding step at any magnitude (a flip) or by up to tol_rms * RMS
    (the hidden-state tolerance) near zero; together only a minority of elements may
    differ at all.  Arrays [nkv][len][d].  Returns (ok, fraction differing, worst)."""
    g = np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    skip = set(skip_positions)
    keep = [p for p in range(r.shape[1]) if p not in skip]
    g, r = g[:, keep], r[:, keep]
    d = np.abs(g - r)
    step = bf16_spacing(np.maximum(np.abs(g), np.abs(r)))
    floor = tol_rms * np.sqrt(np.mean(r * r))
    bad = d > np.maximum(step * 1.0001, floor)
    frac = float((d > 0).mean())
    worst = ""
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, d, 0)), d.shape)
        worst = f"gpu {g[i]!r} oracle {r[i]!r} at {i}"
    return (not bad.any()) and frac < 0.2, frac, worst


def logit_shift(logits_gpu, logits_o, exempt=()):
    """Largest |gpu - oracle| logit over the rows not exempt (0 when none is left)."""
    g = np.asarray(logits_gpu, dtype=np.float64)
    r = np.asarray(logits_o, dtype=np.float64)
    keep = np.ones(r.shape[0], dtype=bool)
    keep[[i for i in exempt if i < r.shape[0]]] = False
    return float(np.abs(g[keep] - r[keep]).max()) if keep.any() else 0.0


def compare_update(canvas_gpu, conf_gpu, upd_o, exempt, n, logit_err=0.0):
    """Canvas after the update, free-running: the GPU's update of its own logits against
    the oracle's update of the oracle's logits, which differ by at most `logit_err` per
    element (measured).  A log-confidence (the top logit minus the log-sum-exp of the
    row) then moves by at most 2 * logit_err on each side, so a position keeps its side
    of the re-noise cut wherever its cut margin exceeds 4 * logit_err, its argmax
    wherever the top-1 minus top-2 logit exceeds 2 * logit_err, and its confidence is
    within a factor exp(2 * logit_err).  Those margins never go below the forced
    check's (1e-3 for the cut, 1e-2 for tokens)."""
    canvas_gpu = np.asarray(canvas_gpu)
    C = canvas_gpu.shape[0]
    cut_m = max(CUT_MARGIN, 4.0 * logit_err * 1.0001)
    tok_m = max(TOKEN_MARGIN, 2.0 * logit_err * 1.0001)
    ren_o = set(upd_o["renoised"].tolist())
    for i in range(C):
        if i in exempt:
            continue
        if upd_o["cut_margin"][i] < cut_m:
            continue
        if i in ren_o:
            assert canvas_gpu[i] == upd_o["canvas"][i], f"re-noised position {i}: {canvas_gpu[i]} vs {upd_o['canvas'][i]}"
        elif upd_o["top_margin"][i] > tok_m:
            assert canvas_gpu[i] == upd_o["canvas"][i], f"position {i}: token {canvas_gpu[i]} vs {upd_o['canvas'][i]}"
    if conf_gpu is not None:
        c = np.asarray(conf_gpu, dtype=np.float64)
        # the set the GPU re-noised, read from its own confidences with the stated rule
        gpu_set = set(np.argsort(c, kind="stable")[:n].tolist())
        for i in gpu_set ^ ren_o:
            assert i in exempt or upd_o["cut_margin"][i] < cut_m, (
                f"re-noise set differs at {i}: cut margin {upd_o['cut_margin'][i]:.3e} (bound {cut_m:.3e})")
        keep = [i for i in range(C) if i not in exempt]
        rtol = max(CONF_RTOL, float(np.expm1(2.0 * logit_err)) * 1.0001)
        np.testing.assert_allclose(c[keep], upd_o["conf"][keep], rtol=rtol)


# ---------------------------------------------------------------- several canvases

class BatchSetup:
    """One model, B caches with prefixes of the given lengths (each its own seeded K/V)."""

    def __init__(self, dg, cfg, prefixes, capacity):
        self.cfg = cfg
        self.host = synth.Model(cfg)
        self.model = dg.Model(self.host)
        self.prec = O.Precision(cfg["dtype"])
        self.caches, self.ocaches = [], []
        for b, P in enumerate(prefixes):
            c = dg.KVCache(cfg, capacity)
            if P > 0:
                kv = synth.prefix_cache(cfg, P, seed=synth.SEED_WEIGHTS + 100 + b)
                c.load_prefix(kv)
                self.ocaches.append(O.Cache(kv))
            else:
                self.ocaches.append(O.Cache.empty(cfg))
            self.caches.append(c)

    def taps(self, rows):
        return make_taps(self.model, self.cfg, rows)


def batch_canvases(cfg, B, C, first=0):
    return np.stack([synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(first + b), C, cfg["vocab"])
                     for b in range(B)]).astype(np.int32)


def check_batched_pass(dg, cfg, prefixes, C, prepare=None):
    """One batched pass (each canvas with its own prefix) and each canvas's update against
    the oracle; `prepare(setup)` may change the model first (e.g. 8-bit experts)."""
    B = len(prefixes)
    bt = BatchSetup(dg, cfg, prefixes, round_up(max(prefixes) + C + 8, 8))
    if prepare is not None:
        prepare(bt)
    V = cfg["vocab"]
    canv = batch_canvases(cfg, B, C)
    taps = bt.taps(B * C)
    ws = dg.Workspace(cfg, B * C)
    logits = torch.empty(B, C, V, device="cuda")
    dg.denoise_pass_batched(bt.model, bt.caches, torch.from_numpy(canv).cuda(), logits, ws)
    # each canvas's own update from its slice of the logits
    n = O.renoise_count(C, 1, 0, 0.25, 0.25)
    out = torch.from_numpy(canv).cuda()
    conf = torch.empty(B, C, device="cuda")
    for b in range(B):
        dg.canvas_update(logits[b], n, synth.SEED_RENOISE + b, 0, out[b], ws, conf[b])
    dg.device_status(ws)
    lg_np, out_np, conf_np = logits.cpu().numpy(), out.cpu().numpy(), conf.cpu().numpy()
    stats = forced_batched_pass_check(cfg, bt.host, bt.prec, bt.ocaches, list(canv), taps, lg_np, out_np, conf_np,
                                      n, [synth.SEED_RENOISE + b for b in range(B)], 0)
    print("forced:", summary(stats))
    res = O.denoise_pass_batched(bt.host, bt.ocaches, list(canv), bt.prec)
    merged = O.merge_batch_taps([t for _, t in res], cfg["n_experts"])
    logits_o = np.concatenate([lg for lg, _ in res], axis=0)
    report = []
    exempt = compare_pass(cfg, taps, logits.reshape(B * C, V).cpu().numpy(), merged, logits_o, report)
    for b in range(B):
        upd_o = O.canvas_update(res[b][0], n, synth.SEED_RENOISE + b, 0)
        ex_b = {r - b * C for r in exempt if b * C <= r < (b + 1) * C}
        compare_update(out_np[b], conf_np[b], upd_o, ex_b, n, logit_shift(lg_np[b], res[b][0], ex_b))
    print(report, "exempt rows:", len(exempt))
    # the caches' committed prefixes are untouched and their lengths unchanged
    for c, P in zip(bt.caches, prefixes):
        assert c.len == P
    return bt, canv, logits


# ---------------------------------------------------------------- teacher-forced stage checks

def oracle_cache_from_gpu(cache, upto=None) -> "O.Cache":
    """The GPU cache's stored K/V [0, len) (or [0, upto)) as an oracle cache (exact upcast)."""
    oc = O.Cache([])
    oc.k, oc.v = [], []
    for l in range(len(cache.k)):
        k, v = cache.logical(l, upto)
        oc.k.append(k)
        oc.v.append(v)
    return oc


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64) if isinstance(t, torch.Tensor) else np.asarray(t)


def _check_structure(gi, counts, perm, union, k, E, label):
    """The GPU's counts, permutation and union are those of its own routing."""
    assert counts.sum() == gi.shape[0] * k, label
    np.testing.assert_array_equal(counts, np.bincount(gi.reshape(-1), minlength=E), err_msg=label)
    flat = gi.reshape(-1)
    want = sorted(range(flat.size), key=lambda a: (int(flat[a]), a))
    np.testing.assert_array_equal(perm, want, err_msg=label)
    assert union == int((counts > 0).sum()), label
    for row in range(gi.shape[0]):
        assert len(set(gi[row].tolist())) == k and gi[row].min() >= 0 and gi[row].max() < E, (label, row)


def _forced_moe(cfg, host, prec, l, rows, taps_gpu, label, stats):
    """The MoE stage of layer l on the GPU's post-attention residual (rows = tokens tapped).
    Returns the rows exempt at this stage (near-tie routing differences)."""
    k, E, t = cfg["top_k"], cfg["n_experts"], tol(cfg)
    xa = _np(taps_gpu["x_attn"][l])[:rows]
    m = O.moe_block(host, l, xa, prec)
    gi = taps_gpu["topk_idx"][l][:rows].cpu().numpy()
    gw = taps_gpu["topk_w"][l][:rows].cpu().numpy().astype(np.float64)
    counts = taps_gpu["counts"][l].cpu().numpy()
    perm = taps_gpu["perm"][l][:rows * k].cpu().numpy()
    _check_structure(gi, counts, perm, int(taps_gpu["unions"][l].item()), k, E, f"{label} layer {l}")
    oi, ow, om = m["topk_idx"], m["topk_w"], m["router_margin"]
    exempt = set()
    w_err = 0.0
    for row in range(rows):
        if set(gi[row].tolist()) != set(oi[row].tolist()):
            assert om[row] < ROUTE_MARGIN, (f"{label} layer {l} row {row}: routing {sorted(gi[row])} vs oracle "
                                            f"{sorted(oi[row])} on the same input, margin {om[row]:.3e}")
            exempt.add(row)
            continue
        gmap = dict(zip(gi[row].tolist(), gw[row].tolist()))
        for e, w in zip(oi[row].tolist(), ow[row].tolist()):
            err = abs(gmap[e] - w) / w
            w_err = max(w_err, err)
            assert err <= WEIGHT_RTOL, (label, l, row, e, gmap[e], w)
    # tokens of each expert segment, in order, over the rows routed alike
    go = [a // k for a in perm if a // k not in exempt]
    oo = [a // k for a in np.asarray(m["perm"]) if a // k not in exempt]
    np.testing.assert_array_equal(go, oo, err_msg=f"{label} layer {l}: expert grouping")
    if not exempt:
        np.testing.assert_array_equal(counts, m["counts"], err_msg=f"{label} layer {l}: counts")
    e_out = rel_err(_np(taps_gpu["x_out"][l])[:rows], m["x_out"], exempt)
    assert e_out <= t, f"{label} layer {l} MoE stage: rel err {e_out:.3e} > {t}"
    stats.setdefault("moe", []).append(e_out)
    stats["weights"] = max(stats.get("weights", 0.0), w_err)
    stats["route_exempt"] = stats.get("route_exempt", 0) + len(exempt)
    return exempt


def forced_pass_check(cfg, host, prec, cache_o, canvas, taps_gpu, logits_gpu, canvas_out=None, conf_gpu=None,
                      n=0, seed=0, step=0, label="pass", upd_fn=None):
    """Every stage of one GPU denoising pass against the oracle's stage on the GPU's own
    stage input.  cache_o: the cache as the GPU read it (stored values); canvas: the
    pass's input tokens; taps_gpu: the pass's taps; logits_gpu [C][V] (numpy or None
    for a pass without logits); canvas_out / conf_gpu: the update's result, checked with
    `upd_fn(logits) -> oracle update` (default: the re-noising update with n, seed,
    step).  Returns a dict of the largest errors seen."""
    t = tol(cfg)
    L = cfg["n_layers"]
    C = len(canvas)
    stats = {}
    x_in = O.embed(host, canvas)
    for l in range(L):
        if l > 0:
            x_in = _np(taps_gpu["x_out"][l - 1])[:C]
        a = O.attention_block(host, l, cache_o, x_in, False, prec)
        e_attn = rel_err(_np(taps_gpu["x_attn"][l])[:C], a["x_attn"])
        assert e_attn <= t, f"{label} layer {l} attention stage: rel err {e_attn:.3e} > {t}"
        stats.setdefault("attn", []).append(e_attn)
        _forced_moe(cfg, host, prec, l, C, taps_gpu, label, stats)
    if logits_gpu is not None:
        lg = np.asarray(logits_gpu, dtype=np.float64)
        lo = O.vocab_logits(host, _np(taps_gpu["x_out"][L - 1])[:C], prec)
        e_log = rel_err(lg, lo)
        assert e_log <= t, f"{label} vocabulary stage: rel err {e_log:.3e} > {t}"
        stats["logits"] = e_log
        if canvas_out is not None:
            upd = upd_fn(lg) if upd_fn else O.canvas_update(lg, n, seed, step)
            stats.update(forced_update_check(upd, canvas_out, conf_gpu, label))
    return stats


def forced_batched_pass_check(cfg, host, prec, caches_o, canvases, taps_gpu, logits_gpu, outs=None, confs=None,
                              n=0, seeds=None, step=0, label="batched pass"):
    """forced_pass_check for B canvases in one pass: the attention stage per canvas (each
    against its own cache), the MoE stage over all B*C rows at once (the batch groups its
    rows by expert together), the vocabulary stage over all rows, the update per canvas.
    logits_gpu [B][C][V]."""
    t = tol(cfg)
    L = cfg["n_layers"]
    B, C = len(canvases), len(canvases[0])
    stats = {}
    x_in = np.concatenate([O.embed(host, c) for c in canvases], axis=0)
    for l in range(L):
        if l > 0:
            x_in = _np(taps_gpu["x_out"][l - 1])[:B * C]
        xa_g = _np(taps_gpu["x_attn"][l])[:B * C]
        for b in range(B):
            a = O.attention_block(host, l, caches_o[b], x_in[b * C:(b + 1) * C], False, prec)
            e_attn = rel_err(xa_g[b * C:(b + 1) * C], a["x_attn"])
            assert e_attn <= t, f"{label} canvas {b} layer {l} attention stage: rel err {e_attn:.3e} > {t}"
            stats.setdefault("attn", []).append(e_attn)
        _forced_moe(cfg, host, prec, l, B * C, taps_gpu, label, stats)
    lg = np.asarray(logits_gpu, dtype=np.float64).reshape(B * C, -1)
    lo = O.vocab_logits(host, _np(taps_gpu["x_out"][L - 1])[:B * C], prec)
    e_log = rel_err(lg, lo)
    assert e_log <= t, f"{label} vocabulary stage: rel err {e_log:.3e} > {t}"
    stats["logits"] = e_log
    if outs is not None:
        for b in range(B):
            upd = O.canvas_update(lg[b * C:(b + 1) * C], n, seeds[b], step)
            r = forced_update_check(upd, outs[b], None if confs is None else confs[b], f"{label} canvas {b}")
            stats["cut_exempt"] = stats.get("cut_exempt", 0) + r["cut_exempt"]
            if "conf" in r:
                stats["conf"] = max(stats.get("conf", 0.0), r["conf"])
    return stats


def forced_update_check(upd, canvas_out, conf_gpu, label="update"):
    """The GPU's update against the oracle's update of the same (GPU) logits: identical
    tokens, except positions within 1e-3 of the re-noise (or keep) cut in log-confidence;
    confidences within 1e-5."""
    g = np.asarray(canvas_out)
    near_cut = np.asarray(upd["cut_margin"]) < CUT_MARGIN
    bad = np.nonzero((g != upd["canvas"]) & ~near_cut)[0]
    assert bad.size == 0, (f"{label}: tokens differ from the oracle's update of the same logits at "
                           f"{bad[:8].tolist()} (gpu {g[bad[:8]].tolist()}, oracle {upd['canvas'][bad[:8]].tolist()})")
    out = {"cut_exempt": int(near_cut.sum())}
    if conf_gpu is not None:
        c = np.asarray(conf_gpu, dtype=np.float64)
        err = float(np.max(np.abs(c - upd["conf"]) / upd["conf"]))
        assert err <= CONF_RTOL, f"{label}: confidence rel err {err:.3e} > {CONF_RTOL}"
        out["conf"] = err
    return out


def forced_prefill_check(cfg, host, prec, cache_before, tokens, taps_gpu, cache_after, P, label="prefill"):
    """Every stage of one GPU prefill of `tokens` at positions P.. against the oracle's
    stage on the GPU's own stage input: per layer the stored K/V (cache_after, slots
    [P, P+T)) and, below the last layer, the attention and MoE stages.  cache_before: the
    cache as the GPU read it.  taps_gpu must cover T rows."""
    t = tol(cfg)
    L, T = cfg["n_layers"], len(tokens)
    stats = {}
    x_in = O.embed(host, tokens)
    for l in range(L):
        if l > 0:
            x_in = _np(taps_gpu["x_out"][l - 1])[:T]
        a = O.attention_block(host, l, cache_before, x_in, True, prec)
        k_g, v_g = cache_after.logical(l, P + T)
        for name, g, r in (("K", k_g[:, P:], a["k_new"]), ("V", v_g[:, P:], a["v_new"])):
            ok, frac, worst = kv_stored_close(g, r, prec)
            assert ok, f"{label} layer {l} stored {name}: {frac:.3%} differ; {worst}"
            stats[f"kv_differ_{l}"] = max(stats.get(f"kv_differ_{l}", 0.0), frac)
        if l == L - 1:
            break
        e_attn = rel_err(_np(taps_gpu["x_attn"][l])[:T], a["x_attn"])
        assert e_attn <= t, f"{label} layer {l} attention stage: rel err {e_attn:.3e} > {t}"
        stats.setdefault("attn", []).append(e_attn)
        _forced_moe(cfg, host, prec, l, T, taps_gpu, label, stats)
    return stats


def kv_stored_close(gpu, exact, prec, max_frac=0.01):
    """K/V the GPU stored against the oracle's unrounded K/V from the same input.  The GPU
    computes the value in fp32 (within the fp32 tolerance, 1e-4 of the rms, of the exact
    value) and bf16 storage holds its rounding (within half a bf16 step of it), so each
    element lies within half a step plus that tolerance of the exact value, and only a
    small fraction differs from the exact value's own rounding; fp32 storage within 1e-4
    relative to the rms."""
    g = np.asarray(gpu, np.float64)
    r = np.asarray(exact, np.float64)
    rms = np.sqrt(np.mean(r * r))
    if prec.dtype != "bf16":
        err = np.abs(g - r).max() / rms
        return err <= 1e-4, float(err), ""
    stored = O.round_bf16(r)
    d = np.abs(g - r)
    half_step = 0.5 * bf16_spacing(np.maximum(np.abs(g), np.abs(r)))
    bad = d > half_step * 1.0001 + 1e-4 * rms
    frac = float((g != stored).mean())
    worst = ""
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, d, 0)), d.shape)
        worst = f"gpu {g[i]!r} exact {r[i]!r} at {i}"
    return (not bad.any()) and frac <= max_frac, frac, worst


def summary(stats):
    """One line of the largest errors of a forced check."""
    parts = []
    for key in ("attn", "moe"):
        if key in stats:
            parts.append(f"{key} {max(stats[key]):.1e}")
    for key in ("logits", "weights", "conf"):
        if key in stats:
            parts.append(f"{key} {stats[key]:.1e}")
    for key in ("route_exempt", "cut_exempt"):
        if stats.get(key):
            parts.append(f"{key} {stats[key]}")
    return ", ".join(parts)
