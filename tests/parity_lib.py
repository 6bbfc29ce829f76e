"""Shared pieces of the GPU parity tests: build the same seeded inputs for the CUDA
path and the oracle, run both, and compare under the stated tolerances.

Comparison rules (the workload's tolerance statement, read as described in the
design notes):
  * routing indices, expert permutations and re-noise sets must match exactly, except
    at positions whose oracle margin is below 1e-3 (router: k-th minus (k+1)-th
    logit; re-noise: log-confidence distance to the cut);
  * a position exempted that way, and which then actually differs, stays exempt in
    every later comparison of the same pass (its hidden state, logits and token);
  * hidden states and logits: max |gpu - oracle| / rms(oracle) <= 2e-2 (bf16) or 1e-4
    (fp32) over the non-exempt rows;
  * canvas tokens: identical wherever the oracle's top-1/top-2 logit margin exceeds 1e-2.
"""
from __future__ import annotations

import numpy as np
import torch

from block_diffusion_lm_masked_b200 import dg, synth
from oracle import dg_oracle as O

ROUTE_MARGIN = 1e-3
CUT_MARGIN = 1e-3
TOKEN_MARGIN = 1e-2


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
        cfg = self.cfg
        L, H, k, E = cfg["n_layers"], cfg["hidden"], cfg["top_k"], cfg["n_experts"]
        dev = self.device
        t = dict(x_attn=[torch.zeros(C, H, device=dev) for _ in range(L)],
                 x_out=[torch.zeros(C, H, device=dev) for _ in range(L)],
                 topk_idx=[torch.zeros(C, k, dtype=torch.int32, device=dev) for _ in range(L)],
                 topk_w=[torch.zeros(C, k, device=dev) for _ in range(L)],
                 counts=[torch.zeros(E, dtype=torch.int32, device=dev) for _ in range(L)],
                 perm=[torch.zeros(C * k, dtype=torch.int32, device=dev) for _ in range(L)],
                 unions=torch.zeros(L, dtype=torch.int32, device=dev))
        self.model.set_taps(t)
        return t


def compare_pass(cfg, taps_gpu, logits_gpu, taps_o, logits_o, report=None, exempt=None):
    """Layer-by-layer comparison of one pass; returns the set of exempt rows.

    `exempt`: rows already exempt on entry (positions whose input token differs)."""
    t = tol(cfg)
    k, E = cfg["top_k"], cfg["n_experts"]
    exempt = set() if exempt is None else set(exempt)
    for l, to in enumerate(taps_o):
        xa = taps_gpu["x_attn"][l].cpu().numpy()
        e_attn = rel_err(xa, to["x_attn"], exempt)
        assert e_attn <= t, f"layer {l} attention residual: rel err {e_attn:.3e} > {t}"
        gi = taps_gpu["topk_idx"][l].cpu().numpy()
        gw = taps_gpu["topk_w"][l].cpu().numpy()
        oi, ow, om = to["topk_idx"], to["topk_w"], to["router_margin"]
        for row in range(gi.shape[0]):
            if row in exempt:
                continue
            if set(gi[row].tolist()) != set(oi[row].tolist()):
                assert om[row] < ROUTE_MARGIN, (
                    f"layer {l} row {row}: routing {sorted(gi[row])} vs oracle {sorted(oi[row])}, margin {om[row]:.3e}")
                exempt.add(row)
                continue
            # weights per expert
            gmap = dict(zip(gi[row].tolist(), gw[row].tolist()))
            for e, w in zip(oi[row].tolist(), ow[row].tolist()):
                assert abs(gmap[e] - w) <= 10 * t, (l, row, e, gmap[e], w)
        counts = taps_gpu["counts"][l].cpu().numpy()
        assert counts.sum() == gi.shape[0] * k
        np.testing.assert_array_equal(counts, np.bincount(gi.reshape(-1), minlength=E))
        # the GPU permutation must be the stable grouping of the GPU's own routing
        perm = taps_gpu["perm"][l].cpu().numpy()
        flat = gi.reshape(-1)
        want = sorted(range(flat.size), key=lambda a: (int(flat[a]), a))
        np.testing.assert_array_equal(perm, want)
        assert int(taps_gpu["unions"][l].item()) == int((counts > 0).sum())
        if not exempt:
            np.testing.assert_array_equal(counts, to["counts"])
            # tokens of each expert segment, in order (independent of the slot order)
            np.testing.assert_array_equal(perm // k, np.asarray(to["perm"]) // k)
        xo = taps_gpu["x_out"][l].cpu().numpy()
        e_out = rel_err(xo, to["x_out"], exempt)
        assert e_out <= t, f"layer {l} MoE residual: rel err {e_out:.3e} > {t}"
        if report is not None:
            report.append(dict(layer=l, attn=e_attn, out=e_out, exempt=len(exempt)))
    e_log = rel_err(logits_gpu, logits_o, exempt)
    assert e_log <= t, f"logits rel err {e_log:.3e} > {t}"
    if report is not None:
        report.append(dict(logits=e_log))
    return exempt


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


def compare_update(canvas_gpu, conf_gpu, upd_o, exempt, n):
    """Canvas after the update: tokens, re-noise set and confidences."""
    canvas_gpu = np.asarray(canvas_gpu)
    C = canvas_gpu.shape[0]
    ren_o = set(upd_o["renoised"].tolist())
    for i in range(C):
        if i in exempt:
            continue
        if upd_o["cut_margin"][i] < CUT_MARGIN:
            continue
        if i in ren_o:
            assert canvas_gpu[i] == upd_o["canvas"][i], f"re-noised position {i}: {canvas_gpu[i]} vs {upd_o['canvas'][i]}"
        elif upd_o["top_margin"][i] > TOKEN_MARGIN:
            assert canvas_gpu[i] == upd_o["canvas"][i], f"position {i}: token {canvas_gpu[i]} vs {upd_o['canvas'][i]}"
    if conf_gpu is not None:
        c = np.asarray(conf_gpu, dtype=np.float64)
        # the set the GPU re-noised, read from its own confidences with the stated rule
        gpu_set = set(np.argsort(c, kind="stable")[:n].tolist())
        for i in gpu_set ^ ren_o:
            assert i in exempt or upd_o["cut_margin"][i] < CUT_MARGIN, (
                f"re-noise set differs at {i}: cut margin {upd_o['cut_margin'][i]:.3e}")
        keep = [i for i in range(C) if i not in exempt]
        np.testing.assert_allclose(c[keep], upd_o["conf"][keep], rtol=5e-2)
