"""The multi-layer workloads at their full sizes, through the C-ABI, against the oracle.

- 8-layer denoise (prefix 2048, canvas 256, 16 passes, re-noise 50% -> 0%): every pass
  compared with the oracle, free running, exemptions carried from pass to pass.
- chained canvases (8 layers, 512-token prompt, 4 canvases x 16 passes + append): the
  prompt's K/V and the first canvas's 16 passes and append against the oracle; all four
  canvases for the properties that hold at any size (cache length, untouched prefix,
  bit-identical repeat run).
- large pass (4 layers, H2816, E128 top-8, F704, V262144, prefix 32768): the first pass
  layer by layer and its update against the oracle; the 8-pass run for its properties.
"""
import numpy as np
import pytest
import torch

from block_diffusion_lm_masked_b200 import configs as CF
from block_diffusion_lm_masked_b200 import synth
from oracle import dg_oracle as O

import parity_lib as PL

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_diffusion_lm_masked_b200 import dg as _dg
    return _dg


def _pass(dg, st, canvas_np, n, step, seed=synth.SEED_RENOISE, taps=True):
    cfg = st.cfg
    C, V = len(canvas_np), cfg["vocab"]
    tp = st.taps(C) if taps else None
    if not taps:
        st.model.set_taps(None)
    ws = st.ws
    canvas = torch.from_numpy(np.asarray(canvas_np, dtype=np.int32)).cuda()
    logits = torch.empty(C, V, device="cuda")
    conf = torch.empty(C, device="cuda")
    dg.denoise_pass(st.model, st.cache, canvas, logits, ws)
    dg.canvas_update(logits, n, seed, step, canvas, ws, conf)
    dg.device_status(ws)
    return tp, logits.cpu().numpy(), canvas.cpu().numpy(), conf.cpu().numpy()


def _free_run(dg, st, oc, noise, S, r0, r1, label):
    """S passes on both sides from the same noise; returns (gpu canvas, oracle canvas, exempt)."""
    C = len(noise)
    cur_g, cur_o = noise.copy(), noise.copy()
    tainted = set()
    for s in range(S):
        n = O.renoise_count(C, S, s, r0, r1)
        taps, logits, nxt_g, conf = _pass(dg, st, cur_g, n, s)
        logits_o, taps_o = O.denoise_pass(st.host, oc, cur_o, st.prec)
        upd = O.canvas_update(logits_o, n, synth.SEED_RENOISE, s)
        report = []
        exempt = PL.compare_pass(st.cfg, taps, logits, taps_o, logits_o, report, exempt=tainted)
        PL.compare_update(nxt_g, conf, upd, exempt, n)
        tainted = exempt | {i for i in range(C) if nxt_g[i] != upd["canvas"][i]}
        print(f"{label} pass {s}: n={n} logits err {report[-1]['logits']:.2e} exempt {len(tainted)}", flush=True)
        cur_g, cur_o = nxt_g, upd["canvas"]
    return cur_g, cur_o, tainted


def test_denoise8_full_size(dg):
    cfg = CF.CONFIGS["denoise8_bf16"]
    P, C, S = cfg["prefix"], cfg["canvas"], cfg["steps"]
    st = PL.Setup(cfg, P, capacity=P + C)
    st.ws = st.workspace(C)
    before = [(k[:, :P].clone(), v[:, :, :P].clone()) for k, v in zip(st.cache.k, st.cache.vt)]
    noise = synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(0), C, cfg["vocab"])
    g, o, exempt = _free_run(dg, st, st.ocache, noise, S, cfg["renoise_start"], cfg["renoise_end"], "denoise8")
    assert len(exempt) <= C // 8, f"too many exempt positions: {len(exempt)}"
    # the prefix K/V were reused untouched across all passes
    for (k0, v0), k, v in zip(before, st.cache.k, st.cache.vt):
        assert torch.equal(k[:, :P], k0) and torch.equal(v[:, :, :P], v0)
    assert st.cache.len == P
    # dg_generate_canvas gives the same canvas, bit for bit
    can = torch.from_numpy(noise).cuda()
    lg = torch.empty(C, cfg["vocab"], device="cuda")
    st.model.set_taps(None)
    dg.generate_canvas(st.model, st.cache, can, S, cfg["renoise_start"], cfg["renoise_end"], synth.SEED_RENOISE,
                       False, lg, st.ws)
    dg.device_status(st.ws)
    np.testing.assert_array_equal(can.cpu().numpy(), g)


def test_chained8_full_size(dg):
    cfg = CF.CONFIGS["chained8_bf16"]
    T0, C, S, n_can = cfg["prompt"], cfg["canvas"], cfg["steps"], cfg["n_canvases"]
    cap = T0 + n_can * C
    st = PL.Setup(cfg, 0, capacity=cap, with_prefix=False)
    st.ws = st.workspace(max(T0, C))
    prompt = synth.tokens(synth.SEED_TOKENS, synth.TID_PREFIX_TOKENS, T0, cfg["vocab"])
    dg.prefill_append(st.model, st.cache, torch.from_numpy(prompt).cuda(), st.ws)
    taps = []
    oc = O.prefill_append(st.host, st.ocache, prompt, st.prec, taps)
    near_tie = {int(i) for t in taps for i in np.nonzero(t["router_margin"] < PL.ROUTE_MARGIN)[0]}
    for l in range(cfg["n_layers"]):
        k, v = st.cache.logical(l)
        for name, a, b in (("K", k, oc.k[l]), ("V", v, oc.v[l])):
            ok, frac, worst = PL.kv_close(a, b, near_tie)
            assert ok, f"prompt layer {l} {name}: {frac:.2%} differ; {worst}"
    prompt_kv = [(k[:, :T0].clone(), v[:, :, :T0].clone()) for k, v in zip(st.cache.k, st.cache.vt)]
    # first canvas: 16 passes free running against the oracle, then its append
    noise0 = synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(0), C, cfg["vocab"])
    g, o, exempt = _free_run(dg, st, oc, noise0, S, cfg["renoise_start"], cfg["renoise_end"], "chained canvas 0")
    assert len(exempt) <= C // 8
    dg.prefill_append(st.model, st.cache, torch.from_numpy(g.astype(np.int32)).cuda(), st.ws)
    if not exempt:
        oc = O.prefill_append(st.host, oc, o, st.prec)
        for l in range(cfg["n_layers"]):
            k, v = st.cache.logical(l)
            ok, frac, worst = PL.kv_close(k, oc.k[l], near_tie)
            assert ok, f"after append layer {l} K: {frac:.2%} differ; {worst}"
    # the remaining canvases through dg_generate_canvas (append included)
    canvases = [g]
    st.model.set_taps(None)
    lg = torch.empty(C, cfg["vocab"], device="cuda")
    for c in range(1, n_can):
        can = torch.from_numpy(synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(c), C, cfg["vocab"])).cuda()
        dg.generate_canvas(st.model, st.cache, can, S, cfg["renoise_start"], cfg["renoise_end"], synth.SEED_RENOISE,
                           True, lg, st.ws)
        canvases.append(can.cpu().numpy())
    dg.device_status(st.ws)
    assert st.cache.len == cap
    for (k0, v0), k, v in zip(prompt_kv, st.cache.k, st.cache.vt):
        assert torch.equal(k[:, :T0], k0) and torch.equal(v[:, :, :T0], v0)
    for c in canvases:
        assert c.min() >= 0 and c.max() < cfg["vocab"]
    # a second, independent run of the whole chain is bit-identical
    st2 = PL.Setup(cfg, 0, capacity=cap, with_prefix=False)
    st2.ws = st2.workspace(max(T0, C))
    dg.prefill_append(st2.model, st2.cache, torch.from_numpy(prompt).cuda(), st2.ws)
    for c in range(n_can):
        can = torch.from_numpy(synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(c), C, cfg["vocab"])).cuda()
        dg.generate_canvas(st2.model, st2.cache, can, S, cfg["renoise_start"], cfg["renoise_end"],
                           synth.SEED_RENOISE, True, lg, st2.ws)
        np.testing.assert_array_equal(can.cpu().numpy(), canvases[c])
    for a, b in zip(st.cache.k, st2.cache.k):
        assert torch.equal(a, b)


def test_large4_full_size(dg):
    cfg = CF.CONFIGS["large4_bf16"]
    P, C, S = cfg["prefix"], cfg["canvas"], cfg["steps"]
    st = PL.Setup(cfg, P, capacity=P + C)
    st.ws = st.workspace(C)
    noise = synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(0), C, cfg["vocab"])
    n0 = O.renoise_count(C, S, 0, cfg["renoise_start"], cfg["renoise_end"])
    taps, logits, nxt, conf = _pass(dg, st, noise, n0, 0)
    logits_o, taps_o = O.denoise_pass(st.host, st.ocache, noise, st.prec)
    upd = O.canvas_update(logits_o, n0, synth.SEED_RENOISE, 0)
    report = []
    exempt = PL.compare_pass(cfg, taps, logits, taps_o, logits_o, report)
    PL.compare_update(nxt, conf, upd, exempt, n0)
    print("large4 first pass:", report, "exempt", sorted(exempt))
    unions = taps["unions"].cpu().numpy()
    assert (unions >= cfg["top_k"]).all() and (unions <= cfg["n_experts"]).all()
    assert [t["union"] for t in taps_o] == list(unions) or exempt
    # the 8-pass run: untouched prefix, tokens in range, bit-identical repeat
    before = [(k[:, :P].clone(), v[:, :, :P].clone()) for k, v in zip(st.cache.k, st.cache.vt)]
    st.model.set_taps(None)
    lg = torch.empty(C, cfg["vocab"], device="cuda")
    runs = []
    for _ in range(2):
        can = torch.from_numpy(noise).cuda()
        dg.generate_canvas(st.model, st.cache, can, S, cfg["renoise_start"], cfg["renoise_end"], synth.SEED_RENOISE,
                           False, lg, st.ws)
        runs.append(can.cpu().numpy())
    dg.device_status(st.ws)
    np.testing.assert_array_equal(runs[0], runs[1])
    assert runs[0].min() >= 0 and runs[0].max() < cfg["vocab"]
    for (k0, v0), k, v in zip(before, st.cache.k, st.cache.vt):
        assert torch.equal(k[:, :P], k0) and torch.equal(v[:, :, :P], v0)
