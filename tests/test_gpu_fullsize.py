"""The multi-layer workloads at their full sizes, through the C-ABI, against the oracle.

Every pass of every run is compared stage by stage with the oracle, teacher-forced (the
oracle's stage applied to the GPU's own stage input; parity_lib states the rules): the
GPU runs its own chain of passes, updates and appends, and each of its stages is checked.
- 8-layer denoise (prefix 2048, canvas 256, 16 passes, re-noise 50% -> 0%): all 16
  passes; the run with taps equals the run without them and dg_generate_canvas, bit for
  bit; the prefix is untouched; the free-running token agreement with the oracle's own
  16-pass run is reported.
- chained canvases (8 layers, 512-token prompt, 4 canvases x 16 passes + append): the
  prompt's prefill, all 64 passes and all 4 appends; an independent run through
  dg_generate_canvas reproduces the chain bit for bit.
- large pass (4 layers, H2816, E128 top-8, F704, V262144, prefix 32768): all 8 passes;
  the run with taps equals dg_generate_canvas; the prefix is untouched.
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


def _pass(dg, st, canvas_np, n, step, seed=synth.SEED_RENOISE):
    """One GPU pass + update with taps on; returns (taps, logits, canvas out, conf)."""
    cfg = st.cfg
    C, V = len(canvas_np), cfg["vocab"]
    tp = st.taps(C)
    canvas = torch.from_numpy(np.asarray(canvas_np, dtype=np.int32)).cuda()
    logits = torch.empty(C, V, device="cuda")
    conf = torch.empty(C, device="cuda")
    dg.denoise_pass(st.model, st.cache, canvas, logits, st.ws)
    dg.canvas_update(logits, n, seed, step, canvas, st.ws, conf)
    dg.device_status(st.ws)
    return tp, logits.cpu().numpy(), canvas.cpu().numpy(), conf.cpu().numpy()


def _forced_run(dg, st, noise, S, r0, r1, label):
    """The GPU's own S passes from `noise`, each teacher-forced against the oracle on the
    cache as the GPU holds it; returns the GPU's final canvas."""
    C = len(noise)
    oc = PL.oracle_cache_from_gpu(st.cache)
    cur = np.asarray(noise, dtype=np.int32).copy()
    for s in range(S):
        n = O.renoise_count(C, S, s, r0, r1)
        taps, logits, nxt, conf = _pass(dg, st, cur, n, s)
        stats = PL.forced_pass_check(st.cfg, st.host, st.prec, oc, cur, taps, logits, nxt, conf, n,
                                     synth.SEED_RENOISE, s, label=f"{label} pass {s}")
        print(f"{label} pass {s}: n={n} forced {PL.summary(stats)}; unions "
              f"{taps['unions'].cpu().numpy().tolist()}", flush=True)
        cur = nxt
    return cur


def _forced_append(dg, st, toks, label):
    P0 = st.cache.len
    before = PL.oracle_cache_from_gpu(st.cache)
    tp = st.taps(len(toks))
    dg.prefill_append(st.model, st.cache, torch.from_numpy(np.asarray(toks, dtype=np.int32)).cuda(), st.ws)
    dg.device_status(st.ws)
    stats = PL.forced_prefill_check(st.cfg, st.host, st.prec, before, toks, tp, st.cache, P0, label=label)
    print(f"{label} at {P0}: forced {PL.summary(stats)}", flush=True)


def _gpu_loop(dg, st, noise, S, r0, r1):
    """The GPU's own S passes (pass + update), no taps."""
    C, V = len(noise), st.cfg["vocab"]
    st.model.set_taps(None)
    can = torch.from_numpy(np.asarray(noise, dtype=np.int32)).cuda()
    lg = torch.empty(C, V, device="cuda")
    for s in range(S):
        dg.denoise_pass(st.model, st.cache, can, lg, st.ws)
        dg.canvas_update(lg, dg.renoise_count(C, S, s, r0, r1), synth.SEED_RENOISE, s, can, st.ws)
    dg.device_status(st.ws)
    return can.cpu().numpy()


def _generate(dg, st, noise, S, r0, r1, append):
    C, V = len(noise), st.cfg["vocab"]
    st.model.set_taps(None)
    can = torch.from_numpy(np.asarray(noise, dtype=np.int32)).cuda()
    lg = torch.empty(C, V, device="cuda")
    dg.generate_canvas(st.model, st.cache, can, S, r0, r1, synth.SEED_RENOISE, append, lg, st.ws)
    dg.device_status(st.ws)
    return can.cpu().numpy()


def test_denoise8_full_size(dg):
    cfg = CF.CONFIGS["denoise8_bf16"]
    P, C, S = cfg["prefix"], cfg["canvas"], cfg["steps"]
    r0, r1 = cfg["renoise_start"], cfg["renoise_end"]
    st = PL.Setup(cfg, P, capacity=P + C)
    st.ws = st.workspace(C)
    before = [(k[:, :P].clone(), v[:, :, :P].clone()) for k, v in zip(st.cache.k, st.cache.vt)]
    noise = synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(0), C, cfg["vocab"])
    final = _forced_run(dg, st, noise, S, r0, r1, "denoise8")
    # taps change nothing: the plain loop and dg_generate_canvas give the same canvas
    g = _gpu_loop(dg, st, noise, S, r0, r1)
    np.testing.assert_array_equal(g, final)
    np.testing.assert_array_equal(_generate(dg, st, noise, S, r0, r1, False), g)
    assert g.min() >= 0 and g.max() < cfg["vocab"]
    for (k0, v0), k, v in zip(before, st.cache.k, st.cache.vt):
        assert torch.equal(k[:, :P], k0) and torch.equal(v[:, :, :P], v0)
    assert st.cache.len == P
    # reported: how many final tokens the oracle's own free-running 16 passes share
    oracle_final, _ = O.generate_canvas(st.host, st.ocache, noise, S, r0, r1, synth.SEED_RENOISE, st.prec, False)
    print(f"denoise8 free-running agreement with the oracle: {np.mean(oracle_final == g):.1%} of final tokens",
          flush=True)


def test_chained8_full_size(dg):
    cfg = CF.CONFIGS["chained8_bf16"]
    T0, C, S, n_can = cfg["prompt"], cfg["canvas"], cfg["steps"], cfg["n_canvases"]
    r0, r1 = cfg["renoise_start"], cfg["renoise_end"]
    cap = T0 + n_can * C
    st = PL.Setup(cfg, 0, capacity=cap, with_prefix=False)
    st.ws = st.workspace(max(T0, C))
    prompt = synth.tokens(synth.SEED_TOKENS, synth.TID_PREFIX_TOKENS, T0, cfg["vocab"])
    _forced_append(dg, st, prompt, "prompt prefill")
    canvases = []
    for c in range(n_can):
        noise = synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(c), C, cfg["vocab"])
        done = _forced_run(dg, st, noise, S, r0, r1, f"chained canvas {c}")
        assert done.min() >= 0 and done.max() < cfg["vocab"]
        canvases.append(done)
        _forced_append(dg, st, done, f"append {c}")
    assert st.cache.len == cap
    # an independent run through the public loop reproduces the chain bit for bit
    st2 = PL.Setup(cfg, 0, capacity=cap, with_prefix=False)
    st2.ws = st2.workspace(max(T0, C))
    st2.model.set_taps(None)
    dg.prefill_append(st2.model, st2.cache, torch.from_numpy(prompt).cuda(), st2.ws)
    for c in range(n_can):
        noise = synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(c), C, cfg["vocab"])
        np.testing.assert_array_equal(_generate(dg, st2, noise, S, r0, r1, True), canvases[c])
    assert st2.cache.len == cap
    for a, b, va, vb in zip(st.cache.k, st2.cache.k, st.cache.vt, st2.cache.vt):
        assert torch.equal(a, b) and torch.equal(va, vb)


def test_large4_full_size(dg):
    cfg = CF.CONFIGS["large4_bf16"]
    P, C, S = cfg["prefix"], cfg["canvas"], cfg["steps"]
    r0, r1 = cfg["renoise_start"], cfg["renoise_end"]
    st = PL.Setup(cfg, P, capacity=P + C)
    st.ws = st.workspace(C)
    before = [(k[:, :P].clone(), v[:, :, :P].clone()) for k, v in zip(st.cache.k, st.cache.vt)]
    noise = synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(0), C, cfg["vocab"])
    final = _forced_run(dg, st, noise, S, r0, r1, "large4")
    np.testing.assert_array_equal(_generate(dg, st, noise, S, r0, r1, False), final)
    assert final.min() >= 0 and final.max() < cfg["vocab"]
    for (k0, v0), k, v in zip(before, st.cache.k, st.cache.vt):
        assert torch.equal(k[:, :P], k0) and torch.equal(v[:, :, :P], v0)
    assert st.cache.len == P
