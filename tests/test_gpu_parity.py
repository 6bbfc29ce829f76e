"""The CUDA path against the CPU oracle on the same seeded inputs, through the C-ABI.

Sizes: the tiny fp32 model and the single-layer bf16 pass at their full workload
sizes; reduced bf16 models whose canvas and prefix lengths are ragged (not
multiples of the 128-row tiles) and span several key chunks; a chained run of
prefill + denoise + append.  Comparison rules are in parity_lib.
"""
import numpy as np
import pytest
import torch

from block_diffusion_lm_masked_b200 import configs as CF
from block_diffusion_lm_masked_b200 import synth
from oracle import dg_oracle as O

import parity_lib as PL

pytestmark = pytest.mark.gpu

SMALL_BF16 = dict(n_layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=128, n_experts=8, top_k=2,
                  expert_ffn=192, vocab=2048, rope_theta=10000.0, rms_eps=1e-6, dtype="bf16")


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_diffusion_lm_masked_b200 import dg as _dg
    return _dg


def _gpu_pass(dg, st, canvas_np, n, step=0, taps=True):
    cfg = st.cfg
    C, V = len(canvas_np), cfg["vocab"]
    tp = st.taps(C) if taps else None
    ws = st.workspace(C)
    canvas = torch.from_numpy(np.asarray(canvas_np, dtype=np.int32)).cuda()
    logits = torch.empty(C, V, device="cuda")
    conf = torch.empty(C, device="cuda")
    dg.denoise_pass(st.model, st.cache, canvas, logits, ws)
    dg.canvas_update(logits, n, synth.SEED_RENOISE, step, canvas, ws, conf)
    dg.device_status(ws)
    return tp, logits.cpu().numpy(), canvas.cpu().numpy(), conf.cpu().numpy()


def _check_one_pass(dg, cfg, P, C):
    """One pass + update: every stage teacher-forced against the oracle, and the whole
    pass free-running against the oracle's pass from the same canvas."""
    st = PL.Setup(cfg, P)
    canvas0 = synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(0), C, cfg["vocab"])
    n = O.renoise_count(C, 1, 0, 0.25, 0.25)
    taps, logits, canvas, conf = _gpu_pass(dg, st, canvas0, n)
    stats = PL.forced_pass_check(cfg, st.host, st.prec, st.ocache, canvas0, taps, logits, canvas, conf, n,
                                 synth.SEED_RENOISE, 0)
    logits_o, taps_o = O.denoise_pass(st.host, st.ocache, canvas0, st.prec)
    upd_o = O.canvas_update(logits_o, n, synth.SEED_RENOISE, 0)
    report = []
    exempt = PL.compare_pass(cfg, taps, logits, taps_o, logits_o, report)
    PL.compare_update(canvas, conf, upd_o, exempt, n, PL.logit_shift(logits, logits_o, exempt))
    print("forced:", PL.summary(stats), "| free-running:", report, "exempt rows:", sorted(exempt))
    return st


def test_tiny_fp32_pass(dg):
    cfg = CF.CONFIGS["tiny_fp32"]
    _check_one_pass(dg, cfg, cfg["prefix"], cfg["canvas"])


def test_small_bf16_pass_ragged(dg):
    # 200 cached + 100 canvas positions: one partial 128-row query tile, 3 key chunks (ragged tail)
    _check_one_pass(dg, SMALL_BF16, 200, 100)


def test_small_bf16_pass_empty_prefix(dg):
    _check_one_pass(dg, dict(SMALL_BF16, n_layers=1), 0, 37)


def test_layer1_bf16_full_size(dg):
    cfg = CF.CONFIGS["layer1_bf16"]
    _check_one_pass(dg, cfg, cfg["prefix"], cfg["canvas"])


def test_prefill_append_matches_oracle(dg):
    """Two prefills (77 tokens into an empty cache, then 150 more): every layer's stored
    K/V and every stage teacher-forced against the oracle; the whole chain free-running
    up to the causal reach of a near-tie routing difference."""
    cfg = SMALL_BF16
    st = PL.Setup(cfg, 0, capacity=512, with_prefix=False)
    ws = st.workspace(300)
    prompt = synth.tokens(synth.SEED_TOKENS, synth.TID_PREFIX_TOKENS, 77, cfg["vocab"])
    more = synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(9), 150, cfg["vocab"])
    runs = []
    for toks in (prompt, more):
        P0 = st.ocache.len
        before = PL.oracle_cache_from_gpu(st.cache)
        tp = st.taps(len(toks))
        dg.prefill_append(st.model, st.cache, torch.from_numpy(toks).cuda(), ws)
        dg.device_status(ws)
        stats = PL.forced_prefill_check(cfg, st.host, st.prec, before, toks, tp, st.cache, P0)
        print(f"prefill at {P0}: forced", PL.summary(stats))
        taps = []
        st.ocache = O.prefill_append(st.host, st.ocache, toks, st.prec, taps)
        runs.append((P0, [t.cpu().numpy() for t in tp["topk_idx"]], taps))
    assert st.cache.len == 227 == st.ocache.len
    seen = PL.kv_close_causal(st.cache, st.ocache, PL.causal_reach(runs, cfg["n_layers"]), "prefill")
    assert seen >= 0.5


def test_mask_worked_example_on_gpu(dg):
    """The 7x7 prefix/block example: 3 prefix tokens prefilled (causal rows), then a
    4-token block denoised against them (bidirectional rows); the logits must equal
    the oracle's recomputation of all 7 positions under the printed mask."""
    cfg = dict(SMALL_BF16, n_layers=2)
    st = PL.Setup(cfg, 0, capacity=64, with_prefix=False)
    ws = st.workspace(8)
    pre = np.array([11, 400, 7], dtype=np.int32)
    blk = np.array([5, 1999, 64, 300], dtype=np.int32)
    dg.prefill_append(st.model, st.cache, torch.from_numpy(pre).cuda(), ws)
    logits = torch.empty(4, cfg["vocab"], device="cuda")
    dg.denoise_pass(st.model, st.cache, torch.from_numpy(blk).cuda(), logits, ws)
    dg.device_status(ws)
    _, _, full = O.full_sequence_states(st.host, pre, blk, st.prec)
    assert PL.rel_err(logits.cpu().numpy(), full) < 2e-2


def test_chained_canvases_small(dg):
    """prompt prefill -> (S denoising steps with re-noising -> append) x 2, the GPU running
    its own chain: every pass and every append teacher-forced against the oracle, each
    stage on the GPU's own input (its canvas, its cache)."""
    cfg = dict(SMALL_BF16, n_layers=2)
    C, S, n_can = 64, 3, 2
    st = PL.Setup(cfg, 0, capacity=512, with_prefix=False)
    ws = st.workspace(96)
    prompt = synth.tokens(synth.SEED_TOKENS, synth.TID_PREFIX_TOKENS, 96, cfg["vocab"])
    _forced_append(dg, st, prompt, ws, "prompt")
    for c in range(n_can):
        cur = synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(c), C, cfg["vocab"])
        oc = PL.oracle_cache_from_gpu(st.cache)
        for s in range(S):
            n = O.renoise_count(C, S, s, 0.5, 0.0)
            taps, logits, nxt_g, conf = _gpu_pass(dg, st, cur, n, step=s)
            stats = PL.forced_pass_check(cfg, st.host, st.prec, oc, cur, taps, logits, nxt_g, conf, n,
                                         synth.SEED_RENOISE, s, label=f"canvas {c} pass {s}")
            print(f"canvas {c} pass {s}: forced", PL.summary(stats))
            cur = nxt_g
        _forced_append(dg, st, cur, ws, f"append {c}")
    dg.device_status(ws)
    assert st.cache.len == 96 + n_can * C


def _forced_append(dg, st, toks, ws, label):
    P0 = st.cache.len
    before = PL.oracle_cache_from_gpu(st.cache)
    tp = st.taps(len(toks))
    dg.prefill_append(st.model, st.cache, torch.from_numpy(np.asarray(toks, dtype=np.int32)).cuda(), ws)
    dg.device_status(ws)
    stats = PL.forced_prefill_check(st.cfg, st.host, st.prec, before, toks, tp, st.cache, P0, label=label)
    print(f"{label}: forced", PL.summary(stats))


def test_generate_canvas_equals_step_loop(dg):
    """dg_generate_canvas runs exactly the documented pass / update / append sequence."""
    cfg = dict(SMALL_BF16, n_layers=1)
    C, S = 48, 4
    a = PL.Setup(cfg, 40, capacity=256)
    b = PL.Setup(cfg, 40, capacity=256)
    noise = torch.from_numpy(synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(3), C, cfg["vocab"])).cuda()
    ws_a, ws_b = a.workspace(C), b.workspace(C)
    lg = torch.empty(C, cfg["vocab"], device="cuda")
    can_a = noise.clone()
    dg.generate_canvas(a.model, a.cache, can_a, S, 0.5, 0.0, 77, True, lg, ws_a)
    can_b = noise.clone()
    for s in range(S):
        dg.denoise_pass(b.model, b.cache, can_b, lg, ws_b)
        dg.canvas_update(lg, dg.renoise_count(C, S, s, 0.5, 0.0), 77, s, can_b, ws_b)
    dg.prefill_append(b.model, b.cache, can_b, ws_b)
    dg.device_status(ws_a)
    assert torch.equal(can_a, can_b)
    assert a.cache.len == b.cache.len == 40 + C
    for l in range(cfg["n_layers"]):
        assert torch.equal(a.cache.k[l], b.cache.k[l]) and torch.equal(a.cache.vt[l], b.cache.vt[l])


def test_prefix_cache_unchanged_and_deterministic(dg):
    """Denoising passes never touch cache slots [0, P); two runs are bit-identical."""
    cfg = SMALL_BF16
    st = PL.Setup(cfg, 300, capacity=640)
    before_k = [t[:, :300].clone() for t in st.cache.k]
    before_v = [t[:, :, :300].clone() for t in st.cache.vt]
    C = 256
    ws = st.workspace(C)
    noise = torch.from_numpy(synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(0), C, cfg["vocab"])).cuda()
    outs = []
    for _ in range(2):
        can = noise.clone()
        lg = torch.empty(C, cfg["vocab"], device="cuda")
        dg.generate_canvas(st.model, st.cache, can, 5, 0.5, 0.0, 1236, False, lg, ws)
        outs.append((can.clone(), lg.clone()))
    dg.device_status(ws)
    assert st.cache.len == 300
    for l in range(cfg["n_layers"]):
        assert torch.equal(st.cache.k[l][:, :300], before_k[l])
        assert torch.equal(st.cache.vt[l][:, :, :300], before_v[l])
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_capacity_error_leaves_cache_unchanged(dg):
    cfg = dict(SMALL_BF16, n_layers=1)
    st = PL.Setup(cfg, 100, capacity=128)
    ws = st.workspace(64)
    toks = torch.zeros(64, dtype=torch.int32, device="cuda")
    with pytest.raises(dg.DGError) as ei:
        dg.prefill_append(st.model, st.cache, toks, ws)
    assert ei.value.status == dg.DG_ERR_CAPACITY and st.cache.len == 100
    with pytest.raises(dg.DGError):
        dg.denoise_pass(st.model, st.cache, toks, torch.empty(64, cfg["vocab"], device="cuda"), ws)


def test_out_of_range_token_is_reported(dg):
    cfg = dict(SMALL_BF16, n_layers=1)
    st = PL.Setup(cfg, 16, capacity=64)
    ws = st.workspace(8)
    toks = torch.tensor([1, 2, cfg["vocab"] + 5, 3], dtype=torch.int32, device="cuda")
    dg.denoise_pass(st.model, st.cache, toks, torch.empty(4, cfg["vocab"], device="cuda"), ws)
    with pytest.raises(dg.DGError) as ei:
        dg.device_status(ws)
    assert ei.value.status == dg.DG_ERR_INVALID_ARG
    dg.device_status(ws)   # the error word was cleared
