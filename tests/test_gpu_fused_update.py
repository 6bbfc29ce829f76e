"""dg_denoise_update (the pass with the update's statistics as the vocabulary
projection's epilogue, no logits) against the two-call path and against the oracle."""

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


def _both(dg, st, canvas_np, n, mask_id=-1, step=3):
    """(two-call canvas, conf, logits), (fused canvas, conf) from the same input."""
    C, V = len(canvas_np), st.cfg["vocab"]
    ws = st.workspace(C)
    logits = torch.empty(C, V, device="cuda")
    a = torch.from_numpy(np.asarray(canvas_np, dtype=np.int32)).cuda()
    ca = torch.empty(C, device="cuda")
    dg.denoise_pass(st.model, st.cache, a, logits, ws)
    if mask_id < 0:
        dg.canvas_update(logits, n, synth.SEED_RENOISE, step, a, ws, ca)
    else:
        dg.canvas_update_masked(logits, n, mask_id, a, ws, ca)
    b = torch.from_numpy(np.asarray(canvas_np, dtype=np.int32)).cuda()
    cb = torch.empty(C, device="cuda")
    dg.denoise_update(st.model, st.cache, b, n, ws, seed=synth.SEED_RENOISE, step=step, mask_id=mask_id, conf=cb)
    dg.device_status(ws)
    return (a.cpu().numpy(), ca.cpu().numpy(), logits.cpu().numpy()), (b.cpu().numpy(), cb.cpu().numpy())


@pytest.mark.parametrize("cfg,P,C", [(SMALL_BF16, 200, 100), (SMALL_BF16, 0, 37), (CF.CONFIGS["layer1_bf16"], 1024, 256),
                                     (CF.CONFIGS["large4_bf16"], 32768, 256)])
def test_fused_update_equals_the_two_call_path(dg, cfg, P, C):
    """The same accumulators feed both paths, so ids agree exactly and confidences to fp32
    summation order; the re-noise sets agree except where two confidences are that close."""
    st = PL.Setup(cfg, P)
    canvas0 = synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(2), C, cfg["vocab"])
    n = C // 4
    (ta, ca, logits), (tb, cb) = _both(dg, st, canvas0, n)
    np.testing.assert_allclose(cb, ca, rtol=2e-5)
    order = np.argsort(ca, kind="stable")
    cut_lo, cut_hi = ca[order[n - 1]], (ca[order[n]] if n < C else np.inf)
    close = (np.abs(ca - cut_lo) < 1e-4 * cut_lo) | (np.abs(ca - cut_hi) < 1e-4 * cut_hi)
    # the two paths' GEMMs may round the logits differently: a position whose top two
    # logits are that close may take either id
    top2 = np.sort(logits, axis=1)[:, -2:]
    near_tie = (top2[:, 1] - top2[:, 0]) <= 1e-5 * np.maximum(np.abs(top2[:, 1]), 1e-30)
    for i in range(C):
        if not close[i] and not near_tie[i]:
            assert ta[i] == tb[i], i


def test_fused_masked_update_equals_the_two_call_path(dg):
    cfg = SMALL_BF16
    st = PL.Setup(cfg, 64)
    C, mask_id = 64, cfg["vocab"] - 1
    canvas0 = np.where(np.arange(C) % 3 == 0, mask_id, synth.tokens(synth.SEED_TOKENS, 90, C, mask_id))
    (ta, ca, _), (tb, cb) = _both(dg, st, canvas0, 5, mask_id=mask_id)
    np.testing.assert_allclose(cb, ca, rtol=2e-5)
    masked = canvas0 == mask_id
    np.testing.assert_array_equal(tb[~masked], canvas0[~masked])
    assert (tb[masked] == mask_id).sum() == 5


def test_fused_update_matches_the_oracle_full_size(dg):
    """The fused call against the oracle's pass and update.  The rows exempt from the
    comparison (routing at a near tie, under the pass's parity rules) come from a tapped
    two-call pass over the same input: the layer stack is the same in both calls."""
    cfg = CF.CONFIGS["layer1_bf16"]
    st = PL.Setup(cfg, cfg["prefix"])
    C, V = cfg["canvas"], cfg["vocab"]
    canvas0 = synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(0), C, cfg["vocab"])
    n = O.renoise_count(C, 1, 0, 0.25, 0.25)
    ws = st.workspace(C)
    taps = st.taps(C)
    logits = torch.empty(C, V, device="cuda")
    dg.denoise_pass(st.model, st.cache, torch.from_numpy(canvas0.astype(np.int32)).cuda(), logits, ws)
    logits_o, taps_o = O.denoise_pass(st.host, st.ocache, canvas0, st.prec)
    exempt = PL.compare_pass(cfg, taps, logits.cpu().numpy(), taps_o, logits_o)
    out = torch.from_numpy(canvas0.astype(np.int32)).cuda()
    conf = torch.empty(C, device="cuda")
    taps_f = st.taps(C)   # the fused call's own layer stack, teacher-forced stage by stage
    dg.denoise_update(st.model, st.cache, out, n, ws, seed=synth.SEED_RENOISE, step=0, conf=conf)
    dg.device_status(ws)
    stats = PL.forced_pass_check(cfg, st.host, st.prec, st.ocache, canvas0, taps_f, None, label="fused pass")
    print("forced layers of the fused call:", PL.summary(stats))
    upd_o = O.canvas_update(logits_o, n, synth.SEED_RENOISE, 0)
    # the fused call's logits (never written) come from the same single-term input and
    # weights as the separate pass's, in another fp32 summation order: 1% slack
    shift = 1.01 * PL.logit_shift(logits.cpu().numpy(), logits_o, exempt)
    PL.compare_update(out.cpu().numpy(), conf.cpu().numpy(), upd_o, exempt, n, shift)
