"""Several canvases in one call (dg_denoise_pass_batched, dg_prefill_append_batched,
dg_generate_canvases) against the oracle and against the single-canvas calls.

Each canvas has its own cache with its own prefix length, including an empty one and
ragged ones.  The batch's taps hold all B C rows; the oracle's per-canvas taps are
merged the same way (rows stacked, experts grouped over the batch) and compared with
the single-pass rules of parity_lib.
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


def test_tiny_fp32_batched_pass(dg):
    cfg = CF.CONFIGS["tiny_fp32"]
    PL.check_batched_pass(dg, cfg, [cfg["prefix"], 0, 17], cfg["canvas"])


def test_small_bf16_batched_pass_ragged(dg):
    # ragged prefixes (one empty) and a canvas that is not a multiple of the 128-row tiles
    PL.check_batched_pass(dg, SMALL_BF16, [200, 0, 131, 64], 100)


def test_layer1_bf16_batched_full_size(dg):
    cfg = CF.CONFIGS["layer1_bf16"]
    PL.check_batched_pass(dg, cfg, [cfg["prefix"], cfg["prefix"] // 2], cfg["canvas"])


def test_layer1_bf16_four_canvases_as_the_bench_runs_them(dg):
    """The bench variant's shape: four canvases over full prefixes (1024 rows, four
    vocabulary chunks of 256)."""
    cfg = CF.CONFIGS["layer1_bf16"]
    PL.check_batched_pass(dg, cfg, [cfg["prefix"]] * 4, cfg["canvas"])


def test_batched_pass_equals_single_passes(dg):
    """Canvas b of a batch against the single-canvas call on the same cache: the fp32
    model's kernels compute every row alone, so the logits agree to fp32 rounding; the
    bf16 model's split-K factors follow the row count, so its logits agree to the
    hidden-state tolerance."""
    for cfg, prefixes, C in ((CF.CONFIGS["tiny_fp32"], [64, 0, 9], 32), (SMALL_BF16, [150, 0], 70)):
        B = len(prefixes)
        bt = PL.BatchSetup(dg, cfg, prefixes, PL.round_up(max(prefixes) + C + 8, 8))
        V = cfg["vocab"]
        canv = PL.batch_canvases(cfg, B, C, first=5)
        ws = dg.Workspace(cfg, B * C)
        lb = torch.empty(B, C, V, device="cuda")
        dg.denoise_pass_batched(bt.model, bt.caches, torch.from_numpy(canv).cuda(), lb, ws)
        for b in range(B):
            ls = torch.empty(C, V, device="cuda")
            dg.denoise_pass(bt.model, bt.caches[b], torch.from_numpy(canv[b]).cuda(), ls, ws)
            err = PL.rel_err(lb[b].cpu().numpy(), ls.cpu().numpy())
            assert err <= (1e-6 if cfg["dtype"] == "f32" else PL.tol(cfg)), (cfg["dtype"], b, err)
        dg.device_status(ws)


def test_prefill_append_batched_matches_oracle(dg):
    cfg = SMALL_BF16
    prefixes = [0, 40, 0]
    B, T = len(prefixes), 77
    bt = PL.BatchSetup(dg, cfg, prefixes, 256)
    prompts = np.stack([synth.tokens(synth.SEED_TOKENS, synth.TID_PREFIX_TOKENS + 50 + b, T, cfg["vocab"])
                        for b in range(B)]).astype(np.int32)
    topk = bt.taps(B * T)["topk_idx"]
    ws = dg.Workspace(cfg, B * T)
    dg.prefill_append_batched(bt.model, bt.caches, torch.from_numpy(prompts).cuda(), ws)
    dg.device_status(ws)
    for b in range(B):
        P0 = bt.ocaches[b].len
        taps = []
        oc = O.prefill_append(bt.host, bt.ocaches[b], prompts[b], bt.prec, taps)
        assert bt.caches[b].len == P0 + T == oc.len
        rows = [t.cpu().numpy()[b * T:(b + 1) * T] for t in topk]
        seen = PL.kv_close_causal(bt.caches[b], oc, PL.causal_reach([(P0, rows, taps)], cfg["n_layers"]),
                                  f"batched prefill canvas {b}")
        assert seen >= 0.5


def test_generate_canvases_equals_single_generation_fp32(dg):
    """dg_generate_canvases on the fp32 model: each canvas's final tokens and appended
    K/V are those of dg_generate_canvas on its own (rows are computed alone there)."""
    cfg = CF.CONFIGS["tiny_fp32"]
    prefixes, C, S = [64, 0], 32, 4
    B = len(prefixes)
    seeds = [synth.SEED_RENOISE, synth.SEED_RENOISE + 7]
    a = PL.BatchSetup(dg, cfg, prefixes, 256)
    s = PL.BatchSetup(dg, cfg, prefixes, 256)
    canv = PL.batch_canvases(cfg, B, C, first=11)
    ws = dg.Workspace(cfg, B * C)
    lb = torch.empty(B, C, cfg["vocab"], device="cuda")
    out = torch.from_numpy(canv).cuda()
    dg.generate_canvases(a.model, a.caches, out, S, 0.5, 0.0, seeds, True, lb, ws)
    for b in range(B):
        one = torch.from_numpy(canv[b]).cuda()
        ls = torch.empty(C, cfg["vocab"], device="cuda")
        dg.generate_canvas(s.model, s.caches[b], one, S, 0.5, 0.0, seeds[b], True, ls, ws)
        np.testing.assert_array_equal(out[b].cpu().numpy(), one.cpu().numpy())
        assert a.caches[b].len == s.caches[b].len == prefixes[b] + C
        for l in range(cfg["n_layers"]):
            ka, va = a.caches[b].logical(l)
            ks, vs = s.caches[b].logical(l)
            np.testing.assert_allclose(ka, ks, rtol=1e-5, atol=1e-6)
            np.testing.assert_allclose(va, vs, rtol=1e-5, atol=1e-6)
    dg.device_status(ws)


def test_generate_canvases_masked_equals_single_generation_fp32(dg):
    """The masked batched generation against the single-canvas masked generation on the
    fp32 model: each canvas ends fully unmasked with the tokens of its own run."""
    cfg = CF.CONFIGS["tiny_fp32"]
    prefixes, C, S, mask_id = [64, 0], 32, 4, cfg["vocab"] - 1
    a = PL.BatchSetup(dg, cfg, prefixes, 256)
    s = PL.BatchSetup(dg, cfg, prefixes, 256)
    ws = dg.Workspace(cfg, len(prefixes) * C)
    lb = torch.empty(len(prefixes), C, cfg["vocab"], device="cuda")
    out = torch.empty(len(prefixes), C, dtype=torch.int32, device="cuda")
    dg.generate_canvases_masked(a.model, a.caches, out, S, (S - 1) / S, 0.0, mask_id, True, lb, ws)
    for b in range(len(prefixes)):
        one = torch.empty(C, dtype=torch.int32, device="cuda")
        ls = torch.empty(C, cfg["vocab"], device="cuda")
        dg.generate_canvas_masked(s.model, s.caches[b], one, S, (S - 1) / S, 0.0, mask_id, True, ls, ws)
        np.testing.assert_array_equal(out[b].cpu().numpy(), one.cpu().numpy())
        assert not (out[b] == mask_id).any()
        assert a.caches[b].len == s.caches[b].len == prefixes[b] + C
    dg.device_status(ws)
