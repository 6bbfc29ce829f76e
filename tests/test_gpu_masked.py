"""The masked-diffusion update and generation loop on the GPU against the oracle."""
import numpy as np
import pytest
import torch

from block_diffusion_lm_masked_b200 import configs as CF
from block_diffusion_lm_masked_b200 import synth
from oracle import dg_oracle as O

import parity_lib as PL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_diffusion_lm_masked_b200 import dg as _dg
    return _dg


@pytest.mark.parametrize("C,V,frac,n_keep,mask_id", [(256, 32768, 0.6, 64, 32767), (100, 4100, 0.3, 7, 0),
                                                     (37, 1024, 1.0, 0, 512), (64, 2048, 0.5, 64, 5)])
def test_masked_update_matches_oracle(dg, C, V, frac, n_keep, mask_id):
    g = torch.Generator(device="cuda").manual_seed(C + V)
    logits = torch.randn(C, V, generator=g, device="cuda") * 3.0
    # the mask id's own logit is often the largest: it must never be used as a fill
    logits[: C // 3, mask_id] += 20.0
    rng = np.random.default_rng(C)
    canvas_np = np.where(rng.random(C) < frac, mask_id, rng.integers(0, V, C)).astype(np.int32)
    canvas = torch.from_numpy(canvas_np).cuda()
    conf = torch.empty(C, device="cuda")
    ws = torch.zeros(dg.update_workspace_bytes(C, V), dtype=torch.uint8, device="cuda")
    dg.canvas_update_masked(logits, n_keep, mask_id, canvas, ws, conf)
    got = canvas.cpu().numpy()
    want = O.canvas_update_masked(logits.double().cpu().numpy(), canvas_np, n_keep, mask_id)
    locked = canvas_np != mask_id
    np.testing.assert_array_equal(got[locked], canvas_np[locked])
    masked = np.nonzero(~locked)[0]
    assert int((got[masked] == mask_id).sum()) == min(n_keep, len(masked))
    kept_o = set(want["kept"].tolist())
    kept_g = {int(i) for i in masked if got[i] == mask_id}
    for i in kept_g ^ kept_o:
        assert want["cut_margin"][i] < PL.CUT_MARGIN, (i, want["cut_margin"][i])
    for i in masked:
        if i in kept_g or i in kept_o:
            continue
        # both sides take the argmax of the same logits (ties to the lowest id): identical
        assert got[i] == want["canvas"][i], (i, got[i], want["canvas"][i])
        assert got[i] != mask_id
    # confidences of identical logits: fp32 against fp64 arithmetic
    np.testing.assert_allclose(conf.cpu().numpy()[masked], want["conf"][masked], rtol=PL.CONF_RTOL, atol=1e-30)


def test_generate_masked_matches_oracle_and_step_loop(dg):
    """From an all-[MASK] canvas: the loop unmasks C/S positions per pass, ends with none,
    never changes a filled position, equals the documented pass / update loop, and its
    first pass matches the oracle."""
    cfg = CF.CONFIGS["tiny_fp32"]
    C, S, mask_id = cfg["canvas"], 4, cfg["vocab"] - 1
    a = PL.Setup(cfg, 16, capacity=16 + 2 * C)
    b = PL.Setup(cfg, 16, capacity=16 + 2 * C)
    ws_a, ws_b = a.workspace(C), b.workspace(C)
    lg = torch.empty(C, cfg["vocab"], device="cuda")
    can_a = torch.zeros(C, dtype=torch.int32, device="cuda")
    dg.generate_canvas_masked(a.model, a.cache, can_a, S, (S - 1) / S, 0.0, mask_id, True, lg, ws_a)
    dg.device_status(ws_a)
    # the step loop through the public calls
    can_b = torch.full((C,), mask_id, dtype=torch.int32, device="cuda")
    prev = can_b.cpu().numpy()
    for s in range(S):
        dg.denoise_pass(b.model, b.cache, can_b, lg, ws_b)
        if s == 0:
            logits_o, _ = O.denoise_pass(b.host, b.ocache, prev, b.prec)
            assert PL.rel_err(lg.cpu().numpy(), logits_o) <= PL.tol(cfg)
        n = dg.renoise_count(C, S, s, (S - 1) / S, 0.0)
        dg.canvas_update_masked(lg, n, mask_id, can_b, ws_b)
        cur = can_b.cpu().numpy()
        filled = prev != mask_id
        np.testing.assert_array_equal(cur[filled], prev[filled])
        assert int((cur == mask_id).sum()) == n
        prev = cur
    dg.prefill_append(b.model, b.cache, can_b, ws_b)
    dg.device_status(ws_b)
    assert torch.equal(can_a, can_b)
    assert not (can_a == mask_id).any()
    assert a.cache.len == b.cache.len == 16 + C
    for l in range(cfg["n_layers"]):
        assert torch.equal(a.cache.k[l], b.cache.k[l]) and torch.equal(a.cache.vt[l], b.cache.vt[l])
