"""No kernel reads workspace it has not written in the same call: a pass and its update
with the workspace filled with NaN bytes (the error word cleared) give bit-identical
logits and canvas to a zero-filled workspace."""

import numpy as np
import pytest
import torch

from block_diffusion_lm_masked_b200 import configs as CF
from block_diffusion_lm_masked_b200 import synth

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


def _run(dg, st, canvas0, fill):
    C, V = len(canvas0), st.cfg["vocab"]
    ws = st.workspace(C)
    ws.buf.fill_(fill)
    ws.buf[:4].zero_()                               # the error word
    logits = torch.empty(C, V, device="cuda")
    canvas = torch.from_numpy(canvas0.astype(np.int32)).cuda()
    dg.denoise_pass(st.model, st.cache, canvas, logits, ws)
    dg.canvas_update(logits, C // 4, synth.SEED_RENOISE, 0, canvas, ws)
    dg.device_status(ws)
    return logits.cpu().numpy(), canvas.cpu().numpy()


@pytest.mark.parametrize("cfg,P,C", [(CF.CONFIGS["tiny_fp32"], 64, 32), (SMALL_BF16, 200, 100),
                                     (CF.CONFIGS["layer1_bf16"], 1024, 256)])
def test_poisoned_workspace_changes_nothing(dg, cfg, P, C):
    st = PL.Setup(cfg, P)
    canvas0 = synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(4), C, cfg["vocab"])
    l0, c0 = _run(dg, st, canvas0, 0)
    l1, c1 = _run(dg, st, canvas0, 0xFF)             # every fp32 / bf16 scratch value a NaN
    assert np.isfinite(l1).all()
    np.testing.assert_array_equal(l1, l0)
    np.testing.assert_array_equal(c1, c0)
