"""dg_canvas_update_noalloc (scratch in libdg's fixed device array) against
dg_canvas_update (scratch in a caller workspace): same canvas and confidences, bit for
bit, on two different calls issued back to back.  The file name sorts last so that the
check also runs after every other test has used the library on this device."""
import pytest
import torch

from block_diffusion_lm_masked_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_diffusion_lm_masked_b200 import dg as _dg
    return _dg


# (C, V, n_renoise, step): the single-layer workload's update, then a ragged one that
# uses a different slice count, so the second call rewrites the scratch differently
CALLS = [(256, 32768, 128, 0), (100, 4100, 7, 3)]


def _inputs(C, V, i):
    g = torch.Generator(device="cuda").manual_seed(1000 + i)
    logits = torch.randn(C, V, generator=g, device="cuda") * 3.0
    canvas = torch.from_numpy(synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(20 + i), C, V)).cuda()
    return logits, canvas


def test_noalloc_update_equals_workspace_update(dg):
    want = []
    for i, (C, V, n, step) in enumerate(CALLS):
        logits, canvas = _inputs(C, V, i)
        ws = torch.zeros(dg.update_workspace_bytes(C, V), dtype=torch.uint8, device="cuda")
        conf = torch.empty(C, device="cuda")
        dg.canvas_update(logits, n, synth.SEED_RENOISE, step, canvas, ws, conf)
        want.append((canvas, conf))
    got = []
    for i, (C, V, n, step) in enumerate(CALLS):   # back to back, no synchronisation between
        logits, canvas = _inputs(C, V, i)
        conf = torch.empty(C, device="cuda")
        dg.canvas_update_noalloc(logits, n, synth.SEED_RENOISE, step, canvas, conf)
        got.append((canvas, conf))
    torch.cuda.synchronize()
    for (wc, wf), (gc, gf) in zip(want, got):
        assert torch.equal(wc, gc)
        assert torch.equal(wf, gf)


def test_noalloc_update_rejects_bad_shapes(dg):
    logits = torch.zeros(1025, 8, device="cuda")
    canvas = torch.zeros(1025, dtype=torch.int32, device="cuda")
    with pytest.raises(dg.DGError, match="C must be"):
        dg.canvas_update_noalloc(logits, 0, 1, 0, canvas)
    logits = torch.zeros(4, 6, device="cuda")
    with pytest.raises(dg.DGError, match="multiple of 4"):
        dg.canvas_update_noalloc(logits, 0, 1, 0, canvas[:4])
