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


def _update_in_new_context(dg, logits_h, n, step, canvas_h):
    """The no-alloc update run inside a CUDA context created for it (not the primary
    context torch uses), on its own host thread, with buffers from the driver API: the
    array's address there is not the primary context's, so the library must look it up
    again for this context."""
    import ctypes
    import threading

    import numpy as np
    from cuda.bindings import driver as cu

    out = {}

    def ok(r):
        err = r[0] if isinstance(r, tuple) else r
        assert err == cu.CUresult.CUDA_SUCCESS, err
        return r[1] if isinstance(r, tuple) and len(r) > 1 else None

    def body():
        ctx = ok(cu.cuCtxCreate(0, ok(cu.cuDeviceGet(0))))
        bufs = []
        try:
            C, V = logits_h.shape
            d_log = ok(cu.cuMemAlloc(logits_h.nbytes)); bufs.append(d_log)
            d_can = ok(cu.cuMemAlloc(canvas_h.nbytes)); bufs.append(d_can)
            d_conf = ok(cu.cuMemAlloc(C * 4)); bufs.append(d_conf)
            ok(cu.cuMemcpyHtoD(d_log, logits_h.ctypes.data, logits_h.nbytes))
            ok(cu.cuMemcpyHtoD(d_can, canvas_h.ctypes.data, canvas_h.nbytes))
            for _ in range(2):   # the second call finds this context's cached address
                st = dg.lib.dg_canvas_update_noalloc(ctypes.c_void_p(int(d_log)), C, V, n, synth.SEED_RENOISE,
                                                     step, ctypes.c_void_p(int(d_can)),
                                                     ctypes.c_void_p(int(d_conf)), None)
                assert st == 0, dg.lib.dg_last_error()
                ok(cu.cuMemcpyHtoD(d_can, canvas_h.ctypes.data, canvas_h.nbytes))
            st = dg.lib.dg_canvas_update_noalloc(ctypes.c_void_p(int(d_log)), C, V, n, synth.SEED_RENOISE, step,
                                                 ctypes.c_void_p(int(d_can)), ctypes.c_void_p(int(d_conf)), None)
            assert st == 0, dg.lib.dg_last_error()
            ok(cu.cuCtxSynchronize())
            can = np.empty_like(canvas_h)
            conf = np.empty(C, dtype=np.float32)
            ok(cu.cuMemcpyDtoH(can.ctypes.data, d_can, can.nbytes))
            ok(cu.cuMemcpyDtoH(conf.ctypes.data, d_conf, conf.nbytes))
            out["canvas"], out["conf"] = can, conf
        except BaseException as e:  # reported on the main thread
            out["error"] = e
        finally:
            for b in bufs:
                cu.cuMemFree(b)
            cu.cuCtxDestroy(ctx)

    t = threading.Thread(target=body)
    t.start()
    t.join()
    if "error" in out:
        raise out["error"]
    return out["canvas"], out["conf"]


def test_noalloc_update_in_a_second_context(dg):
    """A context other than the primary one gets its own scratch address (the cache is
    keyed by context, not by device), and the result equals the workspace path's."""
    C, V, n, step = 256, 32768, 64, 5
    logits, canvas = _inputs(C, V, 7)
    logits_h = logits.cpu().numpy()
    canvas_h = canvas.cpu().numpy()
    dg.canvas_update_noalloc(logits, n, synth.SEED_RENOISE, step, canvas.clone())  # primary context first
    torch.cuda.synchronize()
    ws = torch.zeros(dg.update_workspace_bytes(C, V), dtype=torch.uint8, device="cuda")
    conf = torch.empty(C, device="cuda")
    want = canvas.clone()
    dg.canvas_update(logits, n, synth.SEED_RENOISE, step, want, ws, conf)
    got_canvas, got_conf = _update_in_new_context(dg, logits_h, n, step, canvas_h)
    assert (got_canvas == want.cpu().numpy()).all()
    assert (got_conf == conf.cpu().numpy()).all()
