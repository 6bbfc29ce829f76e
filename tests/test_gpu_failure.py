"""Failure detection on the GPU without a fault: a bounded device-side wait that runs
out is reported as DG_ERR_TIMEOUT, and the context stays usable afterwards."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_cleanly():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_diffusion_lm_masked_b200 import dg
    ws = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    dg.device_status(ws)                       # clean to start with
    dg.debug_bounded_wait(ws, 200)             # nothing completes the barrier: gives up after 0.2 s
    with pytest.raises(dg.DGError) as ei:
        dg.device_status(ws)
    assert ei.value.status == dg.DG_ERR_TIMEOUT
    dg.device_status(ws)                       # the error word was cleared
    x = torch.arange(10, device="cuda").sum()  # the context still works
    assert int(x) == 45
