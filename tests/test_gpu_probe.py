"""The tensor-pipe rate probe (dg_debug_mma_rate) runs and reports a plausible rate."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_mma_rate_probe_reports_cycles_per_instruction():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_diffusion_lm_masked_b200 import dg
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for a_tmem in (False, True):
        per = {}
        for n in (128, 256):
            cyc, ms = dg.debug_mma_rate(a_tmem, n, 2048, sms)
            assert cyc > 0 and ms > 0
            per[n] = cyc / 2048
            # at least the nominal time (64 cycles per 128 columns), at most a few times it
            assert n / 2 <= per[n] <= 8 * n, (a_tmem, n, per[n])
        assert per[256] / 256 <= per[128] / 128 * 1.05   # wider instructions are not slower per column
