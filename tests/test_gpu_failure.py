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


# device error codes the kernels record when a bounded wait gives up (TMA stage full /
# empty, accumulator hand-off, attention); dg_device_status maps them to DG_ERR_TIMEOUT
TIMEOUT_CODES = (1, 2, 3, 4)


def _gemm_case(dg, g):
    # long enough that the epilogue's first wait (for the first tile's MMAs over 128
    # k-blocks) lasts tens of microseconds, far beyond the timer's resolution
    K, M, n = 8192, 2048, 70
    W = (torch.randn(1, M, K, generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    X = torch.randn(n, K, generator=g, device="cuda").to(torch.bfloat16)
    out = torch.full((n, M), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    return W, X, out, err


def test_pre_expired_wait_limit_ends_gemm_and_attention_with_a_timeout():
    """With every bounded wait's limit at 0, a GEMM launch and an attention launch give up
    at their first wait that is not already satisfied: each records a timeout code, winds
    down (loads and MMAs in flight drained, TMEM freed) and returns; with the limit back
    at 2 s the same launches run correctly in the same context."""
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_diffusion_lm_masked_b200 import dg
    from block_diffusion_lm_masked_b200 import configs as CF
    g = torch.Generator(device="cuda").manual_seed(5)
    W, X, out, err = _gemm_case(dg, g)
    scratch = dg.debug_gemm_scratch(X.shape[0], 1)
    d, n_q, n_keys, nq, nkv = 128, 128, 1024, 4, 2
    q = torch.randn(nq, n_q, d, generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn(nkv, n_keys + 8, d, generator=g, device="cuda").to(torch.bfloat16)
    vt = torch.randn(nkv, d, n_keys + 8, generator=g, device="cuda").to(torch.bfloat16)
    cfg = dict(CF.CONFIGS["layer1_bf16"], n_q_heads=nq, n_kv_heads=nkv, hidden=128, expert_ffn=64, n_experts=1,
               top_k=1, vocab=128, n_layers=1)
    ws = dg.Workspace(cfg, n_q)
    o = torch.zeros(n_q, nq * d, dtype=torch.bfloat16, device="cuda")
    dg.device_status(ws)
    try:
        dg.debug_set_wait_limit(0)
        dg.debug_gemm_bf16(W, X, out, W.shape[1], err, scratch)
        torch.cuda.synchronize()
        assert err.item() in TIMEOUT_CODES, err.item()
        dg.debug_attention_bf16(q, k, vt, n_keys, n_keys - n_q, False, o, ws)
        with pytest.raises(dg.DGError) as ei:
            dg.device_status(ws)
        assert ei.value.status == dg.DG_ERR_TIMEOUT
    finally:
        dg.debug_set_wait_limit(dg.WAIT_LIMIT_DEFAULT_NS)
    torch.cuda.synchronize()
    # the same launches again, in the same context, complete and are right
    err.zero_()
    dg.debug_gemm_bf16(W, X, out, W.shape[1], err, scratch)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = X.double() @ W[0].double().T
    torch.testing.assert_close(out.double(), ref, rtol=1e-4, atol=1e-3 * ref.abs().max().item())
    dg.debug_attention_bf16(q, k, vt, n_keys, n_keys - n_q, False, o, ws)
    dg.device_status(ws)
    assert torch.isfinite(o.float()).all()
