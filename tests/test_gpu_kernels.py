"""Single-kernel checks of the tcgen05 GEMM and attention launches against plain
PyTorch fp32 on the same device (the GPU's own reference of the same op), on
shapes with ragged token counts, several tiles and empty groups."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_diffusion_lm_masked_b200 import dg as _dg
    return _dg


def _bf(*shape, scale=1.0, gen=None):
    return (torch.randn(*shape, generator=gen, device="cuda") * scale).to(torch.bfloat16)


def _scratch(dg, rows, groups):
    return dg.debug_gemm_scratch(rows, groups)


@pytest.mark.parametrize("M,K,n", [(128, 64, 1), (256, 128, 16), (384, 512, 100), (128, 2048, 256), (256, 256, 300),
                                   (1408, 2816, 37), (704, 128, 50)])
def test_dense_gemm_store(dg, M, K, n):
    g = torch.Generator(device="cuda").manual_seed(M * 7 + n)
    W, X = _bf(1, M, K, gen=g), _bf(n, K, gen=g)
    out = torch.full((n, M), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dg.debug_gemm_bf16(W, X, out, M, err, _scratch(dg, n, 1))
    torch.cuda.synchronize()
    ref = X.float() @ W[0].float().T
    assert err.item() == 0
    torch.testing.assert_close(out, ref, rtol=1e-4, atol=1e-3 * ref.abs().max().item())


def test_two_term_gemm_is_fp32_accurate(dg):
    """X given as bf16 hi + lo: the product matches the fp32 X to ~16 significant bits."""
    g = torch.Generator(device="cuda").manual_seed(11)
    M, K, n = 256, 1024, 200
    W = _bf(1, M, K, gen=g)
    Xf = torch.randn(n, K, generator=g, device="cuda")
    hi = Xf.to(torch.bfloat16)
    lo = (Xf - hi.float()).to(torch.bfloat16)
    out = torch.full((n, M), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dg.debug_gemm_bf16(W, hi, out, M, err, _scratch(dg, n, 1), X_lo=lo)
    torch.cuda.synchronize()
    ref = (Xf.double() @ W[0].double().T).float()
    single = hi.float() @ W[0].float().T
    e2 = ((out - ref).abs().max() / ref.abs().max()).item()
    e1 = ((single - ref).abs().max() / ref.abs().max()).item()
    assert e2 < 2e-5 and e2 < e1 / 20, (e2, e1)


def _groups(counts):
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return torch.from_numpy(off).cuda(), int(off[-1])


@pytest.mark.parametrize("counts,M", [([0, 3, 17, 40, 1], 256), ([16, 0, 0, 256, 5, 33], 128), ([300, 2], 704),
                                      ([64, 65, 0, 129], 2816)])
def test_grouped_gemm(dg, counts, M):
    g = torch.Generator(device="cuda").manual_seed(sum(counts) + M)
    E, K = len(counts), 192
    off, rows = _groups(counts)
    W, X = _bf(E, M, K, gen=g), _bf(rows, K, gen=g)
    out = torch.full((rows, M), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dg.debug_gemm_bf16(W, X, out, M, err, _scratch(dg, rows, E), group_off=off)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = torch.empty_like(out)
    o = off.cpu().numpy()
    for e in range(E):
        ref[o[e]:o[e + 1]] = X[o[e]:o[e + 1]].float() @ W[e].float().T
    torch.testing.assert_close(out, ref, rtol=1e-4, atol=1e-3 * ref.abs().max().item())


def test_grouped_gemm_rejects_decreasing_offsets(dg):
    """Group offsets are device data in this entry; decreasing ones give no work and the
    bad-count error code instead of a launch over negative row counts."""
    W, X = _bf(3, 128, 64), _bf(40, 64)
    off = torch.tensor([0, 30, 10, 40], dtype=torch.int32, device="cuda")
    out = torch.full((40, 128), 7.0, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dg.debug_gemm_bf16(W, X, out, 128, err, _scratch(dg, 40, 3), group_off=off)
    torch.cuda.synchronize()
    assert err.item() == 5
    assert (out == 7.0).all()


@pytest.mark.parametrize("F", [128, 704])
def test_gate_up_swiglu_epilogue(dg, F):
    g = torch.Generator(device="cuda").manual_seed(5 + F)
    counts = [5, 0, 70, 16, 130]
    E, K = len(counts), 256
    off, rows = _groups(counts)
    gate, up = _bf(E, F, K, scale=0.1, gen=g), _bf(E, F, K, scale=0.1, gen=g)
    Xf = torch.randn(rows, K, generator=g, device="cuda")
    X, X_lo = Xf.to(torch.bfloat16), (Xf - Xf.to(torch.bfloat16).float()).to(torch.bfloat16)
    h = torch.zeros(rows, F, dtype=torch.bfloat16, device="cuda")
    h_lo = torch.zeros(rows, F, dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dg.debug_gemm_bf16(gate, X, h, F, err, _scratch(dg, rows, E), W2=up, X_lo=X_lo, group_off=off, out_lo=h_lo)
    torch.cuda.synchronize()
    assert err.item() == 0
    o = off.cpu().numpy()
    ref = torch.empty(rows, F, device="cuda", dtype=torch.float64)
    for e in range(E):
        xs = Xf[o[e]:o[e + 1]].double()
        a, b = xs @ gate[e].double().T, xs @ up[e].double().T
        ref[o[e]:o[e + 1]] = torch.nn.functional.silu(a) * b
    got = h.double() + h_lo.double()
    torch.testing.assert_close(got, ref, rtol=1e-4, atol=1e-5 * ref.abs().max().item())


def _attn_ref(q, k, vt, n_keys, pos0, causal):
    """The definition in fp64 on the same bf16 inputs."""
    nq, n_q, d = q.shape
    nkv = k.shape[0]
    g = nq // nkv
    out = torch.empty(n_q, nq * d, device="cuda", dtype=torch.float64)
    kk = k[:, :n_keys].double()
    vv = vt[:, :, :n_keys].double().transpose(1, 2)
    pos = torch.arange(n_q, device="cuda") + pos0
    keys = torch.arange(n_keys, device="cuda")
    mask = keys[None, :] <= pos[:, None] if causal else torch.ones(n_q, n_keys, dtype=torch.bool, device="cuda")
    for h in range(nq):
        s = (q[h].double() @ kk[h // g].T) / d ** 0.5
        s = s.masked_fill(~mask, float("-inf"))
        out[:, h * d:(h + 1) * d] = torch.softmax(s, dim=1) @ vv[h // g]
    return out


# Error budget of the attention kernel against the exact result, from its arithmetic:
# scores are exact products of bf16 operands summed in fp32 (relative 2^-24 per add);
# the probabilities and the output each pass through a two-term bf16 representation
# (hi + lo, 16 significant bits: relative error at most 2^-17 each); the exponential is
# the hardware approximation (relative error about 2^-22).  Four 2^-17 terms bound it,
# relative to the element and to the output's rms (diffuse attention averages many keys).
ATTN_TOL = 4 * 2.0 ** -17


@pytest.mark.parametrize("n_q,pos0,n_keys,causal,nq,nkv", [
    (100, 200, 300, False, 4, 2),      # canvas rows over a ragged prefix + canvas
    (256, 1024, 1280, False, 16, 4),   # the single-layer workload's shape
    (200, 50, 250, True, 4, 1),        # prefill rows, causal, ragged
    (64, 4900, 4964, False, 2, 2),     # long keys: split-KV + merge
    (300, 0, 300, True, 2, 1),         # prefill from an empty cache
])
def test_attention(dg, n_q, pos0, n_keys, causal, nq, nkv):
    from block_diffusion_lm_masked_b200 import configs as CF
    g = torch.Generator(device="cuda").manual_seed(n_q + n_keys)
    d, cap = 128, ((n_keys + 7) // 8) * 8 + 8
    q = _bf(nq, n_q, d, gen=g)
    k = _bf(nkv, cap, d, gen=g)
    vt = _bf(nkv, d, cap, gen=g)
    cfg = dict(CF.CONFIGS["layer1_bf16"], n_q_heads=nq, n_kv_heads=nkv, hidden=128, expert_ffn=64, n_experts=1,
               top_k=1, vocab=128, n_layers=1)
    ws = dg.Workspace(cfg, n_q)
    out = torch.zeros(n_q, nq * d, dtype=torch.bfloat16, device="cuda")
    out_lo = torch.zeros(n_q, nq * d, dtype=torch.bfloat16, device="cuda")
    dg.debug_attention_bf16(q, k, vt, n_keys, pos0, causal, out, ws, out_lo=out_lo)
    dg.device_status(ws)
    ref = _attn_ref(q, k, vt, n_keys, pos0, causal)
    rms = ref.pow(2).mean().sqrt().item()
    # hi + lo carries the fp32 result; hi alone is it rounded to bf16 (within one bf16 ulp)
    full = out.double() + out_lo.double()
    err = ((full - ref).abs() / (ref.abs() + rms)).max().item()
    print(f"attention max error / (|ref| + rms): {err:.2e} (bound {ATTN_TOL:.2e})")
    assert err <= ATTN_TOL
    assert ((out.double() - ref).abs() <= 2 ** -8 * ref.abs() + ATTN_TOL * rms).all()
