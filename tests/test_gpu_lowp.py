"""The low-precision-weight GEMMs (dg_debug_gemm_mx8: MX-FP8; dg_debug_gemm_nv4: 4-bit
E2M1 with E4M3 block scales and a tensor scale) against the oracle: weights quantised by
the oracle's quantisers, the expected products computed in fp64 from the oracle's
decoding of the same codes.  Exact where the arithmetic allows it (decoding: identity
activations give the decoded weights themselves), fp32-accumulation close elsewhere;
and whole passes with 8-bit experts."""

import numpy as np
import pytest
import torch

from block_diffusion_lm_masked_b200 import configs as CF
from oracle import dg_oracle as O

import parity_lib as PL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_diffusion_lm_masked_b200 import dg as _dg
    return _dg


def _quantised(rng, G, rows, K, std=0.02):
    w = rng.standard_normal((G, rows, K)) * std
    codes, exps = O.mx_e4m3_quantize(w)
    return codes, exps, O.mx_e4m3_dequantize(codes, exps)


def _upload(dg, codes, exps):
    return (torch.from_numpy(np.ascontiguousarray(codes)).cuda(),
            torch.from_numpy(dg.pack_mx8_scales(exps)).cuda())


def _bf16_pair(rng, n, K):
    x = rng.standard_normal((n, K))
    hi = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    lo = (torch.from_numpy(x.astype(np.float32)) - hi.float()).to(torch.bfloat16)
    return x, hi.cuda(), lo.cuda()


def _run(dg, codes, exps, X, out_cols, X_lo=None, group_off=None, codes2=None, exps2=None, out_lo=None):
    W, S = _upload(dg, codes, exps)
    W2, S2 = _upload(dg, codes2, exps2) if codes2 is not None else (None, None)
    n = X.shape[0]
    dt = torch.bfloat16 if codes2 is not None else torch.float32
    out = torch.full((n, out_cols), float("nan"), device="cuda", dtype=dt)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    G = codes.shape[0]
    dg.debug_gemm_mx8(W, S, X, out, out_cols, err, dg.debug_gemm_scratch(n, G), W2=W2, W2_scales=S2, X_lo=X_lo,
                      group_off=group_off, out_lo=out_lo)
    torch.cuda.synchronize()
    assert err.item() == 0
    return out


def test_decoding_is_exact_for_every_code_and_scale(dg):
    """Rows hold every valid E4M3 code (0x7F / 0xFF excluded) under block scales from
    2^-27 to 2^7; with X = I the output is the decoded weight matrix itself, which must
    equal the oracle's decoding bit for bit (signs, subnormal codes and all)."""
    valid = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    K, rows = 256, 128
    codes = np.resize(valid, (1, rows, K)).astype(np.uint8)
    for r in range(rows):
        codes[0, r] = np.roll(codes[0, r], 3 * r)
    exps = np.array([[[(-27 + (r + 5 * b) % 35) for b in range(K // 32)] for r in range(rows)]], dtype=np.int64)
    want = O.mx_e4m3_dequantize(codes, exps)[0]                     # [rows][K]
    X = torch.eye(K, dtype=torch.bfloat16, device="cuda")
    out = _run(dg, codes, exps, X, rows)                           # out[k][f] = dec(W)[f][k]
    np.testing.assert_array_equal(out.double().cpu().numpy(), want.T)


@pytest.mark.parametrize("M,K,n", [(128, 64, 1), (256, 512, 50), (704, 2816, 37), (1024, 2048, 64), (384, 1024, 200)])
def test_dense_mx8_gemm(dg, M, K, n):
    rng = np.random.default_rng(M + K + n)
    codes, exps, wq = _quantised(rng, 1, M, K)
    x, hi, _ = _bf16_pair(rng, n, K)
    out = _run(dg, codes, exps, hi, M)
    ref = hi.double().cpu().numpy() @ wq[0].T
    err = np.abs(out.double().cpu().numpy() - ref).max() / np.abs(ref).max()
    assert err < 1e-5, err


@pytest.mark.parametrize("counts,M", [([0, 3, 17, 40, 1], 256), ([64, 65, 0, 129], 2048), ([300, 2], 704)])
def test_grouped_two_term_mx8_gemm(dg, counts, M):
    """Groups with empty, ragged and multi-item row counts; weight rows not a multiple of
    128 (zero-filled past the group); tokens as two bf16 terms (fp32 precision)."""
    rng = np.random.default_rng(sum(counts) + M)
    E, K = len(counts), 1024
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    codes, exps, wq = _quantised(rng, E, M, K)
    x, hi, lo = _bf16_pair(rng, int(off[-1]), K)
    out = _run(dg, codes, exps, hi, M, X_lo=lo, group_off=torch.from_numpy(off).cuda())
    got = out.double().cpu().numpy()
    for e in range(E):
        ref = x[off[e]:off[e + 1]] @ wq[e].T
        if ref.size:
            assert np.abs(got[off[e]:off[e + 1]] - ref).max() / np.abs(ref).max() < 2e-5, e


def test_gate_up_swiglu_mx8(dg):
    rng = np.random.default_rng(5)
    counts, F, K = [20, 0, 64, 7], 512, 1024
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    cg, eg, wg = _quantised(rng, 4, F, K)
    cu, eu, wu = _quantised(rng, 4, F, K)
    x, hi, lo = _bf16_pair(rng, int(off[-1]), K)
    out_lo = torch.zeros(int(off[-1]), F, dtype=torch.bfloat16, device="cuda")
    out = _run(dg, cg, eg, hi, F, X_lo=lo, group_off=torch.from_numpy(off).cuda(), codes2=cu, exps2=eu,
               out_lo=out_lo)
    got = out.double().cpu().numpy() + out_lo.double().cpu().numpy()
    for e in range(4):
        xe = x[off[e]:off[e + 1]]
        if not len(xe):
            continue
        g, u = xe @ wg[e].T, xe @ wu[e].T
        ref = O.silu(g) * u
        assert np.abs(got[off[e]:off[e + 1]] - ref).max() / np.abs(ref).max() < 1e-4, e


# ---------------------------------------------------------------- a whole pass with 8-bit experts

SMALL_BF16 = dict(n_layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=128, n_experts=8, top_k=2,
                  expert_ffn=192, vocab=2048, rope_theta=10000.0, rms_eps=1e-6, dtype="bf16")


def _experts_to_mx8(setup):
    """Quantise the model's bf16 experts with the oracle's MX-E4M3 quantiser: the GPU model
    gets the codes, the oracle model the decoded values (the weights the codes define)."""
    layers = []
    for L in setup.host.layers:
        d = {}
        for name, key in (("gate", "w_gate"), ("up", "w_up"), ("down", "w_down")):
            codes, exps = O.mx_e4m3_quantize(O.widen(L[key]))
            d[name] = (codes, exps)
            L[key] = O.mx_e4m3_dequantize(codes, exps)
        layers.append(d)
    setup.model.set_experts_mx8(layers)


@pytest.mark.parametrize("cfg,prefixes,C", [(SMALL_BF16, [200], 100), (SMALL_BF16, [64, 0, 131], 37),
                                            (CF.CONFIGS["layer1_bf16"], [1024], 256)])
def test_pass_with_mx8_experts_matches_oracle(dg, cfg, prefixes, C):
    """The pass with 8-bit experts against the oracle pass over the decoded weights, under
    the bf16 path's parity rules (the decode is exact, so nothing else changes)."""
    PL.check_batched_pass(dg, cfg, prefixes, C, prepare=_experts_to_mx8)


# ---------------------------------------------------------------- 4-bit weights

def _nv4(rng, G, rows, K, std=0.02):
    w = rng.standard_normal((G, rows, K)) * std
    codes, sc, g = O.nvfp4_quantize(w)
    return codes, sc, g, O.nvfp4_dequantize(codes, sc, g)


def _run_nv4(dg, codes, sc, g, X, out_cols, X_lo=None, group_off=None, c2=None, sc2=None, g2=1.0, out_lo=None):
    W = torch.from_numpy(dg.pack_nv4_codes(codes)).cuda()
    S = torch.from_numpy(dg.pack_nv4_scales(sc)).cuda()
    W2 = torch.from_numpy(dg.pack_nv4_codes(c2)).cuda() if c2 is not None else None
    S2 = torch.from_numpy(dg.pack_nv4_scales(sc2)).cuda() if c2 is not None else None
    n = X.shape[0]
    dt = torch.bfloat16 if c2 is not None else torch.float32
    out = torch.full((n, out_cols), float("nan"), device="cuda", dtype=dt)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dg.debug_gemm_nv4(W, S, g, X, out, out_cols, err, dg.debug_gemm_scratch(n, codes.shape[0]), W2=W2, W2_scales=S2,
                      g2=g2, X_lo=X_lo, group_off=group_off, out_lo=out_lo)
    torch.cuda.synchronize()
    assert err.item() == 0
    return out


def test_nv4_decoding_is_exact_for_every_code_and_scale(dg):
    """Every 4-bit code under block scales across the E4M3 range, tensor scale 1: with X = I
    the output is the decoded weight matrix, bit for bit the oracle's."""
    K, rows = 256, 128
    codes = np.array([[(r + 7 * k) % 16 for k in range(K)] for r in range(rows)], dtype=np.uint8)[None]
    sc = np.array([[[(3 + 11 * r + 5 * b) % 0x7F for b in range(K // 16)] for r in range(rows)]], dtype=np.uint8)
    want = O.nvfp4_dequantize(codes, sc, 1.0)[0]
    X = torch.eye(K, dtype=torch.bfloat16, device="cuda")
    out = _run_nv4(dg, codes, sc, 1.0, X, rows)
    np.testing.assert_array_equal(out.double().cpu().numpy(), want.T)


@pytest.mark.parametrize("counts,M", [([0, 3, 17, 40, 1], 256), ([64, 65, 0, 129], 2048), ([300, 2], 704)])
def test_grouped_two_term_nv4_gemm(dg, counts, M):
    rng = np.random.default_rng(sum(counts) + M + 1)
    E, K = len(counts), 1024
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    codes, sc, g, wq = _nv4(rng, E, M, K)
    x, hi, lo = _bf16_pair(rng, int(off[-1]), K)
    out = _run_nv4(dg, codes, sc, g, hi, M, X_lo=lo, group_off=torch.from_numpy(off).cuda())
    got = out.double().cpu().numpy()
    for e in range(E):
        ref = x[off[e]:off[e + 1]] @ wq[e].T
        if ref.size:
            assert np.abs(got[off[e]:off[e + 1]] - ref).max() / np.abs(ref).max() < 2e-5, e


def test_gate_up_swiglu_nv4(dg):
    rng = np.random.default_rng(6)
    counts, F, K = [20, 0, 64, 7], 512, 1024
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    cg, sg, gg, wg = _nv4(rng, 4, F, K)
    cu, su, gu, wu = _nv4(rng, 4, F, K)
    x, hi, lo = _bf16_pair(rng, int(off[-1]), K)
    out_lo = torch.zeros(int(off[-1]), F, dtype=torch.bfloat16, device="cuda")
    out = _run_nv4(dg, cg, sg, gg, hi, F, X_lo=lo, group_off=torch.from_numpy(off).cuda(), c2=cu, sc2=su, g2=gu,
                   out_lo=out_lo)
    got = out.double().cpu().numpy() + out_lo.double().cpu().numpy()
    for e in range(4):
        xe = x[off[e]:off[e + 1]]
        if len(xe):
            ref = O.silu(xe @ wg[e].T) * (xe @ wu[e].T)
            assert np.abs(got[off[e]:off[e + 1]] - ref).max() / np.abs(ref).max() < 1e-4, e


def _experts_to_nv4(setup):
    """Quantise the model's bf16 experts with the oracle's NVFP4 quantiser (one tensor
    scale per expert tensor of a layer): codes to the GPU model, decoded weights to the
    oracle model."""
    layers = []
    for L in setup.host.layers:
        d = {}
        for name, key in (("gate", "w_gate"), ("up", "w_up"), ("down", "w_down")):
            codes, sc, g = O.nvfp4_quantize(O.widen(L[key]))
            d[name] = (codes, sc, g)
            L[key] = O.nvfp4_dequantize(codes, sc, g)
        layers.append(d)
    setup.model.set_experts_nv4(layers)


@pytest.mark.parametrize("cfg,prefixes,C", [(SMALL_BF16, [200], 100), (SMALL_BF16, [64, 0, 131], 37),
                                            (CF.CONFIGS["layer1_bf16"], [1024], 256)])
def test_pass_with_nv4_experts_matches_oracle(dg, cfg, prefixes, C):
    """The pass with 4-bit experts against the oracle pass over the decoded weights (the
    tensor scale applied once to the accumulator on the GPU, to every weight in the oracle:
    rounding differences only)."""
    PL.check_batched_pass(dg, cfg, prefixes, C, prepare=_experts_to_nv4)


# ---------------------------------------------------------------- low-precision output matrix

def _vocab_to_mx8(setup):
    """Quantise the output matrix with the oracle's MX-E4M3 quantiser: codes to the GPU model
    (the batched calls' vocabulary projection), decoded weights to the oracle model."""
    codes, exps = O.mx_e4m3_quantize(O.widen(setup.host.w_out))
    setup.host.w_out = O.mx_e4m3_dequantize(codes, exps)
    setup.model.set_vocab_mx8((codes, exps))


def _vocab_to_nv4(setup):
    codes, sc, g = O.nvfp4_quantize(O.widen(setup.host.w_out))
    setup.host.w_out = O.nvfp4_dequantize(codes, sc, g)
    setup.model.set_vocab_nv4((codes, sc, g))


@pytest.mark.parametrize("fmt", ["mx8", "nv4"])
@pytest.mark.parametrize("cfg,prefixes,C", [(SMALL_BF16, [200], 100), (SMALL_BF16, [64, 0, 131], 37),
                                            (CF.CONFIGS["layer1_bf16"], [1024], 256)])
def test_pass_with_low_precision_vocab_matches_oracle(dg, fmt, cfg, prefixes, C):
    """The batched pass projecting to the vocabulary from an 8- or 4-bit output matrix
    (dense mode of the low-precision GEMM, tiles weight tile major) against the oracle
    pass over the decoded matrix, under the bf16 path's parity rules."""
    PL.check_batched_pass(dg, cfg, prefixes, C, prepare=_vocab_to_mx8 if fmt == "mx8" else _vocab_to_nv4)


def test_pass_with_8bit_experts_and_vocab_matches_oracle(dg):
    def prep(setup):
        _experts_to_mx8(setup)
        _vocab_to_mx8(setup)
    PL.check_batched_pass(dg, SMALL_BF16, [64, 0, 131], 37, prepare=prep)
