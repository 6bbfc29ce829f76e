"""Mutation check of the oracle's pins: each plausible mistake below (a dropped term, a
wrong sign, index, operand or tie rule) is planted in the oracle on the CPU, and at
least one of the named pins must fail under it.  The oracle is only as trustworthy as
its pins; this file shows that they see each of these mistakes.

Nothing here changes the oracle on disk.  A mistake in the C++ arithmetic is one
textual edit of a copy of `oracle/dg_oracle.cpp`, built into a library of its own
(under `_build/oracle_mutants/`, keyed by the edited source's hash) and bound as a
module of its own; the pins then run against that module.  A mistake in the binding's
compositions (the multi-step loops and the batch helpers of `oracle/dg_oracle.py`)
replaces that function in the bound module for the duration of one test.
"""
from __future__ import annotations

import hashlib
import importlib.util
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest

from oracle import build as OB
from oracle import dg_oracle as O
import test_oracle_pins as PINS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
MUT_DIR = os.path.join(ROOT, "_build", "oracle_mutants")
SRC = open(OB.SRC).read()
_orig = {name: getattr(O, name) for name in dir(O)}


# ---------------------------------------------------------------- mistakes in the C++ arithmetic
# name -> ([(original text, replacement, occurrences)], pins that must see it)

def _e(old, new, n=1):
    return (old, new, n)


CPP_MUTANTS = {
    "widen shifts bf16 bits by 8": (
        [_e("uint32_t u = (uint32_t)b << 16;", "uint32_t u = (uint32_t)b << 8;")], ["test_widen_bf16_bits"]),
    "bf16 rounding truncates": (
        [_e("std::nearbyint(m * 256.0)", "std::trunc(m * 256.0)")], ["test_round_bf16_ties_and_library"]),
    "rms_norm drops eps": (
        [_e("std::sqrt(ss / H + eps)", "std::sqrt(ss / H)")], ["test_rms_norm_closed_forms"]),
    "rms_norm sum instead of mean": (
        [_e("std::sqrt(ss / H + eps)", "std::sqrt(ss + eps)")], ["test_rms_norm_closed_forms"]),
    "rope rotates the wrong way": (
        [_e("r[i] = a * c - b * s;\n        r[i + half] = b * c + a * s;",
            "r[i] = a * c + b * s;\n        r[i + half] = b * c - a * s;")],
        ["test_rope_closed_form_and_relative_position"]),
    "rope interleaved pairs": (
        [_e("const double a = r[i], b = r[i + half];\n        r[i] = a * c - b * s;\n"
            "        r[i + half] = b * c + a * s;",
            "const double a = r[2 * i], b = r[2 * i + 1];\n        r[2 * i] = a * c - b * s;\n"
            "        r[2 * i + 1] = b * c + a * s;")],
        ["test_rope_closed_form_and_relative_position"]),
    "rope frequency exponent halved": (
        [_e("std::pow(theta, -(2.0 * i) / d)", "std::pow(theta, -(1.0 * i) / d)")],
        ["test_rope_closed_form_and_relative_position"]),
    "silu sign": ([_e("z / (1.0 + std::exp(-z))", "z / (1.0 + std::exp(z))")], ["test_silu_closed_forms"]),
    "prefix rows see block keys": (
        [_e("(i < P) ? (j <= i) : 1", "1")], ["test_block_mask_matches_worked_example"]),
    "block rows causal": (
        [_e("(i < P) ? (j <= i) : 1", "(j <= i)")], ["test_block_mask_matches_worked_example"]),
    "prefill row misses its own key": (
        [_e("= j <= P + i;", "= j < P + i || (i == 0 && j == 0);")],
        ["test_causal_rows_are_prefix_rows_of_mask"]),
    "prefill bidirectional": (
        [_e("= j <= P + i;", "= 1;")],
        ["test_causal_rows_are_prefix_rows_of_mask", "test_chunked_prefill_equals_single_prefill"]),
    "attention scale 1/d": (
        [_e("const double scale = 1.0 / std::sqrt((double)d);", "const double scale = 1.0 / (double)d;")],
        ["test_attention_two_keys_logistic_scale"]),
    "attention unscaled": (
        [_e("const double scale = 1.0 / std::sqrt((double)d);", "const double scale = 1.0;")],
        ["test_attention_two_keys_logistic_scale"]),
    "gqa interleaved head map": (
        [_e("(size_t)(h / g) * Tk * d", "(size_t)(h % nkv) * Tk * d", 2)], ["test_attention_gqa_head_mapping"]),
    "attention ignores the mask": (
        [_e("(!a || a[j]) ?", "true ?")], ["test_attention_closed_forms"]),
    "softmax not normalised": (
        [_e("const double p = s[j] / sum;", "const double p = s[j];")], ["test_attention_closed_forms"]),
    "router ties to the higher id": (
        [_e("return l[a] > l[b]; });", "return l[a] > l[b] || (l[a] == l[b] && a > b); });")],
        ["test_router_topk_special_cases"]),
    "router weights not renormalised": (
        [_e("for (int j = 0; j < k; ++j) w[(size_t)t * k + j] /= sum;",
            "sum = 0.0;\n    for (int e = 0; e < E; ++e) sum += std::exp(l[e] - mx);\n"
            "    for (int j = 0; j < k; ++j) w[(size_t)t * k + j] /= sum;")],
        ["test_router_topk_brute_force_subsets"]),
    "permutation (expert, slot, token)": (
        [_e("for (int64_t a = 0; a < n; ++a) perm[fill[idx[a]]++] = a;",
            "for (int jj = 0; jj < k; ++jj)\n    for (int tt = 0; tt < T; ++tt) {\n"
            "      const int64_t a = (int64_t)tt * k + jj;\n      perm[fill[idx[a]]++] = a;\n    }")],
        ["test_expert_permutation_invariants"]),
    "router reads the un-normed residual": (
        [_e("matmul_xwt(xn.data(), T, H, W.w_router[l], 0, E, logits.data());",
            "matmul_xwt(x, T, H, W.w_router[l], 0, E, logits.data());")],
        ["test_moe_router_reads_the_normed_residual"]),
    "moe gate and up swapped": (
        [_e("h[i] = oc_silu(g[i]) * up[i];", "h[i] = oc_silu(up[i]) * g[i];")],
        ["test_moe_identical_experts_equals_dense_swiglu"]),
    "moe combine weights reversed": (
        [_e("const double wj = w[(size_t)t * k + j];", "const double wj = w[(size_t)t * k + (k - 1 - j)];")],
        ["test_moe_combine_pairs_each_weight_with_its_expert"]),
    "moe experts read the un-normed residual": (
        [_e("std::copy(xn.begin() + t * H, xn.begin() + (t + 1) * H, xe.begin() + (size_t)r * H);",
            "std::copy(x + t * H, x + (t + 1) * H, xe.begin() + (size_t)r * H);")],
        ["test_moe_identical_experts_equals_dense_swiglu"]),
    "moe rows gathered from the slot index": (
        [_e("const int64_t t = perm[offsets[e] + r] / k;", "const int64_t t = perm[offsets[e] + r] % k;")],
        ["test_moe_combine_pairs_each_weight_with_its_expert"]),
    "embedding scaled by sqrt(H)": (
        [_e("for (int t = 0; t < T; ++t) widen_row(Wp->embed, (size_t)tokens[t] * H, H, x + (size_t)t * H);",
            "for (int t = 0; t < T; ++t) widen_row(Wp->embed, (size_t)tokens[t] * H, H, x + (size_t)t * H);\n"
            "  for (size_t i = 0; i < (size_t)T * H; ++i) x[i] *= std::sqrt((double)H);")],
        ["test_single_token_pass_closed_form"]),
    "no final norm": (
        [_e("oc_rms_norm(x, T, H, cp->rms_eps, xn.data());\n  matmul_xwt(xn.data(), T, H, Wp->w_out",
            "std::copy(x, x + (size_t)T * H, xn.begin());\n  matmul_xwt(xn.data(), T, H, Wp->w_out")],
        ["test_single_token_pass_closed_form"]),
    "pass positions start at 0": (
        [_e("for (int t = 0; t < T; ++t) pos[t] = (int64_t)P + t;\n  std::vector<double> q, k, v;\n"
            "  qkv(c, W,",
            "for (int t = 0; t < T; ++t) pos[t] = causal ? (int64_t)P + t : t;\n  std::vector<double> q, k, v;\n"
            "  qkv(c, W,")],
        ["test_prefix_kv_reuse_equals_full_recompute"]),
    "denoising rows causal": (
        [_e("  if (causal) {\n    oc_causal_rows(P, T, mask.data());", "  if (true) {\n    oc_causal_rows(P, T, mask.data());")],
        ["test_prefix_kv_reuse_equals_full_recompute"]),
    "canvas K/V rounded in flight": (
        [_e("  qkv(c, W, l, x, T, pos.data(), q, k, v);\n",
            "  qkv(c, W, l, x, T, pos.data(), q, k, v);\n  if (c.bf16_storage) {\n"
            "    oc_round_bf16(k.data(), (int64_t)k.size(), k.data());\n"
            "    oc_round_bf16(v.data(), (int64_t)v.size(), v.data());\n  }\n")],
        ["test_bf16_storage_rounds_what_prefill_writes_and_nothing_in_flight"]),
    "prefill stores unrounded K/V": (
        [_e("if (cp->bf16_storage) {   // what later calls read", "if (false) {   // what later calls read")],
        ["test_bf16_storage_rounds_what_prefill_writes_and_nothing_in_flight"]),
    "splitmix64 counter off by one": (
        [_e("uint64_t z = seed + (n + 1) * kGamma;", "uint64_t z = seed + n * kGamma;")],
        ["test_splitmix64_known_answers"]),
    "re-noise token from the low bits": (
        [_e("((x >> 32) * (uint64_t)vocab) >> 32", "((x & 0xFFFFFFFFULL) * (uint64_t)vocab) >> 32")],
        ["test_renoise_token_is_the_top_bits_of_the_published_draw"]),
    "re-noise count rounds up": (
        [_e("return (int64_t)std::floor(C * r_start + 1e-9);", "return (int64_t)std::ceil(C * r_start - 1e-9);"),
         _e("return (int64_t)std::floor(C * f + 1e-9);", "return (int64_t)std::ceil(C * f - 1e-9);")],
        ["test_renoise_schedule_golden"]),
    "re-noise the most confident": (
        [_e("return conf[a] < conf[b]; });\n  for (int i = 0; i < C; ++i) {\n    renoised[i] = 0;",
            "return conf[a] > conf[b]; });\n  for (int i = 0; i < C; ++i) {\n    renoised[i] = 0;")],
        ["test_canvas_update_renoise_set_brute_force"]),
    "re-noise ties to the higher position": (
        [_e("return conf[a] < conf[b]; });\n  for (int i = 0; i < C; ++i) {\n    renoised[i] = 0;",
            "return conf[a] < conf[b] || (conf[a] == conf[b] && a > b); });\n  for (int i = 0; i < C; ++i) {\n"
            "    renoised[i] = 0;")],
        ["test_canvas_update_special_cases"]),
    "argmax ties to the last id": (
        [_e("if (l[v] > m) {", "if (l[v] >= m) {")], ["test_canvas_update_special_cases"]),
    "confidence is the max logit": (
        [_e("conf[i] = 1.0 / denom;", "conf[i] = std::exp(m);")],
        ["test_canvas_update_renoise_set_brute_force"]),
    "masked: the mask id may win": (
        [_e("if (v != mask_id && (a < 0 || l[v] > best)) {", "if ((a < 0 || l[v] > best)) {")],
        ["test_masked_update_worked_example"]),
    "masked: locked positions re-decided": (
        [_e("if (canvas_in[i] == mask_id) masked.push_back(i);", "masked.push_back(i);")],
        ["test_masked_update_worked_example"]),
    "masked: confidence normalised without the mask id": (
        [_e("for (int v = 0; v < V; ++v) denom += std::exp(l[v] - m);\n    int a = -1;",
            "for (int v = 0; v < V; ++v)\n      if (v != mask_id) denom += std::exp(l[v] - m);\n    int a = -1;")],
        ["test_masked_update_worked_example"]),
    "e4m3 bias 8": (
        [_e("return s * (1.0 + m / 8.0) * std::ldexp(1.0, e - 7);", "return s * (1.0 + m / 8.0) * std::ldexp(1.0, e - 8);")],
        ["test_e4m3_decode_closed_forms"]),
    "e4m3 subnormal scale": (
        [_e("if (e == 0) return s * m * std::ldexp(1.0, -9);", "if (e == 0) return s * m * std::ldexp(1.0, -10);")],
        ["test_e4m3_decode_closed_forms"]),
    "nearest code ties away from even": (
        [_e("c = (dlo < dhi || (dlo == dhi && lo % 2 == 0)) ? lo : hi;", "c = (dlo < dhi) ? lo : hi;")],
        ["test_e4m3_encode_round_trip_rounding_saturation", "test_e2m1_codes_rounding_saturation"]),
    "array e4m3 encoder drops the sign": (
        [_e("codes[i] = (uint8_t)oc_e4m3_encode(x[i]);", "codes[i] = (uint8_t)oc_e4m3_encode(std::fabs(x[i]));")],
        ["test_e4m3_array_encoder_is_the_scalar_rule"]),
    "array e2m1 encoder drops the sign": (
        [_e("codes[i] = (uint8_t)oc_e2m1_encode(x[i]);", "codes[i] = (uint8_t)oc_e2m1_encode(std::fabs(x[i]));")],
        ["test_e2m1_array_encoder_is_the_scalar_rule"]),
    "mx scale exponent off by one": (
        [_e("(int)std::floor(std::log2(amax)) - 8", "(int)std::floor(std::log2(amax)) - 7")],
        ["test_mx_e4m3_block_scaling"]),
    "e2m1 subnormal value": (
        [_e("if (e == 0) return s * 0.5 * m;", "if (e == 0) return s * 1.0 * m;")],
        ["test_e2m1_codes_rounding_saturation"]),
    "nvfp4 tensor scale without the 6": (
        [_e("amax_t / (448.0 * 6.0)", "amax_t / 448.0"), _e("oc_e4m3_encode(amax / (6.0 * g))", "oc_e4m3_encode(amax / g)")],
        ["test_nvfp4_block_scaling"]),
    "mx dequantised with the neighbouring block's scale": (
        [_e("std::ldexp(1.0, exps[r * nb + i / 32])", "std::ldexp(1.0, exps[r * nb + (i / 32 + nb - 1) % nb])")],
        ["test_block_scales_stay_with_their_blocks"]),
    "mx dequantised with one scale per row": (
        [_e("std::ldexp(1.0, exps[r * nb + i / 32])",
            "std::ldexp(1.0, *std::max_element(exps + r * nb, exps + (r + 1) * nb))")],
        ["test_block_scales_stay_with_their_blocks"]),
    "nvfp4 dequantised with the neighbouring block's scale": (
        [_e("oc_e4m3_decode(scale_codes[r * nb + i / 16])", "oc_e4m3_decode(scale_codes[r * nb + (i / 16 + nb - 1) % nb])")],
        ["test_block_scales_stay_with_their_blocks"]),
    "RoPE applied to v": (
        [_e("  oc_rope(k.data(), nkv, T, d, pos, c.rope_theta);\n",
            "  oc_rope(k.data(), nkv, T, d, pos, c.rope_theta);\n  oc_rope(v.data(), nkv, T, d, pos, c.rope_theta);\n")],
        ["test_attention_sees_relative_positions_only"]),
    "no RoPE on k": (
        [_e("  oc_rope(k.data(), nkv, T, d, pos, c.rope_theta);\n", "")],
        ["test_attention_sees_relative_positions_only"]),
    "no RoPE at all": (
        [_e("  oc_rope(q.data(), nq, T, d, pos, c.rope_theta);\n", ""),
         _e("  oc_rope(k.data(), nkv, T, d, pos, c.rope_theta);\n", "")],
        ["test_attention_sees_relative_positions_only"]),
    "heads not gathered before the output projection": (
        [_e("oc[(size_t)t * nq * d + h * d + i] = o[((size_t)h * T + t) * d + i];",
            "oc[(size_t)t * nq * d + h * d + i] = o[(size_t)t * nq * d + h * d + i];")],
        ["test_prefix_kv_reuse_equals_full_recompute"]),
    "full recompute with a causal mask over the canvas": (
        [_e("oc_block_mask(P, C, mask.data());", "oc_causal_rows(0, P + C, mask.data());")],
        ["test_prefix_kv_reuse_equals_full_recompute"]),
}


def _mutant_source(edits) -> str:
    s = SRC
    for old, new, n in edits:
        assert s.count(old) == n, f"edit anchor found {s.count(old)} times, expected {n}: {old!r}"
        s = s.replace(old, new)
    return s


def _build(name: str) -> str:
    src = _mutant_source(CPP_MUTANTS[name][0])
    h = hashlib.sha256((src + " ".join(OB.FLAGS)).encode()).hexdigest()[:16]
    lib = os.path.join(MUT_DIR, f"m_{h}.so")
    if not os.path.exists(lib):
        cpp = os.path.join(MUT_DIR, f"m_{h}.cpp")
        with open(cpp, "w") as f:
            f.write(src)
        OB.compile_source(cpp, lib)
    return lib


def _bind(lib_path: str, tag: str):
    """The binding module executed afresh against another build of the oracle."""
    spec = importlib.util.spec_from_file_location(f"oracle_mutant_{tag}", O.__file__)
    mod = importlib.util.module_from_spec(spec)
    mod._LIB_OVERRIDE = lib_path
    spec.loader.exec_module(mod)
    assert mod.LIB_PATH == lib_path
    return mod


@pytest.fixture(scope="module")
def mutant_libs():
    """Every C++ mutant built once (in parallel; cached by source hash across runs)."""
    os.makedirs(MUT_DIR, exist_ok=True)
    names = sorted(CPP_MUTANTS)
    with ThreadPoolExecutor(max_workers=max(1, min(len(names), os.cpu_count() or 1))) as ex:
        libs = list(ex.map(_build, names))
    return dict(zip(names, libs))


def _run_pins(names):
    failed = []
    for n in names:
        try:
            getattr(PINS, n)()
        except AssertionError:
            failed.append(n)
    return failed


def test_every_edit_anchor_is_in_the_oracle_source():
    for name, (edits, pins) in CPP_MUTANTS.items():
        _mutant_source(edits)
        for p in pins:
            assert hasattr(PINS, p), (name, p)


def test_unmutated_rebuild_passes_every_named_pin(tmp_path, monkeypatch):
    """Control: the binding re-bound to a fresh build of the unedited source passes the pins."""
    lib = OB.compile_source(OB.SRC, str(tmp_path / "control.so"))
    monkeypatch.setattr(PINS, "O", _bind(lib, "control"))
    pins = sorted({p for _, ps in CPP_MUTANTS.values() for p in ps})
    assert _run_pins(pins) == []


@pytest.mark.parametrize("name", sorted(CPP_MUTANTS))
def test_pins_see_the_cpp_mutant(name, mutant_libs, monkeypatch):
    _, pins = CPP_MUTANTS[name]
    mod = _bind(mutant_libs[name], hashlib.sha256(name.encode()).hexdigest()[:8])
    monkeypatch.setattr(PINS, "O", mod)
    assert _run_pins(pins), f"no pin sees the mutant '{name}' (ran {pins})"


# ---------------------------------------------------------------- mistakes in the binding's compositions

def _denoise_writes_cache(model, cache, canvas, prec, logit_rows=None):
    """The pass appending the canvas K/V to the caller's cache."""
    out = _orig["denoise_pass"](model, cache, canvas, prec, logit_rows)
    grown = _orig["prefill_append"](model, cache, canvas, prec)
    cache.k, cache.v = grown.k, grown.v
    return out


def _merge_taps_per_canvas(per_canvas_taps, n_experts):
    """Rows stacked, but the permutation kept per canvas (offset) instead of grouped over the batch."""
    out = []
    for layer_taps in zip(*per_canvas_taps):
        m = {key: np.concatenate([t[key] for t in layer_taps], axis=0)
             for key in ("x_in", "attn_o", "x_attn", "x_out", "router_logits", "topk_idx", "topk_w", "router_margin")}
        perms, base = [], 0
        for t in layer_taps:
            perms.append(np.asarray(t["perm"]) + base)
            base += t["topk_idx"].size
        counts = sum(t["counts"] for t in layer_taps)
        m.update(counts=counts, offsets=np.concatenate([[0], np.cumsum(counts)]), perm=np.concatenate(perms),
                 union=int((counts > 0).sum()))
        out.append(m)
    return out


def _batched_shared_cache(model, caches, canvases, prec):
    """Every canvas attends to the first canvas's cache."""
    return [O.denoise_pass(model, caches[0], np.asarray(x), prec) for x in canvases]


def _generate_first_seed(model, caches, canvases, S, r_start, r_end, seeds, prec, append):
    res = [O.generate_canvas(model, c, x, S, r_start, r_end, seeds[0], prec, append)
           for c, x in zip(caches, canvases)]
    return [r[0] for r in res], [r[1] for r in res]


def _generate_no_append(model, caches, canvases, S, r_start, r_end, seeds, prec, append):
    res = [O.generate_canvas(model, c, x, S, r_start, r_end, sd, prec, False)
           for c, x, sd in zip(caches, canvases, seeds)]
    return [r[0] for r in res], [r[1] for r in res]


def _generate_step_plus_one(model, cache, canvas, S, r_start, r_end, seed, prec, append, record=None):
    C = len(canvas)
    cur = np.asarray(canvas, dtype=np.int32).copy()
    for s in range(S):
        logits, taps = O.denoise_pass(model, cache, cur, prec)
        n = O.renoise_count(C, S, s, r_start, r_end)
        upd = O.canvas_update(logits, n, seed, s + 1)
        if record is not None:
            record.append(dict(step=s, canvas_in=cur.copy(), logits=logits, taps=taps, update=upd, n=n))
        cur = upd["canvas"]
    if append:
        cache = O.prefill_append(model, cache, cur, prec)
    return cur, cache


def _masked_generation_from_noise(model, cache, C, S, keep_start, keep_end, mask_id, prec, append, record=None):
    cur = np.arange(C, dtype=np.int32) % mask_id            # not an all-[MASK] canvas
    for s in range(S):
        logits, taps = O.denoise_pass(model, cache, cur, prec)
        n = O.renoise_count(C, S, s, keep_start, keep_end)
        upd = O.canvas_update_masked(logits, cur, n, mask_id)
        if record is not None:
            record.append(dict(step=s, canvas_in=cur.copy(), logits=logits, taps=taps, update=upd, n=n))
        cur = upd["canvas"]
    if append:
        cache = O.prefill_append(model, cache, cur, prec)
    return cur, cache


# name -> (attribute, replacement, pins that must see it)
PY_MUTANTS = {
    "pass writes the cache": ("denoise_pass", _denoise_writes_cache, ["test_denoise_pass_leaves_cache_untouched"]),
    "batch permutation kept per canvas": ("merge_batch_taps", _merge_taps_per_canvas,
                                          ["test_batch_reads_the_union_of_the_canvases_experts"]),
    "batched canvases share a cache": ("denoise_pass_batched", _batched_shared_cache,
                                       ["test_batched_canvases_do_not_see_each_other"]),
    "batched generation with one seed": ("generate_canvases", _generate_first_seed,
                                         ["test_batched_canvases_do_not_see_each_other"]),
    "batched generation skips the append": ("generate_canvases", _generate_no_append,
                                            ["test_batched_canvases_do_not_see_each_other"]),
    "generation re-noises with the next step's draws": ("generate_canvas", _generate_step_plus_one,
                                                        ["test_resume_from_a_middle_pass_reproduces_the_run"]),
    "masked generation starts from noise": ("generate_canvas_masked", _masked_generation_from_noise,
                                            ["test_generate_masked_loop_properties"]),
}


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_pins_see_the_binding_mutant(name, monkeypatch):
    attr, fn, pins = PY_MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    assert _run_pins(pins), f"no pin sees the mutant '{name}' (ran {pins})"
