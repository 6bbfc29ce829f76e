"""The C-ABI library: it loads, exports every symbol the headers declare, and its
host-side validation and arithmetic work without a GPU (no compute calls here)."""
import ctypes
import itertools
import glob
import os
import re

import numpy as np
import pytest

from conftest import ROOT, golden_path
from block_diffusion_lm_masked_b200 import configs as CF
from block_diffusion_lm_masked_b200 import dg


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \t\*]*?\b(dg_[a-z0-9_]+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return names


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert {"dg_prefill_append", "dg_denoise_pass", "dg_canvas_update", "dg_generate_canvas"} <= names
    lib = ctypes.CDLL(dg.LIB_PATH)
    missing = [n for n in sorted(names) if not hasattr(lib, n)]
    assert not missing, missing


def test_workspace_sizes_for_every_config():
    for name in CF.ORDER:
        cfg = CF.CONFIGS[name]
        n = dg.workspace_bytes(cfg, max(cfg["canvas"], cfg.get("prompt", 0)))
        assert n > 0 and n % 256 == 0
    assert dg.update_workspace_bytes(256, 262144) > 256


def test_invalid_configs_rejected_on_host():
    bad = dict(CF.CONFIGS["layer1_bf16"], head_dim=64)          # bf16 path needs d = 128
    assert dg.workspace_bytes(bad, 256) == 0
    c = dg.make_config(bad)
    w = dg.Weights(None, None, None)
    h = ctypes.c_void_p()
    assert dg.lib.dg_model_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h)) == dg.DG_ERR_INVALID_ARG
    assert "head_dim" in dg.lib.dg_last_error().decode()
    for over in (dict(n_q_heads=6, n_kv_heads=4), dict(top_k=17), dict(n_experts=300), dict(expert_ffn=100)):
        assert dg.workspace_bytes(dict(CF.CONFIGS["tiny_fp32"], **over), 32) == 0, over


def test_null_arguments_rejected_on_host():
    assert dg.lib.dg_canvas_update(None, 4, 8, 1, 0, 0, None, None, None, 0, None) == dg.DG_ERR_INVALID_ARG
    assert dg.lib.dg_denoise_pass(None, None, None, 4, None, None, 0, None) == dg.DG_ERR_INVALID_ARG
    assert dg.lib.dg_prefill_append(None, None, None, 4, None, 0, None) == dg.DG_ERR_INVALID_ARG
    assert dg.lib.dg_device_status(None, None) == dg.DG_ERR_INVALID_ARG
    assert dg.lib.dg_canvas_update_noalloc(None, 4, 8, 1, 0, 0, None, None, None) == dg.DG_ERR_INVALID_ARG
    assert dg.lib.dg_canvas_update_masked(None, 4, 8, 1, 7, None, None, None, 0, None) == dg.DG_ERR_INVALID_ARG
    assert dg.lib.dg_generate_canvas_masked(None, None, None, 4, 2, 0.5, 0.0, 7, 0, None, None, 0,
                                            None) == dg.DG_ERR_INVALID_ARG


def test_masked_update_validation_on_host():
    """Every bad argument of the masked entry points is rejected before any CUDA call
    (the placeholder pointers below are never dereferenced)."""
    p = ctypes.c_void_p(4096)
    L = dg.lib

    def upd(C, V, n_keep, mask_id, ws_bytes=1 << 20):
        return L.dg_canvas_update_masked(p, C, V, n_keep, mask_id, p, None, p, ws_bytes, None)

    for args in ((0, 8, 0, 1), (1025, 8, 0, 1), (4, 6, 0, 1), (4, 8, 0, 8), (4, 8, 0, -1), (4, 8, 5, 1),
                 (4, 8, -1, 1)):
        assert upd(*args) == dg.DG_ERR_INVALID_ARG, args
    assert upd(4, 8, 0, 1, ws_bytes=16) == dg.DG_ERR_CAPACITY
    assert L.dg_canvas_update_masked(ctypes.c_void_p(4100), 4, 8, 0, 1, p, None, p, 1 << 20,
                                     None) == dg.DG_ERR_INVALID_ARG        # logits not 16-byte aligned
    assert L.dg_generate_canvas_masked(None, None, p, 4, 2, 0.5, 0.0, 1, 0, p, p, 1 << 20,
                                       None) == dg.DG_ERR_INVALID_ARG     # no model


def test_renoise_schedule_matches_golden():
    g = {}
    for line in open(golden_path("renoise_schedule.txt")):
        if line.strip() and not line.startswith("#"):
            k, *v = line.split()
            g[k] = [int(x) for x in v]
    assert [dg.renoise_count(256, 16, s, 0.5, 0.0) for s in range(16)] == g["S16"]
    assert [dg.renoise_count(256, 8, s, 0.5, 0.0) for s in range(8)] == g["S8"]
    assert dg.renoise_count(256, 1, 0, 0.25, 0.25) == g["S1_C256_q25"][0]
    assert dg.renoise_count(32, 1, 0, 0.25, 0.25) == g["S1_C32_q25"][0]
    assert dg.renoise_count(256, 4, 4, 0.5, 0.0) == -1


def _fake_model(cfg, misalign=None):
    """A model over placeholder device addresses (never dereferenced).  fp32 models encode
    no tensor maps, so dg_model_create needs no GPU for them."""
    base = [1 << 20]

    def addr(name):
        base[0] += 1 << 16
        return base[0] + (8 if name == misalign else 0)

    L = cfg["n_layers"]
    lw = (dg.LayerWeights * L)(*[dg.LayerWeights(*[addr(n) for n in ("w_qkv", "w_o", "w_router", "w_gate", "w_up",
                                                                      "w_down")]) for _ in range(L)])
    w = dg.Weights(addr("embed"), addr("w_out"), lw)
    c = dg.make_config(cfg)
    h = ctypes.c_void_p()
    st = dg.lib.dg_model_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h))
    return st, h


@pytest.mark.parametrize("name", ["embed", "w_out", "w_qkv", "w_o", "w_router", "w_gate", "w_up", "w_down"])
def test_misaligned_weights_rejected_on_host(name):
    """Kernels read the embedding and router rows with 16-byte vector loads and TMA needs
    16-byte aligned bases, so a weight that is not 16-byte aligned is refused at creation."""
    st, h = _fake_model(CF.CONFIGS["tiny_fp32"], misalign=name)
    assert st == dg.DG_ERR_INVALID_ARG and not h.value
    assert "aligned" in dg.lib.dg_last_error().decode()


def test_generation_rejects_bad_arguments_before_any_launch():
    """The generation calls check what their passes, updates and append would check
    before the first launch, so a rejected call launches nothing (the model and cache
    here are placeholders that a launch would fault on)."""
    cfg = CF.CONFIGS["tiny_fp32"]
    st, h = _fake_model(cfg)
    assert st == dg.DG_OK and h.value
    try:
        L = cfg["n_layers"]
        ka = (ctypes.c_void_p * L)(*[(1 << 30) + (i << 16) for i in range(L)])
        va = (ctypes.c_void_p * L)(*[(1 << 31) + (i << 16) for i in range(L)])
        cache = dg.KVCacheS(ka, va, 256, 64)
        C, S = 32, 2
        ws_need = dg.workspace_bytes(cfg, C)
        p, ws = ctypes.c_void_p(1 << 24), ctypes.c_void_p(1 << 25)
        G, GM = dg.lib.dg_generate_canvas, dg.lib.dg_generate_canvas_masked

        def gen(canvas=p, C=C, logits=p, ws=ws, ws_bytes=ws_need, S=S):
            return G(h, ctypes.byref(cache), canvas, C, S, 0.5, 0.0, 7, 1, logits, ws, ws_bytes, None)

        def genm(canvas=p, C=C, logits=p, ws=ws, ws_bytes=ws_need):
            return GM(h, ctypes.byref(cache), canvas, C, S, 0.5, 0.0, 3, 1, logits, ws, ws_bytes, None)

        launches = dg.lib.dg_launch_count()
        for f in (gen, genm):
            assert f(logits=ctypes.c_void_p((1 << 24) + 4)) == dg.DG_ERR_INVALID_ARG      # misaligned logits
            assert "aligned" in dg.lib.dg_last_error().decode()
            assert f(logits=None) == dg.DG_ERR_INVALID_ARG
            assert f(canvas=None) == dg.DG_ERR_INVALID_ARG
            assert f(C=0) == dg.DG_ERR_INVALID_ARG
            assert f(C=1025) == dg.DG_ERR_INVALID_ARG
            assert f(ws=None) == dg.DG_ERR_INVALID_ARG
            assert f(ws=ctypes.c_void_p((1 << 25) + 128)) == dg.DG_ERR_INVALID_ARG     # workspace alignment
            assert f(ws_bytes=ws_need - 256) == dg.DG_ERR_CAPACITY
            assert f(C=256 - 64 + 8) == dg.DG_ERR_CAPACITY                              # no room in the cache
        assert gen(S=0) == dg.DG_ERR_INVALID_ARG
        assert dg.lib.dg_launch_count() == launches          # no launch was even attempted
    finally:
        dg.lib.dg_model_destroy(h)


def test_batched_calls_reject_bad_arguments_before_any_launch():
    """The batched entry points check every cache (valid, room for the canvas, no buffer
    shared with another canvas of the batch) and the workspace for B * C rows before the
    first launch."""
    cfg = CF.CONFIGS["tiny_fp32"]
    st, h = _fake_model(cfg)
    assert st == dg.DG_OK
    try:
        L, C, B = cfg["n_layers"], 16, 3

        def cache(i, length=8, cap=64, share_with=None):
            j = i if share_with is None else share_with
            ka = (ctypes.c_void_p * L)(*[(1 << 32) + (j << 24) + (l << 16) for l in range(L)])
            va = (ctypes.c_void_p * L)(*[(1 << 33) + (j << 24) + (l << 16) for l in range(L)])
            return dg.KVCacheS(ka, va, cap, length), (ka, va)

        def batch(*specs):
            made = [cache(i, **kw) for i, kw in enumerate(specs)]
            return (dg.KVCacheS * len(made))(*[m[0] for m in made]), made

        good, keep = batch({}, {}, {})
        ws_need = dg.workspace_bytes(cfg, B * C)
        p, ws = ctypes.c_void_p(1 << 24), ctypes.c_void_p(1 << 25)
        seeds = (ctypes.c_uint64 * B)(1, 2, 3)
        lib = dg.lib
        launches = lib.dg_launch_count()

        def den(caches=good, B=B, C=C, ws_bytes=ws_need, logits=p):
            return lib.dg_denoise_pass_batched(h, caches, B, p, C, logits, ws, ws_bytes, None)

        def pre(caches=good, B=B, C=C, ws_bytes=ws_need):
            return lib.dg_prefill_append_batched(h, caches, B, p, C, ws, ws_bytes, None)

        def gen(caches=good, B=B, C=C, ws_bytes=ws_need, logits=p, sd=seeds):
            return lib.dg_generate_canvases(h, caches, B, p, C, 2, 0.5, 0.0, sd, 1, logits, ws, ws_bytes, None)

        def genm(caches=good, B=B, C=C, ws_bytes=ws_need, logits=p):
            return lib.dg_generate_canvases_masked(h, caches, B, p, C, 2, 0.5, 0.0, 7, 1, logits, ws, ws_bytes, None)

        shared, k2 = batch({}, {"share_with": 0}, {})
        full, k3 = batch({}, {}, {"length": 60})
        for f in (den, pre, gen, genm):
            assert f(caches=None) == dg.DG_ERR_INVALID_ARG
            assert f(B=0) == dg.DG_ERR_INVALID_ARG
            assert f(C=0) == dg.DG_ERR_INVALID_ARG
            assert f(caches=shared) == dg.DG_ERR_INVALID_ARG
            assert "share" in lib.dg_last_error().decode()
            assert f(caches=full) == dg.DG_ERR_CAPACITY
            assert "cache 2" in lib.dg_last_error().decode()
            assert f(ws_bytes=dg.workspace_bytes(cfg, C)) == dg.DG_ERR_CAPACITY     # sized for one canvas
        assert gen(logits=ctypes.c_void_p((1 << 24) + 8)) == dg.DG_ERR_INVALID_ARG
        assert genm(logits=ctypes.c_void_p((1 << 24) + 8)) == dg.DG_ERR_INVALID_ARG
        assert lib.dg_generate_canvases_masked(h, good, B, p, C, 2, 0.5, 0.0, cfg["vocab"], 1, p, ws, ws_need,
                                               None) == dg.DG_ERR_INVALID_ARG     # mask id outside the vocabulary
        assert gen(sd=None) == dg.DG_ERR_INVALID_ARG
        assert gen(C=1025) == dg.DG_ERR_INVALID_ARG
        assert lib.dg_launch_count() == launches
        assert [good[i].len for i in range(B)] == [8, 8, 8]                        # nothing advanced
    finally:
        dg.lib.dg_model_destroy(h)


def test_mx8_scale_packing_layout():
    """The binding's scale packing puts the exponent of elements 64 j + 32 h .. + 31 of row
    f in group g at [g][j][f][h], biased by 127 (E8M0), as include/dg_debug.h states."""
    rng = np.random.default_rng(3)
    e = rng.integers(-127, 8, size=(3, 16, 8))
    p = dg.pack_mx8_scales(e)
    assert p.dtype == np.uint8 and p.shape == (3, 4, 16, 2) and p.flags["C_CONTIGUOUS"]
    for g, j, f, h in itertools.product(range(3), range(4), range(16), range(2)):
        assert p[g, j, f, h] == e[g, f, 2 * j + h] + 127
    with pytest.raises(ValueError):
        dg.pack_mx8_scales(np.full((1, 2, 2), 8))
    with pytest.raises(ValueError):
        dg.pack_mx8_scales(np.zeros((1, 2, 3), dtype=int))


def test_mx8_gemm_validation_on_host():
    """Every bad argument of dg_debug_gemm_mx8 is rejected before any CUDA call (the
    placeholder addresses are never dereferenced)."""
    p = ctypes.c_void_p(1 << 24)
    err = ctypes.c_void_p(1 << 25)
    sc = ctypes.c_void_p(1 << 26)
    L = dg.lib
    launches = L.dg_launch_count()

    def call(W=p, S=p, W2=None, S2=None, rows=128, G=1, X=p, X_lo=None, n=16, K=128, off=None, ld=128,
             scratch=sc, sbytes=1 << 20):
        return L.dg_debug_gemm_mx8(W, S, W2, S2, rows, G, X, X_lo, n, K, off, p, None, ld, scratch, sbytes, err, None)

    for kw in (dict(W=None), dict(S=None), dict(X=None), dict(scratch=None), dict(W2=p), dict(S2=p),
               dict(K=96), dict(K=0), dict(rows=100), dict(rows=0), dict(n=0), dict(G=2), dict(ld=64),
               dict(W=ctypes.c_void_p((1 << 24) + 8)), dict(X_lo=ctypes.c_void_p((1 << 24) + 4)),
               dict(scratch=ctypes.c_void_p((1 << 26) + 16))):
        assert call(**kw) == dg.DG_ERR_INVALID_ARG, kw
    assert call(sbytes=8) == dg.DG_ERR_CAPACITY
    assert L.dg_launch_count() == launches


@pytest.mark.parametrize("fmt", ["mx8", "nv4"])
def test_set_vocab_lowp_validation_on_host(fmt):
    """dg_model_set_vocab_mx8 / _nv4 refuse an fp32 model and a NULL model before encoding
    anything; NULL codes turns the low-precision output matrix off."""
    st, h = _fake_model(CF.CONFIGS["tiny_fp32"])
    assert st == dg.DG_OK
    P = ctypes.c_void_p(1 << 28)
    try:
        if fmt == "mx8":
            f = lambda m, c, s: dg.lib.dg_model_set_vocab_mx8(m, c, s)
        else:
            f = lambda m, c, s: dg.lib.dg_model_set_vocab_nv4(m, c, s, 0.5)
        assert f(h, P, P) == dg.DG_ERR_INVALID_ARG                           # fp32 model
        assert "bf16" in dg.lib.dg_last_error().decode()
        assert f(h, None, None) == dg.DG_OK
        assert f(None, P, P) == dg.DG_ERR_INVALID_ARG
    finally:
        dg.lib.dg_model_destroy(h)


def test_set_experts_mx8_validation_on_host():
    """dg_model_set_experts_mx8 refuses an fp32 model, NULL or misaligned pointers before
    encoding anything; NULL layers turns the 8-bit experts off."""
    cfg = CF.CONFIGS["tiny_fp32"]
    st, h = _fake_model(cfg)
    assert st == dg.DG_OK
    try:
        L = cfg["n_layers"]
        good = (dg.ExpertsMx8 * L)(*[dg.ExpertsMx8(*[(1 << 28) + (l << 20) + (i << 16) for i in range(6)])
                                     for l in range(L)])
        assert dg.lib.dg_model_set_experts_mx8(h, good) == dg.DG_ERR_INVALID_ARG      # fp32 model
        assert "bf16" in dg.lib.dg_last_error().decode()
        assert dg.lib.dg_model_set_experts_mx8(h, None) == dg.DG_OK
        assert dg.lib.dg_model_set_experts_mx8(None, good) == dg.DG_ERR_INVALID_ARG
    finally:
        dg.lib.dg_model_destroy(h)


def test_nv4_gemm_validation_on_host():
    p = ctypes.c_void_p(1 << 24)
    err, sc = ctypes.c_void_p(1 << 25), ctypes.c_void_p(1 << 26)
    L = dg.lib
    launches = L.dg_launch_count()

    def call(g=1.0, W2=None, S2=None, g2=1.0, K=128, rows=128):
        return L.dg_debug_gemm_nv4(p, p, g, W2, S2, g2, rows, 1, p, None, 16, K, None, p, None, rows, sc, 1 << 20,
                                   err, None)

    for kw in (dict(g=float("nan")), dict(g=float("inf")), dict(W2=p, S2=p, g2=float("nan")), dict(W2=p),
               dict(K=96), dict(rows=12)):
        assert call(**kw) == dg.DG_ERR_INVALID_ARG, kw
    assert L.dg_launch_count() == launches


def test_set_experts_nv4_validation_on_host():
    cfg = CF.CONFIGS["tiny_fp32"]
    st, h = _fake_model(cfg)
    assert st == dg.DG_OK
    try:
        L = cfg["n_layers"]
        good = (dg.ExpertsMx8 * L)(*[dg.ExpertsMx8(*[(1 << 28) + (l << 20) + (i << 16) for i in range(6)])
                                     for l in range(L)])
        gs = (ctypes.c_float * (3 * L))(*([0.01] * (3 * L)))
        assert dg.lib.dg_model_set_experts_nv4(h, good, None) == dg.DG_ERR_INVALID_ARG       # no tensor scales
        assert dg.lib.dg_model_set_experts_nv4(h, good, gs) == dg.DG_ERR_INVALID_ARG         # fp32 model
        assert dg.lib.dg_model_set_experts_nv4(h, None, None) == dg.DG_OK
    finally:
        dg.lib.dg_model_destroy(h)


def test_denoise_update_validation_on_host():
    """dg_denoise_update: an fp32 model is unsupported (the fused epilogue is a tcgen05
    kernel); bad sizes and a missing canvas are rejected before any launch."""
    cfg = CF.CONFIGS["tiny_fp32"]
    st, h = _fake_model(cfg)
    assert st == dg.DG_OK
    try:
        L = cfg["n_layers"]
        ka = (ctypes.c_void_p * L)(*[(1 << 30) + (i << 16) for i in range(L)])
        va = (ctypes.c_void_p * L)(*[(1 << 31) + (i << 16) for i in range(L)])
        cs = dg.KVCacheS(ka, va, 256, 64)
        p, ws = ctypes.c_void_p(1 << 24), ctypes.c_void_p(1 << 25)
        launches = dg.lib.dg_launch_count()
        assert dg.lib.dg_denoise_update(h, ctypes.byref(cs), p, 32, 8, 1, 0, -1, None, ws, 1 << 30,
                                        None) == dg.DG_ERR_UNSUPPORTED
        assert dg.lib.dg_denoise_update(None, ctypes.byref(cs), p, 32, 8, 1, 0, -1, None, ws, 1 << 30,
                                        None) == dg.DG_ERR_INVALID_ARG
        assert dg.lib.dg_launch_count() == launches
    finally:
        dg.lib.dg_model_destroy(h)


def test_checked_build_is_selected_by_the_environment():
    """DG_CHECKED=1 makes the binding load libdg_checked.so (the kernels' bounds and
    alignment checks compiled in); without it the product library loads."""
    import subprocess
    import sys
    code = "from block_diffusion_lm_masked_b200 import dg; print(dg.LIB_PATH)"
    env = dict(os.environ, PYTHONPATH=ROOT)
    env.pop("DG_CHECKED", None)
    plain = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, cwd=ROOT)
    assert plain.returncode == 0 and plain.stdout.strip().endswith("libdg.so")
    checked_path = os.path.join(ROOT, "block_diffusion_lm_masked_b200", "libdg_checked.so")
    if not os.path.exists(checked_path):
        pytest.skip("the checked build is made on demand (build --checked)")
    env["DG_CHECKED"] = "1"
    chk = subprocess.run([sys.executable, "-c", code + "; print(dg.lib.dg_launch_count())"], env=env,
                         capture_output=True, text=True, cwd=ROOT)
    assert chk.returncode == 0 and chk.stdout.split()[0].endswith("libdg_checked.so"), chk.stderr


_INJECT = r"""
import ctypes, sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
from block_diffusion_lm_masked_b200 import configs as CF, dg
import test_abi as T
cfg = CF.CONFIGS["tiny_fp32"]
st, h = T._fake_model(cfg)
L = cfg["n_layers"]
ka = (ctypes.c_void_p * L)(*[(1 << 30) + (i << 16) for i in range(L)])
va = (ctypes.c_void_p * L)(*[(1 << 31) + (i << 16) for i in range(L)])
cache = dg.KVCacheS(ka, va, 256, 64)
n = dg.workspace_bytes(cfg, 32)
r = dg.lib.dg_prefill_append(h, ctypes.byref(cache), ctypes.c_void_p(1 << 24), 32, ctypes.c_void_p(1 << 25), n, None)
print(r, cache.len, dg.lib.dg_launch_count(), dg.lib.dg_last_error().decode(), sep="|")
"""


def test_injected_launch_failure_is_a_clean_error_with_the_cache_unchanged():
    """DG_FAULT_INJECT=launch:1: the first launch of a prefill fails on the host (no kernel
    runs, no GPU is involved); the call returns DG_ERR_CUDA with the injected message and
    the cache length does not advance."""
    import subprocess
    import sys
    code = _INJECT.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    env = dict(os.environ, DG_FAULT_INJECT="launch:1")
    env.pop("DG_CHECKED", None)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    status, length, launches, msg = r.stdout.strip().split("|", 3)
    assert int(status) == dg.DG_ERR_CUDA
    assert int(length) == 64
    assert "injected launch failure" in msg
    assert int(launches) == 0                          # failed before any launch was attempted


@pytest.mark.parametrize("name", ["dg_debug_attention_bf16", "dg_debug_attention_pair_bf16"])
def test_debug_attention_validation_on_host(name):
    """Both attention entry points refuse bad shapes before touching any pointer."""
    f = getattr(dg.lib, name)
    P = ctypes.c_void_p(256)                     # never dereferenced: every call below is refused first
    launches = dg.lib.dg_launch_count()
    #        q     k  vt  cap  n_q pos0 n_keys causal nq nkv out out_lo ws   bytes
    bad = [(None, P, P, 64, 8, 0, 8, 0, 2, 1, P, None, P, 1 << 20),      # NULL q
           (P, P, P, 64, 8, 0, 8, 0, 3, 2, P, None, P, 1 << 20),         # nq not a multiple of nkv
           (P, P, P, 60, 8, 0, 8, 0, 2, 1, P, None, P, 1 << 20),         # cap not a multiple of 8
           (P, P, P, 64, 8, 0, 72, 0, 2, 1, P, None, P, 1 << 20),        # n_keys beyond cap
           (P, P, P, 64, 8, 4, 8, 1, 2, 1, P, None, P, 1 << 20),         # causal rows past the keys
           (P, P, P, 64, 0, 0, 8, 0, 2, 1, P, None, P, 1 << 20)]         # no query rows
    for args in bad:
        assert f(*args, None) == dg.DG_ERR_INVALID_ARG, args
    assert dg.lib.dg_launch_count() == launches


def test_mma_rate_probe_validation_on_host():
    """The tensor-pipe probe refuses bad shapes and NULL outputs before any CUDA call."""
    c, m = ctypes.c_uint64(), ctypes.c_float()
    C, M = ctypes.byref(c), ctypes.byref(m)
    launches = dg.lib.dg_launch_count()
    bad = [(0, 96, 16, 1, C, M),        # n not 64, 128 or 256
           (0, 128, 0, 1, C, M),        # no MMAs
           (0, 128, 1 << 21, 1, C, M),  # too many
           (1, 128, 16, 0, C, M),       # no CTAs
           (1, 128, 16, 2048, C, M),    # too many CTAs
           (0, 128, 16, 1, None, M)]    # NULL output
    for args in bad:
        assert dg.lib.dg_debug_mma_rate(*args, None) == dg.DG_ERR_INVALID_ARG, args
    assert dg.lib.dg_launch_count() == launches
