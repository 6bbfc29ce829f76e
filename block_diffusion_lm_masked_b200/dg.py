"""ctypes binding of libdg.so: argument marshalling only.

Every step of the denoising pass runs inside the library's CUDA kernels; this
module turns torch tensors into device pointers and Python values into the C
structs of include/dg.h, and raises on any non-OK status.  PyTorch provides the
device memory and the stream.  Importing this module fails loudly if the library
has not been built: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# DG_CHECKED=1 loads the build with the kernels' bounds and alignment checks compiled in
# (python -m block_diffusion_lm_masked_b200.build --checked)
LIB_PATH = os.path.join(_HERE, "libdg_checked.so" if os.environ.get("DG_CHECKED") == "1" else "libdg.so")

DG_OK, DG_ERR_INVALID_ARG, DG_ERR_CAPACITY, DG_ERR_CUDA, DG_ERR_TIMEOUT, DG_ERR_UNSUPPORTED = 0, -1, -2, -3, -4, -5
DTYPE = {"bf16": 0, "f32": 1}
KERNEL_KINDS = ["embed_norm", "rms_norm", "gemm_qkv", "rope_kv", "attention", "attn_merge", "gemm_o", "router", "topk",
                "permute", "gather", "gemm_gate_up", "swiglu", "gemm_down", "combine", "gemm_vocab", "update_partial",
                "update_select"]


class DGError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"dg status {status}: {msg}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("hidden", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("expert_ffn", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("rope_theta", ctypes.c_float), ("rms_eps", ctypes.c_float), ("dtype", ctypes.c_int32)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("w_qkv", ctypes.c_void_p), ("w_o", ctypes.c_void_p), ("w_router", ctypes.c_void_p),
                ("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p)]


class Weights(ctypes.Structure):
    _fields_ = [("embed", ctypes.c_void_p), ("w_out", ctypes.c_void_p), ("layers", ctypes.POINTER(LayerWeights))]


class KVCacheS(ctypes.Structure):
    _fields_ = [("k", ctypes.POINTER(ctypes.c_void_p)), ("vt", ctypes.POINTER(ctypes.c_void_p)),
                ("capacity", ctypes.c_int32), ("len", ctypes.c_int32)]


class ExpertsMx8(ctypes.Structure):
    _fields_ = [("gate", ctypes.c_void_p), ("gate_scales", ctypes.c_void_p), ("up", ctypes.c_void_p),
                ("up_scales", ctypes.c_void_p), ("down", ctypes.c_void_p), ("down_scales", ctypes.c_void_p)]


class Taps(ctypes.Structure):
    _fields_ = [("x_attn", ctypes.POINTER(ctypes.c_void_p)), ("x_out", ctypes.POINTER(ctypes.c_void_p)),
                ("topk_idx", ctypes.POINTER(ctypes.c_void_p)), ("topk_w", ctypes.POINTER(ctypes.c_void_p)),
                ("counts", ctypes.POINTER(ctypes.c_void_p)), ("perm", ctypes.POINTER(ctypes.c_void_p)),
                ("unions", ctypes.c_void_p), ("rows", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m block_diffusion_lm_masked_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, U32, U64, F32, SZ = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32, ctypes.c_uint64,
                                 ctypes.c_float, ctypes.c_size_t)
    sig = {
        "dg_model_create": (I32, [ctypes.POINTER(Config), ctypes.POINTER(Weights), ctypes.POINTER(P)]),
        "dg_model_destroy": (None, [P]),
        "dg_workspace_bytes": (SZ, [ctypes.POINTER(Config), I32]),
        "dg_update_workspace_bytes": (SZ, [I32, I32]),
        "dg_prefill_append": (I32, [P, ctypes.POINTER(KVCacheS), P, I32, P, SZ, P]),
        "dg_denoise_pass": (I32, [P, ctypes.POINTER(KVCacheS), P, I32, P, P, SZ, P]),
        "dg_canvas_update": (I32, [P, I32, I32, I32, U64, U32, P, P, P, SZ, P]),
        "dg_denoise_update": (I32, [P, ctypes.POINTER(KVCacheS), P, I32, I32, U64, U32, I32, P, P, SZ, P]),
        "dg_canvas_update_noalloc": (I32, [P, I32, I32, I32, U64, U32, P, P, P]),
        "dg_canvas_update_masked": (I32, [P, I32, I32, I32, I32, P, P, P, SZ, P]),
        "dg_generate_canvas_masked": (I32, [P, ctypes.POINTER(KVCacheS), P, I32, I32, F32, F32, I32, I32, P, P, SZ,
                                            P]),
        "dg_generate_canvas": (I32, [P, ctypes.POINTER(KVCacheS), P, I32, I32, F32, F32, U64, I32, P, P, SZ, P]),
        "dg_prefill_append_batched": (I32, [P, P, I32, P, I32, P, SZ, P]),
        "dg_denoise_pass_batched": (I32, [P, P, I32, P, I32, P, P, SZ, P]),
        "dg_generate_canvases": (I32, [P, P, I32, P, I32, I32, F32, F32, P, I32, P, P, SZ, P]),
        "dg_generate_canvases_masked": (I32, [P, P, I32, P, I32, I32, F32, F32, I32, I32, P, P, SZ, P]),
        "dg_model_set_experts_mx8": (I32, [P, P]),
        "dg_model_set_experts_nv4": (I32, [P, P, P]),
        "dg_model_set_vocab_mx8": (I32, [P, P, P]),
        "dg_model_set_vocab_nv4": (I32, [P, P, P, F32]),
        "dg_device_status": (I32, [P, P]),
        "dg_last_error": (ctypes.c_char_p, []),
        "dg_set_taps": (I32, [P, ctypes.POINTER(Taps)]),
        "dg_profile_enable": (I32, [I32]),
        "dg_profile_read": (I32, [I32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(I32)]),
        "dg_profile_reset": (None, []),
        "dg_kernel_name": (ctypes.c_char_p, [I32]),
        "dg_launch_count": (ctypes.c_int64, []),
        "dg_renoise_count": (I32, [I32, I32, I32, F32, F32]),
        "dg_debug_bounded_wait": (I32, [P, I32, P]),
        "dg_debug_set_wait_limit": (I32, [U64]),
        "dg_debug_mma_rate": (I32, [I32, I32, I32, I32, P, P, P]),
        "dg_debug_gemm_bf16": (I32, [P, P, I32, I32, P, P, I32, I32, P, P, P, I32, P, SZ, P, P]),
        "dg_debug_gemm_scratch_bytes": (SZ, [I32, I32]),
        "dg_debug_gemm_mx8": (I32, [P, P, P, P, I32, I32, P, P, I32, I32, P, P, P, I32, P, SZ, P, P]),
        "dg_debug_gemm_nv4": (I32, [P, P, F32, P, P, F32, I32, I32, P, P, I32, I32, P, P, P, I32, P, SZ, P, P]),
        "dg_debug_attention_bf16": (I32, [P, P, P, I32, I32, I32, I32, I32, I32, I32, P, P, P, SZ, P]),
        "dg_debug_attention_pair_bf16": (I32, [P, P, P, I32, I32, I32, I32, I32, I32, I32, P, P, P, SZ, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def _check(status):
    if status != DG_OK:
        raise DGError(status, lib.dg_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def make_config(cfg: dict) -> Config:
    return Config(cfg["n_layers"], cfg["hidden"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"],
                  cfg["n_experts"], cfg["top_k"], cfg["expert_ffn"], cfg["vocab"], cfg["rope_theta"], cfg["rms_eps"],
                  DTYPE[cfg["dtype"]])


def act_torch_dtype(cfg):
    return torch.bfloat16 if cfg["dtype"] == "bf16" else torch.float32


def _upload(arr: np.ndarray, device) -> torch.Tensor:
    """Stored weights (uint16 bf16 bit patterns or float32) -> device tensor of that dtype."""
    if arr.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).to(device)


class Model:
    """Device copy of a synthetic model in the library's weight layouts, plus its dg_model handle."""

    def __init__(self, host_model, device="cuda"):
        cfg = host_model.cfg
        self.cfg = cfg
        self.device = device
        self.embed = _upload(host_model.embed, device)
        self.w_out = _upload(host_model.w_out, device)
        self.layers = []
        for L in host_model.layers:
            wqkv = _upload(np.concatenate([L["w_q"], L["w_k"], L["w_v"]], axis=0), device)
            self.layers.append(dict(w_qkv=wqkv, w_o=_upload(L["w_o"], device),
                                    w_router=torch.from_numpy(np.ascontiguousarray(L["w_router"], np.float32)).to(device),
                                    w_gate=_upload(L["w_gate"], device), w_up=_upload(L["w_up"], device),
                                    w_down=_upload(L["w_down"], device)))
        self._lw = (LayerWeights * len(self.layers))(*[
            LayerWeights(L["w_qkv"].data_ptr(), L["w_o"].data_ptr(), L["w_router"].data_ptr(),
                         L["w_gate"].data_ptr(), L["w_up"].data_ptr(), L["w_down"].data_ptr()) for L in self.layers])
        self._w = Weights(self.embed.data_ptr(), self.w_out.data_ptr(), self._lw)
        self._cfg = make_config(cfg)
        h = ctypes.c_void_p()
        _check(lib.dg_model_create(ctypes.byref(self._cfg), ctypes.byref(self._w), ctypes.byref(h)))
        self.handle = h
        self._taps = None

    def __del__(self):
        if getattr(self, "handle", None):
            lib.dg_model_destroy(self.handle)
            self.handle = None

    def set_experts_mx8(self, layers: list | None):
        """layers: per layer dict(gate=(codes, exps), up=(codes, exps), down=(codes, exps)) with
        codes uint8 [E][rows][K] and block exponents [E][rows][K / 32] (scale 2^x); None
        returns to the bf16 experts.  Used by the batched calls."""
        if layers is None:
            _check(lib.dg_model_set_experts_mx8(self.handle, None))
            self._lowp = None
            return
        dev, keep, structs = self.device, [], []
        for L in layers:
            ptrs = []
            for name in ("gate", "up", "down"):
                codes, exps = L[name]
                c = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).to(dev)
                sc = torch.from_numpy(pack_mx8_scales(exps)).to(dev)
                keep += [c, sc]
                ptrs += [c.data_ptr(), sc.data_ptr()]
            structs.append(ExpertsMx8(*ptrs))
        arr = (ExpertsMx8 * len(structs))(*structs)
        _check(lib.dg_model_set_experts_mx8(self.handle, arr))
        self._lowp = keep

    def set_experts_nv4(self, layers: list | None):
        """layers: per layer dict(gate=(codes, scale_codes, g), up=..., down=...) with codes
        uint8 [E][rows][K] (one 4-bit code per byte), E4M3 block-scale codes
        [E][rows][K / 16] and the tensor scale g; None returns to the bf16 experts."""
        if layers is None:
            _check(lib.dg_model_set_experts_nv4(self.handle, None, None))
            self._lowp = None
            return
        dev, keep, structs, gs = self.device, [], [], []
        for L in layers:
            ptrs = []
            for name in ("gate", "up", "down"):
                codes, sc, g = L[name]
                c = torch.from_numpy(pack_nv4_codes(codes)).to(dev)
                s_ = torch.from_numpy(pack_nv4_scales(sc)).to(dev)
                keep += [c, s_]
                ptrs += [c.data_ptr(), s_.data_ptr()]
                gs.append(float(g))
            structs.append(ExpertsMx8(*ptrs))
        arr = (ExpertsMx8 * len(structs))(*structs)
        g_arr = (ctypes.c_float * len(gs))(*gs)
        _check(lib.dg_model_set_experts_nv4(self.handle, arr, g_arr))
        self._lowp = keep

    def set_vocab_mx8(self, vocab: tuple | None):
        """vocab: (codes uint8 [V][H], block exponents [V][H / 32]) for the output matrix;
        None returns to the bf16 W_out.  Used by the batched calls."""
        if vocab is None:
            _check(lib.dg_model_set_vocab_mx8(self.handle, None, None))
            self._lowp_vocab = None
            return
        codes, exps = vocab
        c = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).to(self.device)
        sc = torch.from_numpy(pack_mx8_scales(np.asarray(exps)[None])[0]).to(self.device)
        _check(lib.dg_model_set_vocab_mx8(self.handle, ctypes.c_void_p(c.data_ptr()), ctypes.c_void_p(sc.data_ptr())))
        self._lowp_vocab = (c, sc)

    def set_vocab_nv4(self, vocab: tuple | None):
        """vocab: (codes uint8 [V][H] one 4-bit code per byte, E4M3 block-scale codes
        [V][H / 16], tensor scale g); None returns to the bf16 W_out."""
        if vocab is None:
            _check(lib.dg_model_set_vocab_nv4(self.handle, None, None, 1.0))
            self._lowp_vocab = None
            return
        codes, sc, g = vocab
        c = torch.from_numpy(pack_nv4_codes(np.asarray(codes)[None])[0]).to(self.device)
        s_ = torch.from_numpy(pack_nv4_scales(np.asarray(sc)[None])[0]).to(self.device)
        _check(lib.dg_model_set_vocab_nv4(self.handle, ctypes.c_void_p(c.data_ptr()), ctypes.c_void_p(s_.data_ptr()),
                                          float(g)))
        self._lowp_vocab = (c, s_)

    def set_taps(self, taps: dict | None):
        """taps: name -> list (per layer) of device tensors sized for taps['rows'] tokens,
        'unions' -> int32 tensor [L]; None turns off.  Calls of more tokens take no taps."""
        if taps is None:
            _check(lib.dg_set_taps(self.handle, None))
            self._taps = None
            return
        L = self.cfg["n_layers"]
        keep = {}

        def arr(name):
            if name not in taps:
                return None
            a = (ctypes.c_void_p * L)(*[t.data_ptr() for t in taps[name]])
            keep[name] = a
            return ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p))

        t = Taps(arr("x_attn"), arr("x_out"), arr("topk_idx"), arr("topk_w"), arr("counts"), arr("perm"),
                 taps["unions"].data_ptr() if "unions" in taps else None, int(taps["rows"]))
        _check(lib.dg_set_taps(self.handle, ctypes.byref(t)))
        self._taps = (taps, keep)


class KVCache:
    """Per-layer K [nkv][capacity][d] and V^T [nkv][d][capacity] device buffers."""

    def __init__(self, cfg, capacity, device="cuda"):
        nkv, d = cfg["n_kv_heads"], cfg["head_dim"]
        dt = act_torch_dtype(cfg)
        self.cfg = cfg
        self.k = [torch.zeros((nkv, capacity, d), dtype=dt, device=device) for _ in range(cfg["n_layers"])]
        self.vt = [torch.zeros((nkv, d, capacity), dtype=dt, device=device) for _ in range(cfg["n_layers"])]
        self._ka = (ctypes.c_void_p * len(self.k))(*[t.data_ptr() for t in self.k])
        self._va = (ctypes.c_void_p * len(self.vt))(*[t.data_ptr() for t in self.vt])
        self.s = KVCacheS(ctypes.cast(self._ka, ctypes.POINTER(ctypes.c_void_p)),
                          ctypes.cast(self._va, ctypes.POINTER(ctypes.c_void_p)), capacity, 0)

    @property
    def len(self):
        return self.s.len

    @len.setter
    def len(self, v):
        self.s.len = v

    @property
    def capacity(self):
        return self.s.capacity

    def load_prefix(self, layers_kv):
        """Place given prefix K/V (logical [nkv][P][d] per layer, stored arrays) at positions [0, P)."""
        P = layers_kv[0][0].shape[1]
        for l, (k, v) in enumerate(layers_kv):
            self.k[l][:, :P].copy_(_upload(k, "cpu"))
            self.vt[l][:, :, :P].copy_(_upload(np.ascontiguousarray(np.swapaxes(v, 1, 2)), "cpu"))
        self.len = P

    def logical(self, l, upto=None):
        """(K, V) of layer l as host float64 arrays [nkv][len][d] (test read-back)."""
        n = self.len if upto is None else upto
        k = self.k[l][:, :n].float().cpu().numpy().astype(np.float64)
        v = self.vt[l][:, :, :n].float().cpu().numpy().astype(np.float64).swapaxes(1, 2)
        return k, np.ascontiguousarray(v)


class Workspace:
    def __init__(self, cfg, max_tokens, device="cuda"):
        c = make_config(cfg)
        n = lib.dg_workspace_bytes(ctypes.byref(c), max_tokens)
        if n == 0:
            raise DGError(DG_ERR_INVALID_ARG, "bad config for workspace sizing")
        self.nbytes = int(n)
        self.buf = torch.zeros(self.nbytes, dtype=torch.uint8, device=device)

    @property
    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr())


def workspace_bytes(cfg, max_tokens):
    c = make_config(cfg)
    return int(lib.dg_workspace_bytes(ctypes.byref(c), max_tokens))


def update_workspace_bytes(C, V):
    return int(lib.dg_update_workspace_bytes(C, V))


def prefill_append(model: Model, cache: KVCache, tokens: torch.Tensor, ws: Workspace, stream=None):
    _check(lib.dg_prefill_append(model.handle, ctypes.byref(cache.s), _ptr(tokens), tokens.numel(), ws.ptr,
                                 ws.nbytes, _stream(stream)))


def denoise_pass(model: Model, cache: KVCache, canvas: torch.Tensor, logits: torch.Tensor, ws: Workspace,
                 stream=None):
    _check(lib.dg_denoise_pass(model.handle, ctypes.byref(cache.s), _ptr(canvas), canvas.numel(), _ptr(logits),
                               ws.ptr, ws.nbytes, _stream(stream)))


def denoise_update(model: Model, cache: KVCache, canvas: torch.Tensor, n: int, ws: Workspace, seed: int = 0,
                   step: int = 0, mask_id: int = -1, conf: torch.Tensor | None = None, stream=None):
    """One pass and its update without logits (include/dg.h); canvas int32 [C] in/out."""
    _check(lib.dg_denoise_update(model.handle, ctypes.byref(cache.s), _ptr(canvas), canvas.numel(), n,
                                 seed & 0xFFFFFFFFFFFFFFFF, step, mask_id, _ptr(conf), ws.ptr, ws.nbytes,
                                 _stream(stream)))


def canvas_update(logits: torch.Tensor, n_renoise: int, seed: int, step: int, canvas: torch.Tensor, ws,
                  conf: torch.Tensor | None = None, stream=None):
    C, V = logits.shape
    ptr = ws.ptr if isinstance(ws, Workspace) else ctypes.c_void_p(ws.data_ptr())
    nb = ws.nbytes if isinstance(ws, Workspace) else ws.numel()
    _check(lib.dg_canvas_update(_ptr(logits), C, V, n_renoise, seed & 0xFFFFFFFFFFFFFFFF, step, _ptr(canvas),
                                _ptr(conf), ptr, nb, _stream(stream)))


def canvas_update_noalloc(logits: torch.Tensor, n_renoise: int, seed: int, step: int, canvas: torch.Tensor,
                          conf: torch.Tensor | None = None, stream=None):
    """dg_canvas_update without a workspace: the scratch is libdg's fixed per-device array
    (calls on one device must be ordered; see include/dg_noalloc.h)."""
    C, V = logits.shape
    _check(lib.dg_canvas_update_noalloc(_ptr(logits), C, V, n_renoise, seed & 0xFFFFFFFFFFFFFFFF, step,
                                        _ptr(canvas), _ptr(conf), _stream(stream)))


def generate_canvas(model: Model, cache: KVCache, canvas: torch.Tensor, S: int, r_start: float, r_end: float,
                    seed: int, append: bool, logits: torch.Tensor, ws: Workspace, stream=None):
    _check(lib.dg_generate_canvas(model.handle, ctypes.byref(cache.s), _ptr(canvas), canvas.numel(), S, r_start,
                                  r_end, seed & 0xFFFFFFFFFFFFFFFF, 1 if append else 0, _ptr(logits), ws.ptr,
                                  ws.nbytes, _stream(stream)))


def canvas_update_masked(logits: torch.Tensor, n_keep: int, mask_id: int, canvas: torch.Tensor, ws,
                         conf: torch.Tensor | None = None, stream=None):
    C, V = logits.shape
    ptr = ws.ptr if isinstance(ws, Workspace) else ctypes.c_void_p(ws.data_ptr())
    nb = ws.nbytes if isinstance(ws, Workspace) else ws.numel()
    _check(lib.dg_canvas_update_masked(_ptr(logits), C, V, n_keep, mask_id, _ptr(canvas), _ptr(conf), ptr, nb,
                                       _stream(stream)))


def generate_canvas_masked(model: Model, cache: KVCache, canvas: torch.Tensor, S: int, keep_start: float,
                           keep_end: float, mask_id: int, append: bool, logits: torch.Tensor, ws: Workspace,
                           stream=None):
    _check(lib.dg_generate_canvas_masked(model.handle, ctypes.byref(cache.s), _ptr(canvas), canvas.numel(), S,
                                         keep_start, keep_end, mask_id, 1 if append else 0, _ptr(logits), ws.ptr,
                                         ws.nbytes, _stream(stream)))


def _caches(caches):
    """Host array of the caches' C structs (copies; lens are copied back after a call that advances them)."""
    return (KVCacheS * len(caches))(*[c.s for c in caches])


def prefill_append_batched(model: Model, caches: list, tokens: torch.Tensor, ws: Workspace, stream=None):
    """tokens int32 [B][T]: row b is appended to caches[b]."""
    B, T = tokens.shape
    arr = _caches(caches)
    _check(lib.dg_prefill_append_batched(model.handle, arr, B, _ptr(tokens), T, ws.ptr, ws.nbytes, _stream(stream)))
    for c, s in zip(caches, arr):
        c.len = s.len


def denoise_pass_batched(model: Model, caches: list, canvases: torch.Tensor, logits: torch.Tensor, ws: Workspace,
                         stream=None):
    """canvases int32 [B][C], logits fp32 [B][C][V]; canvas b attends to caches[b] only."""
    B, C = canvases.shape
    _check(lib.dg_denoise_pass_batched(model.handle, _caches(caches), B, _ptr(canvases), C, _ptr(logits), ws.ptr,
                                       ws.nbytes, _stream(stream)))


def generate_canvases(model: Model, caches: list, canvases: torch.Tensor, S: int, r_start: float, r_end: float,
                      seeds, append: bool, logits: torch.Tensor, ws: Workspace, stream=None):
    """generate_canvas for B canvases at once; canvas b re-noised from seeds[b]."""
    B, C = canvases.shape
    arr = _caches(caches)
    sd = (ctypes.c_uint64 * B)(*[int(x) & 0xFFFFFFFFFFFFFFFF for x in seeds])
    _check(lib.dg_generate_canvases(model.handle, arr, B, _ptr(canvases), C, S, r_start, r_end, sd,
                                    1 if append else 0, _ptr(logits), ws.ptr, ws.nbytes, _stream(stream)))
    for c, s in zip(caches, arr):
        c.len = s.len


def generate_canvases_masked(model: Model, caches: list, canvases: torch.Tensor, S: int, keep_start: float,
                             keep_end: float, mask_id: int, append: bool, logits: torch.Tensor, ws: Workspace,
                             stream=None):
    """generate_canvas_masked for B canvases at once (canvases int32 [B][C], written by the call)."""
    B, C = canvases.shape
    arr = _caches(caches)
    _check(lib.dg_generate_canvases_masked(model.handle, arr, B, _ptr(canvases), C, S, keep_start, keep_end, mask_id,
                                           1 if append else 0, _ptr(logits), ws.ptr, ws.nbytes, _stream(stream)))
    for c, s in zip(caches, arr):
        c.len = s.len


def device_status(ws, stream=None):
    ptr = ws.ptr if isinstance(ws, Workspace) else ctypes.c_void_p(ws.data_ptr())
    _check(lib.dg_device_status(ptr, _stream(stream)))


def renoise_count(C, S, step, r_start, r_end) -> int:
    return int(lib.dg_renoise_count(C, S, step, r_start, r_end))


def profile_enable(on: bool):
    _check(lib.dg_profile_enable(1 if on else 0))


def profile_reset():
    lib.dg_profile_reset()


def profile_read(kind) -> tuple[float, int]:
    k = KERNEL_KINDS.index(kind) if isinstance(kind, str) else int(kind)
    ms = ctypes.c_double()
    n = ctypes.c_int32()
    _check(lib.dg_profile_read(k, ctypes.byref(ms), ctypes.byref(n)))
    return ms.value, n.value


def launch_count() -> int:
    return int(lib.dg_launch_count())


def debug_gemm_scratch(x_rows, n_groups, device="cuda"):
    n = int(lib.dg_debug_gemm_scratch_bytes(x_rows, n_groups))
    return torch.zeros(n, dtype=torch.uint8, device=device)


def debug_gemm_bf16(W, X, out, ld_out, err, scratch, W2=None, X_lo=None, group_off=None, out_lo=None,
                    stream=None):
    """One persistent tcgen05 GEMM launch (see include/dg_debug.h). W [groups][rows][K]."""
    G, rows, K = W.shape
    _check(lib.dg_debug_gemm_bf16(_ptr(W), _ptr(W2), rows, G, _ptr(X), _ptr(X_lo), X.shape[0], K, _ptr(group_off),
                                  _ptr(out), _ptr(out_lo), ld_out, _ptr(scratch),
                                  scratch.numel(), _ptr(err), _stream(stream)))


def pack_mx8_scales(exponents: np.ndarray) -> np.ndarray:
    """Block exponents x of weights [groups][rows][K] (one per 32 consecutive K elements,
    array [groups][rows][K / 32], block scale 2^x) -> the library's scale bytes
    [groups][K / 64][rows][2] (E8M0: x + 127)."""
    e = np.asarray(exponents, dtype=np.int64)
    G, R, nb = e.shape
    if nb % 2 or e.min() < -127 or e.max() > 7:
        raise ValueError("block exponents must come in pairs per 64 K elements and lie in [-127, 7]")
    return np.ascontiguousarray((e + 127).astype(np.uint8).reshape(G, R, nb // 2, 2).transpose(0, 2, 1, 3))


def debug_gemm_mx8(W, W_scales, X, out, ld_out, err, scratch, W2=None, W2_scales=None, X_lo=None, group_off=None,
                   out_lo=None, stream=None):
    """One launch of the 8-bit-weight GEMM (see include/dg_debug.h): W uint8 codes
    [groups][rows][K], W_scales uint8 [groups][K / 64][rows][2]."""
    G, rows, K = W.shape
    _check(lib.dg_debug_gemm_mx8(_ptr(W), _ptr(W_scales), _ptr(W2), _ptr(W2_scales), rows, G, _ptr(X), _ptr(X_lo),
                                 X.shape[0], K, _ptr(group_off), _ptr(out), _ptr(out_lo), ld_out, _ptr(scratch),
                                 scratch.numel(), _ptr(err), _stream(stream)))


def pack_nv4_codes(codes: np.ndarray) -> np.ndarray:
    """4-bit codes, one per byte [groups][rows][K] -> two per byte [groups][rows][K / 2]
    (element 2 i in the low nibble of byte i)."""
    c = np.asarray(codes, dtype=np.uint8)
    if c.shape[-1] % 2 or (c > 0xF).any():
        raise ValueError("4-bit codes in [0, 16) with an even row length")
    return np.ascontiguousarray(c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def pack_nv4_scales(scale_codes: np.ndarray) -> np.ndarray:
    """E4M3 block-scale codes [groups][rows][K / 16] -> the library's [groups][K / 64][rows][4]."""
    sc = np.asarray(scale_codes, dtype=np.uint8)
    G, R, nb = sc.shape
    if nb % 4:
        raise ValueError("four block scales per 64 K elements")
    return np.ascontiguousarray(sc.reshape(G, R, nb // 4, 4).transpose(0, 2, 1, 3))


def debug_gemm_nv4(W, W_scales, g, X, out, ld_out, err, scratch, W2=None, W2_scales=None, g2=1.0, X_lo=None,
                   group_off=None, out_lo=None, stream=None):
    """One launch of the 4-bit-weight GEMM (see include/dg_debug.h): W uint8 packed codes
    [groups][rows][K / 2], W_scales uint8 [groups][K / 64][rows][4], g the tensor scale."""
    G, rows, K2 = W.shape
    _check(lib.dg_debug_gemm_nv4(_ptr(W), _ptr(W_scales), float(g), _ptr(W2), _ptr(W2_scales), float(g2), rows, G,
                                 _ptr(X), _ptr(X_lo), X.shape[0], 2 * K2, _ptr(group_off), _ptr(out), _ptr(out_lo),
                                 ld_out, _ptr(scratch), scratch.numel(), _ptr(err), _stream(stream)))


def debug_attention_bf16(q, k, vt, n_keys, pos0, causal, out, ws: Workspace, out_lo=None, stream=None):
    """One attention launch (see include/dg_debug.h): q [nq][n_q][128], k [nkv][cap][128], vt [nkv][128][cap]."""
    nq, n_q, _ = q.shape
    nkv, cap, _ = k.shape
    _check(lib.dg_debug_attention_bf16(_ptr(q), _ptr(k), _ptr(vt), cap, n_q, pos0, n_keys, 1 if causal else 0, nq,
                                       nkv, _ptr(out), _ptr(out_lo), ws.ptr, ws.nbytes, _stream(stream)))


def debug_attention_pair_bf16(q, k, vt, n_keys, pos0, causal, out, ws: Workspace, out_lo=None, stream=None):
    """The same attention through the head-pair kernel (see include/dg_debug.h)."""
    nq, n_q, _ = q.shape
    nkv, cap, _ = k.shape
    _check(lib.dg_debug_attention_pair_bf16(_ptr(q), _ptr(k), _ptr(vt), cap, n_q, pos0, n_keys, 1 if causal else 0,
                                            nq, nkv, _ptr(out), _ptr(out_lo), ws.ptr, ws.nbytes, _stream(stream)))


def debug_bounded_wait(ws, timeout_ms, stream=None):
    """Launch the bounded-wait self-test kernel (see include/dg_debug.h)."""
    ptr = ws.ptr if isinstance(ws, Workspace) else ctypes.c_void_p(ws.data_ptr())
    _check(lib.dg_debug_bounded_wait(ptr, timeout_ms, _stream(stream)))


WAIT_LIMIT_DEFAULT_NS = 2_000_000_000


def debug_mma_rate(a_tmem: bool, n: int, count: int, blocks: int, stream=None):
    """Tensor-pipe rate probe (include/dg_debug.h): returns (block 0's cycles from the first
    MMA issue to the completion, the launch's milliseconds)."""
    cyc = ctypes.c_uint64()
    ms = ctypes.c_float()
    _check(lib.dg_debug_mma_rate(1 if a_tmem else 0, int(n), int(count), int(blocks), ctypes.byref(cyc),
                                 ctypes.byref(ms), _stream(stream)))
    return int(cyc.value), float(ms.value)


def debug_set_wait_limit(limit_ns: int):
    """Limit of the tensor-core kernels' bounded waits for later launches (see include/dg_debug.h)."""
    _check(lib.dg_debug_set_wait_limit(int(limit_ns)))
