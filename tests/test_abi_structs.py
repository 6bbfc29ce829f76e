"""The binding's ctypes structs against the C structs of include/*.h: a small C program,
compiled here with the host compiler against the headers, prints each struct's size and
every field's offset; the ctypes layouts must agree, so the library reads exactly the
fields the binding writes."""
import ctypes
import os
import shutil
import subprocess

import pytest

from block_diffusion_lm_masked_b200 import dg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

STRUCTS = {
    "dg_config": (dg.Config, ["n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "n_experts", "top_k",
                              "expert_ffn", "vocab", "rope_theta", "rms_eps", "dtype"]),
    "dg_layer_weights": (dg.LayerWeights, ["w_qkv", "w_o", "w_router", "w_gate", "w_up", "w_down"]),
    "dg_weights": (dg.Weights, ["embed", "w_out", "layers"]),
    "dg_kv_cache": (dg.KVCacheS, ["k", "vt", "capacity", "len"]),
    "dg_expert_weights_mx8": (dg.ExpertsMx8, ["gate", "gate_scales", "up", "up_scales", "down", "down_scales"]),
    "dg_taps": (dg.Taps, ["x_attn", "x_out", "topk_idx", "topk_w", "counts", "perm", "unions", "rows"]),
}


def c_layouts(tmp_path):
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "dg.h"', '#include "dg_debug.h"',
             'int main(void) {']
    for s, (_, fields) in STRUCTS.items():
        lines.append(f'  printf("{s} size %zu\\n", sizeof({s}));')
        for f in fields:
            lines.append(f'  printf("{s} {f} %zu\\n", offsetof({s}, {f}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layouts.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layouts"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines():
        s, f, v = line.split()
        out[(s, f)] = int(v)
    return out


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs the host C compiler")
def test_ctypes_structs_match_the_headers(tmp_path):
    c = c_layouts(tmp_path)
    for s, (cls, fields) in STRUCTS.items():
        assert [f for f, _ in cls._fields_] == fields, f"{s}: field order"
        assert ctypes.sizeof(cls) == c[(s, "size")], f"{s}: size {ctypes.sizeof(cls)} vs C {c[(s, 'size')]}"
        for f in fields:
            assert getattr(cls, f).offset == c[(s, f)], f"{s}.{f}: offset {getattr(cls, f).offset} vs C {c[(s, f)]}"
