"""The ctypes binding against the C headers: every function include/*.h declares is bound,
with the declared number of parameters, each of the declared kind (pointer, 32- or 64-bit
integer, float, size), and the declared return type.  A binding that drifted from a
header would place arguments wrongly in calls that only a GPU run would make."""
import ctypes
import glob
import os
import re

from block_diffusion_lm_masked_b200 import dg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCALARS = {"int32_t": ctypes.c_int32, "uint32_t": ctypes.c_uint32, "uint64_t": ctypes.c_uint64,
           "int64_t": ctypes.c_int64, "float": ctypes.c_float, "double": ctypes.c_double, "size_t": ctypes.c_size_t}
RETURNS = {"dg_status": ctypes.c_int32, "size_t": ctypes.c_size_t, "void": None, "const char*": ctypes.c_char_p,
           "int32_t": ctypes.c_int32, "int64_t": ctypes.c_int64}


def declarations():
    out = {}
    for h in sorted(glob.glob(os.path.join(ROOT, "include", "*.h"))):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        src = re.sub(r"#[^\n]*", " ", src)
        for m in re.finditer(r"([A-Za-z_][\w\s\*]*?)\b(dg_\w+)\s*\(([^;{}()]*)\)\s*;", src):
            ret, name, params = " ".join(m.group(1).split()), m.group(2), m.group(3).strip()
            if ret.startswith("typedef") or "typedef" in ret:
                continue
            plist = [] if params in ("", "void") else [" ".join(p.split()) for p in params.split(",")]
            out[name] = (ret.replace(" *", "*"), plist)
    return out


def kind_ok(param, ctype):
    if "*" in param or param.split()[0] == "dg_stream":
        return ctype in (ctypes.c_void_p, ctypes.c_char_p) or issubclass(ctype, ctypes._Pointer)
    base = [t for t in param.replace("const ", "").split() if t in SCALARS]
    return bool(base) and SCALARS[base[0]] is ctype


def test_every_declared_function_is_bound_with_its_signature():
    decls = declarations()
    assert len(decls) >= 30, sorted(decls)
    for name, (ret, params) in decls.items():
        f = getattr(dg.lib, name)
        assert f.argtypes is not None, f"{name} has no argtypes in the binding"
        assert len(f.argtypes) == len(params), f"{name}: header {len(params)} parameters, binding {len(f.argtypes)}"
        for i, (p, t) in enumerate(zip(params, f.argtypes)):
            assert kind_ok(p, t), f"{name} parameter {i} '{p}' bound as {t.__name__}"
        want = RETURNS.get(ret, "?")
        assert want != "?", f"{name}: unexpected return type '{ret}'"
        assert f.restype is want, f"{name}: returns {ret}, bound as {f.restype}"


def test_the_parser_sees_the_known_shapes():
    """The header parser itself: a few declarations checked by hand."""
    d = declarations()
    assert d["dg_model_set_vocab_nv4"] == ("dg_status", ["dg_model* m", "const void* codes", "const void* scales",
                                                         "float tensor_scale"])
    assert d["dg_launch_count"][1] == [] and d["dg_last_error"][0] == "const char*"
    assert len(d["dg_debug_attention_pair_bf16"][1]) == 15


def test_kernel_kinds_follow_the_library_numbering():
    """The binding's kernel-kind names (used to label the bench's per-kernel times) are the
    library's, in its order, and cover every kind."""
    got = [dg.lib.dg_kernel_name(i).decode() for i in range(len(dg.KERNEL_KINDS))]
    assert got == dg.KERNEL_KINDS
    assert dg.lib.dg_kernel_name(len(dg.KERNEL_KINDS)).decode() == "?"
