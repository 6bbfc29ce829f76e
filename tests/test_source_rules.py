"""Static checks of the CUDA sources and the committed profiling commands (no GPU).

They guard rules that keep the kernels safe to run on a shared GPU:
  * no bulk or tensor copy with cluster multicast anywhere in the library (a multicast
    load whose source could be another GPU's memory is never built);
  * no device trap or assert: a failure is reported through the status word and the
    kernel returns;
  * every spin on an mbarrier lives in the bounded helpers of dg_common.cuh (a wait that
    gives up after a time limit, or the wind-down wait with a fixed limit), and each of
    them reads the clock;
  * no register reallocation (setmaxnreg), whose split must add up against the launch;
  * every ncu command committed under profiles/ leaves the GPU's clocks alone.
"""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_diffusion_lm_masked_b200", "csrc")


def _sources():
    out = {}
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(CSRC, name)) as f:
                out[name] = f.read()
    return out


def _strip_comments(text):
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.sub(r"//[^\n]*", "", text)


def test_sources_found():
    src = _sources()
    for name in ("dg_common.cuh", "k_tc_attn.cu", "k_tc_gemm.cu", "k_simt.cu", "dg_api.cu"):
        assert name in src, name


def test_no_multicast_copies():
    for name, text in _sources().items():
        assert "multicast" not in _strip_comments(text), name


def test_no_device_trap_or_assert():
    for name, text in _sources().items():
        code = _strip_comments(text)
        assert "__trap" not in code, name
        assert "trap;" not in code, name
        assert not re.search(r"(?<![_\w])assert\s*\(", code), name


def test_no_register_reallocation():
    for name, text in _sources().items():
        assert "setmaxnreg" not in _strip_comments(text), name


def _function_bodies(code):
    """(name, body) of every brace-delimited function definition at namespace level."""
    out = []
    for m in re.finditer(r"([A-Za-z_]\w*)\s*\([^;{}]*\)\s*(?:const\s*)?\{", code):
        depth, i = 1, m.end()
        while depth and i < len(code):
            depth += {"{": 1, "}": -1}.get(code[i], 0)
            i += 1
        out.append((m.group(1), code[m.end():i - 1]))
    return out


def test_mbarrier_spins_only_in_bounded_helpers():
    src = _sources()
    for name, text in src.items():
        code = _strip_comments(text)
        if name == "dg_common.cuh":
            continue
        # the raw try-wait is wrapped once, in dg_common.cuh; everything else calls the
        # bounded helpers
        assert "mbarrier.try_wait" not in code, name
        assert "mbar_try_wait" not in code, name
        assert not re.search(r"while\s*\(\s*(true|1)\s*\)|for\s*\(\s*;\s*;\s*\)", code), name
    common = _strip_comments(src["dg_common.cuh"])
    spinning = [(fn, body) for fn, body in _function_bodies(common)
                if re.search(r"while\s*\([^)]*mbar_try_wait|while\s*\(\s*true\s*\)", body)]
    assert {fn for fn, _ in spinning} >= {"mbar_wait", "mbar_wait_drain"}, [fn for fn, _ in spinning]
    for fn, body in spinning:
        assert "globaltimer" in body, fn          # every spin reads the clock ...
        assert re.search(r"return\s*(false)?\s*;", body), fn  # ... and gives up


def test_profiled_ncu_commands_leave_clocks_alone():
    pdir = os.path.join(ROOT, "profiles")
    seen = 0
    for name in sorted(os.listdir(pdir)):
        with open(os.path.join(pdir, name)) as f:
            text = f.read()
        # join continuation lines, then check every ncu invocation on a line
        text = text.replace("\\\n", " ")
        for line in text.splitlines():
            for m in re.finditer(r"\bncu\s+-", line):  # an ncu invocation (not the prose's "ncu")
                cmd = line[m.start():]
                if re.match(r"ncu\s+-i\s", cmd):      # reading a saved report runs nothing
                    continue
                seen += 1
                assert "--clock-control none" in cmd, (name, line)
    assert seen >= 5
