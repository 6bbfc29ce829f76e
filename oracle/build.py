"""Build the C++ oracle (oracle/dg_oracle.cpp) into oracle/libdg_oracle.so -- TEST
INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU baseline load it.

    python -m oracle.build [--force]

Plain g++ with OpenMP; x86-64-v3 (AVX2 + FMA) so that the library built here also runs
on the GPU machines' host cores.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "dg_oracle.cpp")
LIB = os.path.join(HERE, "libdg_oracle.so")
# the system compiler (its OpenMP runtime is installed); $DG_ORACLE_CXX overrides
CXX = os.environ.get("DG_ORACLE_CXX") or shutil.which("g++") or "g++"
FLAGS = ["-O2", "-std=c++17", "-march=x86-64-v3", "-fopenmp", "-fPIC", "-shared", "-Wall"]


def compile_source(src_path: str, out_path: str) -> str:
    """Compile one oracle source file into a shared library at out_path."""
    tmp = out_path + f".tmp{os.getpid()}"
    r = subprocess.run([CXX] + FLAGS + [src_path, "-o", tmp], capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"oracle build failed ({src_path}):\n{r.stdout}{r.stderr}")
    os.replace(tmp, out_path)   # atomic: a concurrent loader never sees a half-written file
    return out_path


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        compile_source(SRC, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
