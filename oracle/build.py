"""Compile the C oracle into oracle/_build/libdflash_oracle.so (gcc + OpenMP)."""
from __future__ import annotations

import os
import subprocess

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dflash_oracle.c")
_HDR = os.path.join(_HERE, "dflash_oracle.h")
_OUT_DIR = os.path.join(_HERE, "_build")


def oracle_lib_path() -> str:
    return os.path.join(_OUT_DIR, "libdflash_oracle.so")


def build_oracle(force: bool = False, verbose: bool = False) -> str:
    out = oracle_lib_path()
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))):
        return out
    os.makedirs(_OUT_DIR, exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    # Portable x86-64 flags: the oracle may run on a different host CPU than it was built on.
    cmd = ["gcc", "-O3", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-mavx2", "-mfma",
           "-Wall", "-Wno-unused-function", _SRC, "-o", tmp, "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out
