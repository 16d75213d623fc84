"""Host-side fast path of the synthetic weight generator (synthetic/fastgen.c).

Produces exactly the tensors synthetic.weights.make_weight produces on the CPU
(checked by tests), in a few seconds for an 8B-parameter model.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from typing import Optional

import torch

from .configs import SpecConfig
from .weights import (QUANT_KINDS, SIGMA_S, _layer_base_shape, quantized, split_part, storage_dtype, tensor_key,
                      weight_shapes)

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    src = os.path.join(_HERE, "fastgen.c")
    out_dir = os.path.join(_HERE, "_build")
    out = os.path.join(out_dir, "libfastgen.so")
    if not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        os.makedirs(out_dir, exist_ok=True)
        tmp = out + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", src, "-o", tmp], check=True)
        os.replace(tmp, out)
    lib = C.CDLL(out)
    lib.fastgen_f32.argtypes = [C.c_void_p, C.c_uint64, C.c_uint32, C.c_float, C.c_float, C.c_int]
    lib.fastgen_bf16.argtypes = [C.c_void_p, C.c_uint64, C.c_uint32, C.c_float]
    _lib = lib
    return lib


def make_weight_host(cfg: SpecConfig, name: str, random_gains: bool = False, seed: Optional[int] = None) -> torch.Tensor:
    lib = _load()
    shape, kind = weight_shapes(cfg)[name]
    seed = cfg.seed if seed is None else seed
    n = 1
    for d in shape:
        n *= d
    key = tensor_key(name, seed)
    if kind == "norm":
        if not random_gains:
            return torch.ones(shape, dtype=torch.float32)
        t = torch.empty(shape, dtype=torch.float32)
        lib.fastgen_f32(t.data_ptr(), n, key, float(torch.tensor(0.1 / SIGMA_S, dtype=torch.float32)), 1.0, 1)
        return t
    scale = float(torch.tensor(cfg.weight_std / SIGMA_S, dtype=torch.float32))
    if kind in QUANT_KINDS:
        base, part = split_part(name, kind)
        bshape = _layer_base_shape(cfg, base)
        bn = 1
        for d in bshape:
            bn *= d

        def make_base():
            t = torch.empty(bshape, dtype=torch.bfloat16)
            lib.fastgen_bf16(t.data_ptr(), bn, tensor_key(base, seed), scale)
            return t
        return quantized(base, (cfg.name, seed, "cpu", cfg.weight_std), make_base, cfg.dtype)[part]
    if storage_dtype(cfg) == torch.bfloat16:
        t = torch.empty(shape, dtype=torch.bfloat16)
        lib.fastgen_bf16(t.data_ptr(), n, key, scale)
    else:
        t = torch.empty(shape, dtype=torch.float32)
        lib.fastgen_f32(t.data_ptr(), n, key, scale, 0.0, 0)
    return t


def make_weights_host(cfg: SpecConfig, random_gains: bool = False, seed: Optional[int] = None):
    return {n: make_weight_host(cfg, n, random_gains, seed) for n in weight_shapes(cfg)}
