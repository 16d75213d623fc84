"""Counter-based synthetic weights, bit-identical on CPU and GPU.

Every matrix entry is a function of (seed, tensor name, flat index):

  k  = crc32(name) XOR lowbias32(seed)
  h1 = lowbias32(lowbias32(i) XOR k),  h2 = lowbias32(h1 XOR 0x9E3779B9)
  S  = sum of the four 16-bit halves of h1 and h2, minus their mean 131070
  w  = round_to_storage_type( float32(S) * float32(std / sigma_S) )

lowbias32 is the 32-bit integer hash published by C. Wellons ("Prospecting
for hash functions", 2018): x ^= x>>16; x *= 0x7feb352d; x ^= x>>15;
x *= 0x846ca68b; x ^= x>>16.  S is an Irwin-Hall sum of four uniform 16-bit
integers: mean 0, standard deviation sigma_S = sqrt((65536^2 - 1)/3), tails cut
at 3.46 sigma.  It stands in for N(0, std): same mean and variance, close shape.
Every step is integer arithmetic, one int->fp32 conversion, one fp32 multiply
and one round-to-nearest-even cast, all exactly specified by IEEE-754, so CPU
and CUDA tensors come out identical.

RMSNorm gains are 1 (the plain reading of "random init"); tests can ask for
random gains 1 + 0.1*z to exercise the gain path.
"""
from __future__ import annotations

import math
import zlib
from collections import OrderedDict
from typing import Dict, Optional, Tuple

import torch

from .configs import ModelDims, SpecConfig

M32 = 0xFFFFFFFF
SIGMA_S = math.sqrt((65536.0 ** 2 - 1.0) / 3.0)
_CHUNK = 1 << 24


def _mul32(x: torch.Tensor, c: int) -> torch.Tensor:
    """(x * c) mod 2^32 for int64 x in [0, 2^32), without int64 overflow."""
    c_lo = c & 0xFFFF
    return ((x & 0xFFFF) * c + ((((x >> 16) * c_lo) & 0xFFFF) << 16)) & M32


def hash32(x: torch.Tensor) -> torch.Tensor:
    """lowbias32 on an int64 tensor holding uint32 values."""
    x = x ^ (x >> 16)
    x = _mul32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


def _hash32_int(x: int) -> int:
    x &= M32
    x ^= x >> 16
    x = (x * 0x7FEB352D) & M32
    x ^= x >> 15
    x = (x * 0x846CA68B) & M32
    x ^= x >> 16
    return x


def tensor_key(name: str, seed: int) -> int:
    return (zlib.crc32(name.encode()) ^ _hash32_int(seed * 0x9E3779B1 + 0x632BE5AB)) & M32


def centered_irwin_hall(idx: torch.Tensor, key: int) -> torch.Tensor:
    """Integer S in [-131070, 131070] for flat indices idx (int64)."""
    h1 = hash32(hash32(idx & M32) ^ key)
    h2 = hash32(h1 ^ 0x9E3779B9)
    s = (h1 & 0xFFFF) + (h1 >> 16) + (h2 & 0xFFFF) + (h2 >> 16)
    return s - 131070


def _fill(shape: Tuple[int, ...], name: str, seed: int, scale: float, offset: float,
          dtype: torch.dtype, device) -> torch.Tensor:
    n = 1
    for d in shape:
        n *= d
    if n >= (1 << 32):
        raise ValueError(f"{name}: {n} elements exceed the 32-bit counter")
    key = tensor_key(name, seed)
    out = torch.empty(n, dtype=dtype, device=device)
    c = torch.tensor(scale, dtype=torch.float32, device=device)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        idx = torch.arange(s, e, dtype=torch.int64, device=device)
        v = centered_irwin_hall(idx, key).to(torch.float32) * c
        if offset != 0.0:
            v = v + torch.tensor(offset, dtype=torch.float32, device=device)
        out[s:e] = v.to(dtype)
    return out.view(shape)


def _layer_shapes(prefix: str, d: ModelDims) -> "OrderedDict[str, Tuple[Tuple[int, ...], str]]":
    H = d.hidden
    s: "OrderedDict[str, Tuple[Tuple[int, ...], str]]" = OrderedDict()
    for l in range(d.n_layers):
        p = f"{prefix}.L{l}."
        s[p + "attn_norm"] = ((H,), "norm")
        s[p + "wqkv"] = ((d.qkv_dim, H), "matrix")      # rows: [Wq; Wk; Wv]
        s[p + "wo"] = ((H, d.q_dim), "matrix")
        if d.qk_norm:
            s[p + "q_norm"] = ((d.head_dim,), "norm")
            s[p + "k_norm"] = ((d.head_dim,), "norm")
        s[p + "ffn_norm"] = ((H,), "norm")
        if d.is_moe:
            s[p + "w_router"] = ((d.n_experts, H), "matrix")
            s[p + "we_gate_up"] = ((d.n_experts, 2 * d.expert_ffn, H), "matrix")  # per expert [gate; up]
            s[p + "we_down"] = ((d.n_experts, H, d.expert_ffn), "matrix")
        else:
            s[p + "w_gate_up"] = ((2 * d.ffn, H), "matrix")   # rows: [W_gate; W_up]
            s[p + "w_down"] = ((H, d.ffn), "matrix")
    s[prefix + ".final_norm"] = ((H,), "norm")
    return s


def weight_shapes(cfg: SpecConfig) -> "OrderedDict[str, Tuple[Tuple[int, ...], str]]":
    """Logical, row-major tensors of one workload, in a fixed order.

    With cfg.dtype == "fp8" every matrix but the embedding is stored as E4M3
    codes (kind "fp8", uint8) plus "<name>.scale" (kind "scale", fp32, one
    value per row); see synthetic.fp8.  With cfg.dtype == "fp4" the same
    matrices are MXFP4: packed E2M1 codes (kind "fp4", uint8 [rows, K/2]),
    "<name>.bscale" (kind "bscale", uint8 [K/128, rows, 4]) and "<name>.scale";
    see synthetic.fp4."""
    t, dr = cfg.target, cfg.drafter
    s: "OrderedDict[str, Tuple[Tuple[int, ...], str]]" = OrderedDict()
    s["embed"] = ((t.vocab, t.hidden), "matrix")
    s["lm_head"] = ((t.vocab, t.hidden), "matrix")
    s.update(_layer_shapes("target", t))
    s.update(_layer_shapes("drafter", dr))
    s["fuse.w_fc"] = ((dr.hidden, cfg.n_taps * t.hidden), "matrix")
    s["fuse.norm"] = ((dr.hidden,), "norm")
    if cfg.dtype not in ("fp8", "fp4"):
        return s
    if t.is_moe:
        raise ValueError(f"{cfg.dtype} weights are built for dense targets only")
    q: "OrderedDict[str, Tuple[Tuple[int, ...], str]]" = OrderedDict()
    for name, (shape, kind) in s.items():
        if kind == "matrix" and name != "embed":
            if cfg.dtype == "fp8":
                q[name] = (shape, "fp8")
            else:
                rows, K = shape
                q[name] = ((rows, K // 2), "fp4")
                q[name + ".bscale"] = ((K // 128, rows, 4), "bscale")
            q[name + ".scale"] = (shape[:-1], "scale")
        else:
            q[name] = (shape, kind)
    return q


def _layer_base_shape(cfg: SpecConfig, base: str) -> Tuple[int, ...]:
    """Logical shape [rows, K] of a quantised matrix (its codes' shape for fp8)."""
    shape, kind = weight_shapes(cfg)[base]
    return (shape[0], shape[1] * 2) if kind == "fp4" else shape


def weight_names(cfg: SpecConfig):
    return list(weight_shapes(cfg).keys())


def storage_dtype(cfg: SpecConfig) -> torch.dtype:
    """Type of the generated matrices (fp8 and fp4 models quantise bf16 ones)."""
    return torch.bfloat16 if cfg.dtype in ("bf16", "fp8", "fp4") else torch.float32


_QCACHE: dict = {}


QUANT_KINDS = ("fp8", "fp4", "bscale", "scale")


def quantized(name: str, key, make_base, fmt: str = "fp8"):
    """The stored parts of matrix `name` quantised to `fmt`: {"": codes, ".scale":
    row scales} (+ ".bscale" for fp4), cached while the parts are fetched."""
    k = (name, key, fmt)
    if k not in _QCACHE:
        _QCACHE.clear()
        if fmt == "fp8":
            from .fp8 import quantize_rows
            codes, scale = quantize_rows(make_base())
            _QCACHE[k] = {"": codes, ".scale": scale}
        else:
            from .fp4 import quantize_mx
            codes, bscale, scale = quantize_mx(make_base())
            _QCACHE[k] = {"": codes, ".bscale": bscale, ".scale": scale}
    return _QCACHE[k]


def split_part(name: str, kind: str) -> Tuple[str, str]:
    """(matrix name, part suffix) of a stored tensor of a quantised matrix."""
    for suf in (".scale", ".bscale"):
        if kind in ("scale", "bscale") and name.endswith(suf):
            return name[:-len(suf)], suf
    return name, ""


def make_weight(cfg: SpecConfig, name: str, device="cpu", random_gains: bool = False,
                seed: Optional[int] = None) -> torch.Tensor:
    shape, kind = weight_shapes(cfg)[name]
    seed = cfg.seed if seed is None else seed
    if kind == "norm":
        if not random_gains:
            return torch.ones(shape, dtype=torch.float32, device=device)
        return _fill(shape, name, seed, 0.1 / SIGMA_S, 1.0, torch.float32, device)
    if kind in QUANT_KINDS:
        base, part = split_part(name, kind)
        bshape = _layer_base_shape(cfg, base)
        parts = quantized(base, (cfg.name, seed, str(device), cfg.weight_std),
                          lambda: _fill(bshape, base, seed, cfg.weight_std / SIGMA_S, 0.0, torch.bfloat16, device),
                          cfg.dtype)
        return parts[part]
    return _fill(shape, name, seed, cfg.weight_std / SIGMA_S, 0.0, storage_dtype(cfg), device)


def make_weights(cfg: SpecConfig, device="cpu", random_gains: bool = False,
                 seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    return OrderedDict((n, make_weight(cfg, n, device, random_gains, seed))
                       for n in weight_shapes(cfg))
