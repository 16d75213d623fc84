"""MXFP4 weight codes: FP4 (E2M1) elements sharing one power-of-two scale per
32 values along K (the OCP Microscaling form), plus one fp32 scale per output row.

The quantised form of a bf16 matrix W[rows, K] (K a multiple of 128) is a
triple (codes, bscale, scale):

  E[r, b]    = floor(log2(max_{k in block b} |W[r, k]|)) - 2, clamped to [-127, 127]
               (block b holds k = 32b .. 32b + 31; an all-zero block takes -127)
  code[r, k] = E2M1 code of W[r, k] / 2^E[r, k // 32], rounded to nearest even,
               magnitudes above 6 saturated to 6
  scale[r]   = 1

and the quantised model's weight is W_q[r, k] = scale[r] * 2^E[r, k // 32] *
e2m1_value(code[r, k]).  The "- 2" is the exponent of E2M1's largest normal
magnitude (6 = 1.5 * 2^2), so a block's largest element lands in [4, 8) before
the rounding.  E2M1 (4-bit float): sign bit, 2 exponent bits with bias 1, 1
mantissa bit; magnitudes 0, 0.5 (subnormal), 1, 1.5, 2, 3, 4, 6.

Storage (what the weight arena holds):
  codes   uint8 [rows, K/2]        element k in byte k // 2, the low nibble for even k
  bscale  uint8 [K/128, rows, 4]   byte (k // 128, r, (k // 32) % 4) = E[r, k // 32] + 127 (UE8M0)
  scale   fp32  [rows]

This module only prepares inputs: it turns the seeded bf16 weights into the
codes and scales both implementations read, with exact integer and IEEE fp32
operations (power-of-two scalings and comparisons) that give the same bits on a
CPU and a GPU.  The dequantised arithmetic itself lives in each implementation.
"""
from __future__ import annotations

from typing import Tuple

import torch

E2M1_MAX = 6.0
EMAX_ELEM = 2  # exponent of the largest E2M1 normal magnitude


def e2m1_encode(x: torch.Tensor) -> torch.Tensor:
    """4-bit E2M1 codes (uint8, 0..15) of fp32 values, nearest even, saturating at 6."""
    if x.dtype != torch.float32:
        raise TypeError("fp32 input expected")
    a = x.abs()
    # the magnitude code counts the rounding thresholds below |x|; at a tie (the
    # midpoint of two grid values) the even code wins, so the comparison is >=
    # where the upper code is even and > where it is odd
    code = (a > 0.25).to(torch.uint8)
    code += (a >= 0.75).to(torch.uint8)
    code += (a > 1.25).to(torch.uint8)
    code += (a >= 1.75).to(torch.uint8)
    code += (a > 2.5).to(torch.uint8)
    code += (a >= 3.5).to(torch.uint8)
    code += (a > 5.0).to(torch.uint8)
    return code | (torch.signbit(x).to(torch.uint8) << 3)


def e2m1_decode(codes: torch.Tensor) -> torch.Tensor:
    """fp64 value of 4-bit E2M1 codes (0..15)."""
    c = codes.to(torch.int64)
    s, e, m = (c >> 3) & 1, (c >> 1) & 3, c & 1
    mag = torch.where(e == 0, m.double() * 0.5, (1.0 + m.double() * 0.5) * torch.pow(2.0, (e - 1).double()))
    return torch.where(s == 1, -mag, mag)


def block_exponents(w: torch.Tensor) -> torch.Tensor:
    """E [rows, K/32] (int32) of a matrix [rows, K]."""
    wf = w.float()
    rows, K = wf.shape
    amax = wf.abs().view(rows, K // 32, 32).amax(-1)
    _, ex = torch.frexp(amax)  # amax = mant * 2^ex, mant in [0.5, 1): floor(log2 amax) = ex - 1
    e = (ex.to(torch.int32) - 1) - EMAX_ELEM
    e = torch.where(amax > 0, e, torch.full_like(e, -127))
    return e.clamp(-127, 127)


def quantize_mx(w: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """(codes uint8 [rows, K/2], bscale uint8 [K/128, rows, 4], scale fp32 [rows])
    of a bf16 / fp32 matrix [rows, K], K a multiple of 128."""
    if w.dim() != 2 or w.shape[1] % 128:
        raise ValueError("MXFP4 needs a matrix with K a multiple of 128")
    rows, K = w.shape
    e = block_exponents(w)
    wf = w.float().view(rows, K // 32, 32)
    # w / 2^E: a multiplication by the fp32 power of two 2^-E (E <= 125 for
    # finite inputs, so 2^-E is a normal number built from its exponent bits);
    # exact unless the product underflows, which only values that round to code 0
    # can do
    inv = ((127 - e).to(torch.int32) << 23).view(torch.float32)
    y = (wf * inv.unsqueeze(-1)).view(rows, K)
    c = e2m1_encode(y)
    codes = (c[:, 0::2] | (c[:, 1::2] << 4)).contiguous()
    bscale = (e + 127).to(torch.uint8).view(rows, K // 128, 4).permute(1, 0, 2).contiguous()
    scale = torch.ones(rows, dtype=torch.float32, device=w.device)
    return codes, bscale, scale


def unpack_codes(codes: torch.Tensor) -> torch.Tensor:
    """4-bit codes [rows, K] of the packed bytes [rows, K/2]."""
    lo, hi = codes & 15, codes >> 4
    return torch.stack([lo, hi], dim=-1).view(codes.shape[0], codes.shape[1] * 2)


def dequantize_mx(codes: torch.Tensor, bscale: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    """fp64 W_q[r, k] = scale[r] * 2^(bscale byte - 127) * e2m1_value(code[r, k])."""
    c = unpack_codes(codes)
    rows, K = c.shape
    e = bscale.permute(1, 0, 2).reshape(rows, K // 32).to(torch.int64) - 127
    p2 = torch.pow(2.0, e.double()).repeat_interleave(32, dim=1)
    return scale.double().unsqueeze(-1) * p2 * e2m1_decode(c)
