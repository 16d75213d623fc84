"""FP8 (E4M3) weight codes with one fp32 scale per output row.

The quantised form of a bf16 matrix W[..., K] (rows = every index but the
last) is a pair (codes, scale):

  scale[r]    = fp32(max_k |W[r, k]|) / fp32(448)          (1 for an all-zero row)
  codes[r, k] = E4M3 code of fp32(W[r, k]) / scale[r], rounded to nearest even

and the quantised model's weight is W_q[r, k] = scale[r] * e4m3_value(codes[r, k]).
E4M3 (the OCP 8-bit float with 4 exponent and 3 mantissa bits): sign bit,
exponent bias 7, subnormals 0.mmm * 2^-6, largest finite 448 (code 0x7E), no
infinities, 0x7F / 0xFF are NaN (never produced here).

This module only prepares inputs: it turns the seeded bf16 weights into the
codes and scales both implementations read, with integer and IEEE fp32
operations that give the same bits on a CPU and a GPU.  The dequantised
arithmetic itself lives in each implementation.
"""
from __future__ import annotations

from typing import Tuple

import torch

E4M3_MAX = 448.0
_MIN_NORMAL_BITS = 121 << 23  # fp32 bit pattern of 2^-6, the smallest normal E4M3 magnitude


def e4m3_encode(x: torch.Tensor) -> torch.Tensor:
    """Round fp32 values (|x| <= 448) to E4M3 codes, ties to even."""
    if x.dtype != torch.float32:
        raise TypeError("fp32 input expected")
    u = x.contiguous().view(torch.int32)
    sign = (u >> 31) & 1
    a = u & 0x7FFFFFFF
    # normal range: keep 3 of the 23 fp32 mantissa bits, round to nearest even,
    # then move the exponent bias from 127 to 7 ((127 - 7) << 3 = 960)
    normal = ((a + 0x7FFFF + ((a >> 20) & 1)) >> 20) - 960
    # below 2^-6: multiples of 2^-9 (the scaling by 512 is exact), ties to even
    sub = torch.round(x.abs() * 512.0).to(torch.int32)
    code = torch.where(a >= _MIN_NORMAL_BITS, normal, sub).clamp(max=0x7E)
    return (code | (sign << 7)).to(torch.uint8)


def e4m3_decode(codes: torch.Tensor) -> torch.Tensor:
    """fp64 value of E4M3 codes (NaN for 0x7F / 0xFF)."""
    c = codes.to(torch.int64)
    s, e, m = (c >> 7) & 1, (c >> 3) & 15, c & 7
    mag = torch.where(e == 0, m.double() * 2.0 ** -9, (1.0 + m.double() / 8.0) * torch.pow(2.0, (e - 7).double()))
    mag = torch.where((e == 15) & (m == 7), torch.full_like(mag, float("nan")), mag)
    return torch.where(s == 1, -mag, mag)


def quantize_rows(w: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """(codes uint8 [..., K], scale fp32 [...]) of a bf16 / fp32 matrix."""
    wf = w.float()
    amax = wf.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / torch.tensor(E4M3_MAX, dtype=torch.float32, device=w.device),
                        torch.ones_like(amax))
    return e4m3_encode(wf / scale.unsqueeze(-1)), scale


def dequantize_rows(codes: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    """fp64 W_q = scale[r] * e4m3_value(codes[r, k])."""
    return scale.double().unsqueeze(-1) * e4m3_decode(codes)
