"""Number formats of the KV cache, decoded exactly into float64.

Test infrastructure only (see the package docstring).

* bfloat16: the upper 16 bits of an IEEE-754 binary32.
* e4m3 ("fn" variant, the OCP 8-bit floating-point format): 1 sign bit,
  4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 encodes
  subnormals m/8 * 2^-6; the all-ones exponent with all-ones mantissa is NaN;
  there is no infinity, so the largest finite magnitude is 1.75 * 2^8 = 448.
* FP8 cache row (FlashMLA walkthrough (sao.pub), section "二、核心功能与架构",
  KV-cache format list): 512 e4m3 NoPE values, then 4 float32 scales (one per
  128 NoPE values), then 64 unquantised bfloat16 RoPE values -- 656 bytes.
  A dequantised NoPE value is code value * scale of its group.
"""
from __future__ import annotations

import numpy as np

D_NOPE = 512
D_ROPE = 64
GROUP = 128
ROW_BYTES = D_NOPE + 16 + 2 * D_ROPE


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bfloat16 bit patterns (uint16) as float64."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u32.view(np.float32).astype(np.float64)


def e4m3_value(code: int) -> float:
    """Value of one e4m3fn code, from the field definition."""
    sign = -1.0 if (code >> 7) & 1 else 1.0
    exp = (code >> 3) & 0xF
    man = code & 0x7
    if exp == 0xF and man == 0x7:
        return float("nan")
    if exp == 0:
        return sign * (man / 8.0) * 2.0 ** (1 - 7)
    return sign * (1.0 + man / 8.0) * 2.0 ** (exp - 7)


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def fp8_rows_to_f64(rows: np.ndarray) -> np.ndarray:
    """Dequantise FP8 cache rows uint8 [..., 656] into float64 [..., 576]:
    NoPE[d] = e4m3(byte[d]) * scale[d // 128] for d < 512, then the 64
    bfloat16 RoPE values."""
    rows = np.asarray(rows, dtype=np.uint8)
    assert rows.shape[-1] == ROW_BYTES
    lead = rows.shape[:-1]
    nope = E4M3_TABLE[rows[..., :D_NOPE]]
    scales = np.ascontiguousarray(rows[..., D_NOPE:D_NOPE + 16]).view("<f4").astype(np.float64)
    scales = scales.reshape(lead + (4,))
    nope = nope * np.repeat(scales, GROUP, axis=-1)
    rope = bf16_bits_to_f64(np.ascontiguousarray(rows[..., D_NOPE + 16:]).view("<u2").reshape(lead + (D_ROPE,)))
    return np.concatenate([nope, rope], axis=-1)
