"""FP8 cache writer, restated plainly: quantise new key rows into the FP8
cache row format and store them at their cache slots.

Test infrastructure only (see the package docstring): the CUDA writer is
checked against this byte for byte.

The row format is the FlashMLA walkthrough's (sao.pub), section
"二、核心功能与架构", KV-cache format list: 512 e4m3 NoPE values with one
float32 scale per 128 of them, then 64 unquantised bfloat16 RoPE values
(656 bytes).  The pages fix the format, not how a writer chooses the scales.
The reading taken here (the plainest one):

* per 128-value group, scale = max |x| / 448 computed in float32 (448 is the
  largest e4m3 magnitude), so the group's largest value maps to +-448;
* code = e4m3 of x / scale (float32 IEEE division), rounded to nearest with
  ties to the even code, saturating at +-448; the sign of zero is kept;
* a group whose values are all zero gets scale 0 and codes 0;
* RoPE values are copied bit for bit.
"""
from __future__ import annotations

import numpy as np

from .formats import D_NOPE, D_ROPE, E4M3_TABLE, GROUP, ROW_BYTES

E4M3_MAX = 448.0
_MAG_VALUES = E4M3_TABLE[:0x7F]          # codes 0x00..0x7e: 0 .. 448, increasing


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """e4m3 code (uint8) of each value: nearest finite e4m3 magnitude, ties
    to the even code (even mantissa), saturating at 448, sign bit from x."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    i = np.searchsorted(_MAG_VALUES, a, side="right") - 1          # largest magnitude <= a
    j = np.minimum(i + 1, len(_MAG_VALUES) - 1)
    d_lo = a - _MAG_VALUES[i]
    d_hi = _MAG_VALUES[j] - a
    up = (d_hi < d_lo) | ((d_hi == d_lo) & (i % 2 == 1))
    code = np.where(up, j, i).astype(np.uint8)
    return code | np.where(np.signbit(x), 0x80, 0).astype(np.uint8)


def quantize_rows(k_bits: np.ndarray) -> np.ndarray:
    """bf16 key rows (uint16 bits [n, 576]) -> FP8 cache rows uint8 [n, 656]."""
    k_bits = np.asarray(k_bits, dtype=np.uint16)
    n = k_bits.shape[0]
    assert k_bits.shape == (n, D_NOPE + D_ROPE)
    nope = (k_bits[:, :D_NOPE].astype(np.uint32) << 16).view(np.float32)      # exact
    out = np.zeros((n, ROW_BYTES), dtype=np.uint8)
    scales = np.zeros((n, D_NOPE // GROUP), dtype=np.float32)
    for g in range(D_NOPE // GROUP):
        grp = nope[:, g * GROUP:(g + 1) * GROUP]
        amax = np.max(np.abs(grp), axis=1)                                     # float32, exact
        scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)               # float32 division
        nz = amax > 0
        q = np.zeros_like(grp)
        q[nz] = grp[nz] / scale[nz, None]                                      # float32 division
        codes = e4m3_round(q)
        codes[~nz] = 0
        out[:, g * GROUP:(g + 1) * GROUP] = codes
        scales[:, g] = np.where(nz, scale, np.float32(0))
    out[:, D_NOPE:D_NOPE + 16] = scales.astype("<f4").view(np.uint8).reshape(n, 16)
    out[:, D_NOPE + 16:] = np.ascontiguousarray(k_bits[:, D_NOPE:]).astype("<u2").view(np.uint8).reshape(n, 2 * D_ROPE)
    return out


def write_cache(cache: np.ndarray, k_bits: np.ndarray, slot_mapping: np.ndarray):
    """Store the quantised rows of k_bits into a copy of the FP8 cache
    (uint8 [num_blocks, 64, 1, 656]) at slot = page * 64 + row of each token.
    Slot -1 skips a token; a slot outside the cache is skipped and reported.
    Returns (new cache, any slot out of range)."""
    cache = np.array(cache, dtype=np.uint8, copy=True)
    rows = quantize_rows(k_bits)
    bad = False
    for i, slot in enumerate(np.asarray(slot_mapping, dtype=np.int64)):
        if slot == -1:
            continue
        if slot < 0 or slot >= cache.shape[0] * 64:
            bad = True
            continue
        cache[slot // 64, slot % 64, 0, :] = rows[i]
    return cache, bad
