"""The decode definition as pure-Python loops (math.exp, math.fsum), for tiny
inputs only.  Test infrastructure only (see the package docstring).

It is written independently of ``mla_oracle`` and ``formats``: it decodes
bf16 bits with ``struct``, e4m3 codes from their bit fields and the FP8 row's
scales with ``struct``, walks the block table page by page (or the index
list, on the sparse path), and forms the log-sum-exp and the weighted sum
with explicit loops, so that a slip in the vectorised oracle (a transposed
operand, a wrong slice, a missing scale, a bad page or index lookup) shows up
as a disagreement.

FP8 row (FlashMLA walkthrough (sao.pub), section "二、核心功能与架构"): bytes
0..511 are e4m3 codes, 512..527 four little-endian float32 scales (one per
128 codes), 528..655 sixty-four little-endian bf16 RoPE values.
"""
from __future__ import annotations

import math
import struct
from typing import List, Tuple


def _bf16(bits: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (int(bits) & 0xFFFF) << 16))[0]


def _e4m3(byte: int) -> float:
    """e4m3fn: sign bit, 4 exponent bits (bias 7), 3 mantissa bits; a zero
    exponent field is subnormal (m * 2^-9); S.1111.111 is NaN."""
    sign = -1.0 if byte & 0x80 else 1.0
    e, m = (byte >> 3) & 15, byte & 7
    if e == 15 and m == 7:
        return math.nan
    if e == 0:
        return sign * m * 2.0 ** -9
    return sign * (8 + m) * 2.0 ** (e - 10)


def _key_row(kv_bits, block_table, b: int, t: int) -> List[float]:
    page = int(block_table[b][t // 64])
    slot = t % 64
    return [_bf16(v) for v in kv_bits[page][slot][0]]


def _fp8_key_row(kv_fp8, block_table, b: int, t: int) -> List[float]:
    page = int(block_table[b][t // 64])
    row = bytes(int(v) for v in kv_fp8[page][t % 64][0])
    scales = struct.unpack("<4f", row[512:528])
    nope = [_e4m3(row[d]) * scales[d // 128] for d in range(512)]
    rope = [_bf16(v) for v in struct.unpack("<64H", row[528:656])]
    return nope + rope


def decode_token(q_bits_row, kv_bits, block_table, b: int, L: int, limit: int,
                 scale: float, kv_fp8=None) -> Tuple[List[List[float]], List[float]]:
    """All heads of one query token against keys t < min(L, limit), from the
    bf16 cache or, with kv_fp8, the FP8 cache.  q_bits_row: [h_q][576] bf16
    bits.  Returns (out [h_q][512], lse [h_q])."""
    n = min(L, limit)
    if kv_fp8 is not None:
        keys = [_fp8_key_row(kv_fp8, block_table, b, t) for t in range(n)]
    else:
        keys = [_key_row(kv_bits, block_table, b, t) for t in range(n)]
    return _attend(q_bits_row, keys, scale)


def decode_token_sparse(q_bits_row, kv_fp8, block_table, b: int, L: int, index_row,
                        scale: float) -> Tuple[List[List[float]], List[float]]:
    """All heads of one query token against the FP8 cache positions its
    index list names: -1 is padding, a position outside [0, L) is skipped, a
    position listed twice is two keys."""
    keys = [_fp8_key_row(kv_fp8, block_table, b, int(i)) for i in index_row if 0 <= int(i) < L]
    return _attend(q_bits_row, keys, scale)


def _attend(q_bits_row, keys, scale: float) -> Tuple[List[List[float]], List[float]]:
    n = len(keys)
    outs, lses = [], []
    for qb in q_bits_row:
        q = [_bf16(v) for v in qb]
        if n == 0:
            outs.append([0.0] * 512)
            lses.append(-math.inf)
            continue
        logits = []
        for k in keys:
            acc = math.fsum(q[d] * k[d] for d in range(576))
            logits.append(scale * acc)
        top = max(logits)
        weights = [math.exp(s - top) for s in logits]
        denom = math.fsum(weights)
        lses.append(top + math.log(denom))
        out = []
        for d in range(512):
            out.append(math.fsum(weights[t] * keys[t][d] for t in range(n)) / denom)
        outs.append(out)
    return outs, lses
