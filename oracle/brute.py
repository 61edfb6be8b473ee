"""The decode definition as pure-Python loops (math.exp, math.fsum), for tiny
inputs only.  Test infrastructure only (see the package docstring).

It is written independently of ``mla_oracle``: it decodes bf16 bits with
``struct``, walks the block table page by page, and forms the log-sum-exp and
the weighted sum with explicit loops, so that a slip in the vectorised
oracle (a transposed operand, a wrong slice, a missing scale, a bad page
lookup) shows up as a disagreement.
"""
from __future__ import annotations

import math
import struct
from typing import List, Tuple


def _bf16(bits: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (int(bits) & 0xFFFF) << 16))[0]


def _key_row(kv_bits, block_table, b: int, t: int) -> List[float]:
    page = int(block_table[b][t // 64])
    slot = t % 64
    return [_bf16(v) for v in kv_bits[page][slot][0]]


def decode_token(q_bits_row, kv_bits, block_table, b: int, L: int, limit: int,
                 scale: float) -> Tuple[List[List[float]], List[float]]:
    """All heads of one query token against keys t < min(L, limit).
    q_bits_row: [h_q][576] bf16 bits.  Returns (out [h_q][512], lse [h_q])."""
    n = min(L, limit)
    keys = [_key_row(kv_bits, block_table, b, t) for t in range(n)]
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
