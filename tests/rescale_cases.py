"""Workloads whose running max jumps mid-sequence.

The GPU parity tests that exercise the decode kernel's O rescale use them.
So does a CPU test that replays the kernel's lazy-rescale rule on them to
check that they really rescale.  N(0, 1) data alone never moves a row's max
past the threshold after the first page, so a few key rows on later pages are
boosted:
- bf16 rows are scaled x12;
- FP8 rows either get group scales 2^-5 (7-28 times the workload's scales),
  or keep their own non-power-of-two scales multiplied by 17 (float32); the
  second kind is the general case, whose dequantised values have up to 28
  significant bits, and its boosted logits reach 30-50."""
from __future__ import annotations

import numpy as np

from mla_decode_attention_get_b200 import inputs as I

BOOST_SCALE = 2.0 ** -5


def _boost_bf16(w, phys, row):
    bits = w.kv_bits[phys, row, 0, :].astype(np.uint32) << 16
    w.kv_bits[phys, row, 0, :] = I.f32_to_bf16_bits(bits.view(np.float32) * 12.0)


def _boost_fp8(w, phys, row):
    # the four group scales sit in bytes 512..527 (little-endian f32)
    w.kv_fp8[phys, row, 0, 512:528] = np.full(4, BOOST_SCALE, "<f4").view(np.uint8)


def _boost_fp8_x17(w, phys, row):
    # the row's own scales x17: not powers of two, so code x scale is not a
    # short binary number
    raw = w.kv_fp8[phys, row, 0, 512:528].copy().view("<f4")
    w.kv_fp8[phys, row, 0, 512:528] = (raw * np.float32(17.0)).astype("<f4").view(np.uint8)


def _boost_dense_positions(w, boost):
    for b, L in enumerate(w.cache_seqlens):
        for tok in (700 + b, 1500, int(L) - 3):
            boost(w, w.block_table[b, tok // 64], tok % 64)
    return w


def bf16_case(h_q: int, s_q: int, causal: bool):
    w = I.make_workload("rescale", 2, s_q, h_q, [3000, 2000], causal=causal, seed=50 + h_q)
    return _boost_dense_positions(w, _boost_bf16)


def fp8_dense_case(x17: bool = False):
    w = I.make_workload("fp8dresc", 2, 1, 64, [3000, 2000], fp8=True, seed=47)
    return _boost_dense_positions(w, _boost_fp8_x17 if x17 else _boost_fp8)


def fp8_sparse_case(x17: bool = False):
    # the rows named at index slots 700 and 1500 of every token
    w = I.make_workload("rescale8", 2, 1, 128, [4000, 3000], fp8=True, topk=2048, seed=53)
    boost = _boost_fp8_x17 if x17 else _boost_fp8
    for b in range(w.batch):
        for slot in (700, 1500):
            pos = int(w.indices[b, 0, slot])
            boost(w, w.block_table[b, pos // 64], pos % 64)
    return w
