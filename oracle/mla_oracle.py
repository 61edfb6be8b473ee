"""Reference MLA decode over a paged KV cache, in float64.

Test infrastructure only (see the package docstring).

What is computed (one shared latent KV head, h_kv = 1):

* The call returns ``o_i, lse_i`` for queries ``q``, the paged cache, the
  ``block_table``, ``cache_seqlens``, the output width ``dv`` and a ``causal``
  flag ("Was ist FlashMLA?" (topnet.top), section "3. MLA-Decodierung
  ausführen").  The cache is paged with block size 64 (same page, section
  "Hauptmerkmale von FlashMLA").
* A cache row holds 576 dims: 512 latent (NoPE) dims and 64 RoPE dims (the
  split the FlashMLA walkthrough (sao.pub), section "二、核心功能与架构", gives
  for its cache rows).  Keys use all 576 dims; values are the first 512 dims
  of the same rows (dv = 512).
* The sparse path attends only to the positions named by an ``indices``
  tensor (walkthrough, section "二、核心功能与架构", DSA paragraph).

Readings where the pages say nothing (each is listed in the design notes):

1. logits s_t = scale * (q . K_t), default scale = 576 ** -0.5;
   lse = ln(sum_t exp(s_t)) over the visible keys, natural log, of the
   *scaled* logits; out = sum_t exp(s_t - lse) * K_t[:512].
2. Causal with s_q > 1: the s_q new tokens are the last s_q cache positions;
   token i sees keys t <= L - s_q + i.  With s_q = 1 causal changes nothing.
3. Empty key set: out = 0 and lse = -inf.
4. Sparse indices are logical positions in [0, L_b) of sequence b, resolved
   through the block_table; -1 is padding; other values outside [0, L_b) are
   skipped as invalid; duplicates count as separate keys; all h_q heads of a
   token share its index list; ``causal`` is ignored on the sparse path.
"""
from __future__ import annotations

from typing import Optional, Sequence, Tuple

import numpy as np

from .formats import bf16_bits_to_f64, fp8_rows_to_f64

PAGE = 64
D_QK = 576
D_V = 512


def gather_rows(block_table: np.ndarray, b: int, positions: np.ndarray, *,
                kv_bits: Optional[np.ndarray] = None,
                kv_fp8: Optional[np.ndarray] = None) -> np.ndarray:
    """Cache rows of logical positions ``positions`` of sequence ``b`` as
    float64 [n, 576]: row t lives in physical page block_table[b, t // 64] at
    slot t % 64."""
    positions = np.asarray(positions, dtype=np.int64)
    pages = block_table[b, positions // PAGE].astype(np.int64)
    slots = positions % PAGE
    if kv_fp8 is not None:
        return fp8_rows_to_f64(kv_fp8[pages, slots, 0, :])
    return bf16_bits_to_f64(kv_bits[pages, slots, 0, :])


def attend(q_rows: np.ndarray, keys: np.ndarray, scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """softmax(scale * q K^T) V and the log-sum-exp for query rows
    q_rows [h, 576] against keys [n, 576] (V = keys[:, :512]).

    Returns out [h, 512] and lse [h] in float64; an empty key set gives
    out = 0 and lse = -inf."""
    h = q_rows.shape[0]
    if keys.shape[0] == 0:
        return np.zeros((h, D_V)), np.full(h, -np.inf)
    s = scale * (q_rows @ keys.T)                      # [h, n]
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    out = (p @ keys[:, :D_V]) / l
    lse = (m + np.log(l))[:, 0]
    return out, lse


def visible_positions(L: int, s_q: int, i: int, causal: bool) -> np.ndarray:
    """Dense key set of query token i: t < L, and t <= L - s_q + i if causal."""
    hi = L if not causal else max(0, min(L, L - s_q + i + 1))
    return np.arange(hi, dtype=np.int64)


def sparse_positions(indices_row: np.ndarray, L: int) -> np.ndarray:
    """Sparse key multiset of one query token: its indices that lie in
    [0, L), in index order (-1 padding and out-of-range values skipped)."""
    idx = np.asarray(indices_row, dtype=np.int64)
    return idx[(idx >= 0) & (idx < L)]


def decode(q_bits: np.ndarray, block_table: np.ndarray, cache_seqlens: np.ndarray, *,
           kv_bits: Optional[np.ndarray] = None, kv_fp8: Optional[np.ndarray] = None,
           indices: Optional[np.ndarray] = None, causal: bool = False,
           softmax_scale: Optional[float] = None,
           batches: Optional[Sequence[int]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Decode every sequence (or only ``batches``).

    q_bits uint16 [b, s_q, h_q, 576] (bf16 bits).  Returns out float64
    [b, s_q, h_q, 512] and lse float64 [b, h_q, s_q]; rows of sequences not in
    ``batches`` are left NaN."""
    assert (kv_bits is None) != (kv_fp8 is None)
    bsz, s_q, h_q, d = q_bits.shape
    assert d == D_QK
    scale = D_QK ** -0.5 if softmax_scale is None else float(softmax_scale)
    out = np.full((bsz, s_q, h_q, D_V), np.nan)
    lse = np.full((bsz, h_q, s_q), np.nan)
    for b in (range(bsz) if batches is None else batches):
        L = int(cache_seqlens[b])
        keys_all = None
        for i in range(s_q):
            if indices is not None:
                pos = sparse_positions(indices[b, i], L)
                keys = gather_rows(block_table, b, pos, kv_bits=kv_bits, kv_fp8=kv_fp8)
            else:
                if keys_all is None:
                    keys_all = gather_rows(block_table, b, np.arange(L), kv_bits=kv_bits, kv_fp8=kv_fp8)
                keys = keys_all[:len(visible_positions(L, s_q, i, causal))]
            o, l_ = attend(bf16_bits_to_f64(q_bits[b, i]), keys, scale)
            out[b, i] = o
            lse[b, :, i] = l_
    return out, lse


def merge_splits(outs: Sequence[np.ndarray], lses: Sequence[np.ndarray]) -> Tuple[np.ndarray, np.ndarray]:
    """Merge attention results computed over disjoint key subsets.

    Each part j has normalised out_j [h, 512] and lse_j [h].  With
    L = max_j lse_j, lse = L + ln sum_j exp(lse_j - L) and
    out = sum_j exp(lse_j - lse) * out_j.  Parts with lse = -inf weigh 0;
    if every part is empty the result is out = 0, lse = -inf."""
    lse_stack = np.stack(lses)                       # [k, h]
    out_stack = np.stack(outs)                       # [k, h, 512]
    mx = lse_stack.max(axis=0)
    safe = np.where(np.isfinite(mx), mx, 0.0)
    tot = np.exp(lse_stack - safe).sum(axis=0)
    with np.errstate(divide="ignore"):
        lse = np.where(tot > 0, safe + np.log(tot), -np.inf)
    w = np.where(np.isfinite(lse)[None], np.exp(lse_stack - np.where(np.isfinite(lse), lse, 0.0)[None]), 0.0)
    out = (w[..., None] * out_stack).sum(axis=0)
    return out, lse
