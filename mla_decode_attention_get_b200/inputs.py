"""Seeded synthetic inputs for MLA decoding over a paged KV cache.

This module is shared by the tests, the benchmark and the CPU oracle's
callers.  It only draws random numbers and lays them out in the storage
formats the decode path consumes; it holds none of the attention arithmetic.

Storage formats (all little-endian, raw bits so that both the CUDA path and
the oracle start from identical bytes):

* ``q_bits``      uint16 [batch, s_q, h_q, 576]  -- bfloat16 bit patterns
* ``kv_bits``     uint16 [num_blocks, 64, 1, 576] -- bfloat16 cache rows
                  (512 latent "NoPE" dims followed by 64 RoPE dims)
* ``kv_fp8``      uint8  [num_blocks, 64, 1, 656] -- FP8 cache rows:
                  512 e4m3 NoPE codes | 4 float32 scales | 64 bfloat16 RoPE
                  values (row format from the FlashMLA walkthrough (sao.pub),
                  section "二、核心功能与架构", KV-cache format list)
* ``block_table`` int32 [batch, max_blocks] -- physical page of each logical
                  64-token page, -1 where unused
* ``cache_seqlens`` int32 [batch]
* ``indices``     int32 [batch, s_q, topk] -- logical token positions, -1 pads

Workload recipes follow the five decode configurations of the project
(tiny, memory-bound, variable-length, MTP causal, FP8 sparse); see
``CONFIGS``.  Every array comes from its own PCG64 stream spawned from
``SeedSequence(seed)``, so arrays do not depend on each other's draw order.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np
import torch

PAGE = 64
D_QK = 576
D_V = 512
D_NOPE = 512
D_ROPE = 64
FP8_ROW_BYTES = D_NOPE + 4 * 4 + D_ROPE * 2  # 656
E4M3_MAX = 448.0

# Number of pages generated per chunk when filling large caches; fixed so the
# bytes of a given seed never depend on available memory.
_CHUNK_PAGES = 2048


@dataclasses.dataclass
class Workload:
    name: str
    batch: int
    s_q: int
    h_q: int
    causal: bool
    fp8: bool
    topk: int
    seed: int
    cache_seqlens: np.ndarray          # int32 [batch]
    block_table: np.ndarray            # int32 [batch, max_blocks]
    q_bits: np.ndarray                 # uint16 [batch, s_q, h_q, 576]
    kv_bits: Optional[np.ndarray]      # uint16 [nblk, 64, 1, 576] (bf16 cache)
    kv_fp8: Optional[np.ndarray]       # uint8  [nblk, 64, 1, 656] (fp8 cache)
    indices: Optional[np.ndarray]      # int32 [batch, s_q, topk]
    softmax_scale: float

    @property
    def num_blocks(self) -> int:
        kv = self.kv_fp8 if self.fp8 else self.kv_bits
        return int(kv.shape[0])

    def kv_rows_visible(self) -> int:
        """Number of cache rows the decode reads (one per key and sequence,
        or one per valid index for the sparse path)."""
        if self.indices is not None:
            return int((self.indices >= 0).sum())
        return int(self.cache_seqlens.astype(np.int64).sum())


def _rngs(seed: int, n: int) -> List[np.random.Generator]:
    return [np.random.Generator(np.random.PCG64(s))
            for s in np.random.SeedSequence(seed).spawn(n)]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round-to-nearest-even, by torch) and
    return the 16-bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def f32_to_e4m3_codes(x: np.ndarray) -> np.ndarray:
    """Saturate to +-448, then round to e4m3fn (round-to-nearest-even, by
    torch).  Saturating first matters: torch maps out-of-range values to NaN."""
    x = np.clip(np.asarray(x, dtype=np.float32), -E4M3_MAX, E4M3_MAX)
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    return f32_to_bf16_bits(rng.standard_normal(size=shape, dtype=np.float32))


def _page_layout(rng_perm: np.random.Generator, seqlens: np.ndarray, min_blocks: int = 0):
    """Assign a shuffled physical page to every logical page of every sequence."""
    pages_per_seq = [(int(L) + PAGE - 1) // PAGE for L in seqlens]
    total = sum(pages_per_seq)
    nblk = max(total, min_blocks, 1)
    perm = rng_perm.permutation(nblk).astype(np.int32)
    width = max(max(pages_per_seq) if pages_per_seq else 0, 1)
    bt = np.full((len(seqlens), width), -1, dtype=np.int32)
    pos = 0
    for b, n in enumerate(pages_per_seq):
        bt[b, :n] = perm[pos:pos + n]
        pos += n
    return bt, nblk


def _fill_bf16_cache(rng: np.random.Generator, nblk: int) -> np.ndarray:
    kv = np.empty((nblk, PAGE, 1, D_QK), dtype=np.uint16)
    for p0 in range(0, nblk, _CHUNK_PAGES):
        p1 = min(nblk, p0 + _CHUNK_PAGES)
        kv[p0:p1] = _normal_bf16(rng, (p1 - p0, PAGE, 1, D_QK))
    return kv


def _fill_fp8_cache(rng_scale: np.random.Generator, rng_nope: np.random.Generator,
                    rng_rope: np.random.Generator, nblk: int) -> np.ndarray:
    """FP8 rows: scales ~ U[0.5, 2]/448 per 128-value group; NoPE codes are
    sat_e4m3(N(0,1)/scale); RoPE ~ N(0,1) rounded to bf16."""
    kv = np.empty((nblk, PAGE, 1, FP8_ROW_BYTES), dtype=np.uint8)
    for p0 in range(0, nblk, _CHUNK_PAGES):
        p1 = min(nblk, p0 + _CHUNK_PAGES)
        n = p1 - p0
        scales = (rng_scale.uniform(0.5, 2.0, size=(n, PAGE, 1, 4)) / E4M3_MAX).astype(np.float32)
        x = rng_nope.standard_normal(size=(n, PAGE, 1, D_NOPE), dtype=np.float32)
        x /= np.repeat(scales, D_NOPE // 4, axis=-1)
        kv[p0:p1, :, :, :D_NOPE] = f32_to_e4m3_codes(x)
        kv[p0:p1, :, :, D_NOPE:D_NOPE + 16] = scales.view(np.uint8).reshape(n, PAGE, 1, 16)
        rope = _normal_bf16(rng_rope, (n, PAGE, 1, D_ROPE))
        kv[p0:p1, :, :, D_NOPE + 16:] = rope.view(np.uint8).reshape(n, PAGE, 1, 2 * D_ROPE)
    return kv


def make_workload(name: str, batch: int, s_q: int, h_q: int, seqlens, *, causal: bool = False,
                  fp8: bool = False, topk: int = 0, seed: int = 0, pad_rows_per_token: int = 0,
                  num_padded_rows: int = 0, softmax_scale: Optional[float] = None,
                  min_blocks: int = 0) -> Workload:
    """Build one seeded workload.

    ``seqlens`` is a list of cache lengths.  For the sparse path (``topk`` >
    0) every query token draws ``topk`` distinct positions from [0, L_b); then
    ``num_padded_rows`` seeded (b, token) rows get their last
    ``pad_rows_per_token`` entries set to -1.
    """
    r_len, r_perm, r_q, r_kv, r_scale, r_rope, r_idx, r_pad = _rngs(seed, 8)
    del r_len  # lengths are given explicitly here; kept for stream stability
    seqlens = np.asarray(seqlens, dtype=np.int32)
    assert seqlens.shape == (batch,)
    bt, nblk = _page_layout(r_perm, seqlens, min_blocks)
    q_bits = _normal_bf16(r_q, (batch, s_q, h_q, D_QK))
    kv_bits = kv_fp8 = None
    if fp8:
        kv_fp8 = _fill_fp8_cache(r_scale, r_kv, r_rope, nblk)
    else:
        kv_bits = _fill_bf16_cache(r_kv, nblk)
    indices = None
    if topk > 0:
        indices = np.empty((batch, s_q, topk), dtype=np.int32)
        for b in range(batch):
            L = int(seqlens[b])
            for i in range(s_q):
                if L >= topk:
                    indices[b, i] = r_idx.choice(L, size=topk, replace=False).astype(np.int32)
                else:
                    row = np.full(topk, -1, dtype=np.int32)
                    row[:L] = r_idx.permutation(L).astype(np.int32)
                    indices[b, i] = row
        if num_padded_rows > 0 and pad_rows_per_token > 0:
            flat = indices.reshape(batch * s_q, topk)
            rows = r_pad.choice(batch * s_q, size=min(num_padded_rows, batch * s_q), replace=False)
            for r in rows:
                flat[r, topk - pad_rows_per_token:] = -1
    if softmax_scale is None:
        softmax_scale = D_QK ** -0.5
    return Workload(name=name, batch=batch, s_q=s_q, h_q=h_q, causal=causal, fp8=fp8, topk=topk,
                    seed=seed, cache_seqlens=seqlens, block_table=bt, q_bits=q_bits,
                    kv_bits=kv_bits, kv_fp8=kv_fp8, indices=indices,
                    softmax_scale=float(softmax_scale))


def _varlen_lengths(seed: int, batch: int, lo: int, hi: int, n_min: int, n_max: int) -> np.ndarray:
    rng = _rngs(seed, 8)[0]
    L = rng.integers(lo, hi + 1, size=batch).astype(np.int32)
    forced = rng.choice(batch, size=n_min + n_max, replace=False)
    L[forced[:n_min]] = lo
    L[forced[n_min:]] = hi
    return L


# The five decode configurations.  Each entry builds its Workload; the
# seed is 1000 + config number.
CONFIG_NAMES = {
    1: "tiny bf16 decode b=2 s_q=1 h_q=16 L={100,37}",
    2: "memory-bound bf16 decode b=128 s_q=1 h_q=16 L=4096",
    3: "varlen bf16 decode b=64 s_q=1 h_q=128 L~U[1,8192]",
    4: "MTP causal bf16 decode b=132 s_q=2 h_q=128 L=16384",
    5: "fp8 sparse decode b=64 s_q=1 h_q=128 L=32768 topk=2048",
}


def make_config(cfg: int, *, batch: Optional[int] = None, seqlen: Optional[int] = None) -> Workload:
    """Workload of decode configuration ``cfg`` (1..5).  ``batch`` /
    ``seqlen`` shrink the configuration (same recipe, smaller sizes) for tests
    the oracle must finish in seconds."""
    seed = 1000 + cfg
    if cfg == 1:
        return make_workload("tiny", 2, 1, 16, [100, 37], seed=seed)
    if cfg == 2:
        b = batch or 128
        L = seqlen or 4096
        return make_workload("membound", b, 1, 16, [L] * b, seed=seed)
    if cfg == 3:
        b = batch or 64
        hi = seqlen or 8192
        n_force = min(4, b // 2)
        L = _varlen_lengths(seed, b, 1, hi, n_force, n_force)
        return make_workload("varlen", b, 1, 128, L, seed=seed)
    if cfg == 4:
        b = batch or 132
        L = seqlen or 16384
        return make_workload("mtp_causal", b, 2, 128, [L] * b, causal=True, seed=seed)
    if cfg == 5:
        b = batch or 64
        L = seqlen or 32768
        topk = min(2048, L)
        return make_workload("fp8_sparse", b, 1, 128, [L] * b, fp8=True, topk=topk, seed=seed,
                             pad_rows_per_token=64, num_padded_rows=min(4, b))
    raise ValueError(f"unknown config {cfg}")


def with_queries(w: Workload, name: str, s_q: int, h_q: int, *, causal: bool, seed: int) -> Workload:
    """The same cache, block table and lengths as ``w`` (dense path) with new
    seeded N(0,1) bf16 queries of another shape: the multi-token and head-count
    variants of a configuration without drawing its cache again."""
    assert w.indices is None
    q_bits = _normal_bf16(_rngs(seed, 1)[0], (w.batch, s_q, h_q, D_QK))
    return dataclasses.replace(w, name=name, s_q=s_q, h_q=h_q, causal=causal, seed=seed, q_bits=q_bits)


def flops_and_bytes(w: Workload):
    """Algorithmic work of one decode call: 2*(576+512) FLOPs per unmasked
    (query row, key) pair, and 1152 B per visible bf16 cache row or 656 B per
    fp8 row (each row counted once per sequence on the dense paths, or once
    per valid index of a query token on the sparse path)."""
    pairs = 0
    if w.indices is not None:
        pairs = int((w.indices >= 0).sum()) * w.h_q
        kv_bytes = int((w.indices >= 0).sum()) * FP8_ROW_BYTES
    else:
        for L in w.cache_seqlens.tolist():
            for i in range(w.s_q):
                vis = L if not w.causal else max(0, min(L, L - w.s_q + i + 1))
                pairs += vis * w.h_q
        kv_bytes = int(w.cache_seqlens.astype(np.int64).sum()) * (FP8_ROW_BYTES if w.fp8 else D_QK * 2)
    return 2 * (D_QK + D_V) * pairs, kv_bytes


def to_device(w: Workload, dev="cuda") -> dict:
    """Copy a workload's arrays to the device as the tensors the decode API
    takes: q / bf16 cache as bfloat16 views of the bits, the FP8 cache as
    uint8, tables and indices as int32."""
    t = {"q": torch.from_numpy(w.q_bits.view(np.int16)).view(torch.bfloat16).to(dev)}
    if w.fp8:
        t["kv"] = torch.from_numpy(w.kv_fp8).to(dev)
    else:
        t["kv"] = torch.from_numpy(w.kv_bits.view(np.int16)).view(torch.bfloat16).to(dev)
    t["bt"] = torch.from_numpy(w.block_table).to(dev)
    t["sl"] = torch.from_numpy(w.cache_seqlens).to(dev)
    t["idx"] = torch.from_numpy(w.indices).to(dev) if w.indices is not None else None
    return t
