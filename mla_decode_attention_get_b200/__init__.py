"""MLA decode attention over a paged KV cache, native to B200 (sm_100a).

Python face of the C-ABI library ``libmla_decode_b200.so`` (declared in
include/mla_decode.h).  The two user calls mirror the pages' API ("Was ist
FlashMLA?" (topnet.top), sections "2. MLA-Metadaten abrufen" and
"3. MLA-Decodierung ausführen")::

    tile_scheduler_metadata, num_splits = get_mla_metadata(
        cache_seqlens, s_q * h_q // h_kv, h_kv)
    for layer in range(num_layers):
        o, lse = flash_mla_with_kvcache(q[layer], kv_cache[layer], block_table,
                                        cache_seqlens, dv, tile_scheduler_metadata,
                                        num_splits, causal=True)

PyTorch only supplies device memory and the current stream; every step of
the computation runs in the library's CUDA kernels.  There is no CPU path.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Tuple

import torch

from . import _abi
from ._abi import MlaError, D_QK, D_V, PAGE_SIZE, FP8_ROW_BYTES

__all__ = ["get_mla_metadata", "flash_mla_with_kvcache", "MlaError", "mla_get_metadata", "mla_decode",
           "mla_decode_attention", "mla_decode_combine", "mla_decode_noalloc", "mla_metadata_shape",
           "mla_workspace_bytes", "DecodeCall", "fp8_cache_write"]


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream_ptr(device) -> int:
    """Handle of the current CUDA stream of ``device`` (a torch.device)."""
    if _raw_stream is not None:
        idx = device.index
        return _raw_stream(torch.cuda.current_device() if idx is None else idx)
    return torch.cuda.current_stream(device).cuda_stream


# Host-side plan sizes are pure functions of the shapes (and of the device's
# SM count): cache them, so that a decode step costs no extra library calls.
_shape_cache = {}
_ws_cache = {}
# Error word of calls made with check=False: nobody reads it, so all such
# calls on a device share one (the kernels only OR bits into it).
_discard_err = {}


def _require(cond: bool, msg: str) -> None:
    if not cond:
        raise ValueError(msg)


# ----------------------------------------------------------------- C-ABI names

def mla_metadata_shape(batch: int, s_q: int, h_q: int, h_kv: int = 1, topk: int = 0,
                       num_sm_parts: int = 0) -> Tuple[int, int]:
    """(num_parts, num_splits_len) of the split plan (host only)."""
    return _abi.metadata_shape(batch, s_q, h_q, h_kv, topk, num_sm_parts)


def mla_workspace_bytes(batch: int, s_q: int, h_q: int, topk: int, num_parts: int) -> int:
    return _abi.workspace_bytes(batch, s_q, h_q, topk, num_parts)


def _metadata_shape_of(batch, s_q, h_q, h_kv, topk, num_sm_parts, device) -> Tuple[int, int]:
    key = (batch, s_q, h_q, h_kv, topk, num_sm_parts, device.index)
    r = _shape_cache.get(key)
    if r is None:
        with torch.cuda.device(device):
            r = mla_metadata_shape(batch, s_q, h_q, h_kv, topk, num_sm_parts)
        _shape_cache[key] = r
    return r


def _workspace_bytes_of(batch, s_q, h_q, topk, num_parts) -> int:
    key = (batch, s_q, h_q, topk, num_parts)
    r = _ws_cache.get(key)
    if r is None:
        r = mla_workspace_bytes(batch, s_q, h_q, topk, num_parts)
        _ws_cache[key] = r
    return r


def _discard_err_word(device) -> torch.Tensor:
    e = _discard_err.get(device.index)
    if e is None:
        e = torch.zeros((1,), dtype=torch.int32, device=device)
        _discard_err[device.index] = e
    return e


def mla_get_metadata(cache_seqlens: torch.Tensor, batch: int, s_q: int, h_q: int, h_kv: int, topk: int,
                     tile_md: torch.Tensor, num_splits: torch.Tensor) -> None:
    """Fill ``tile_md`` [num_parts, 8] and ``num_splits`` [units + 1] (int32, device)."""
    _abi.check(_abi.lib().mla_get_metadata(
        cache_seqlens.data_ptr(), batch, s_q, h_q, h_kv, topk, tile_md.shape[0],
        tile_md.data_ptr(), num_splits.data_ptr(), ctypes.c_void_p(_stream_ptr(cache_seqlens.device))),
        "mla_get_metadata")


class DecodeCall:
    """Marshalled arguments of one decode call (reusable across launches on
    the same tensors, e.g. inside a timing loop or a CUDA graph capture)."""

    def __init__(self, q, k_cache, block_table, cache_seqlens, tile_md, num_splits, out, lse, workspace,
                 err, softmax_scale: float, causal: bool, is_fp8: bool, indices=None, h_kv: int = 1):
        b, s_q, h_q, d = q.shape
        a = _abi.DecodeArgs()
        a.q = q.data_ptr()
        a.q_batch_stride = q.stride(0)
        a.k_cache = k_cache.data_ptr()
        a.k_block_stride = k_cache.stride(0) * k_cache.element_size()
        a.num_blocks = k_cache.shape[0]
        a.block_table = block_table.data_ptr()
        a.block_table_stride = block_table.stride(0)
        a.block_table_width = block_table.shape[1]
        a.cache_seqlens = cache_seqlens.data_ptr()
        a.indices = indices.data_ptr() if indices is not None else None
        a.topk = indices.shape[-1] if indices is not None else 0
        a.tile_md = tile_md.data_ptr()
        a.num_splits = num_splits.data_ptr()
        a.num_parts = tile_md.shape[0]
        a.out = out.data_ptr()
        a.lse = lse.data_ptr()
        a.workspace = workspace.data_ptr()
        a.workspace_bytes = workspace.numel() * workspace.element_size()
        a.err_word = err.data_ptr()
        a.batch, a.s_q, a.h_q, a.h_kv, a.d_v = b, s_q, h_q, h_kv, D_V
        a.softmax_scale = float(softmax_scale)
        a.causal = 1 if causal else 0
        a.is_fp8 = 1 if is_fp8 else 0
        self.args = a
        self.device = q.device
        # keep the tensors alive as long as the marshalled pointers
        self._keep = (q, k_cache, block_table, cache_seqlens, tile_md, num_splits, out, lse, workspace, err,
                      indices)

    def _call(self, fn, name, stream=None):
        s = _stream_ptr(self.device) if stream is None else stream
        _abi.check(fn(ctypes.byref(self.args), ctypes.c_void_p(s)), name)

    def decode(self, stream=None):
        self._call(_abi.lib().mla_decode, "mla_decode", stream)

    def decode_noalloc(self, stream=None):
        """The same decode through mla_decode_noalloc: the library's built-in
        scratch array replaces this call's workspace tensor."""
        self._call(_abi.lib().mla_decode_noalloc, "mla_decode_noalloc", stream)

    def attention(self, stream=None):
        self._call(_abi.lib().mla_decode_attention, "mla_decode_attention", stream)

    def combine(self, stream=None):
        self._call(_abi.lib().mla_decode_combine, "mla_decode_combine", stream)


def mla_decode(call: DecodeCall) -> None:
    call.decode()


def mla_decode_noalloc(call: DecodeCall) -> None:
    call.decode_noalloc()


def mla_decode_attention(call: DecodeCall) -> None:
    call.attention()


def mla_decode_combine(call: DecodeCall) -> None:
    call.combine()


# ----------------------------------------------------------------- user API

def get_mla_metadata(cache_seqlens: torch.Tensor, num_q_tokens_per_head_k: int, num_heads_k: int, *,
                     s_q: int = 1, topk: Optional[int] = None,
                     num_sm_parts: Optional[int] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Split plan for one decode step, reused by every layer.

    ``num_q_tokens_per_head_k`` is ``s_q * h_q // h_kv`` as in the pages' call.
    The sparse path (``topk`` = indices per query token) plans per (sequence,
    token) unit and needs ``s_q``.  Returns (tile_scheduler_metadata int32
    [num_parts, 8], num_splits int32 [units + 1]) on the device of
    ``cache_seqlens``."""
    _require(cache_seqlens.is_cuda and cache_seqlens.dtype == torch.int32 and cache_seqlens.dim() == 1,
             "cache_seqlens must be a 1-D int32 CUDA tensor")
    if cache_seqlens.stride(0) != 1:
        cache_seqlens = cache_seqlens.contiguous()
    batch = cache_seqlens.shape[0]
    rows = num_q_tokens_per_head_k * num_heads_k
    _require(rows % s_q == 0, "s_q must divide s_q*h_q")
    h_q = rows // s_q
    tk = int(topk or 0)
    dev = cache_seqlens.device
    parts, nlen = _metadata_shape_of(batch, s_q, h_q, num_heads_k, tk, int(num_sm_parts or 0), dev)
    # one allocation: tile_md [parts, 8] then num_splits [nlen]
    buf = torch.empty((parts * _abi.MD_WORDS + nlen,), dtype=torch.int32, device=dev)
    tile_md = buf[:parts * _abi.MD_WORDS].view(parts, _abi.MD_WORDS)
    num_splits = buf[parts * _abi.MD_WORDS:]
    _abi.check(_abi.lib().mla_get_metadata(
        cache_seqlens.data_ptr(), batch, s_q, h_q, num_heads_k, tk, parts, tile_md.data_ptr(),
        num_splits.data_ptr(), _stream_ptr(dev)), "mla_get_metadata")
    return tile_md, num_splits


def _check_decode_inputs(q, k_cache, block_table, cache_seqlens, head_dim_v, is_fp8_kvcache, indices):
    """Validate the decode inputs (host checks only); returns the cache as
    the library reads it (the FP8 cache viewed as bytes)."""
    _require(q.is_cuda and q.dtype == torch.bfloat16 and q.dim() == 4 and q.shape[-1] == D_QK,
             "q must be bf16 [batch, s_q, h_q, 576] on CUDA")
    b, s_q, h_q, _ = q.shape
    qs = q.stride()
    _require(qs[3] == 1 and (h_q == 1 or qs[2] == D_QK) and (s_q == 1 or qs[1] == h_q * D_QK),
             "q must be contiguous within a batch entry")
    _require(head_dim_v == D_V, "head_dim_v must be 512")
    _require(k_cache.dim() == 4 and k_cache.shape[1] == PAGE_SIZE, "k_cache must be [blocks, 64, h_kv, d]")
    if is_fp8_kvcache:
        if k_cache.dtype != torch.uint8:
            k_cache = k_cache.view(torch.uint8)
        _require(k_cache.shape[-1] == FP8_ROW_BYTES, "fp8 cache rows must be 656 bytes")
    else:
        _require(k_cache.dtype == torch.bfloat16 and k_cache.shape[-1] == D_QK, "bf16 cache rows must be 576 wide")
    ks = k_cache.stride()
    d = k_cache.shape[3]
    _require(ks[3] == 1 and (k_cache.shape[2] == 1 or ks[2] == d) and ks[1] == k_cache.shape[2] * d,
             "each cache page must be contiguous")
    _require(block_table.dtype == torch.int32 and block_table.dim() == 2 and block_table.stride(1) == 1,
             "block_table must be int32 [batch, max_blocks] with unit column stride")
    _require(cache_seqlens.dtype == torch.int32 and cache_seqlens.dim() == 1 and cache_seqlens.stride(0) == 1,
             "cache_seqlens must be contiguous int32")
    if indices is not None:
        _require(is_fp8_kvcache, "sparse indices are read with the fp8 cache only")
        _require(indices.dtype == torch.int32 and indices.dim() == 3 and indices.shape[:2] == (b, s_q)
                 and indices.is_contiguous(), "indices must be contiguous int32 [batch, s_q, topk]")
    return k_cache


def prepare_decode(q: torch.Tensor, k_cache: torch.Tensor, block_table: torch.Tensor,
                   cache_seqlens: torch.Tensor, head_dim_v: int, tile_scheduler_metadata: torch.Tensor,
                   num_splits: torch.Tensor, softmax_scale: Optional[float] = None, causal: bool = False,
                   is_fp8_kvcache: bool = False, indices: Optional[torch.Tensor] = None) -> DecodeCall:
    """Validate shapes, allocate out / lse / workspace / error word, and
    marshal one decode call."""
    k_cache = _check_decode_inputs(q, k_cache, block_table, cache_seqlens, head_dim_v, is_fp8_kvcache, indices)
    b, s_q, h_q, _ = q.shape
    topk = indices.shape[-1] if indices is not None else 0
    if softmax_scale is None:
        softmax_scale = D_QK ** -0.5
    dev = q.device
    out = torch.empty((b, s_q, h_q, D_V), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((b, h_q, s_q), dtype=torch.float32, device=dev)
    ws = torch.empty((_workspace_bytes_of(b, s_q, h_q, topk, tile_scheduler_metadata.shape[0]),),
                     dtype=torch.uint8, device=dev)
    err = torch.zeros((1,), dtype=torch.int32, device=dev)
    return DecodeCall(q, k_cache, block_table, cache_seqlens, tile_scheduler_metadata, num_splits, out, lse,
                      ws, err, softmax_scale, causal, is_fp8_kvcache, indices, k_cache.shape[2])


def flash_mla_with_kvcache(q: torch.Tensor, k_cache: torch.Tensor, block_table: torch.Tensor,
                           cache_seqlens: torch.Tensor, head_dim_v: int, tile_scheduler_metadata: torch.Tensor,
                           num_splits: torch.Tensor, softmax_scale: Optional[float] = None, causal: bool = False,
                           is_fp8_kvcache: bool = False, indices: Optional[torch.Tensor] = None, *,
                           check: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """MLA decode: returns (out bf16 [batch, s_q, h_q, 512], lse fp32
    [batch, h_q, s_q]).  With ``check=True`` the call synchronises and raises
    if a kernel reported a data error (bad block_table entry or index);
    without it the error bits go to a word nobody reads."""
    k_cache = _check_decode_inputs(q, k_cache, block_table, cache_seqlens, head_dim_v, is_fp8_kvcache, indices)
    b, s_q, h_q, _ = q.shape
    topk = indices.shape[-1] if indices is not None else 0
    if softmax_scale is None:
        softmax_scale = D_QK ** -0.5
    dev = q.device
    num_parts = tile_scheduler_metadata.shape[0]
    out = torch.empty((b, s_q, h_q, D_V), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((b, h_q, s_q), dtype=torch.float32, device=dev)
    ws_bytes = _workspace_bytes_of(b, s_q, h_q, topk, num_parts)
    ws = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    err = torch.zeros((1,), dtype=torch.int32, device=dev) if check else _discard_err_word(dev)
    a = _abi.DecodeArgs(q.data_ptr(), q.stride(0), k_cache.data_ptr(), k_cache.stride(0) * k_cache.element_size(),
                        k_cache.shape[0], block_table.data_ptr(), block_table.stride(0), block_table.shape[1],
                        cache_seqlens.data_ptr(), indices.data_ptr() if indices is not None else None, topk,
                        tile_scheduler_metadata.data_ptr(), num_splits.data_ptr(), num_parts, out.data_ptr(),
                        lse.data_ptr(), ws.data_ptr(), ws_bytes, err.data_ptr(), b, s_q, h_q, k_cache.shape[2],
                        D_V, float(softmax_scale), 1 if causal else 0, 1 if is_fp8_kvcache else 0)
    _abi.check(_abi.lib().mla_decode(ctypes.byref(a), _stream_ptr(dev)), "mla_decode")
    if check:
        e = int(err.item())
        if e:
            raise MlaError(_abi.MLA_ERR_INVALID_ARG, f"device error word 0x{e:x}")
    return out, lse


def fp8_cache_write(k_new: torch.Tensor, slot_mapping: torch.Tensor, kv_cache: torch.Tensor,
                    err: Optional[torch.Tensor] = None, check: bool = False) -> torch.Tensor:
    """Quantise new key rows into the FP8 cache (C ABI ``mla_fp8_cache_write``).

    ``k_new`` bf16 [n, 576] on CUDA (rows contiguous); ``slot_mapping`` int32
    [n] (page * 64 + row; -1 skips a row); ``kv_cache`` uint8
    [num_blocks, 64, 1, 656], written in place.  Returns the int32 error word
    (``err`` if given); with ``check=True`` it synchronises and raises if a
    slot was out of range."""
    _require(k_new.is_cuda and k_new.dtype == torch.bfloat16 and k_new.dim() == 2 and k_new.shape[1] == D_QK
             and k_new.stride(1) == 1, "k_new must be bf16 [n, 576] with contiguous rows")
    _require(slot_mapping.dtype == torch.int32 and slot_mapping.is_contiguous()
             and slot_mapping.shape == (k_new.shape[0],), "slot_mapping must be contiguous int32 [n]")
    if kv_cache.dtype != torch.uint8:
        kv_cache = kv_cache.view(torch.uint8)
    _require(kv_cache.dim() == 4 and kv_cache.shape[1] == PAGE_SIZE and kv_cache.shape[2] == 1
             and kv_cache.shape[3] == FP8_ROW_BYTES and kv_cache[0].is_contiguous(),
             "kv_cache must be uint8 [num_blocks, 64, 1, 656] with contiguous pages")
    if err is None:
        err = torch.zeros((1,), dtype=torch.int32, device=k_new.device)
    st = _abi.lib().mla_fp8_cache_write(k_new.data_ptr(), k_new.stride(0), k_new.shape[0], slot_mapping.data_ptr(),
                                        kv_cache.data_ptr(), kv_cache.stride(0), kv_cache.shape[0], err.data_ptr(),
                                        torch.cuda.current_stream(k_new.device).cuda_stream)
    _abi.check(st, "mla_fp8_cache_write")
    if check:
        torch.cuda.synchronize(k_new.device)
        if int(err.item()) != 0:
            raise RuntimeError(f"fp8_cache_write: device error word {int(err.item())}")
    return err
