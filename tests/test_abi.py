"""The C-ABI library loads and exports every declared symbol; host-only entry
points validate their arguments (CPU only: no kernel is launched)."""
import ctypes
import os
import re

import pytest

from mla_decode_attention_get_b200 import _abi
from mla_decode_attention_get_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return _abi.lib()


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:MLA_API\s+)?(?:const\s+)?\w+\s*\*?\s*(mla_\w+)\s*\(", text, flags=re.M)
    return names


def test_header_declares_the_abi():
    names = _declared_functions()
    assert set(_abi.EXPORTS) <= set(names), names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings(lib):
    assert _abi.status_string(0) == "MLA_OK"
    assert "workspace" in _abi.status_string(_abi.MLA_ERR_WORKSPACE)
    assert "UNKNOWN" in _abi.status_string(99)


def test_metadata_shape_host_only(lib):
    # forced partition counts need no device
    assert _abi.metadata_shape(128, 1, 16, 1, 0, 148) == (148, 129)
    assert _abi.metadata_shape(64, 1, 128, 1, 2048, 74) == (74, 65)
    assert _abi.metadata_shape(4, 2, 8, 1, 64, 3) == (3, 9)       # sparse: units = batch * s_q
    with pytest.raises(_abi.MlaError) as e:
        _abi.metadata_shape(4, 1, 16, 2, 0, 8)
    assert e.value.status == _abi.MLA_ERR_UNSUPPORTED
    with pytest.raises(_abi.MlaError) as e:
        _abi.metadata_shape(0, 1, 16, 1, 0, 8)
    assert e.value.status == _abi.MLA_ERR_INVALID_ARG


def test_workspace_bytes(lib):
    # (units + parts) splits x rows x (512 + 1) floats, lse block rounded to 256 B
    n = _abi.workspace_bytes(128, 1, 16, 0, 148)
    splits = 128 + 148
    assert n == splits * 16 * 512 * 4 + ((splits * 16 * 4 + 255) // 256) * 256
    n = _abi.workspace_bytes(64, 1, 128, 2048, 74)
    splits = 64 + 74
    assert n == splits * 128 * 512 * 4 + ((splits * 128 * 4 + 255) // 256) * 256
    base = (132 + 37) * 256 * 512 * 4 + (((132 + 37) * 256 * 4 + 255) // 256) * 256
    assert _abi.workspace_bytes(132, 2, 128, 0, 37) == base


def test_row_counts_beyond_the_combine_grid_are_unsupported(lib):
    # the combine kernel covers a unit's rows 4 to a CTA in grid y (<= 65535)
    assert _abi.metadata_shape(1, 1, 4 * 65535, 1, 0, 8) == (8, 2)
    with pytest.raises(_abi.MlaError) as e:
        _abi.metadata_shape(1, 1, 4 * 65535 + 1, 1, 0, 8)
    assert e.value.status == _abi.MLA_ERR_UNSUPPORTED
    with pytest.raises(_abi.MlaError) as e:
        _abi.workspace_bytes(1, 2, 4 * 65535, 0, 8)             # dense rows = s_q * h_q
    assert e.value.status == _abi.MLA_ERR_UNSUPPORTED
    assert _abi.workspace_bytes(1, 2, 4 * 65535, 64, 8) > 0     # sparse rows = h_q


def test_decode_rejects_bad_arguments_before_launch(lib):
    L = _abi.lib()
    assert L.mla_decode(None, None) == _abi.MLA_ERR_INVALID_ARG
    a = _abi.DecodeArgs()
    a.batch, a.s_q, a.h_q, a.h_kv, a.d_v = 2, 1, 16, 1, 512
    assert L.mla_decode(ctypes.byref(a), None) == _abi.MLA_ERR_INVALID_ARG   # null pointers
    a.h_kv = 2
    assert L.mla_decode(ctypes.byref(a), None) == _abi.MLA_ERR_UNSUPPORTED
    a.h_kv, a.d_v = 1, 256
    assert L.mla_decode(ctypes.byref(a), None) == _abi.MLA_ERR_UNSUPPORTED
    a.d_v, a.is_fp8 = 512, 0
    a.indices, a.topk = 1 << 20, 64                                         # sparse indices, bf16 cache
    assert L.mla_decode(ctypes.byref(a), None) == _abi.MLA_ERR_UNSUPPORTED
    a.indices, a.topk = None, 0
    assert L.mla_get_metadata(None, 2, 1, 16, 1, 0, 4, None, None, None) == _abi.MLA_ERR_INVALID_ARG
    assert L.mla_get_metadata(None, 2, 1, 16, 3, 0, 4, None, None, None) == _abi.MLA_ERR_UNSUPPORTED


def test_decode_checks_alignment_and_workspace(lib):
    """Every pointer is a fake non-null host address; validation must stop
    before any CUDA call."""
    L = _abi.lib()
    a = _abi.DecodeArgs()
    fake = 1 << 20
    for f in ("q", "k_cache", "block_table", "cache_seqlens", "tile_md", "num_splits", "out", "lse",
              "workspace", "err_word"):
        setattr(a, f, fake)
    a.batch, a.s_q, a.h_q, a.h_kv, a.d_v = 2, 1, 16, 1, 512
    a.q_batch_stride = 16 * 576
    a.k_block_stride = 64 * 576 * 2
    a.num_blocks, a.block_table_stride, a.block_table_width, a.num_parts = 3, 2, 2, 4
    a.softmax_scale = 576 ** -0.5
    a.workspace_bytes = 0
    assert L.mla_decode(ctypes.byref(a), None) == _abi.MLA_ERR_WORKSPACE
    a.workspace_bytes = 1 << 30
    a.q = fake + 8                                                          # not 16-B aligned
    assert L.mla_decode(ctypes.byref(a), None) == _abi.MLA_ERR_INVALID_ARG
    a.q = fake
    a.k_block_stride = 64 * 576 * 2 - 16                                    # page overlaps the next
    assert L.mla_decode(ctypes.byref(a), None) == _abi.MLA_ERR_INVALID_ARG
    a.k_block_stride = 64 * 576 * 2
    for bad in (0.0, -0.04, float("nan"), float("inf")):                    # softmax_scale finite, > 0
        a.softmax_scale = bad
        assert L.mla_decode(ctypes.byref(a), None) == _abi.MLA_ERR_INVALID_ARG
    a.softmax_scale = 576 ** -0.5
    a.k_block_stride = 64 * 576 * 2
    a.q_batch_stride = 16 * 576 - 8
    assert L.mla_decode(ctypes.byref(a), None) == _abi.MLA_ERR_INVALID_ARG


def test_fp8_cache_write_validates_before_launch(lib):
    L = _abi.lib()
    fake = 1 << 20
    ok = dict(k=fake, rs=576, n=4, slots=fake, cache=fake, bs=64 * 656, nb=8, err=fake)

    def call(**kw):
        a = {**ok, **kw}
        return L.mla_fp8_cache_write(a["k"], a["rs"], a["n"], a["slots"], a["cache"], a["bs"], a["nb"], a["err"], None)

    assert call(n=0) == _abi.MLA_OK                       # nothing to do: no launch
    assert call(n=-1) == _abi.MLA_ERR_INVALID_ARG
    assert call(k=0) == _abi.MLA_ERR_INVALID_ARG
    assert call(k=fake + 8) == _abi.MLA_ERR_INVALID_ARG   # not 16-B aligned
    assert call(rs=572) == _abi.MLA_ERR_INVALID_ARG       # rows overlap
    assert call(rs=580) == _abi.MLA_ERR_INVALID_ARG       # row starts not 16-B aligned
    assert call(bs=64 * 656 - 16) == _abi.MLA_ERR_INVALID_ARG
    assert call(nb=0) == _abi.MLA_ERR_INVALID_ARG
