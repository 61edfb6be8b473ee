"""Pins of the FP8 cache writer oracle (oracle/fp8_writer_ref.py): a
hand-worked row, e4m3 rounding against torch's float8_e4m3fn cast, the
round-trip error bound of the format, and slot handling."""
import os

import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import fp8_writer_ref as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fp8_writer_example.txt")


def _bf16_bits(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_hand_worked_row():
    entries = []
    for line in open(GOLDEN):
        if line.strip() and not line.startswith("#"):
            g, d, x, code = line.split()[:4]
            entries.append((int(g), int(d), float(x), int(code, 16)))
    row = np.zeros(576, np.float32)
    for g, d, x, _ in entries:
        row[128 * g + d] = x
    row[512:] = 1.0
    bits = _bf16_bits(row)
    assert np.array_equal(F.bf16_bits_to_f64(bits), row.astype(np.float64))   # all exact in bf16
    out = W.quantize_rows(bits[None, :])[0]
    for g, d, _, code in entries:
        assert out[128 * g + d] == code, (g, d, hex(out[128 * g + d]), hex(code))
    listed = {128 * g + d for g, d, _, _ in entries}
    others = [i for i in range(512) if i not in listed]
    assert (out[others] == 0).all()
    scales = out[512:528].view("<f4")
    assert scales[0] == np.float32(2.0) / np.float32(448.0)
    assert scales[1] == 0.0
    assert scales[2] == 1.0
    assert scales[3] == np.float32(1000.0) / np.float32(448.0)
    assert bytes(out[528:]) == b"\x80\x3f" * 64


def test_rounding_matches_torch_cast():
    rng = np.random.default_rng(0)
    mags = W._MAG_VALUES
    mids = (mags[:-1] + mags[1:]) / 2                      # every tie between neighbours
    x = np.concatenate([rng.uniform(-448, 448, 20000), rng.uniform(-0.02, 0.02, 5000), mids, -mids,
                        mags, -mags, [0.0, -0.0, 448.0, -448.0]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = W.e4m3_round(x)
    assert np.array_equal(got, ref)


def test_round_trip_error_bound():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((64, 576)) * rng.uniform(0.01, 100, (64, 1))).astype(np.float32)
    x[3, 128:256] = 0                                       # an all-zero group
    bits = _bf16_bits(x)
    xv = F.bf16_bits_to_f64(bits)
    rows = W.quantize_rows(bits)
    back = F.fp8_rows_to_f64(rows)
    scales = rows[:, 512:528].view("<f4").astype(np.float64)
    s = np.repeat(scales, 128, axis=1)
    err = np.abs(back[:, :512] - xv[:, :512])
    # half an e4m3 ulp: 2^-4 relative for normals, 2^-10 * scale for subnormals
    bound = np.maximum(np.abs(xv[:, :512]) * 2.0 ** -4, s * 2.0 ** -10) * 1.001 + 1e-30
    assert (err <= bound).all()
    assert np.array_equal(back[:, 512:], xv[:, 512:])      # RoPE exact
    assert (rows[3, 128:256] == 0).all() and scales[3, 1] == 0


def test_group_max_maps_to_448():
    rng = np.random.default_rng(2)
    bits = _bf16_bits(rng.standard_normal((16, 576)).astype(np.float32))
    rows = W.quantize_rows(bits)
    xv = F.bf16_bits_to_f64(bits)
    for r in range(16):
        for g in range(4):
            d = 128 * g + int(np.argmax(np.abs(xv[r, 128 * g:128 * (g + 1)])))
            assert rows[r, d] & 0x7F == 0x7E


def test_write_cache_slots():
    rng = np.random.default_rng(3)
    cache = rng.integers(0, 256, size=(4, 64, 1, 656), dtype=np.uint8)
    bits = _bf16_bits(rng.standard_normal((4, 576)).astype(np.float32))
    new, bad = W.write_cache(cache, bits, np.array([5, -1, 64 * 3 + 63, 64 * 4], np.int32))
    assert bad                                              # slot 256 is past the cache
    rows = W.quantize_rows(bits)
    assert np.array_equal(new[0, 5, 0], rows[0])
    assert np.array_equal(new[3, 63, 0], rows[2])
    mask = np.ones((4, 64), bool)
    mask[0, 5] = mask[3, 63] = False
    assert np.array_equal(new[:, :, 0][mask], cache[:, :, 0][mask])   # nothing else touched
