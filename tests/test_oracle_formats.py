"""Pins of the oracle's number-format decoding (CPU only)."""
import math
import os

import numpy as np
import pytest
import torch

from oracle import formats

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_spec_points.txt")


def test_e4m3_spec_points():
    """Code points printed from the OCP FP8 format definition."""
    n = 0
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            code, val = line.split()
            got = formats.E4M3_TABLE[int(code, 16)]
            if val == "nan":
                assert math.isnan(got)
            else:
                assert got == float(val), (code, got, val)
                assert math.copysign(1.0, got) == math.copysign(1.0, float(val))
            n += 1
    assert n >= 10


def test_e4m3_table_matches_torch_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float32).numpy().astype(np.float64)
    ours = formats.E4M3_TABLE
    nan = np.isnan(ref)
    assert (np.isnan(ours) == nan).all()
    assert (ours[~nan] == ref[~nan]).all()
    assert nan.sum() == 2  # 0x7f, 0xff


def test_e4m3_largest_and_monotone():
    pos = formats.E4M3_TABLE[:0x7F]
    assert pos.max() == 448.0
    assert (np.diff(pos) > 0).all()


@pytest.mark.filterwarnings("ignore::RuntimeWarning")
def test_bf16_decode_matches_torch():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 16, size=4096, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy().astype(np.float64)
    got = formats.bf16_bits_to_f64(bits)
    nan = np.isnan(ref)
    assert (np.isnan(got) == nan).all()
    assert (got[~nan] == ref[~nan]).all()


def test_fp8_row_dequant_hand_example():
    """One row built by hand: group g holds code 0x38 (1.0) at dim 128g and
    code 0x40 (2.0) at dim 128g+1, scale = (g+1)/4; RoPE[r] = bf16(r)."""
    row = np.zeros(656, dtype=np.uint8)
    scales = np.array([0.25, 0.5, 0.75, 1.0], dtype="<f4")
    for g in range(4):
        row[128 * g] = 0x38
        row[128 * g + 1] = 0x40
    row[512:528] = scales.view(np.uint8)
    rope = torch.arange(64, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    row[528:] = rope.view(np.uint8)
    k = formats.fp8_rows_to_f64(row[None])[0]
    assert k.shape == (576,)
    for g in range(4):
        assert k[128 * g] == 0.25 * (g + 1)
        assert k[128 * g + 1] == 0.5 * (g + 1)
        assert (k[128 * g + 2:128 * g + 128] == 0).all()
    assert (k[512:] == np.arange(64)).all()
