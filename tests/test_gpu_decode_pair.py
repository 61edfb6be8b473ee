"""Parity of the two-CTA decode kernel (dense units of more than 64 query
rows, 128-row tiles; selected by MLA_TWO_CTA_DECODE=1) against the fp64
oracle, through the C ABI.

The cases aim at what is particular to that kernel: row counts that leave
part of a 128-row tile empty or need a second tile, causal tiles holding two
query tokens, the hand-off of P / alpha / 1/l through the ring (many pages
per segment, several segments per partition, splits), the O rescale the
value CTA applies when a later page raises a row's running max, and the
zeroed padding rows of a partial page."""
import numpy as np
import pytest

import mla_decode_attention_get_b200 as M
from mla_decode_attention_get_b200 import inputs as I
from gpu_util import assert_close, oracle, run

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def two_cta(monkeypatch):
    monkeypatch.setenv("MLA_TWO_CTA_DECODE", "1")


def test_pair_kernel_is_selected(monkeypatch):
    # >64 dense rows per unit: partitions are counted in CTA pairs
    parts_pair, _ = M.mla_metadata_shape(4, 1, 128, 1, 0)
    parts_single, _ = M.mla_metadata_shape(4, 1, 64, 1, 0)
    assert parts_pair <= parts_single // 2
    monkeypatch.delenv("MLA_TWO_CTA_DECODE")
    assert M.mla_metadata_shape(4, 1, 128, 1, 0)[0] == parts_single // 2   # default: 64-row tiles


@pytest.mark.parametrize("h_q,s_q", [(72, 1), (96, 1), (128, 1), (64, 2), (80, 2), (128, 2), (128, 3), (256, 1)])
def test_row_counts(h_q, s_q):
    w = I.make_workload("pairrows", 3, s_q, h_q, [700, 129, 1], causal=s_q > 1, seed=h_q + 7 * s_q)
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 128, 191, 4097])
def test_lengths_around_page_edges(L):
    w = I.make_workload("pairedge", 2, 1, 128, [L, 64 * 5 + 3], seed=L + 3)
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


def test_causal_two_tokens_per_tile():
    # s_q = 2, h_q = 64: rows 0-63 are token 0, rows 64-127 token 1 of one tile
    w = I.make_workload("paircausal", 4, 2, 64, [1, 2, 65, 1000], causal=True, seed=31)
    out, lse, err = run(w)
    assert err == 0
    ref_out, ref_lse = oracle(w)
    assert np.isneginf(ref_lse[0, :, 0]).all()
    assert_close(out, lse, ref_out, ref_lse)


def test_running_max_rescales():
    # scale a few cache rows on later pages so that many rows' running max
    # jumps by far more than the lazy-rescale threshold mid-sequence
    w = I.make_workload("pairrescale", 2, 1, 128, [3000, 2000], seed=32)
    for b, L in enumerate(w.cache_seqlens):
        for tok in (700 + b, 1500, L - 3):
            phys = w.block_table[b, tok // 64]
            bits = w.kv_bits[phys, tok % 64, 0, :].astype(np.uint32) << 16
            row = bits.view(np.float32) * 12.0
            w.kv_bits[phys, tok % 64, 0, :] = I.f32_to_bf16_bits(row)
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


@pytest.mark.parametrize("parts", [1, 2, 5, 74, 300])
def test_output_independent_of_partition_count(parts):
    w = I.make_config(3, batch=10, seqlen=2500)
    out, lse, err = run(w, num_sm_parts=parts)
    assert err == 0
    assert_close(out, lse, *oracle(w))


def test_nan_padding_past_length_is_ignored():
    w = I.make_workload("pairnan", 2, 1, 128, [100, 37], seed=33)
    nan = I.f32_to_bf16_bits(np.array([np.nan], np.float32))[0]
    for b, L in enumerate(w.cache_seqlens):
        last = w.block_table[b, (L - 1) // 64]
        w.kv_bits[last, L % 64:, 0, :] = nan
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


def test_empty_sequences():
    w = I.make_workload("pairempty", 5, 1, 128, [0, 70, 0, 5, 0], seed=34)
    out, lse, err = run(w)
    assert err == 0
    ref_out, ref_lse = oracle(w)
    assert (out[0] == 0).all() and np.isneginf(lse[0]).all()
    assert (out[4] == 0).all() and np.isneginf(lse[4]).all()
    assert_close(out, lse, ref_out, ref_lse)


def test_bad_block_table_entry_is_flagged_and_masked():
    w = I.make_workload("pairbadbt", 2, 1, 128, [200, 100], seed=35)
    w.block_table[0, 1] = w.num_blocks + 7          # keys 64..127 of sequence 0 become unreadable
    out, lse, err = run(w)
    assert err & 1
    # the same as a sequence whose keys 64..127 carry no weight: drop them
    ref = I.make_workload("pairbadbt", 2, 1, 128, [200, 100], seed=35)
    keep = np.r_[0:64, 128:200]
    q = ref.q_bits
    kv = np.zeros((ref.num_blocks + 4, 64, 1, 576), np.uint16)
    kv[: ref.num_blocks] = ref.kv_bits
    rows = [ref.kv_bits[ref.block_table[0, t // 64], t % 64, 0] for t in keep]
    extra = ref.num_blocks
    for i, r in enumerate(rows):
        kv[extra + i // 64, i % 64, 0] = r
    bt = ref.block_table.copy()
    bt[0, :3] = [extra, extra + 1, extra + 2]
    bt[0, 3:] = -1
    from oracle import mla_oracle as O
    ref_out, ref_lse = O.decode(q, bt, np.array([len(keep), 100], np.int32), kv_bits=kv,
                                softmax_scale=ref.softmax_scale)
    assert_close(out, lse, ref_out, ref_lse)


def test_deterministic():
    w = I.make_config(4, batch=3, seqlen=900)
    from gpu_util import upload
    t = upload(w)
    a = run(w, t)
    b = run(w, t)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
