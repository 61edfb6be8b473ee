"""Dense decode over the FP8 cache (no indices: the block table is walked page
by page, as for the bf16 cache), against the fp64 oracle through the C ABI.

The FP8 row format is the walkthrough's (512 e4m3 + 4 fp32 scales + 64 bf16
RoPE, FlashMLA walkthrough, section "二、核心功能与架构"); the oracle
dequantises it exactly.  Cases: row tilings and causal s_q > 1, lengths
around page edges, NaN codes in the padding past a sequence's length, a bad
block-table entry, empty sequences, partition counts, and a larger sampled
batch."""
import numpy as np
import pytest

from mla_decode_attention_get_b200 import inputs as I
from gpu_util import assert_close, oracle, run
import rescale_cases as RC

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("h_q,s_q", [(16, 1), (64, 1), (128, 1), (16, 2), (128, 2), (40, 3)])
def test_row_tilings(h_q, s_q):
    w = I.make_workload("fp8d", 3, s_q, h_q, [700, 129, 1], fp8=True, causal=s_q > 1, seed=h_q + s_q)
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


@pytest.mark.parametrize("L", [1, 63, 64, 65, 191, 2049])
def test_lengths_around_page_edges(L):
    w = I.make_workload("fp8dedge", 2, 1, 16, [L, 64 * 3 + 5], fp8=True, seed=L)
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


def test_nan_codes_past_length_are_ignored():
    w = I.make_workload("fp8dnan", 2, 1, 16, [100, 37], fp8=True, seed=41)
    for b, L in enumerate(w.cache_seqlens):
        last = w.block_table[b, (L - 1) // 64]
        w.kv_fp8[last, L % 64:, 0, :512] = 0x7F            # e4m3 NaN codes in the padding rows
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


def test_causal_key_set_empty_for_first_token():
    w = I.make_workload("fp8dc1", 2, 2, 16, [1, 2], fp8=True, causal=True, seed=42)
    out, lse, err = run(w)
    assert err == 0
    ref_out, ref_lse = oracle(w)
    assert np.isneginf(ref_lse[0, :, 0]).all()
    assert_close(out, lse, ref_out, ref_lse)


def test_empty_sequences():
    w = I.make_workload("fp8dempty", 4, 1, 16, [0, 70, 0, 5], fp8=True, seed=43)
    out, lse, err = run(w)
    assert err == 0
    assert (out[0] == 0).all() and np.isneginf(lse[0]).all()
    assert_close(out, lse, *oracle(w))


def test_bad_block_table_entry_is_flagged_and_masked():
    w = I.make_workload("fp8dbad", 2, 1, 16, [100, 100], fp8=True, seed=44)
    w.block_table[0, 1] = w.num_blocks + 7                # keys 64..99 of sequence 0 become unreadable
    out, lse, err = run(w)
    assert err & 1
    w2 = I.make_workload("fp8dbad", 2, 1, 16, [100, 100], fp8=True, seed=44)
    w2.cache_seqlens = np.array([64, 100], np.int32)
    assert_close(out, lse, *oracle(w2))


@pytest.mark.parametrize("parts", [1, 7, 148])
def test_output_independent_of_partition_count(parts):
    w = I.make_workload("fp8dparts", 6, 1, 64, [3000, 1, 640, 2500, 77, 1300], fp8=True, seed=45)
    out, lse, err = run(w, num_sm_parts=parts)
    assert err == 0
    assert_close(out, lse, *oracle(w))


def test_running_max_rescales():
    # many rows' running max jumps far past the lazy-rescale threshold
    # mid-sequence (rows boosted with exact power-of-two scales)
    w = RC.fp8_dense_case()
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


def test_larger_batch_sampled():
    rng = np.random.default_rng(46)
    L = rng.integers(1, 6000, size=32)
    w = I.make_workload("fp8dbig", 32, 1, 128, L.tolist(), fp8=True, seed=46)
    out, lse, err = run(w)
    assert err == 0
    batches = sorted({int(np.argmin(L)), int(np.argmax(L)), 3, 11, 20})
    ref_out, ref_lse = oracle(w, batches=batches)
    assert_close(out, lse, ref_out, ref_lse, batches=batches)
    assert np.isfinite(out).all()
