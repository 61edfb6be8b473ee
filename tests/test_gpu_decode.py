"""Decode parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances: max|out - ref| <= 1e-2 * max|ref| over the compared rows, lse
within 1e-3 absolute, rows with an empty key set exactly (0, -inf)."""
import numpy as np
import pytest
import torch

from mla_decode_attention_get_b200 import inputs as I
from gpu_util import assert_close, oracle, run, upload
import rescale_cases as RC

pytestmark = pytest.mark.gpu


def test_tiny_config():
    w = I.make_config(1)
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 127, 128, 129, 1000])
def test_lengths_around_page_edges(L):
    w = I.make_workload("edge", 3, 1, 16, [L, max(1, L // 3), 64 * 3 + 1], seed=L)
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


@pytest.mark.parametrize("h_q,s_q", [(16, 1), (32, 1), (64, 1), (128, 1), (8, 2), (16, 2), (40, 1), (128, 2)])
def test_row_tilings(h_q, s_q):
    w = I.make_workload("rows", 3, s_q, h_q, [300, 77, 1], causal=s_q > 1, seed=h_q * 10 + s_q)
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


@pytest.mark.parametrize("h_q,s_q", [(128, 3), (128, 4), (64, 3), (64, 4)])
def test_mtp_decode_more_tokens(h_q, s_q):
    # s_q in {3, 4} new tokens (causal, bottom-right aligned) and 64-head tiles
    w = I.make_workload("mtp", 3, s_q, h_q, [1000, 130, 2], causal=True, seed=7 * h_q + s_q)
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


def test_membound_small():
    w = I.make_config(2, batch=8, seqlen=1000)
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


def test_varlen_small():
    w = I.make_config(3, batch=24, seqlen=1500)
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


def test_mtp_causal_small():
    w = I.make_config(4, batch=4, seqlen=777)
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


def test_fp8_sparse_small():
    w = I.make_config(5, batch=4, seqlen=5000)
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


@pytest.mark.parametrize("h_q,s_q,causal", [(16, 1, False), (128, 1, False), (64, 2, True)])
def test_running_max_rescales(h_q, s_q, causal):
    # many rows' running max jumps far past the lazy-rescale threshold
    # mid-sequence, while PV of the preceding pages may still be in flight
    w = RC.bf16_case(h_q, s_q, causal)
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


def test_running_max_rescales_fp8_sparse():
    w = RC.fp8_sparse_case()
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


@pytest.mark.parametrize("parts", [1, 2, 7, 148, 592])
def test_output_independent_of_partition_count(parts):
    w = I.make_config(3, batch=12, seqlen=3000)
    out, lse, err = run(w, num_sm_parts=parts)
    assert err == 0
    assert_close(out, lse, *oracle(w))


def test_sparse_prefill_shape():
    # prefill-shaped sparse call: many query tokens, each with its own top-k
    # (one scheduler unit per token)
    w = I.make_workload("sprefill", 1, 96, 64, [5000], fp8=True, topk=512, seed=51,
                        pad_rows_per_token=32, num_padded_rows=10)
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


@pytest.mark.parametrize("topk", [64, 100])
@pytest.mark.parametrize("h_q", [16, 64, 128])
def test_sparse_head_counts_and_topk(h_q, topk):
    # one or two 64-row tiles per token, a whole or a partial last key tile,
    # and a token whose list repeats an index (each copy counts as a key)
    w = I.make_workload(f"sphk{h_q}_{topk}", 2, 2, h_q, [3000, 130], fp8=True, topk=topk, seed=60 + h_q + topk,
                        pad_rows_per_token=7, num_padded_rows=1)
    w.indices[1, 0, 3] = w.indices[1, 0, 2]
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


@pytest.mark.parametrize("parts", [1, 3, 148])
def test_sparse_output_independent_of_partition_count(parts):
    w = I.make_workload("sp", 3, 2, 32, [4000, 700, 90], fp8=True, topk=300, seed=5,
                        pad_rows_per_token=40, num_padded_rows=2)
    out, lse, err = run(w, num_sm_parts=parts)
    assert err == 0
    assert_close(out, lse, *oracle(w))


def test_nan_padding_past_length_is_ignored():
    w = I.make_workload("nanpad", 2, 1, 16, [100, 37], seed=21)
    nan = I.f32_to_bf16_bits(np.array([np.nan], np.float32))[0]
    for b, L in enumerate(w.cache_seqlens):
        last = w.block_table[b, (L - 1) // 64]
        w.kv_bits[last, L % 64:, 0, :] = nan
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))


def test_empty_sequences():
    w = I.make_workload("empty", 4, 1, 16, [0, 70, 0, 5], seed=22)
    out, lse, err = run(w)
    assert err == 0
    ref_out, ref_lse = oracle(w)
    assert (out[0] == 0).all() and np.isneginf(lse[0]).all()
    assert_close(out, lse, ref_out, ref_lse)


def test_causal_key_set_empty_for_first_token():
    # L = 1 with s_q = 2: token 0 sees no key
    w = I.make_workload("c1", 2, 2, 16, [1, 2], causal=True, seed=23)
    out, lse, err = run(w)
    assert err == 0
    ref_out, ref_lse = oracle(w)
    assert np.isneginf(ref_lse[0, :, 0]).all()
    assert_close(out, lse, ref_out, ref_lse)


def test_bad_block_table_entry_is_flagged_and_masked():
    w = I.make_workload("badbt", 2, 1, 16, [100, 100], seed=24)
    w.block_table[0, 1] = w.num_blocks + 7          # keys 64..99 of sequence 0 become unreadable
    out, lse, err = run(w)
    assert err & 1
    w2 = I.make_workload("badbt", 2, 1, 16, [100, 100], seed=24)
    w2.cache_seqlens = np.array([64, 100], np.int32)
    ref_out, ref_lse = oracle(w2)
    assert_close(out, lse, ref_out, ref_lse)


def test_bad_sparse_index_is_flagged_and_skipped():
    w = I.make_workload("badidx", 2, 1, 16, [300, 300], fp8=True, topk=128, seed=25)
    w.indices[0, 0, 5] = 300          # == L: invalid
    w.indices[1, 0, 7] = -5           # negative, not -1: invalid
    out, lse, err = run(w)
    assert err & 2
    assert_close(out, lse, *oracle(w))   # the oracle skips out-of-range indices too


def test_deterministic():
    w = I.make_config(3, batch=8, seqlen=2000)
    t = upload(w)
    a = run(w, t)
    b = run(w, t)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


# --------------------------------------------------------------- full sizes

def _sample(batch, k, seed):
    rng = np.random.default_rng(seed)
    return sorted(rng.choice(batch, size=min(k, batch), replace=False).tolist())


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_full_size_config_sampled(cfg):
    """The bench's launch configuration at full size; the oracle checks a
    seeded sample of sequences (plus every sequence of extreme length)."""
    w = I.make_config(cfg)
    out, lse, err = run(w)
    assert err == 0
    batches = _sample(w.batch, 4 if cfg in (4, 5) else 6, cfg)
    if cfg == 3:
        L = w.cache_seqlens
        batches = sorted(set(batches) | {int(np.argmin(L)), int(np.argmax(L))})
    ref_out, ref_lse = oracle(w, batches=batches)
    assert_close(out, lse, ref_out, ref_lse, batches=batches)
    assert np.isfinite(out).all()
