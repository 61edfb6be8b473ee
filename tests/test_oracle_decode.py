"""Pins of the fp64 decode oracle against brute force, closed forms and
invariants of the definition (CPU only)."""
import math

import numpy as np
import pytest

from mla_decode_attention_get_b200 import inputs as I
from oracle import brute, mla_oracle as O
from oracle.formats import bf16_bits_to_f64, fp8_rows_to_f64

SCALE = 576 ** -0.5


def _bits(x):
    return I.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _dense(w, **kw):
    return O.decode(w.q_bits, w.block_table, w.cache_seqlens, kv_bits=w.kv_bits,
                    causal=w.causal, softmax_scale=w.softmax_scale, **kw)


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("causal,s_q,lens", [(False, 1, [100, 37]), (True, 2, [70, 3]),
                                             (False, 1, [64, 129])])
def test_oracle_matches_brute_force(causal, s_q, lens):
    h_q = 3
    w = I.make_workload("brute", len(lens), s_q, h_q, lens, causal=causal, seed=7 + s_q)
    out, lse = _dense(w)
    for b, L in enumerate(lens):
        for i in range(s_q):
            limit = L - s_q + i + 1 if causal else L
            bo, bl = brute.decode_token(w.q_bits[b, i].tolist(), w.kv_bits.tolist(),
                                        w.block_table.tolist(), b, L, limit, SCALE)
            np.testing.assert_allclose(out[b, i], np.array(bo), rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b, :, i], np.array(bl), rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal,s_q,lens", [(False, 1, [100, 37]), (True, 2, [70, 3])])
def test_oracle_matches_brute_force_fp8_dense(causal, s_q, lens):
    h_q = 2
    w = I.make_workload("brute8", len(lens), s_q, h_q, lens, causal=causal, fp8=True, seed=17 + s_q)
    out, lse = O.decode(w.q_bits, w.block_table, w.cache_seqlens, kv_fp8=w.kv_fp8, causal=causal)
    kv = w.kv_fp8.tolist()
    for b, L in enumerate(lens):
        for i in range(s_q):
            limit = L - s_q + i + 1 if causal else L
            bo, bl = brute.decode_token(w.q_bits[b, i].tolist(), None, w.block_table.tolist(), b, L, limit,
                                        SCALE, kv_fp8=kv)
            np.testing.assert_allclose(out[b, i], np.array(bo), rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b, :, i], np.array(bl), rtol=0, atol=1e-12)


def test_oracle_matches_brute_force_sparse():
    # padding, out-of-range positions and a duplicate in the index lists
    w = I.make_workload("brutes", 2, 2, 2, [150, 90], fp8=True, topk=40, seed=19)
    idx = w.indices.copy()
    idx[0, 0, -5:] = -1
    idx[0, 1, 3] = 150                   # == L: outside the sequence, skipped
    idx[1, 0, 7] = idx[1, 0, 8]          # listed twice
    idx[1, 1, :] = -1
    idx[1, 1, 0] = 89
    out, lse = O.decode(w.q_bits, w.block_table, w.cache_seqlens, kv_fp8=w.kv_fp8, indices=idx)
    kv = w.kv_fp8.tolist()
    for b, L in enumerate(w.cache_seqlens.tolist()):
        for i in range(2):
            bo, bl = brute.decode_token_sparse(w.q_bits[b, i].tolist(), kv, w.block_table.tolist(), b, L,
                                               idx[b, i].tolist(), SCALE)
            np.testing.assert_allclose(out[b, i], np.array(bo), rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b, :, i], np.array(bl), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- closed forms

def test_single_key_gives_its_value_row():
    w = I.make_workload("one", 1, 1, 4, [1], seed=3)
    out, lse = _dense(w)
    k = bf16_bits_to_f64(w.kv_bits[w.block_table[0, 0], 0, 0])
    q = bf16_bits_to_f64(w.q_bits[0, 0])
    np.testing.assert_array_equal(out[0, 0], np.broadcast_to(k[:512], (4, 512)))
    for h in range(4):
        s0 = SCALE * math.fsum(q[h, d] * k[d] for d in range(576))
        assert abs(lse[0, h, 0] - s0) < 1e-12


def test_rope_dims_enter_logits_but_not_values():
    """Queries nonzero only in the 64 RoPE dims: a single key's lse is the
    scaled RoPE dot product; its output is the key's first 512 dims."""
    w = I.make_workload("rope", 1, 1, 2, [1], seed=4)
    q = bf16_bits_to_f64(w.q_bits).copy()
    q[..., :512] = 0
    w.q_bits = _bits(q)
    out, lse = _dense(w)
    k = bf16_bits_to_f64(w.kv_bits[w.block_table[0, 0], 0, 0])
    for h in range(2):
        s0 = SCALE * float(np.dot(q[0, 0, h, 512:], k[512:]))
        assert abs(lse[0, h, 0] - s0) < 1e-12
    np.testing.assert_array_equal(out[0, 0, 0], k[:512])


def test_equal_logits_give_mean_of_values():
    """All keys share their RoPE part and queries are zero in NoPE dims, so
    every logit is equal: out = mean of V, lse = s + ln(n)."""
    L = 150
    w = I.make_workload("eq", 1, 1, 3, [L], seed=5)
    q = bf16_bits_to_f64(w.q_bits).copy()
    q[..., :512] = 0
    w.q_bits = _bits(q)
    kv = w.kv_bits.copy()
    kv[:, :, :, 512:] = kv[0, 0, 0, 512:]
    w.kv_bits = kv
    out, lse = _dense(w)
    keys = np.stack([bf16_bits_to_f64(kv[w.block_table[0, t // 64], t % 64, 0]) for t in range(L)])
    mean_v = keys[:, :512].mean(axis=0)
    for h in range(3):
        np.testing.assert_allclose(out[0, 0, h], mean_v, rtol=0, atol=1e-12)
        s = SCALE * float(np.dot(q[0, 0, h, 512:], keys[0, 512:]))
        assert abs(lse[0, h, 0] - (s + math.log(L))) < 1e-12


def test_one_hot_large_logit_selects_its_row():
    L, star = 90, 71
    w = I.make_workload("hot", 1, 1, 1, [L], seed=6)
    q = np.zeros((1, 1, 1, 576), dtype=np.float32)
    q[..., 512] = 1.0
    w.q_bits = _bits(q)
    kv = w.kv_bits.copy()
    kv[:, :, :, 512:] = 0
    page, slot = w.block_table[0, star // 64], star % 64
    kv[page, slot, 0, 512] = _bits(np.array([50.0 / SCALE], np.float32))[0]
    w.kv_bits = kv
    out, lse = _dense(w)
    v = bf16_bits_to_f64(kv[page, slot, 0, :512])
    s_star = SCALE * bf16_bits_to_f64(kv[page, slot, 0, 512])
    # every other logit is 0, so the others weigh about (L-1)*exp(-50)
    np.testing.assert_allclose(out[0, 0, 0], v, rtol=0, atol=1e-15)
    assert abs(lse[0, 0, 0] - (s_star + math.log1p((L - 1) * math.exp(-s_star)))) < 1e-12


def test_empty_sequence():
    w = I.make_workload("empty", 2, 1, 2, [0, 5], seed=8)
    out, lse = _dense(w)
    assert (out[0] == 0).all() and np.isneginf(lse[0]).all()
    assert np.isfinite(lse[1]).all()


# ---------------------------------------------------------------- invariants

def test_page_permutation_invariance_bit_exact():
    w = I.make_workload("perm", 2, 1, 4, [200, 77], seed=9)
    out, lse = _dense(w)
    rng = np.random.default_rng(1)
    perm = rng.permutation(w.kv_bits.shape[0])           # new position of old page
    kv2 = np.empty_like(w.kv_bits)
    kv2[perm] = w.kv_bits
    bt2 = np.where(w.block_table >= 0, perm[np.maximum(w.block_table, 0)], -1).astype(np.int32)
    out2, lse2 = O.decode(w.q_bits, bt2, w.cache_seqlens, kv_bits=kv2, softmax_scale=SCALE)
    np.testing.assert_array_equal(out, out2)
    np.testing.assert_array_equal(lse, lse2)


def test_padding_and_unused_block_table_entries_have_no_effect():
    w = I.make_workload("pad", 2, 1, 4, [100, 37], seed=10, min_blocks=6)
    out, lse = _dense(w)
    kv = w.kv_bits.copy()
    nan = _bits(np.float32(np.nan))
    for b, L in enumerate(w.cache_seqlens):
        last = w.block_table[b, (L - 1) // 64]
        kv[last, L % 64 or 64:, 0, :] = nan
    bt = np.concatenate([w.block_table, np.full((2, 3), 2 ** 31 - 1, np.int32)], axis=1)
    bt[bt == -1] = 12345
    out2, lse2 = O.decode(w.q_bits, bt, w.cache_seqlens, kv_bits=kv, softmax_scale=SCALE)
    np.testing.assert_array_equal(out, out2)
    np.testing.assert_array_equal(lse, lse2)


def test_causal_token_equals_shorter_noncausal_call():
    L, s_q = 130, 2
    w = I.make_workload("causal", 1, s_q, 4, [L], causal=True, seed=11)
    out, lse = _dense(w)
    for i in range(s_q):
        Li = L - s_q + 1 + i
        o1, l1 = O.decode(w.q_bits[:, i:i + 1], w.block_table, np.array([Li], np.int32),
                          kv_bits=w.kv_bits, softmax_scale=SCALE)
        np.testing.assert_allclose(out[0, i], o1[0, 0], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[0, :, i], l1[0, :, 0], rtol=0, atol=1e-13)


def test_merge_of_key_subranges_equals_whole():
    L = 333
    w = I.make_workload("split", 1, 1, 5, [L], seed=12)
    q = bf16_bits_to_f64(w.q_bits[0, 0])
    keys = O.gather_rows(w.block_table, 0, np.arange(L), kv_bits=w.kv_bits)
    whole_o, whole_l = O.attend(q, keys, SCALE)
    cuts = [0, 64, 65, 200, 333]
    parts = [O.attend(q, keys[a:b], SCALE) for a, b in zip(cuts[:-1], cuts[1:])]
    parts.append(O.attend(q, keys[:0], SCALE))          # an empty split weighs 0
    mo, ml = O.merge_splits([p[0] for p in parts], [p[1] for p in parts])
    np.testing.assert_allclose(mo, whole_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(ml, whole_l, rtol=0, atol=1e-12)
    eo, el = O.merge_splits([parts[-1][0]] * 2, [parts[-1][1]] * 2)
    assert (eo == 0).all() and np.isneginf(el).all()


# ---------------------------------------------------------------- sparse / fp8

def _fp8(L=300, h_q=4, topk=64, s_q=1, seed=13):
    return I.make_workload("fp8", 1, s_q, h_q, [L], fp8=True, topk=topk, seed=seed)


def test_sparse_arange_equals_dense_over_fp8_cache():
    L = 300
    w = _fp8(L=L, topk=L)
    idx = np.arange(L, dtype=np.int32)[None, None]
    so, sl = O.decode(w.q_bits, w.block_table, w.cache_seqlens, kv_fp8=w.kv_fp8, indices=idx)
    do, dl = O.decode(w.q_bits, w.block_table, w.cache_seqlens, kv_fp8=w.kv_fp8)
    np.testing.assert_allclose(so, do, rtol=0, atol=1e-12)
    np.testing.assert_allclose(sl, dl, rtol=0, atol=1e-12)


def test_sparse_index_order_is_irrelevant():
    w = _fp8(topk=128)
    o1, l1 = O.decode(w.q_bits, w.block_table, w.cache_seqlens, kv_fp8=w.kv_fp8, indices=w.indices)
    idx2 = w.indices[..., ::-1].copy()
    o2, l2 = O.decode(w.q_bits, w.block_table, w.cache_seqlens, kv_fp8=w.kv_fp8, indices=idx2)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def test_sparse_single_valid_index_and_all_padding():
    w = _fp8(topk=64)
    idx = np.full_like(w.indices, -1)
    idx[0, 0, 17] = 211
    o, l = O.decode(w.q_bits, w.block_table, w.cache_seqlens, kv_fp8=w.kv_fp8, indices=idx)
    # the key straight from its stored row (page from the block table, slot 211 % 64)
    k = fp8_rows_to_f64(w.kv_fp8[w.block_table[0, 211 // 64], 211 % 64, 0])
    q = bf16_bits_to_f64(w.q_bits[0, 0])
    np.testing.assert_array_equal(o[0, 0], np.broadcast_to(k[:512], o[0, 0].shape))
    np.testing.assert_allclose(l[0, :, 0], SCALE * (q @ k), rtol=0, atol=1e-12)
    idx[:] = -1
    o, l = O.decode(w.q_bits, w.block_table, w.cache_seqlens, kv_fp8=w.kv_fp8, indices=idx)
    assert (o == 0).all() and np.isneginf(l).all()


def test_sparse_duplicate_index_counts_twice():
    """A key listed twice carries twice the weight: lse grows by
    ln(1 + exp(s_k - lse)) compared with listing it once."""
    w = _fp8(topk=64)
    idx = w.indices.copy()
    once_o, once_l = O.decode(w.q_bits, w.block_table, w.cache_seqlens, kv_fp8=w.kv_fp8, indices=idx)
    dup = idx.copy()
    dup[0, 0, -1] = dup[0, 0, 0]
    keep = dup[0, 0, :-1].copy()
    base = np.concatenate([keep, [-1]])[None, None].astype(np.int32)
    bo, bl = O.decode(w.q_bits, w.block_table, w.cache_seqlens, kv_fp8=w.kv_fp8, indices=base)
    do, dl = O.decode(w.q_bits, w.block_table, w.cache_seqlens, kv_fp8=w.kv_fp8, indices=dup)
    k = O.gather_rows(w.block_table, 0, np.array([idx[0, 0, 0]]), kv_fp8=w.kv_fp8)[0]
    s = SCALE * (bf16_bits_to_f64(w.q_bits[0, 0]) @ k)
    np.testing.assert_allclose(dl[0, :, 0], np.logaddexp(bl[0, :, 0], s), rtol=0, atol=1e-12)
    del once_o, once_l, do


def test_sparse_out_of_range_indices_are_skipped():
    w = _fp8(L=200, topk=64)
    idx = w.indices.copy()
    o1, l1 = O.decode(w.q_bits, w.block_table, w.cache_seqlens, kv_fp8=w.kv_fp8, indices=idx)
    bad = np.concatenate([idx, np.array([[[200, 5000, -7]]], np.int32)], axis=-1)
    o2, l2 = O.decode(w.q_bits, w.block_table, w.cache_seqlens, kv_fp8=w.kv_fp8, indices=bad)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
