"""FP8 cache writer (C ABI mla_fp8_cache_write) against its oracle
(oracle/fp8_writer_ref.py): the whole cache must come out byte for byte
identical.  Then a round trip: rows the GPU writes are read back by the dense
FP8 decode and checked against the fp64 oracle."""
import numpy as np
import pytest
import torch

import mla_decode_attention_get_b200 as M
from mla_decode_attention_get_b200 import inputs as I
from oracle import fp8_writer_ref as W
from gpu_util import assert_close, oracle, run

pytestmark = pytest.mark.gpu


def _bf16_bits(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _rows(n, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, 576)).astype(np.float32) * rng.uniform(1e-3, 300, (n, 1)).astype(np.float32)
    x[::7, 128:256] = 0                                  # all-zero groups
    x[::11, 5] = -0.0                                    # negative zeros
    ties = np.array([448, 17, 19, 2.0 ** -10, 3 * 2.0 ** -10, -5, 0.5, -3.25], np.float32)
    x[1::13, 256:264] = ties                             # group 2 keeps max 448 (scale 1): exact ties
    x[1::13, 264:384] = 0
    return _bf16_bits(x)


def _gpu_write(bits, slots, cache):
    k = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    c = torch.from_numpy(cache).cuda()
    err = M.fp8_cache_write(k, torch.from_numpy(slots).cuda(), c)
    torch.cuda.synchronize()
    return c.cpu().numpy(), int(err.item())


@pytest.mark.parametrize("n,nblk", [(1, 1), (37, 2), (1000, 40), (100_000, 2000)])
def test_cache_bytes_match_oracle(n, nblk):
    rng = np.random.default_rng(n)
    cache = rng.integers(0, 256, size=(nblk, 64, 1, 656), dtype=np.uint8)
    slots = rng.choice(nblk * 64, size=n, replace=False).astype(np.int32)
    bits = _rows(n, n + 1)
    got, err = _gpu_write(bits, slots, cache)
    ref, bad = W.write_cache(cache, bits, slots)
    assert err == 0 and not bad
    assert np.array_equal(got, ref)


def test_skipped_and_out_of_range_slots():
    rng = np.random.default_rng(5)
    cache = rng.integers(0, 256, size=(3, 64, 1, 656), dtype=np.uint8)
    slots = np.array([0, -1, 3 * 64, 191, -7, 64], np.int32)
    bits = _rows(len(slots), 6)
    got, err = _gpu_write(bits, slots, cache)
    ref, bad = W.write_cache(cache, bits, slots)
    assert bad and err == 1
    assert np.array_equal(got, ref)


def test_round_trip_through_the_fp8_decode():
    # write every key of a paged bf16 workload into an FP8 cache with the same
    # page layout, then decode it densely and compare with the oracle
    w = I.make_workload("writer", 3, 2, 32, [500, 64, 130], causal=True, seed=9)
    n_pages = w.num_blocks
    keys, slots = [], []
    for b, L in enumerate(w.cache_seqlens):
        for t in range(int(L)):
            page = int(w.block_table[b, t // 64])
            keys.append(w.kv_bits[page, t % 64, 0])
            slots.append(page * 64 + t % 64)
    bits = np.stack(keys)
    cache = np.zeros((n_pages, 64, 1, 656), np.uint8)
    got, err = _gpu_write(bits, np.array(slots, np.int32), cache)
    assert err == 0
    w.kv_fp8, w.kv_bits, w.fp8 = got, None, True
    out, lse, err = run(w)
    assert err == 0
    assert_close(out, lse, *oracle(w))
