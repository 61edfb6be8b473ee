"""The scheduler kernel reproduces the reference plan bit for bit."""
import numpy as np
import pytest
import torch

import mla_decode_attention_get_b200 as M
from oracle import metadata_ref as R

pytestmark = pytest.mark.gpu


def _gpu_plan(seqlens, s_q, h_q, topk, parts):
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    md, ns = M.get_mla_metadata(sl, s_q * h_q, 1, s_q=s_q, topk=topk or None, num_sm_parts=parts)
    torch.cuda.synchronize()
    return md.cpu().numpy(), ns.cpu().numpy()


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("parts", [1, 2, 7, 37, 148, 592])
def test_dense_plan_bit_exact(seed, parts):
    rng = np.random.default_rng(100 + seed)
    b = int(rng.integers(1, 300))
    L = rng.integers(0, 20000, size=b)
    L[rng.random(b) < 0.15] = 0
    L[rng.random(b) < 0.1] = 1
    md, ns = _gpu_plan(L.tolist(), 1, 16, 0, parts)
    ref_md, ref_ns = R.schedule(R.unit_tiles(L), parts)
    np.testing.assert_array_equal(ns, np.array(ref_ns))
    np.testing.assert_array_equal(md, np.array(ref_md))


@pytest.mark.parametrize("parts", [3, 74, 148])
def test_sparse_plan_bit_exact(parts):
    L = [32768, 5, 0, 4000]
    md, ns = _gpu_plan(L, 2, 64, 2048, parts)
    ref_md, ref_ns = R.schedule(R.unit_tiles(L, s_q=2, topk=2048), parts)
    np.testing.assert_array_equal(ns, np.array(ref_ns))
    np.testing.assert_array_equal(md, np.array(ref_md))


def test_large_batch_and_single_sequence():
    L = np.full(5000, 700)
    md, ns = _gpu_plan(L.tolist(), 1, 16, 0, 148)
    ref_md, ref_ns = R.schedule(R.unit_tiles(L), 148)
    np.testing.assert_array_equal(ns, np.array(ref_ns))
    np.testing.assert_array_equal(md, np.array(ref_md))
    md, ns = _gpu_plan([1_000_000], 1, 128, 0, 74)
    ref_md, ref_ns = R.schedule(R.unit_tiles([1_000_000]), 74)
    np.testing.assert_array_equal(md, np.array(ref_md))
    np.testing.assert_array_equal(ns, np.array(ref_ns))


def test_plan_too_large_for_shared_memory():
    # 2 x 30001 + 3 x 1185 ints exceed the on-chip variant: the global-memory kernel runs
    rng = np.random.default_rng(7)
    L = rng.integers(0, 5000, size=30000)
    md, ns = _gpu_plan(L.tolist(), 1, 16, 0, 1184)
    ref_md, ref_ns = R.schedule(R.unit_tiles(L), 1184)
    np.testing.assert_array_equal(ns, np.array(ref_ns))
    np.testing.assert_array_equal(md, np.array(ref_md))


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_config_plans(cfg):
    from mla_decode_attention_get_b200 import inputs as I
    w = I.make_config(cfg, batch=None) if cfg in (1, 3) else None
    if w is None:
        L = {2: [4096] * 128, 4: [16384] * 132, 5: [32768] * 64}[cfg]
        s_q, h_q, topk = {2: (1, 16, 0), 4: (2, 128, 0), 5: (1, 128, 2048)}[cfg]
    else:
        L, s_q, h_q, topk = w.cache_seqlens.tolist(), w.s_q, w.h_q, 0
    parts, _ = M.mla_metadata_shape(len(L), s_q, h_q, 1, topk)
    md, ns = _gpu_plan(L, s_q, h_q, topk, None)
    ref_md, ref_ns = R.schedule(R.unit_tiles(L, s_q=s_q, topk=topk), parts)
    np.testing.assert_array_equal(md, np.array(ref_md))
    np.testing.assert_array_equal(ns, np.array(ref_ns))
