"""The user-facing calls, made the way a serving loop makes them:
get_mla_metadata then flash_mla_with_kvcache, which allocates its outputs and
scratch per call ("Was ist FlashMLA?" (topnet.top), sections
"2. MLA-Metadaten abrufen" and "3. MLA-Decodierung ausführen"), against the
fp64 oracle.  Covers both error-word modes (check=True: a fresh zeroed word,
read back and raised on; check=False: a per-device word nobody reads), the
cached plan sizes across interleaved shapes, and the stride checks that
replaced views of the first batch entry."""
import numpy as np
import pytest
import torch

import mla_decode_attention_get_b200 as M
from mla_decode_attention_get_b200 import inputs as I
from gpu_util import assert_close, oracle, upload

pytestmark = pytest.mark.gpu


def _workload(case):
    if case == "bf16 causal s_q=2":
        return I.make_workload("api_bf16", 3, 2, 32, [700, 64, 1500], causal=True, seed=91)
    if case == "fp8 dense":
        return I.make_workload("api_fp8d", 2, 1, 64, [1300, 400], fp8=True, seed=92)
    return I.make_workload("api_fp8s", 2, 1, 128, [3000, 900], fp8=True, topk=512, seed=93)


def _call(w, t, check):
    md, ns = M.get_mla_metadata(t["sl"], w.s_q * w.h_q, 1, s_q=w.s_q, topk=w.topk if w.fp8 else None)
    out, lse = M.flash_mla_with_kvcache(t["q"], t["kv"], t["bt"], t["sl"], 512, md, ns, w.softmax_scale,
                                        w.causal, w.fp8, t["idx"], check=check)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("check", [False, True])
@pytest.mark.parametrize("case", ["bf16 causal s_q=2", "fp8 dense", "fp8 sparse"])
def test_public_calls_match_the_oracle(case, check):
    w = _workload(case)
    out, lse = _call(w, upload(w), check)
    assert out.shape == (w.batch, w.s_q, w.h_q, 512) and lse.shape == (w.batch, w.h_q, w.s_q)
    assert_close(out, lse, *oracle(w))


def test_interleaved_shapes_use_their_own_plans():
    # the plan sizes are cached per shape: alternate two shapes and a third
    # that shares the batch but not the heads
    ws = [I.make_workload("api_a", 2, 1, 16, [500, 300], seed=94),
          I.make_workload("api_b", 5, 1, 128, [64, 900, 1, 2000, 129], seed=95),
          I.make_workload("api_c", 2, 1, 64, [500, 300], seed=96)]
    ts = [upload(w) for w in ws]
    refs = [oracle(w) for w in ws]
    for _ in range(2):
        for w, t, ref in zip(ws, ts, refs):
            out, lse = _call(w, t, check=False)
            assert_close(out, lse, *ref)


def test_check_raises_on_a_device_error_and_the_next_call_is_clean():
    w = I.make_workload("api_bad", 2, 1, 16, [100, 100], seed=97)
    w.block_table[0, 1] = w.num_blocks + 7          # keys 64..99 of sequence 0 become unreadable
    t = upload(w)
    _call(w, t, check=False)                        # the error goes to the unread word: no raise
    with pytest.raises(M.MlaError):
        _call(w, t, check=True)
    good = I.make_workload("api_good", 2, 1, 16, [100, 100], seed=97)
    out, lse = _call(good, upload(good), check=True)   # a fresh word: the earlier errors do not leak
    assert_close(out, lse, *oracle(good))


def test_layout_checks():
    w = I.make_workload("api_layout", 2, 1, 16, [200, 100], seed=98)
    t = upload(w)
    md, ns = M.get_mla_metadata(t["sl"], w.s_q * w.h_q, 1)
    # s_q = 1: the stride of the size-1 dim does not matter
    q_odd = t["q"].as_strided(t["q"].shape, (t["q"].stride(0), 7, 576, 1))
    out, lse = M.flash_mla_with_kvcache(q_odd, t["kv"], t["bt"], t["sl"], 512, md, ns, w.softmax_scale)
    torch.cuda.synchronize()
    assert_close(out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64), *oracle(w))
    q_strided = torch.empty((2, 1, 16, 1152), dtype=torch.bfloat16, device="cuda")[..., :576]
    with pytest.raises(ValueError):
        M.flash_mla_with_kvcache(q_strided, t["kv"], t["bt"], t["sl"], 512, md, ns, w.softmax_scale)
    kv_strided = torch.empty((t["kv"].shape[0], 64, 1, 1152), dtype=torch.bfloat16, device="cuda")[..., :576]
    with pytest.raises(ValueError):
        M.flash_mla_with_kvcache(t["q"], kv_strided, t["bt"], t["sl"], 512, md, ns, w.softmax_scale)
