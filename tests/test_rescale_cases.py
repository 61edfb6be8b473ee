"""The workloads of the O-rescale parity tests really rescale (CPU).

The decode kernel keeps a row's running max m (in log2 units) from the first
page. It moves m, rescaling O, only when a later page's max exceeds m by more
than 8 (a factor 2^8). This test replays that rule in fp64 on the keys in the
order the kernel walks them (pages of 64 keys, or tiles of 64 index slots).
It checks that rows of every rescale case do jump after the first page, and
that the same workloads without the boosts do not: there the GPU tests would
pass without exercising the branch."""
import numpy as np
import pytest

from mla_decode_attention_get_b200 import inputs as I
from oracle.formats import bf16_bits_to_f64
from oracle.mla_oracle import gather_rows
import rescale_cases as RC

RESCALE_LOG2 = 8.0
LOG2E = 1.0 / np.log(2.0)


def _jumping_rows(w, b):
    """Rows of sequence b whose running max moves after their first tile."""
    L = int(w.cache_seqlens[b])
    q = bf16_bits_to_f64(w.q_bits[b])                       # [s_q, h_q, 576]
    kw = dict(kv_bits=w.kv_bits, kv_fp8=w.kv_fp8)
    n = 0
    for i in range(w.s_q):
        if w.indices is not None:
            slots = w.indices[b, i]
            pos = np.where(slots >= 0, slots, 0)
            s = q[i] @ gather_rows(w.block_table, b, pos, **kw).T
            s[:, slots < 0] = -np.inf
        else:
            s = q[i] @ gather_rows(w.block_table, b, np.arange(L), **kw).T
            if w.causal:
                s[:, np.arange(L) > L - w.s_q + i] = -np.inf
        s = s * w.softmax_scale * LOG2E
        m = s[:, :64].max(1)
        moved = np.zeros(len(m), bool)
        for t0 in range(64, s.shape[1], 64):
            pm = s[:, t0:t0 + 64].max(1)
            jump = pm > m + RESCALE_LOG2
            moved |= jump
            m = np.where(jump, pm, m)
        n += int(moved.sum())
    return n


CASES = {
    "bf16 h16": lambda: RC.bf16_case(16, 1, False),
    "bf16 h128": lambda: RC.bf16_case(128, 1, False),
    "bf16 h64 causal s_q=2": lambda: RC.bf16_case(64, 2, True),
    "fp8 dense": RC.fp8_dense_case,
    "fp8 sparse": RC.fp8_sparse_case,
    "fp8 dense x17 scales": lambda: RC.fp8_dense_case(x17=True),
    "fp8 sparse x17 scales": lambda: RC.fp8_sparse_case(x17=True),
}


@pytest.mark.parametrize("name", list(CASES))
def test_rescale_cases_move_the_running_max(name):
    w = CASES[name]()
    assert _jumping_rows(w, 0) > 0


@pytest.mark.parametrize("name", ["fp8 dense x17 scales", "fp8 sparse x17 scales"])
def test_x17_cases_reach_large_logits(name):
    # the boosted rows give natural-log logits of 30 or more, where a 2^-11
    # relative rounding of a key value would move the lse by ~1e-3 or more
    w = CASES[name]()
    q = bf16_bits_to_f64(w.q_bits[0])
    L = int(w.cache_seqlens[0])
    keys = gather_rows(w.block_table, 0, np.arange(L), kv_fp8=w.kv_fp8)
    s = (q[0] @ keys.T) * w.softmax_scale
    assert s.max() >= 30.0


def test_unboosted_workloads_do_not():
    w = I.make_workload("rescale", 2, 1, 16, [3000, 2000], seed=66)
    assert _jumping_rows(w, 0) == 0
    w = I.make_workload("fp8dresc", 2, 1, 64, [3000, 2000], fp8=True, seed=47)
    assert _jumping_rows(w, 0) == 0
