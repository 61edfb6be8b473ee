"""Failure detection without a GPU fault: the decode kernels' bounded waits
give up, report it, and leave the context usable.

Every pipeline wait of both decode kernels gives up after a limit (2 s by
default); a CTA that gives up sets MLA_DEVERR_TIMEOUT in the error word,
drains its own copies and MMAs (those drains keep the full 2 s bound), frees
its tensor memory and returns.  mla_set_pipeline_wait_limit shortens the
pipeline waits' limit to 1 ns here (the waits then poll without suspending,
so each test sees the clock), and they run out on an ordinary workload: one
partition, tens of pages, where some wait always outlasts a tick of the
clock.  No arrival is withheld and nothing is malformed.  The call must
return with the bit set, and the next call, at the default limit, must match
the fp64 oracle in the same process."""
import numpy as np
import pytest

from mla_decode_attention_get_b200 import _abi
from mla_decode_attention_get_b200 import inputs as I
from gpu_util import assert_close, oracle, run, upload

pytestmark = pytest.mark.gpu


def _workload(case):
    if case == "bf16":
        return I.make_workload("tobf16", 2, 1, 16, [1500, 700], seed=81)
    if case == "fp8 dense":
        return I.make_workload("tofp8d", 2, 1, 16, [1500, 700], fp8=True, seed=82)
    return I.make_workload("tofp8s", 2, 1, 64, [3000, 1000], fp8=True, topk=1024, seed=83)


# the outputs of the call that gave up are undefined (numpy warns on casting
# their garbage); only its error word is checked
@pytest.mark.filterwarnings("ignore:invalid value encountered in cast:RuntimeWarning")
@pytest.mark.parametrize("case", ["bf16", "fp8 dense", "fp8 sparse"])
def test_waits_give_up_and_the_next_call_is_correct(case):
    w = _workload(case)
    t = upload(w)
    _abi.set_pipeline_wait_limit(1)
    try:
        _, _, err = run(w, t, num_sm_parts=1)
    finally:
        _abi.set_pipeline_wait_limit(0)
    assert err & _abi.MLA_DEVERR_TIMEOUT, f"error word {err:#x}"
    out, lse, err = run(w, t)
    assert err == 0
    assert_close(out, lse, *oracle(w))
    out1, lse1, err1 = run(w, t, num_sm_parts=1)
    assert err1 == 0
    assert np.isfinite(out1).all()
    assert_close(out1, lse1, *oracle(w))
