"""mla_decode_noalloc: the decode entry point for callers that may not create
device allocations of their own (code handed its buffers by a host program,
or code that must stay off cudaMalloc / cudaFree because those calls can
synchronise the device).  Its split-KV scratch is an array built into the
library.  Both entry points run the same kernels on the same plan, so the
results must equal mla_decode's (which uses a caller workspace) bit for bit,
and they must also agree with the fp64 oracle within the project tolerance.
A warmed-up call must leave the device's allocations unchanged.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes
import gc

import numpy as np
import pytest
import torch

import mla_decode_attention_get_b200 as M
from mla_decode_attention_get_b200 import _abi
from mla_decode_attention_get_b200 import inputs as I
from gpu_util import assert_close, oracle

pytestmark = pytest.mark.gpu


def _calls(w):
    t = I.to_device(w)
    topk = w.topk if w.fp8 else None
    md, ns = M.get_mla_metadata(t["sl"], w.s_q * w.h_q, 1, s_q=w.s_q, topk=topk)
    ref = M.prepare_decode(t["q"], t["kv"], t["bt"], t["sl"], 512, md, ns, w.softmax_scale, w.causal, w.fp8,
                           t["idx"])
    other = M.prepare_decode(t["q"], t["kv"], t["bt"], t["sl"], 512, md, ns, w.softmax_scale, w.causal, w.fp8,
                             t["idx"])
    # the scratch-free call must not need the caller's workspace: give it 16 bytes
    other.args.workspace_bytes = 16
    return ref, other


def _results(call):
    out = call._keep[6].float().cpu().numpy()
    lse = call._keep[7].cpu().numpy()
    return out, lse, int(call._keep[9].item())


def test_noalloc_matches_mla_decode_on_two_calls():
    workloads = [I.make_config(2, batch=8, seqlen=1000),                  # dense, sequences split
                 I.make_config(5, batch=3, seqlen=3000)]                  # FP8 sparse, another plan
    for w in workloads:                                                   # two calls in a row
        ref, other = _calls(w)
        ref.decode()
        other.decode_noalloc()
        torch.cuda.synchronize()
        ro, rl, rerr = _results(ref)
        no, nl, nerr = _results(other)
        assert rerr == 0 and nerr == 0
        # same kernels, same plan: any difference would mean stale or shared scratch
        assert np.array_equal(no, ro)
        assert np.array_equal(nl, rl)
        batches = [0, w.batch - 1]
        ref_out, ref_lse = oracle(w, batches=batches)
        assert_close(no.astype(np.float64), nl.astype(np.float64), ref_out, ref_lse, batches=batches)


def test_noalloc_allocates_nothing():
    w = I.make_config(2, batch=8, seqlen=1000)
    ref, call = _calls(w)                                                 # both stay alive throughout
    call.decode_noalloc()                                                 # warm-up: module and symbol set up
    torch.cuda.synchronize()
    # no Python garbage collection may free other tests' tensors in between
    gc.collect()
    gc.disable()
    try:
        torch_before = torch.cuda.memory_allocated()
        free_before, _ = torch.cuda.mem_get_info()
        for i in range(3):
            call.decode_noalloc()
        torch.cuda.synchronize()
        free_after, total = torch.cuda.mem_get_info()
        torch_after = torch.cuda.memory_allocated()
    finally:
        gc.enable()
    assert torch_after == torch_before
    assert free_after == free_before
    assert int(call._keep[9].item()) == 0
    del ref


def test_noalloc_rejects_plans_beyond_its_scratch():
    # 132 x 2 x 128 rows over 37 partitions need ~89 MB of split scratch
    need = _abi.workspace_bytes(132, 2, 128, 0, 37)
    assert need > _abi.NOALLOC_SCRATCH_BYTES
    a = _abi.DecodeArgs()
    a.batch, a.s_q, a.h_q, a.h_kv, a.d_v, a.num_parts = 132, 2, 128, 1, 512, 37
    assert _abi.lib().mla_decode_noalloc(ctypes.byref(a), None) == _abi.MLA_ERR_WORKSPACE
