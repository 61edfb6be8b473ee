"""mla_decode_noalloc: the decode entry point for callers that may not create
device allocations of their own (code handed its buffers by a host program,
or code that must stay off cudaMalloc / cudaFree because those calls can
synchronise the device).  Its split-KV scratch is an array built into the
library; the results must match mla_decode, which uses a caller workspace.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import mla_decode_attention_get_b200 as M
from mla_decode_attention_get_b200 import _abi
from mla_decode_attention_get_b200 import inputs as I

pytestmark = pytest.mark.gpu

OUT_RTOL = 1e-2
LSE_ATOL = 1e-3


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
        scale = np.abs(ro).max()
        assert np.abs(no - ro).max() <= OUT_RTOL * scale
        inf = np.isneginf(rl)
        assert (np.isneginf(nl) == inf).all()
        assert np.abs(nl[~inf] - rl[~inf]).max() <= LSE_ATOL


def test_noalloc_rejects_plans_beyond_its_scratch():
    # 132 x 2 x 128 rows over 37 partitions need ~89 MB of split scratch
    need = _abi.workspace_bytes(132, 2, 128, 0, 37)
    assert need > _abi.NOALLOC_SCRATCH_BYTES
    a = _abi.DecodeArgs()
    a.batch, a.s_q, a.h_q, a.h_kv, a.d_v, a.num_parts = 132, 2, 128, 1, 512, 37
    assert _abi.lib().mla_decode_noalloc(ctypes.byref(a), None) == _abi.MLA_ERR_WORKSPACE
