"""Helpers shared by the GPU parity tests: upload a seeded workload, run the
decode through the public API (C ABI underneath), compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import mla_decode_attention_get_b200 as M
from mla_decode_attention_get_b200 import inputs as I
from oracle import mla_oracle as O

OUT_RTOL = 1e-2    # max|out - ref| <= 1e-2 * max|ref|
LSE_ATOL = 1e-3    # |lse - ref| <= 1e-3


def upload(w, dev="cuda"):
    return I.to_device(w, dev)


def run(w, t=None, num_sm_parts=None, check=False, return_call=False):
    t = t or upload(w)
    md, ns = M.get_mla_metadata(t["sl"], w.s_q * w.h_q, 1, s_q=w.s_q,
                                topk=w.topk if w.fp8 else None, num_sm_parts=num_sm_parts)
    call = M.prepare_decode(t["q"], t["kv"], t["bt"], t["sl"], 512, md, ns, w.softmax_scale, w.causal,
                            w.fp8, t["idx"])
    call.decode()
    torch.cuda.synchronize()
    out = call._keep[6].float().cpu().numpy().astype(np.float64)
    lse = call._keep[7].cpu().numpy().astype(np.float64)
    err = int(call._keep[9].item())
    if return_call:
        return out, lse, err, call
    return out, lse, err


def oracle(w, batches=None):
    return O.decode(w.q_bits, w.block_table, w.cache_seqlens,
                    kv_bits=w.kv_bits, kv_fp8=w.kv_fp8, indices=w.indices, causal=w.causal,
                    softmax_scale=w.softmax_scale, batches=batches)


def assert_close(out, lse, ref_out, ref_lse, batches=None):
    if batches is not None:
        out, lse, ref_out, ref_lse = out[batches], lse[batches], ref_out[batches], ref_lse[batches]
    scale = max(np.abs(ref_out).max(), 1e-30)
    err = np.abs(out - ref_out).max()
    assert np.isfinite(out).all(), "non-finite output"
    assert err <= OUT_RTOL * scale, f"out max|d| {err:.3e} > {OUT_RTOL} * {scale:.3e}"
    inf = np.isneginf(ref_lse)
    assert (np.isneginf(lse) == inf).all(), "-inf lse rows differ"
    d = np.abs(lse[~inf] - ref_lse[~inf]).max() if (~inf).any() else 0.0
    assert d <= LSE_ATOL, f"lse max|d| {d:.3e}"
    return err / scale, d
