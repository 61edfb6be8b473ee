"""Benchmark of MLA decode over a paged KV cache on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl native|reference]

One step = one pass of the whole decode path over one batch: the split-KV
scheduler kernel, the attention kernel and the split-combine kernel, with all
inputs resident in HBM.  The default workload is the memory-bound
configuration (batch 128, s_q 1, h_q 16, 4096 cached tokens each, 64-token
pages, shuffled block table); its 604 MB of KV is larger than the 126 MB L2,
so no flush is needed between steps.  Smaller workloads (--config 5) flush L2
with a 256 MB write before every step, outside the timed events.

With N > 1 (torchrun, one process per GPU) every rank decodes its own batch
(batch-sharded replicas: sequences are independent, there is no exchange);
`value` is the KV bytes of all ranks over the slowest rank's time.

On one GPU the same line also carries `per_config`: every decode
configuration (tiny, memory-bound, variable-length, MTP causal, FP8 sparse)
and three decode shapes next to them (s_q = 3 and 4 MTP, h_q = 64), each
timed the same way (kernel and step microseconds, TFLOP/s, KV GB/s, the
attention kernel's roofline fraction against the measured peaks, clocks,
and a bounded sample of the CPU oracle).

`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workload (the project has no other reference implementation).
"""
from __future__ import annotations

import argparse
import gc
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode TFLOPS & KV GB/s at 1 B200, as fraction of roofline, per config"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

# DRAM traffic (read + write bytes) of one attention-kernel launch per
# workload, from one ncu capture of the current kernels (profiles/); None
# where the workload was not captured.  The MTP shapes were captured on 16 of
# their 132 sequences and scaled by 132 / 16 (the same row tiles re-read the
# same pages of every sequence).
ATTN_TRAFFIC_BYTES = {"C1": None, "C2": 612192768, "C3": 330257152, "C4": 2572225920, "C5": 119535616,
                      "MTP s_q=4": 2609194368}
# The sources each attention kernel is built from, and their SHA-256 when the
# figures above were captured: a kernel whose sources have changed since
# reports no traffic (null) until it is captured again.
ATTN_KERNEL_SOURCES = {
    "mla_decode_kernel": ("decode_sm100.cu", "decode_common.cuh", "ptx_sm100.cuh", "mla_kernels.cuh",
                          "mla_api.cu"),
    "mla_decode_fp8_kernel": ("decode_fp8_sm100.cu", "decode_common.cuh", "ptx_sm100.cuh", "mla_kernels.cuh",
                              "mla_api.cu"),
}
ATTN_TRAFFIC_SOURCE_SHA256 = {
    "mla_decode_kernel": "6ed14556c1d04e02372428e056698d7e51bdd43ea699c8e8c43a2f2f6d5c1385",
    "mla_decode_fp8_kernel": "f1eec4739e0e4722b0ffc0743a1864e3251956a1efe280d46b9c9cdf967d7c52",
}


def kernel_sources_sha256(kernel):
    h = hashlib.sha256()
    for name in ATTN_KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "mla_decode_attention_get_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def attn_traffic(key, kernel):
    """The captured traffic of workload `key`, or None if the kernel's
    sources differ from those it was captured with."""
    try:
        current = kernel_sources_sha256(kernel) == ATTN_TRAFFIC_SOURCE_SHA256[kernel]
    except OSError:
        current = False
    return ATTN_TRAFFIC_BYTES.get(key) if current else None


def _env_int(k, d):
    try:
        return int(os.environ.get(k, d))
    except ValueError:
        return d


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int, uuid=None):
        self.index = index
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = None
            if uuid:
                try:
                    self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
                except Exception:
                    self.h = None
            if self.h is None:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


def max_over_ranks(ms: float, device) -> float:
    """The slowest rank's time (every rank passes its own; the process group
    is initialised).  Timing only: the decode itself exchanges nothing."""
    import torch
    import torch.distributed as dist
    x = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(x, op=dist.ReduceOp.MAX)
    return float(x.item())


def whole_job_rates(kv_bytes: int, flops: int, world: int, ms_step: float):
    """(GB/s, TFLOP/s) of all ranks together: every rank decodes its own
    batch of the workload in ms_step (the slowest rank's step time)."""
    return kv_bytes * world / (ms_step * 1e-3) / 1e9, flops * world / (ms_step * 1e-3) / 1e12


def attention_roofline(kv_bytes: int, flops: int, attn_ms: float, hbm_gbs: float, tc_burst: float,
                       tc_sustained: float) -> dict:
    """Roofline of the attention kernel: the resource whose roofline time is
    longer bounds it -- KV bytes at the measured copy bandwidth, or FLOPs at
    the measured bf16 GEMM rate.  The timed loops last milliseconds, so the
    tensor peak is the burst GEMM figure; the fraction of the sustained
    (power-capped, seconds-long) figure is reported beside it."""
    gbs = kv_bytes / (attn_ms * 1e-3) / 1e9
    tfs = flops / (attn_ms * 1e-3) / 1e12
    if flops / (tc_burst * 1e12) > kv_bytes / (hbm_gbs * 1e9):
        return {"bound": "tensor", "achieved": round(tfs, 1), "peak": tc_burst, "unit": "TFLOP/s",
                "frac": round(tfs / tc_burst, 4), "peak_kind": "burst bf16 GEMM (measured)",
                "frac_of_sustained_peak": round(tfs / tc_sustained, 4), "hbm_frac": round(gbs / hbm_gbs, 4)}
    return {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_gbs, "unit": "GB/s",
            "frac": round(gbs / hbm_gbs, 4), "peak_kind": "copy bandwidth (measured)",
            "tensor_frac": round(tfs / tc_burst, 4)}


def _blas_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([x.get("num_threads", 1) for x in info] or [1])
    except Exception:
        return len(os.sched_getaffinity(0))


def _sub_work(w, batches):
    """Algorithmic FLOPs and KV bytes of the listed sequences of workload w."""
    from mla_decode_attention_get_b200 import inputs as I
    sub = I.Workload(**{**w.__dict__})
    sub.cache_seqlens = w.cache_seqlens[batches]
    if w.indices is not None:
        sub.indices = w.indices[batches]
    sub.batch = len(batches)
    return I.flops_and_bytes(sub)


def cpu_oracle_sample(w, budget_s: float):
    """Time the oracle, as it stands, on whole sequences of the workload until
    `budget_s` seconds of CPU work; returns (KV GB/s, TFLOP/s, description, cores)."""
    from oracle import mla_oracle as O
    done, t0 = [], time.perf_counter()
    while time.perf_counter() - t0 < budget_s and len(done) < w.batch:
        done.append(len(done))
        O.decode(w.q_bits, w.block_table, w.cache_seqlens, kv_bits=w.kv_bits, kv_fp8=w.kv_fp8,
                 indices=w.indices, causal=w.causal, softmax_scale=w.softmax_scale, batches=[done[-1]])
    el = time.perf_counter() - t0
    flops, kv_bytes = _sub_work(w, done)
    desc = f"{len(done)} of {w.batch} sequences of the workload, {el:.1f} s wall, numpy fp64"
    return kv_bytes / el / 1e9, flops / el / 1e12, desc, _blas_threads()


def bench_fp8_writer(args) -> int:
    """The FP8 cache writer on one GPU: 2 Mi new key rows (2.3 GB of bf16)
    quantised into a 1.3 GB FP8 cache at shuffled slots.  A row moves 1152 B
    in, 656 B out and a 4-B slot; the inputs exceed L2, so nothing is flushed.
    One JSON line: GB/s against the measured copy bandwidth."""
    import torch
    import mla_decode_attention_get_b200 as M
    hbm = load_peaks()[0]
    n = 2 << 20
    g = torch.Generator(device="cuda").manual_seed(2024)
    k = torch.randn((n, 576), generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)
    slots = torch.randperm(n, generator=g, device="cuda").to(torch.int32)
    cache = torch.zeros((n // 64, 64, 1, 656), dtype=torch.uint8, device="cuda")
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    for _ in range(args.warmup):
        M.fp8_cache_write(k, slots, cache, err)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    sampler = ClockSampler(torch.cuda.current_device(), None)
    with sampler:
        ev[0].record()
        for _ in range(args.steps):
            M.fp8_cache_write(k, slots, cache, err)
        ev[1].record()
        torch.cuda.synchronize()
    ms = ev[0].elapsed_time(ev[1]) / args.steps
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())}")
    moved = n * (1152 + 656 + 4)
    gbs = moved / (ms * 1e-3) / 1e9
    print(json.dumps({
        "metric": "FP8 cache writer GB/s (bytes moved per row: 1152 in, 656 + 4 out)", "value": round(gbs, 1),
        "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "dtype": "bf16->e4m3", "data": "synthetic",
        "config": {"workload": "fp8 cache write n=2097152 rows, shuffled slots", "rows": n},
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(gbs / hbm, 4), "kernel": "fp8_cache_write_kernel", "kernel_ms": round(ms, 5)},
        "gpu_launches": args.steps, "clocks": sampler.summary()}), flush=True)
    return 0


def bench_sparse_prefill(args) -> int:
    """A prefill-shaped sparse call on one GPU: 2 sequences of 32768 cached
    FP8 tokens, 1024 new query tokens each, h_q = 128, a top-k of 2048
    positions per token (the same kernels as the sparse decode: one
    scheduler unit per token).  One JSON line: TFLOP/s against the measured
    sustained bf16 GEMM rate."""
    import torch
    import mla_decode_attention_get_b200 as M
    from mla_decode_attention_get_b200 import inputs as I
    _, tc, tc_sus, _ = load_peaks()
    w = I.make_workload("sparse prefill b=2 s_q=1024 h_q=128 L=32768 topk=2048", 2, 1024, 128, [32768, 32768],
                        fp8=True, topk=2048, seed=3001)
    flops, kv_bytes = I.flops_and_bytes(w)
    t = I.to_device(w)
    md, ns = M.get_mla_metadata(t["sl"], w.s_q * w.h_q, 1, s_q=w.s_q, topk=w.topk)
    call = M.prepare_decode(t["q"], t["kv"], t["bt"], t["sl"], 512, md, ns, w.softmax_scale, False, True, t["idx"])
    for _ in range(args.warmup):
        call.decode()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    sampler = ClockSampler(torch.cuda.current_device(), None)
    with sampler:
        ev[0].record()
        for _ in range(args.steps):
            call.decode()
        ev[1].record()
        torch.cuda.synchronize()
    ms = ev[0].elapsed_time(ev[1]) / args.steps
    if int(call._keep[9].item()) != 0:
        raise RuntimeError(f"device error word {int(call._keep[9].item())}")
    tfs = flops / (ms * 1e-3) / 1e12
    print(json.dumps({
        "metric": "sparse prefill TFLOP/s (2*(576+512) FLOPs per (row, valid index))", "value": round(tfs, 1),
        "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "dtype": "f16 (exact e4m3 codes; fp32 scales after the MMA)", "data": "synthetic",
        "config": {"workload": w.name, "flops": flops, "kv_bytes": kv_bytes},
        "roofline": {"bound": "tensor", "achieved": round(tfs, 1), "peak": tc_sus, "unit": "TFLOP/s",
                     "frac": round(tfs / tc_sus, 4), "peak_kind": "sustained bf16 GEMM",
                     "frac_of_burst_peak": round(tfs / tc, 4)},
        "gpu_launches": 3 * args.steps, "clocks": sampler.summary()}), flush=True)
    return 0


# Workloads of the per-configuration record: the five decode configurations,
# then three decode shapes on the MTP configuration's cache (132 sequences of
# 16384 tokens): 3 and 4 causal query tokens x 128 heads, and 64 heads x 1
# token.
PER_CONFIG = ("C1", "C2", "C3", "C4", "C5", "MTP s_q=3", "MTP s_q=4", "h_q=64")
DERIVED = {"MTP s_q=3": (3, 128, True, 3003), "MTP s_q=4": (4, 128, True, 3004), "h_q=64": (1, 64, False, 3064)}


def _workload_of(key, cache):
    from mla_decode_attention_get_b200 import inputs as I
    if key in DERIVED:
        s_q, h_q, causal, seed = DERIVED[key]
        base = cache.get("C4") or I.make_config(4)
        cache["C4"] = base
        name = f"{key} causal={causal} b=132 h_q={h_q} L=16384 (the MTP configuration's cache)"
        return I.with_queries(base, name, s_q, h_q, causal=causal, seed=seed)
    w = I.make_config(int(key[1:]))
    if key == "C4":
        cache["C4"] = w
    return w


def _workload_name(key, w):
    from mla_decode_attention_get_b200 import inputs as I
    return I.CONFIG_NAMES[int(key[1:])] if key not in DERIVED else w.name


class Timed:
    """One workload resident on the device and timed through the C ABI: the
    scheduler, attention and combine kernels per step."""

    def __init__(self, w, dev):
        import torch
        import mla_decode_attention_get_b200 as M
        from mla_decode_attention_get_b200 import inputs as I
        self.w, self.dev = w, dev
        self.flops, self.kv_bytes = I.flops_and_bytes(w)
        self.t = I.to_device(w, dev)
        self.stream = torch.cuda.current_stream(dev)
        topk = w.topk if w.fp8 else 0
        parts, _ = M.mla_metadata_shape(w.batch, w.s_q, w.h_q, 1, topk)
        self.md = torch.empty((parts, 8), dtype=torch.int32, device=dev)
        self.ns = torch.empty((w.batch * (w.s_q if w.indices is not None else 1) + 1,), dtype=torch.int32,
                              device=dev)
        sl = self.t["sl"]
        self.meta = lambda: M.mla_get_metadata(sl, w.batch, w.s_q, w.h_q, 1, topk, self.md, self.ns)  # noqa: E731
        self.meta()
        self.call = M.prepare_decode(self.t["q"], self.t["kv"], self.t["bt"], sl, 512, self.md, self.ns,
                                     w.softmax_scale, w.causal, w.fp8, self.t["idx"])
        # workloads smaller than L2 flush it with a 256 MB write before every
        # step, outside the timed events
        self.flush = (torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)
                      if self.kv_bytes < 256 * 2 ** 20 else None)

    def step(self, ev=None):
        self.meta()
        if ev is not None:
            ev[0].record(self.stream)
        self.call.attention()
        if ev is not None:
            ev[1].record(self.stream)
        self.call.combine()

    def run(self, steps, warmup, world, uuid):
        """(ms per step, attention-kernel ms per launch, clock summary)."""
        import torch
        # the W warm-up steps, then more until the GPU has been busy for a
        # quarter of a second: an idle GPU (the host-side oracle runs between
        # configurations) comes back at a lower clock and needs that long to
        # ramp up
        t0 = time.perf_counter()
        n = 0
        while n < warmup or (time.perf_counter() - t0 < 0.25 and n < warmup + 5000):
            if self.flush is not None:
                self.flush.zero_()
            self.step()
            n += 1
            if n >= warmup and n % 8 == 0:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        err = int(self.call._keep[9].item())
        if err != 0:
            raise RuntimeError(f"{self.w.name}: device error word {err}")
        # K steps between a barrier and a device synchronisation on both
        # sides, one event pair around the whole loop (per-step pairs when L2
        # is flushed between steps, so that the flushes stay outside)
        step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(steps)]
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        sampler = ClockSampler(self.dev.index if self.dev.index is not None else 0, uuid)
        with sampler:
            whole0 = torch.cuda.Event(enable_timing=True)
            whole1 = torch.cuda.Event(enable_timing=True)
            whole0.record(self.stream)
            for k in range(steps):
                if self.flush is not None:
                    self.flush.zero_()
                    step_ev[k][0].record(self.stream)
                self.step()
                if self.flush is not None:
                    step_ev[k][1].record(self.stream)
            whole1.record(self.stream)
            torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        ms_total = (whole0.elapsed_time(whole1) if self.flush is None
                    else sum(a.elapsed_time(b) for a, b in step_ev))
        # the attention kernel's own duration: the same K steps again, with an
        # event pair around every attention launch
        attn_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(steps)]
        torch.cuda.synchronize()
        for k in range(steps):
            if self.flush is not None:
                self.flush.zero_()
            self.step(attn_ev[k])
        torch.cuda.synchronize()
        attn_ms = sum(a.elapsed_time(b) for a, b in attn_ev) / steps
        return ms_total / steps, attn_ms, sampler.summary()

    def l2_note(self):
        return ("flushed before every step (256 MB write)" if self.flush is not None
                else f"inputs larger than L2 ({self.kv_bytes / 1e6:.0f} MB KV)")


def _gpu_uuid(dev):
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return None


def per_config_record(key, w, tm, ms_step, attn_ms, clocks, peaks, cpu_budget):
    hbm, tc, tc_sus, _ = peaks
    roof = attention_roofline(tm.kv_bytes, tm.flops, attn_ms, hbm, tc, tc_sus)
    roof["traffic"] = attn_traffic(key, "mla_decode_fp8_kernel" if w.fp8 else "mla_decode_kernel")
    rec = {
        "workload": _workload_name(key, w), "batch": w.batch, "s_q": w.s_q, "h_q": w.h_q,
        "causal": bool(w.causal), "cache": "fp8" if w.fp8 else "bf16", "topk": w.topk,
        "flops": tm.flops, "kv_bytes": tm.kv_bytes,
        "kernel": "mla_decode_fp8_kernel" if w.fp8 else "mla_decode_kernel",
        "kernel_us": round(attn_ms * 1e3, 2), "step_us": round(ms_step * 1e3, 2),
        "tflops": round(tm.flops / (attn_ms * 1e-3) / 1e12, 1),
        "kv_gbs": round(tm.kv_bytes / (attn_ms * 1e-3) / 1e9, 1),
        "step_tflops": round(tm.flops / (ms_step * 1e-3) / 1e12, 1),
        "roofline": roof, "clocks": clocks, "l2": tm.l2_note(),
    }
    if cpu_budget > 0:
        gbs, tfl, desc, cores = cpu_oracle_sample(w, cpu_budget)
        rec["cpu_baseline"] = {"value": round(tfl, 6), "unit": "TFLOP/s", "kv_gbs": round(gbs, 4),
                               "cores": cores, "kind": "oracle", "sample": desc}
    return rec


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", type=int, default=2, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--shape", default="", choices=[""] + list(DERIVED),
                    help="one of the extra MTP / h_q shapes on the MTP configuration's cache, instead of --config")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--per-config-cpu-budget", type=float, default=4.0,
                    help="seconds of oracle work per entry of the per-configuration record")
    ap.add_argument("--batch", type=int, default=0, help="shrink the workload's batch (profiling runs)")
    ap.add_argument("--seqlen", type=int, default=0, help="shrink the workload's cache length (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--per-config-steps", type=int, default=0,
                    help="timed steps per per-configuration entry (default: --steps, at most 300)")
    ap.add_argument("--op", default="decode", choices=["decode", "fp8_cache_write", "sparse_prefill"],
                    help="decode (the step: scheduler + attention + combine), the FP8 cache writer alone, "
                         "or a prefill-shaped sparse call")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"
    if args.op == "fp8_cache_write":
        return bench_fp8_writer(args)
    if args.op == "sparse_prefill":
        return bench_sparse_prefill(args)

    world = _env_int("WORLD_SIZE", 1)
    rank = _env_int("RANK", 0)
    local_rank = _env_int("LOCAL_RANK", 0)

    from mla_decode_attention_get_b200 import inputs as I
    peaks = load_peaks()
    hbm, tc, tc_sus, peak_src = peaks

    if args.impl == "reference":
        if rank != 0:
            return 0
        from oracle import mla_oracle as O
        w = I.make_config(args.config)
        cores = _blas_threads()
        done, elapsed = [], 0.0
        for k in range(args.warmup + args.steps):
            b = k % w.batch
            t0 = time.perf_counter()
            O.decode(w.q_bits, w.block_table, w.cache_seqlens, kv_bits=w.kv_bits, kv_fp8=w.kv_fp8,
                     indices=w.indices, causal=w.causal, softmax_scale=w.softmax_scale, batches=[b])
            if k >= args.warmup:
                elapsed += time.perf_counter() - t0
                done.append(b)
        flops, kv_bytes = _sub_work(w, done)
        gbs, tfl = kv_bytes / elapsed / 1e9, flops / elapsed / 1e12
        desc = (f"each step = the oracle on one whole sequence of the workload ({args.steps} timed steps, "
                f"{elapsed:.1f} s), numpy fp64")
        line = {
            "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * elapsed / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": I.CONFIG_NAMES[args.config], "config": args.config},
            "tflops": round(tfl, 6),
            "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return 0

    import torch
    import mla_decode_attention_get_b200 as M

    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    uuid = _gpu_uuid(dev)

    head_key = args.shape or f"C{args.config}"
    wl_cache = {}
    if args.batch or args.seqlen:
        # a smaller case of the same recipe: a profiling run, not a bench line
        base_cfg = 4 if args.shape else args.config
        w = I.make_config(base_cfg, batch=args.batch or None, seqlen=args.seqlen or None)
        if args.shape:
            s_q_, h_q_, causal_, seed_ = DERIVED[args.shape]
            w = I.with_queries(w, args.shape, s_q_, h_q_, causal=causal_, seed=seed_)
        args.no_per_config = True
        head_key = f"{head_key} (reduced: batch {w.batch}, max length {int(w.cache_seqlens.max())})"
    else:
        w = _workload_of(head_key, wl_cache)
    tm = Timed(w, dev)
    flops, kv_bytes = tm.flops, tm.kv_bytes
    ms_step, attn_ms, clocks = tm.run(args.steps, args.warmup, world, uuid)
    if world > 1:
        ms_step = max_over_ranks(ms_step, dev)
    value, tflops = whole_job_rates(kv_bytes, flops, world, ms_step)
    t, stream, flush = tm.t, tm.stream, tm.flush

    # ---- end to end through the public API, host buffers, copies in the region
    # A step's inputs (q, block_table, cache_seqlens and the sparse indices)
    # sit in one pinned host buffer and travel in one copy, as a serving
    # engine would stage them; the device side is a buffer of the same
    # layout, viewed as the four tensors.
    parts = [("q", t["q"]), ("bt", t["bt"]), ("sl", t["sl"])] + ([("idx", t["idx"])] if t["idx"] is not None else [])
    offs, in_bytes = {}, 0
    for name, x in parts:
        offs[name] = in_bytes
        in_bytes += (x.numel() * x.element_size() + 255) // 256 * 256
    in_host = torch.empty((in_bytes,), dtype=torch.uint8).pin_memory()
    for name, x in parts:
        nb = x.numel() * x.element_size()
        in_host[offs[name]:offs[name] + nb].copy_(x.cpu().contiguous().view(-1).view(torch.uint8))

    def device_inputs():
        buf = torch.empty((in_bytes,), dtype=torch.uint8, device=dev)
        views = {name: buf[offs[name]:offs[name] + x.numel() * x.element_size()].view(x.dtype).view(x.shape)
                 for name, x in parts}
        views["buf"] = buf
        views.setdefault("idx", None)
        return views

    out_host = torch.empty((w.batch, w.s_q, w.h_q, 512), dtype=torch.bfloat16).pin_memory()
    lse_host = torch.empty((w.batch, w.h_q, w.s_q), dtype=torch.float32).pin_memory()
    h2d = in_bytes
    d2h = out_host.numel() * 2 + lse_host.numel() * 4
    din = device_inputs()

    def e2e_step():
        din["buf"].copy_(in_host, non_blocking=True)
        md_, ns_ = M.get_mla_metadata(din["sl"], w.s_q * w.h_q, 1, s_q=w.s_q, topk=w.topk if w.fp8 else None)
        o, l = M.flash_mla_with_kvcache(din["q"], t["kv"], din["bt"], din["sl"], 512, md_, ns_, w.softmax_scale,
                                        w.causal, w.fp8, din["idx"])
        out_host.copy_(o, non_blocking=True)
        lse_host.copy_(l, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 200))
    e2e_reps = 1
    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    if flush is not None:
        # inputs smaller than L2: every step alone, L2 flushed before it
        e2e_mode = "serial steps, L2 flushed before each"
        e_ms = []
        for _ in range(e2e_steps):
            flush.zero_()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            e2e_step()
            b.record(stream)
            b.synchronize()
            e_ms.append(a.elapsed_time(b))
        e2e_ms = statistics.mean(e_ms)
    else:
        # A serving loop: every step copies its own inputs in from pinned host
        # memory and its out + lse back.  Two device input sets and two host
        # output sets let one step's copies (their own streams) overlap the
        # neighbouring steps' kernels.  The region ends when the last
        # result is on the host.
        e2e_mode = "pipelined serving loop: 2 buffer sets, copy streams; median of 5 runs of 100 steps"
        cin, cout = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        sets = []
        for _ in range(2):
            S = device_inputs()
            S.update({"out": torch.empty_like(out_host).pin_memory(), "lse": torch.empty_like(lse_host).pin_memory(),
                      "ready": torch.cuda.Event(), "done": torch.cuda.Event()})
            sets.append(S)
        # The loop is host-paced when the host falls behind the GPU, so a
        # pause of the host (a collection, a descheduled thread) lands in it:
        # 100 steps per run, five runs, the median run, collections off.
        e2e_steps, e2e_reps = 100, 5
        runs = []
        gc_was = gc.isenabled()
        gc.disable()
        for _ in range(e2e_reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            a.record(stream)
            cin.wait_event(a)
            for k in range(e2e_steps):
                S = sets[k & 1]
                with torch.cuda.stream(cin):
                    if k >= 2:
                        cin.wait_event(S["done"])          # step k-2 has finished reading this set
                    S["buf"].copy_(in_host, non_blocking=True)
                    S["ready"].record(cin)
                stream.wait_event(S["ready"])
                md_, ns_ = M.get_mla_metadata(S["sl"], w.s_q * w.h_q, 1, s_q=w.s_q, topk=w.topk if w.fp8 else None)
                o, l = M.flash_mla_with_kvcache(S["q"], t["kv"], S["bt"], S["sl"], 512, md_, ns_, w.softmax_scale,
                                                w.causal, w.fp8, S["idx"])
                S["done"].record(stream)
                with torch.cuda.stream(cout):
                    cout.wait_event(S["done"])
                    S["out"].copy_(o, non_blocking=True)
                    S["lse"].copy_(l, non_blocking=True)
                    o.record_stream(cout)
                    l.record_stream(cout)
            stream.wait_stream(cout)
            b.record(stream)
            torch.cuda.synchronize()
            runs.append(a.elapsed_time(b) / e2e_steps)
        if gc_was:
            gc.enable()
        e2e_ms = statistics.median(runs)
    e2e_value = kv_bytes * world / (e2e_ms * 1e-3) / 1e9
    if world > 1:
        e2e_ms_max = max_over_ranks(e2e_ms, dev)
        e2e_value = kv_bytes * world / (e2e_ms_max * 1e-3) / 1e9

    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return 0

    roof = attention_roofline(kv_bytes, flops, attn_ms, hbm, tc, tc_sus)
    roof.update({"traffic": attn_traffic(head_key, "mla_decode_fp8_kernel" if w.fp8 else "mla_decode_kernel"),
                 "peak_source": peak_src,
                 "kernel": "mla_decode_fp8_kernel" if w.fp8 else "mla_decode_kernel",
                 "kernel_ms": round(attn_ms, 5)})
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": I.CONFIG_NAMES[args.config] if head_key == f"C{args.config}" else head_key,
                   "config": args.config, "batch": w.batch,
                   "s_q": w.s_q, "h_q": w.h_q, "seq_len": int(w.cache_seqlens.max()),
                   "page": 64, "topk": w.topk, "kv_bytes": kv_bytes, "flops": flops, "l2": tm.l2_note(),
                   "parallelism": f"batch-sharded replicas x{world}"},
        "tflops": round(tflops, 3),
        "roofline": roof,
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "mode": e2e_mode},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        gbs, tfl, desc, cores = cpu_oracle_sample(w, args.cpu_budget)
        line["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                                "sample": desc}

    if world == 1 and not args.no_per_config:
        # every configuration and shape, one at a time, timed like the headline
        pc_steps = args.per_config_steps or min(args.steps, 300)
        cpu_budget = 0.0 if args.no_cpu_baseline else args.per_config_cpu_budget
        per = {}
        head_rec = per_config_record(head_key, w, tm, ms_step, attn_ms, clocks, peaks, 0.0)
        head_rec["cpu_baseline"] = line.get("cpu_baseline")
        head_rec["steps"] = args.steps
        head_rec["gpu_launches"] = 3 * args.steps
        din = sets = t = tm = None   # release the headline workload's device buffers
        torch.cuda.empty_cache()
        for key in PER_CONFIG:
            if key == head_key:
                per[key] = head_rec
                continue
            wk = _workload_of(key, wl_cache)
            tk = Timed(wk, dev)
            ms_k, attn_k, clk = tk.run(pc_steps, args.warmup, 1, uuid)
            per[key] = per_config_record(key, wk, tk, ms_k, attn_k, clk, peaks, cpu_budget)
            per[key]["steps"] = pc_steps
            per[key]["gpu_launches"] = 3 * pc_steps
            del tk
            torch.cuda.empty_cache()
        wl_cache.clear()
        line["per_config"] = per
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
