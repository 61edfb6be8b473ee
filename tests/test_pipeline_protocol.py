"""The decode kernels' barrier protocols, checked on host-side models (CPU).

`pipeline_model` restates the hand-offs of one CTA of the bf16 decode kernel
(and, in `Fp8Model`, of the FP8 kernel, with its five-part QK^T through a
ring of three TMEM slots and the V' rewrite by the gather warps):
- the page producer: TMA in two parts per page, or 8 gather warps on the FP8
  kernel;
- the MMA warp's event loop;
- four softmax warps, with padding warps, lazy rescales, segment epilogues and
  query-tile staging.
It interleaves them at random, checking parity aliasing, arrivals into the
wrong phase, data hazards on stages, S, P, Q and O, and deadlock; for the bf16
kernel also the drain of a CTA whose TMA warp gives up.  The
current protocol must run clean on every schedule tried.  Each planted
mistake must be caught."""
import random

import pytest

import pipeline_model as PM


def _plan(rng, fp8, live=None, p_rescale=0.3):
    segs = [rng.randint(1, 7) for _ in range(rng.randint(1, 4))]
    live = rng.randint(1, PM.WARPS) if live is None else live
    T = sum(segs)
    resc = {(w, t): rng.random() < p_rescale for w in range(PM.WARPS) for t in range(T)}
    return PM.Plan(segs, live, fp8, resc)


def test_protocol_runs_clean_on_random_schedules():
    for seed in range(150):
        rng = random.Random(seed)
        PM.Model(_plan(rng, False), seed).run()


def test_single_page_and_single_warp_edges():
    for seed in range(50):
        PM.Model(PM.Plan([1], 1, False, {}), seed).run()
        PM.Model(PM.Plan([1, 1, 1, 1, 1], 4, False, {}), seed).run()
        PM.Model(PM.Plan([7], 4, False, {(w, t): True for w in range(4) for t in range(7)}), seed).run()


def test_fp8_protocol_runs_clean_on_random_schedules():
    for seed in range(150):
        rng = random.Random(seed)
        PM.Fp8Model(_plan(rng, True), seed).run()
    for seed in range(30):
        PM.Fp8Model(PM.Plan([1], 1, True, {}), seed).run()
        PM.Fp8Model(PM.Plan([1, 1, 1, 1, 1], 4, True, {}), seed).run()


@pytest.mark.parametrize("mutation", ["no_slot_wait", "early_p", "early_v", "no_seg_end_pv", "early_q"])
def test_fp8_planted_mistakes_are_caught(mutation):
    caught = 0
    for seed in range(60):
        rng = random.Random(seed)
        try:
            PM.Fp8Model(_plan(rng, True, live=PM.WARPS, p_rescale=0.5), seed, mutation=mutation).run()
        except PM.ProtocolError:
            caught += 1
    assert caught > 0


def test_giving_up_drains_every_issued_copy():
    # the TMA warp gives up at a random wait (between a page's parts too);
    # the drain at exit must end, and end with nothing in flight
    for parts in (2, 4):
        for seed in range(200):
            rng = random.Random(seed)
            plan = _plan(rng, False)
            PM.Model(plan, seed, parts=parts, abort_at=(rng.randrange(sum(plan.segments)), rng.randrange(parts))).run()


@pytest.mark.parametrize("mutation", ["no_abort_arrive", "extra_abort_arrive"])
def test_planted_drain_mistakes_are_caught(mutation):
    caught = 0
    for seed in range(40):
        rng = random.Random(seed)
        plan = _plan(rng, False)
        try:
            PM.Model(plan, seed, mutation=mutation, abort_at=(rng.randrange(sum(plan.segments)), 1)).run()
        except PM.ProtocolError:
            caught += 1
    assert caught == 40


@pytest.mark.parametrize("mutation", ["shared_p_full", "no_rescale_wait", "single_pv_barrier", "hi_on_lo",
                                      "lo_before_pv"])
def test_planted_mistakes_are_caught(mutation):
    caught = 0
    for seed in range(60):
        rng = random.Random(seed)
        try:
            PM.Model(_plan(rng, False, live=PM.WARPS, p_rescale=0.5), seed, mutation=mutation).run()
        except PM.ProtocolError:
            caught += 1
    assert caught > 0


def _constants(path):
    import os
    import re
    src = open(os.path.join(os.path.dirname(__file__), "..", "mla_decode_attention_get_b200", "csrc", path)).read()
    return src, {m.group(1): int(m.group(2)) for m in re.finditer(r"constexpr int (k\w+) = (\d+);", src)}


def test_models_mirror_the_kernels():
    """The models' constants are the kernels' own: a protocol change in the
    CUDA source that the model does not follow fails here."""
    import re
    src, k = _constants("decode_sm100.cu")
    assert PM.STAGES == k["kStages"]
    assert re.search(r"mbar_init\(&bars\.kv_full\[s\], %d\)" % PM.REFILL_PARTS, src)
    assert PM.REFILL_PARTS == 2 and k["kLoChunks"] == 4          # chunks 0-3, then 4-8
    src8, k8 = _constants("decode_fp8_sm100.cu")
    assert PM.FP8_STAGES == k8["kStages"]
    assert PM.FP8_PARTS == k8["kParts"] and PM.FP8_SLOTS == k8["kSlots"]
    assert PM.GATHER_WARPS == k8["kGatherWarps"]
    rewriters = sorted(int(gw) for gw, count in re.findall(r"gw == (\d) \? RewriteKeys\{\d+, (\d+)\}", src8)
                       if int(count) > 0)
    assert tuple(rewriters) == tuple(sorted(PM.FP8_REWRITERS)) and len(rewriters) == k8["kRewriteWarps"]
