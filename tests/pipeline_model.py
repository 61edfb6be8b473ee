"""A host-side model of the decode kernels' synchronisation protocols.

Test infrastructure only.  `Model` restates, role by role, the mbarrier
hand-offs of one CTA of the bf16 decode kernel in `csrc/decode_sm100.cu`:
- the page producer, the TMA warp;
- the MMA warp's event loop;
- the four softmax warps, with idle padding warps, lazy rescales, segment
  epilogues and query-tile staging.
A random scheduler then interleaves the roles, the landing of page loads and
the in-order completion of the tensor pipe.  A page is loaded in `parts`
parts (REFILL_PARTS): PV runs in as many slices of the 512 value dims, part i
(of all but the last) holds the chunks only QK^T and PV slice i read and is
loaded once that slice of the stage's previous page has completed
(kv_empty_part[i]); the last part (P's chunk included) once all of PV has
(kv_empty).  kv_full takes one arrival per part.

An mbarrier is modelled by its count, its pending arrivals and the number of
phases it has completed.  A wait on parity P passes when the completed count
has the other parity, as the hardware does.  The model also knows which
phase each wait and each arrival means, and flags:
- a wait that passes on a different phase than the one it means (parity
  aliasing);
- an arrival that lands in another page's phase;
- a data hazard: an MMA that reads a stage, S buffer, P tile or query tile
  its producer has not finished, or a write to one that a reader still needs;
  a rescale or epilogue read of O while PV may still update it;
- a deadlock: nothing can move, and work is left.

`mutation` switches on one planted protocol mistake, to show that the checks
catch it:
- "shared_p_full": one p_full barrier for all pages;
- "no_rescale_wait": rescale O without waiting for PV of the previous page;
- "single_pv_barrier": the epilogue waits for PV through one barrier
  committed per page, with parity t & 1;
- "hi_on_lo": the last part of a page (P's chunk included) is loaded once
  the PV slice before the last has completed, like the part before it;
- "lo_before_pv": the first part's release is committed before the first PV
  slice is issued.

`abort_at=(t, i)` makes the TMA warp give up at its wait for part i of page
t, as on a timeout: the other roles stop at once, the copies and MMAs already
issued complete, and the load lane's drain waits on kv_full for the last page
it issued into each stage.  Giving up between a page's parts, it first makes
the page's remaining arrivals.  The drain must end, and end with no copy in
flight.  Planted mistakes: "no_abort_arrive" (the remaining arrivals are not
made: the drain never ends) and "extra_abort_arrive" (one arrival too many:
the drain ends while a part is still landing).

`Fp8Model` (at the end) does the same for the FP8 kernel in
`csrc/decode_fp8_sm100.cu`, whose protocol differs (three stages filled by 8
gather warps, QK^T in five parts through a ring of three TMEM slots, V'
rewritten in place by the gather warps).
"""
from __future__ import annotations

import random
from dataclasses import dataclass, field
from typing import Dict, List, Optional

STAGES = 3
REFILL_PARTS = 2     # bf16 kernel: parts a stage is refilled in
WARPS = 4            # softmax warps, one per TMEM lane quadrant
GATHER_WARPS = 8     # FP8 kernel
FP8_PARTS = 5        # FP8 kernel: QK^T parts per tile (latent groups 0-3, RoPE)
FP8_SLOTS = 3        # FP8 kernel: partial-S slots in TMEM
FP8_REWRITERS = (0, 1, 2, 4, 5, 6)   # FP8 kernel: the gather warps that rewrite V'


class ProtocolError(AssertionError):
    pass


class Barrier:
    def __init__(self, name: str, count: int):
        self.name, self.count, self.pending, self.completed = name, count, count, 0

    def arrive(self, phase: int):
        if phase != self.completed:
            raise ProtocolError(f"{self.name}: arrival meant for phase {phase} lands in phase {self.completed}")
        self.pending -= 1
        if self.pending == 0:
            self.completed += 1
            self.pending = self.count

    def passes(self, phase: int) -> bool:
        """Hardware parity test of a wait that means "phase `phase` has
        completed" (phase -1: the barrier's initial state)."""
        ok = (self.completed & 1) != (phase & 1)
        if ok and self.completed != phase + 1:
            raise ProtocolError(f"{self.name}: wait for phase {phase} passes at {self.completed} completed phases")
        return ok


@dataclass
class Plan:
    segments: List[int]                 # pages per segment, in order
    live_warps: int                     # softmax warps with at least one real row
    fp8: bool = False                   # (Fp8Model only)
    rescale: Optional[Dict] = None      # (warp, page) -> bool: a rescale is needed


@dataclass
class State:
    stage_page: List[Optional[int]] = field(default_factory=lambda: [None] * STAGES)
    stage_page_part: Dict[int, List[Optional[int]]] = field(default_factory=dict)   # bf16: all but the last part
    pv_part_done: Dict[int, set] = field(default_factory=dict)                       # bf16: PV slices but the last
    stage_writers: List[int] = field(default_factory=lambda: [0] * STAGES)
    qk_done: set = field(default_factory=set)
    pv_done: set = field(default_factory=set)
    p_written: Dict[int, int] = field(default_factory=dict)
    s_reading: Dict[int, set] = field(default_factory=lambda: {0: set(), 1: set()})
    s_page: Dict[int, Optional[int]] = field(default_factory=lambda: {0: None, 1: None})
    o_busy: set = field(default_factory=set)
    q_seg: int = -1                     # segment whose query tile is in TMEM
    q_writes: Dict[int, int] = field(default_factory=dict)
    epilogue_done: Dict[int, int] = field(default_factory=dict)


class Model:
    def __init__(self, plan: Plan, seed: int, mutation: Optional[str] = None, parts: int = REFILL_PARTS,
                 abort_at: Optional[tuple] = None):
        self.plan, self.rng, self.mut, self.parts = plan, random.Random(seed), mutation, parts
        self.abort_at, self.aborted = abort_at, False
        self.T = sum(plan.segments)
        self.seg_of, self.first_of_seg = [], set()
        t = 0
        for k, n in enumerate(plan.segments):
            self.first_of_seg.add(t)
            self.seg_of += [k] * n
            t += n
        S = STAGES
        self.kv_full = [Barrier(f"kv_full[{s}]", parts) for s in range(S)]
        self.kv_empty_part = [[Barrier(f"kv_empty_part[{i}][{s}]", 1) for s in range(S)] for i in range(parts - 1)]
        self.kv_empty = [Barrier(f"kv_empty[{s}]", 1) for s in range(S)]
        self.s_full = [Barrier(f"s_full[{b}]", 1) for b in range(2)]
        self.s_empty = [Barrier(f"s_empty[{b}]", WARPS) for b in range(2)]
        self.q_full = Barrier("q_full", WARPS)
        if mutation == "shared_p_full":
            shared = Barrier("p_full", WARPS)
            self.p_full = [shared] * S
        else:
            self.p_full = [Barrier(f"p_full[{s}]", WARPS) for s in range(S)]
        self.pv_bar = Barrier("pv_done", 1)          # only the planted mistake waits on it
        self.st = State()
        self.st.stage_page_part = {i: [None] * S for i in range(parts - 1)}
        self.st.pv_part_done = {i: set() for i in range(parts - 1)}
        self.pipe: List[tuple] = []                  # tensor pipe, in order
        self.loads: List[tuple] = []                 # (page, part) in flight; part 0: chunks 0-3
        self.last_issued: List[Optional[int]] = [None] * S   # per stage, for the drain after giving up

    # -- phase bookkeeping ---------------------------------------------------
    def p_full_phase(self, t):
        return t if self.mut == "shared_p_full" else t // STAGES

    # -- roles (generators yielding ("wait", pred) or ("step",)) -------------
    def producer(self):
        for t in range(self.T):
            s = t % STAGES
            for i in range(self.parts):
                last = i == self.parts - 1
                if last and self.mut == "hi_on_lo":
                    freed = self.kv_empty_part[i - 1]
                else:
                    freed = self.kv_empty if last else self.kv_empty_part[i]
                if (t, i) == self.abort_at:
                    if i > 0 and self.mut != "no_abort_arrive":
                        for _ in range(self.parts - i + (1 if self.mut == "extra_abort_arrive" else 0)):
                            self.kv_full[s].arrive(t // STAGES)
                    self.aborted = True
                    return
                yield ("wait", lambda s=s, t=t, freed=freed: freed[s].passes(t // STAGES - 1))
                self._stage_write_begin(s, t, i)
                self.loads.append((t, i))
                if i == 0:
                    self.last_issued[s] = t
                yield ("step",)

    def mma(self):
        pv = qk = 0
        o_seg = -1
        while pv < self.T:
            issued = False
            if pv < qk and self.p_full[pv % STAGES].passes(self.p_full_phase(pv)):
                s = pv % STAGES
                first = self.seg_of[pv] != o_seg
                if self.mut == "lo_before_pv":
                    self.pipe.append(("commit", self.kv_empty_part[0][s], pv // STAGES))
                for h in range(self.parts):
                    self.pipe.append(("PV", pv, first, h))
                    if h < self.parts - 1 and not (h == 0 and self.mut == "lo_before_pv"):
                        self.pipe.append(("commit", self.kv_empty_part[h][s], pv // STAGES))
                o_seg = self.seg_of[pv]
                self.pipe.append(("commit", self.kv_empty[s], pv // STAGES))
                if self.mut == "single_pv_barrier":
                    self.pipe.append(("commit", self.pv_bar, pv))
                pv += 1
                issued = True
            if qk < self.T:
                s, sb = qk % STAGES, qk & 1
                first = qk in self.first_of_seg
                if (self.kv_full[s].passes(qk // STAGES)
                        and (not first or self.q_full.passes(self.seg_of[qk]))
                        and self.s_empty[sb].passes((qk >> 1) - 1)):
                    self.pipe.append(("QK", qk))
                    self.pipe.append(("commit", self.s_full[sb], qk >> 1))
                    qk += 1
                    issued = True
            yield ("step",) if issued else ("idle",)

    def softmax(self, w):
        live = w < self.plan.live_warps
        self._stage_q(w, 0)
        yield ("step",)
        self.q_full.arrive(0)
        t = 0
        for k, n in enumerate(self.plan.segments):
            any_pv = False
            for j in range(n):
                s, sb = t % STAGES, t & 1
                yield ("wait", lambda s=s, t=t: self.kv_full[s].passes(t // STAGES))
                yield ("wait", lambda sb=sb, t=t: self.s_full[sb].passes(t >> 1))
                if live:
                    if self.st.s_page[sb] != t:
                        raise ProtocolError(f"softmax {w} reads S[{sb}] for page {t}, holding {self.st.s_page[sb]}")
                    self.st.s_reading[sb].add(w)
                    yield ("step",)
                    self.st.s_reading[sb].discard(w)
                self.s_empty[sb].arrive(t >> 1)
                need = live and any_pv and bool((self.plan.rescale or {}).get((w, t), False))
                if need:
                    if self.mut != "no_rescale_wait":
                        yield ("wait", lambda t=t: self.kv_empty[(t - 1) % STAGES].passes((t - 1) // STAGES))
                    if (t - 1) not in self.st.pv_done:
                        raise ProtocolError(f"softmax {w} rescales O before PV of page {t - 1} completed")
                    self.st.o_busy.add(w)
                    yield ("step",)
                    self.st.o_busy.discard(w)
                if live:
                    if t not in self.st.qk_done or self.st.stage_page[s] != t:
                        raise ProtocolError(f"softmax {w} writes P of page {t} into a stage QK still reads")
                    yield ("step",)
                    self.st.p_written[t] = self.st.p_written.get(t, 0) + 1
                self.p_full[s].arrive(self.p_full_phase(t))
                any_pv = True
                if j == n - 1:
                    if k + 1 < len(self.plan.segments):
                        if t not in self.st.qk_done:
                            raise ProtocolError(f"softmax {w} overwrites the query tile while QK of page {t} runs")
                        self._stage_q(w, k + 1)
                        yield ("step",)
                        self.q_full.arrive(k + 1)
                    if live:
                        if self.mut == "single_pv_barrier":
                            yield ("wait", lambda t=t: self.pv_bar.passes(t))
                        else:
                            yield ("wait", lambda s=s, t=t: self.kv_empty[s].passes(t // STAGES))
                        if t not in self.st.pv_done:
                            raise ProtocolError(f"softmax {w} reads O for segment {k} before PV of page {t} completed")
                        self.st.o_busy.add(w)
                        yield ("step",)
                        self.st.o_busy.discard(w)
                    self.st.epilogue_done[k] = self.st.epilogue_done.get(k, 0) + 1
                t += 1

    # -- helpers ---------------------------------------------------------------
    def _stage_write_begin(self, s, t, part):
        if part < self.parts - 1:
            prev, done = self.st.stage_page_part[part][s], self.st.pv_part_done[part]
        else:
            prev, done = self.st.stage_page[s], self.st.pv_done
        if prev is not None and prev != t and prev not in done:
            raise ProtocolError(f"page {t} overwrites stage {s} (part {part}) while page {prev} is still in use")

    def _stage_q(self, w, seg):
        self.st.q_writes[seg] = self.st.q_writes.get(seg, 0) + 1
        if self.st.q_writes[seg] == WARPS:
            self.st.q_seg = seg

    def _land(self, t, part):
        s = t % STAGES
        if part < self.parts - 1:
            self.st.stage_page_part[part][s] = t
        else:
            self.st.stage_page[s] = t
        self.kv_full[s].arrive(t // STAGES)

    def _pipe_pop(self):
        item = self.pipe.pop(0)
        kind = item[0]
        if kind == "commit":
            item[1].arrive(item[2])
        elif kind == "QK":
            t = item[1]
            s, sb = t % STAGES, t & 1
            held = [self.st.stage_page_part[i][s] for i in range(self.parts - 1)] + [self.st.stage_page[s]]
            if any(x != t for x in held):
                raise ProtocolError(f"QK of page {t} reads stage {s} holding {held}")
            if self.st.q_seg != self.seg_of[t]:
                raise ProtocolError(f"QK of page {t} reads the query tile of segment {self.st.q_seg}")
            if self.st.s_reading[sb]:
                raise ProtocolError(f"QK of page {t} overwrites S[{sb}] while it is being read")
            self.st.s_page[sb] = t
            self.st.qk_done.add(t)
        else:
            t, first, half = item[1], item[2], item[3]
            s = t % STAGES
            # P lives in chunk 8 (the last part): every slice reads it
            own = self.st.stage_page[s] if half == self.parts - 1 else self.st.stage_page_part[half][s]
            if self.st.stage_page[s] != t or own != t:
                raise ProtocolError(f"PV slice {half} of page {t} reads stage {s} holding {own} / {self.st.stage_page[s]}")
            if self.st.p_written.get(t, 0) != self.plan.live_warps:
                raise ProtocolError(f"PV of page {t} reads P before every live warp wrote it")
            if self.st.o_busy:
                raise ProtocolError(f"PV of page {t} updates O while warps {sorted(self.st.o_busy)} use it")
            seg = self.seg_of[t]
            if first and seg > 0 and self.st.epilogue_done.get(seg - 1, 0) != WARPS:
                raise ProtocolError(f"PV of page {t} restarts O before the epilogue of segment {seg - 1}")
            if half < self.parts - 1:
                self.st.pv_part_done[half].add(t)
            else:
                self.st.pv_done.add(t)

    def _drain(self):
        """After the TMA warp gave up: the other roles have stopped; issued
        copies land and issued MMAs complete in any interleaving until the
        load lane's waits (kv_full of the last page issued into each stage)
        all pass."""
        def drained():
            return all(lt is None or self.kv_full[s].passes(lt // STAGES) for s, lt in enumerate(self.last_issued))
        while True:
            if drained():
                if self.loads:
                    raise ProtocolError(f"the drain ends with copies {self.loads} in flight")
                return
            movers = [("land", x) for x in self.loads] + ([("pipe", None)] if self.pipe else [])
            if not movers:
                raise ProtocolError("the drain never ends: an issued page's kv_full cannot complete")
            kind, arg = self.rng.choice(movers)
            if kind == "pipe":
                self._pipe_pop()
            else:
                self.loads.remove(arg)
                self._land(*arg)

    # -- scheduler -------------------------------------------------------------
    def run(self, max_steps: int = 200000):
        roles = [self.mma()] + [self.softmax(w) for w in range(WARPS)] + [self.producer()]
        waiting = [None] * len(roles)        # pending wait predicate, or "idle"
        done = [False] * len(roles)

        def advance(i):
            try:
                cmd = next(roles[i])
            except StopIteration:
                done[i] = True
                return
            waiting[i] = cmd[1] if cmd[0] == "wait" else ("idle" if cmd[0] == "idle" else None)

        for i in range(len(roles)):
            advance(i)
        for _ in range(max_steps):
            if self.aborted:
                self._drain()
                return
            if all(done) and not self.pipe and not self.loads:
                return
            movers, polls = [], []
            for i in range(len(roles)):
                if done[i]:
                    continue
                w = waiting[i]
                if w == "idle":
                    polls.append(("role", i))
                elif w is None or w():
                    movers.append(("role", i))
            if self.pipe:
                movers.append(("pipe", None))
            movers += [("land", x) for x in self.loads]
            if not movers:
                if not polls:
                    raise ProtocolError("deadlock: no role can move and nothing is in flight")
                i = polls[0][1]
                pipe_before = len(self.pipe)
                advance(i)
                if waiting[i] == "idle" and len(self.pipe) == pipe_before:
                    raise ProtocolError("deadlock: the MMA warp polls, nothing else can move")
                continue
            kind, arg = self.rng.choice(movers + polls)
            if kind == "role":
                advance(arg)
            elif kind == "pipe":
                self._pipe_pop()
            else:
                self.loads.remove(arg)
                self._land(*arg)
        raise ProtocolError("no completion within the step budget")


# ---------------------------------------------------------------------------
# The FP8 kernel (`csrc/decode_fp8_sm100.cu`) has its own protocol:
# - three stages, converted by 8 gather warps (kv_full) and freed by the
#   commit after PV of their tile (kv_empty);
# - QK^T in five parts per tile (latent groups 0-3, RoPE), part i of tile t
#   being item n = 5 t + i of a ring of three TMEM slots: the MMA warp writes
#   slot n % 3 once the four softmax warps have read its previous item
#   (slot_empty) and commits slot_full; the first part also waits for the
#   tile (kv_full) and, at a segment's start, the query tile (q_full); the
#   last commits the stage's qk_done as well;
# - the softmax writes the tile's P into the stage's RoPE chunk (which the
#   RoPE part reads) after that part has completed, and arrives p_full;
# - after converting tile t, the six rewriting gather warps rewrite the codes
#   of tile t-1 as V' (waiting on qk_done: QK^T reads the codes) and arrive
#   v_ready;
# - the MMA warp issues, in order per tile: the five parts of QK^T(t),
#   PV(t-1), and PV(t) at the end of a segment; PV waits p_full and v_ready.
FP8_STAGES = 3


class Fp8Model:
    """Random interleavings of the FP8 kernel's roles; the same checks as
    `Model`.  Part i of tile t is QK^T item n = 5 t + i, written into slot
    n % 3 (use n // 3 of the slot).  `mutation`:
    - "no_slot_wait": the MMA writes a slot without waiting for the softmax
      to have read its previous part;
    - "early_p": the softmax writes P before the RoPE part of QK^T (the last
      reader of the chunk P goes to) has completed;
    - "early_v": the gather rewrites V' without waiting for qk_done;
    - "no_seg_end_pv": PV of a segment's last tile waits for the next tile
      (a deadlock only while the ring has fewer slots than a tile has parts);
    - "early_q": the softmax stages the next segment's query tile before the
      QK^T parts of the segment's last tile have completed."""

    def __init__(self, plan: Plan, seed: int, mutation: Optional[str] = None):
        self.plan, self.rng, self.mut = plan, random.Random(seed), mutation
        self.T = sum(plan.segments)
        self.seg_of, self.first_of_seg, self.last_of_seg = [], set(), set()
        t = 0
        for k, n in enumerate(plan.segments):
            self.first_of_seg.add(t)
            self.last_of_seg.add(t + n - 1)
            self.seg_of += [k] * n
            t += n
        S = FP8_STAGES
        self.kv_full = [Barrier(f"kv_full[{s}]", GATHER_WARPS) for s in range(S)]
        self.kv_empty = [Barrier(f"kv_empty[{s}]", 1) for s in range(S)]
        self.p_full = [Barrier(f"p_full[{s}]", WARPS) for s in range(S)]
        self.qk_done = [Barrier(f"qk_done[{s}]", 1) for s in range(S)]
        self.v_ready = [Barrier(f"v_ready[{s}]", len(FP8_REWRITERS)) for s in range(S)]
        self.slot_full = [Barrier(f"slot_full[{r}]", 1) for r in range(FP8_SLOTS)]
        self.slot_empty = [Barrier(f"slot_empty[{r}]", WARPS) for r in range(FP8_SLOTS)]
        self.q_full = Barrier("q_full", WARPS)
        self.pipe: List[tuple] = []
        self.stage_page: List[Optional[int]] = [None] * S
        self.stage_writers = [0] * S
        self.v_writers = [0] * S
        self.codes_are_v = [False] * S        # the stage's codes were rewritten as V'
        self.rope_is_p = [False] * S          # the RoPE chunk holds P (QK^T of its tile is over)
        self.slot = [None] * FP8_SLOTS        # (tile, part) held by each slot
        self.reading = [set() for _ in range(FP8_SLOTS)]
        self.qk_all_done, self.pv_done = set(), set()
        self.p_written: Dict[int, int] = {}
        self.q_writes: Dict[int, int] = {}
        self.q_seg = -1
        self.o_busy = set()
        self.epilogue_done: Dict[int, int] = {}

    # -- roles -------------------------------------------------------------------
    def gather(self, w):
        ph = lambda t: t // FP8_STAGES  # noqa: E731
        tr = 0
        for t in range(self.T):
            s = t % FP8_STAGES
            yield ("wait", lambda s=s, t=t: self.kv_empty[s].passes(ph(t) - 1))
            prev = self.stage_page[s]
            if prev is not None and prev != t and prev not in self.pv_done:
                raise ProtocolError(f"tile {t} overwrites stage {s} while tile {prev} is still in use")
            yield ("step",)
            self.stage_writers[s] += 1
            if self.stage_writers[s] == GATHER_WARPS:
                self.stage_writers[s] = 0
                self.stage_page[s] = t
                self.rope_is_p[s] = False
                self.codes_are_v[s] = False
            self.kv_full[s].arrive(ph(t))
            yield ("step",)
            while w in FP8_REWRITERS and t + 1 - tr > 1:
                yield from self._rewrite(tr)
                tr += 1
        while w in FP8_REWRITERS and tr < self.T:
            yield from self._rewrite(tr)
            tr += 1

    def _rewrite(self, t):
        s = t % FP8_STAGES
        if self.mut != "early_v":
            yield ("wait", lambda s=s, t=t: self.qk_done[s].passes(t // FP8_STAGES))
        if self.stage_page[s] != t:
            raise ProtocolError(f"V' of tile {t} rewrites stage {s} holding {self.stage_page[s]}")
        if t not in self.qk_all_done:
            raise ProtocolError(f"V' of tile {t} rewrites codes that QK^T still reads")
        yield ("step",)
        self.v_writers[s] += 1
        if self.v_writers[s] == len(FP8_REWRITERS):
            self.v_writers[s] = 0
            self.codes_are_v[s] = True
        self.v_ready[s].arrive(t // FP8_STAGES)

    def mma(self):
        ph = lambda t: t // FP8_STAGES  # noqa: E731
        prev = None
        for t in range(self.T):
            s = t % FP8_STAGES
            yield ("wait", lambda s=s, t=t: self.kv_full[s].passes(ph(t)))
            if t in self.first_of_seg:
                yield ("wait", lambda t=t: self.q_full.passes(self.seg_of[t]))
            for i in range(FP8_PARTS):
                n = FP8_PARTS * t + i
                r, use = n % FP8_SLOTS, n // FP8_SLOTS
                if self.mut != "no_slot_wait":
                    yield ("wait", lambda r=r, use=use: self.slot_empty[r].passes(use - 1))
                self.pipe.append(("QK", t, i, r))
                self.pipe.append(("commit", self.slot_full[r], use))
            self.pipe.append(("commit", self.qk_done[s], ph(t)))
            if prev is not None:
                yield from self._pv(prev)
            prev = t
            if t in self.last_of_seg and self.mut != "no_seg_end_pv":
                yield from self._pv(t)
                prev = None
            yield ("step",)
        if prev is not None:
            yield from self._pv(prev)

    def _pv(self, t):
        s = t % FP8_STAGES
        yield ("wait", lambda s=s, t=t: self.p_full[s].passes(t // FP8_STAGES))
        yield ("wait", lambda s=s, t=t: self.v_ready[s].passes(t // FP8_STAGES))
        self.pipe.append(("PV", t))
        self.pipe.append(("commit", self.kv_empty[s], t // FP8_STAGES))

    def _write_p(self, w, t, s):
        if t not in self.qk_all_done or self.stage_page[s] != t:
            raise ProtocolError(f"softmax {w} writes P of tile {t} into a RoPE chunk QK^T still reads")
        yield ("step",)
        self.rope_is_p[s] = True
        self.p_written[t] = self.p_written.get(t, 0) + 1

    def softmax(self, w):
        live = w < self.plan.live_warps
        self._stage_q(0)
        yield ("step",)
        self.q_full.arrive(0)
        t = 0
        for k, n in enumerate(self.plan.segments):
            any_pv = False
            for j in range(n):
                s = t % FP8_STAGES
                yield ("wait", lambda s=s, t=t: self.kv_full[s].passes(t // FP8_STAGES))
                wrote_p = False
                staged_q = False
                if self.mut == "early_q" and j == n - 1 and k + 1 < len(self.plan.segments):
                    yield from self._stage_next_q(w, t, k)
                    staged_q = True
                for i in range(FP8_PARTS):
                    if i == FP8_PARTS - 1 and self.mut == "early_p" and live:
                        yield from self._write_p(w, t, s)
                        wrote_p = True
                    q = FP8_PARTS * t + i
                    r, use = q % FP8_SLOTS, q // FP8_SLOTS
                    yield ("wait", lambda r=r, use=use: self.slot_full[r].passes(use))
                    if live:
                        if self.slot[r] != (t, i):
                            raise ProtocolError(f"softmax {w} reads slot {r} for part {i} of tile {t}, "
                                                f"holding {self.slot[r]}")
                        self.reading[r].add(w)
                        yield ("step",)
                        self.reading[r].discard(w)
                    self.slot_empty[r].arrive(use)
                need = live and any_pv and bool((self.plan.rescale or {}).get((w, t), False))
                if need:
                    yield ("wait", lambda t=t: self.kv_empty[(t - 1) % FP8_STAGES].passes((t - 1) // FP8_STAGES))
                    if (t - 1) not in self.pv_done:
                        raise ProtocolError(f"softmax {w} rescales O before PV of tile {t - 1} completed")
                    self.o_busy.add(w)
                    yield ("step",)
                    self.o_busy.discard(w)
                if live and not wrote_p:
                    yield from self._write_p(w, t, s)
                self.p_full[s].arrive(t // FP8_STAGES)
                any_pv = True
                if j == n - 1:
                    if k + 1 < len(self.plan.segments) and not staged_q:
                        yield from self._stage_next_q(w, t, k)
                    if live:
                        yield ("wait", lambda s=s, t=t: self.kv_empty[s].passes(t // FP8_STAGES))
                        if t not in self.pv_done:
                            raise ProtocolError(f"softmax {w} reads O for segment {k} before PV of tile {t} completed")
                        self.o_busy.add(w)
                        yield ("step",)
                        self.o_busy.discard(w)
                    self.epilogue_done[k] = self.epilogue_done.get(k, 0) + 1
                t += 1

    def _stage_next_q(self, w, t, k):
        if t not in self.qk_all_done:
            raise ProtocolError(f"softmax {w} overwrites the query tile while QK of tile {t} runs")
        self._stage_q(k + 1)
        yield ("step",)
        self.q_full.arrive(k + 1)

    def _stage_q(self, seg):
        self.q_writes[seg] = self.q_writes.get(seg, 0) + 1
        if self.q_writes[seg] == WARPS:
            self.q_seg = seg

    def _pipe_pop(self):
        item = self.pipe.pop(0)
        kind = item[0]
        if kind == "commit":
            item[1].arrive(item[2])
            return
        t = item[1]
        s = t % FP8_STAGES
        if self.stage_page[s] != t:
            raise ProtocolError(f"{kind} of tile {t} reads stage {s} holding {self.stage_page[s]}")
        if kind == "QK":
            i, r = item[2], item[3]
            if self.q_seg != self.seg_of[t]:
                raise ProtocolError(f"QK part {i} of tile {t} reads the query tile of segment {self.q_seg}")
            if self.codes_are_v[s]:
                raise ProtocolError(f"QK part {i} of tile {t} reads codes already rewritten as V'")
            if self.reading[r]:
                raise ProtocolError(f"QK part {i} of tile {t} overwrites slot {r} while it is being read")
            if i == FP8_PARTS - 1 and self.rope_is_p[s]:
                raise ProtocolError(f"QK RoPE part of tile {t} reads a RoPE chunk that holds P")
            self.slot[r] = (t, i)
            if i == FP8_PARTS - 1:
                self.qk_all_done.add(t)
        else:
            if self.p_written.get(t, 0) != self.plan.live_warps:
                raise ProtocolError(f"PV of tile {t} reads P before every live warp wrote it")
            if not self.codes_are_v[s]:
                raise ProtocolError(f"PV of tile {t} reads V' before the gather warps wrote it")
            if self.o_busy:
                raise ProtocolError(f"PV of tile {t} updates O while warps {sorted(self.o_busy)} use it")
            seg = self.seg_of[t]
            if t in self.first_of_seg and seg > 0 and self.epilogue_done.get(seg - 1, 0) != WARPS:
                raise ProtocolError(f"PV of tile {t} restarts O before the epilogue of segment {seg - 1}")
            self.pv_done.add(t)

    def run(self, max_steps: int = 300000):
        roles = [self.mma()] + [self.softmax(w) for w in range(WARPS)]
        roles += [self.gather(g) for g in range(GATHER_WARPS)]
        waiting = [None] * len(roles)
        done = [False] * len(roles)

        def advance(i):
            try:
                cmd = next(roles[i])
            except StopIteration:
                done[i] = True
                return
            waiting[i] = cmd[1] if cmd[0] == "wait" else None

        for i in range(len(roles)):
            advance(i)
        for _ in range(max_steps):
            if all(done) and not self.pipe:
                return
            movers = [("role", i) for i in range(len(roles)) if not done[i] and (waiting[i] is None or waiting[i]())]
            if self.pipe:
                movers.append(("pipe", None))
            if not movers:
                raise ProtocolError("deadlock: no role can move and nothing is in flight")
            kind, arg = self.rng.choice(movers)
            if kind == "role":
                advance(arg)
            else:
                self._pipe_pop()
        raise ProtocolError("no completion within the step budget")
