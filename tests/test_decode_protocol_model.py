"""Model check of the one-token decode kernel's barrier protocol (csrc/decode_sm100.cu) on the CPU.

The kernel's warps hand tiles to one another through mbarriers whose waits test a phase PARITY, so
a wait that runs two phases behind (or ahead) passes early or never.  This model runs every role of
a CTA pair as a Python generator under a random scheduler, together with the asynchronous work
(TMA loads, cp.async gathers, bulk copies between the CTAs, MMA groups):

* producer (warp 0): query TMA into the exchange buffers, the stage ring (dense TMA boxes; top-k
  gathers split with the second gathering warp; FP8 rotary box plus a raw slot), and the early
  split-KV arrival of a segment that does not hold its whole sequence (slot list + decision, after
  the softmax warps have taken that segment's query: the segment count q_seg);
* score-MMA issuer (warp 1), P.V issuer (warp 2; FP8: converts rows 32..63 two tiles ahead),
  FP8 converter (warp 15), second gatherer (warp 15, top-k);
* four exchange warps: S read, fp16 staging, bulk copy into the peer's receive buffer;
* eight softmax warps: query copy, staging + receive read, row-max rendezvous per lane quadrant,
  P into TMEM after the previous P.V, epilogue barriers (sum, merge decision, publish / merge).

Barriers follow the PTX rules (arrival count, transaction count, phase completion).  Every wait
states the phase it needs and fails if the barrier is not within one phase of it; every buffer
records the tile it holds and fails on a read of the wrong tile or a write over an unread one.
Cross-cluster flags and counters are abstracted: the merge decision is random.  Two planted
mistakes check that the model notices: the producer waiting on the query barrier's parity (the
bug the segment count fixed) and an exchange warp not waiting for its staging buffer to be read.
"""

import random

NO_MISTAKE, PARITY_WAIT_ON_QUERY, NO_STAGING_WAIT = 0, 1, 2


class ProtocolViolation(Exception):
    pass


class Barrier:
    """An mbarrier: `count` arrivals and a zero transaction count complete a phase."""

    def __init__(self, name, count, clock):
        self.name, self.count, self.clock = name, count, clock
        self.pending, self.tx, self.phase = count, 0, 0

    def _settle(self):
        self.clock[0] += 1
        if self.pending < 0:
            raise ProtocolViolation(f"{self.name}: more arrivals than its count in phase {self.phase}")
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self):
        self.pending -= 1
        self._settle()

    def arrive_expect_tx(self, n):
        self.tx += n
        self.pending -= 1
        self._settle()

    def complete_tx(self, n):
        self.tx -= n
        self._settle()


class PairDecodeModel:
    def __init__(self, seed, segments, mode, planted=NO_MISTAKE):
        self.rng = random.Random(seed)
        self.segs = segments            # [(tiles, whole)] of the cluster's range
        self.mode = mode                # "dense" | "topk" | "fp8"
        self.planted = planted
        self.NS = 3 if mode == "fp8" else 4
        self.ntiles = sum(k for k, _ in segments)
        self.clock = [0]
        self.async_ops = []
        B = lambda name, count: Barrier(name, count, self.clock)
        per = lambda name, count: [B(f"{name}[{r}]", count) for r in range(2)]
        per2 = lambda name, count: [[B(f"{name}[{r}][{i}]", count) for i in range(2)] for r in range(2)]
        full_count = {"dense": 1, "topk": 2, "fp8": 3}[mode]
        self.full = [[B(f"full[{r}][{s}]", full_count) for s in range(self.NS)] for r in range(2)]
        self.empty = [[B(f"empty[{r}][{s}]", 1) for s in range(self.NS)] for r in range(2)]
        self.q_tma, self.q_full = per("q_tma", 1), per("q_full", 8)
        self.s_full, self.s_empty = per("s_full", 1), per("s_empty", 4)
        self.p_full, self.pv_done = per("p_full", 8), per("pv_done", 1)
        self.x_full, self.x_free = per2("x_full", 1), per2("x_free", 1)
        self.own_ready, self.stg_free = per2("own_ready", 4), per2("stg_free", 8)
        self.red_bar = [[[B(f"red_bar[{r}][{i}][{q}]", 2) for q in range(4)] for i in range(2)] for r in range(2)]
        self.sum_bar, self.pub_bar = per("sum_bar", 8), per("pub_bar", 8)
        self.last_bar, self.mrg_done = per("last_bar", 1), per("mrg_done", 8)
        self.xch_drained = per("xch_drained", 4)
        self.raw_full, self.raw_empty = per2("raw_full", 1), per2("raw_empty", 2)
        self.q_seg = [0, 0]
        # buffer contents
        self.stage = [[None] * self.NS for _ in range(2)]
        self.stage_parts = [[{} for _ in range(self.NS)] for _ in range(2)]
        self.stage_reads = [[set() for _ in range(self.NS)] for _ in range(2)]
        self.raw = [[None, None] for _ in range(2)]
        self.raw_reads = [[0, 0] for _ in range(2)]
        self.S, self.S_reads = [None, None], [set(), set()]
        self.stg = [[[None] * 4 for _ in range(2)] for _ in range(2)]
        self.xr = [[[None] * 4 for _ in range(2)] for _ in range(2)]
        self.stg_read = [[-1, -1] for _ in range(2)]
        self.xr_read = [[-1, -1] for _ in range(2)]
        self.rd_count = [[0, 0] for _ in range(2)]
        self.q_copied = [False, False]
        self.P, self.P_read, self.p_writes = [None, None], [True, True], [{}, {}]
        self.qk_exec, self.pv_exec = [-1, -1], [-1, -1]
        self.Q_seg = [[None] * 8 for _ in range(2)]
        self.slots_of, self.slots_read, self.is_last = [None, None], [set(), set()], [False, False]
        self.copies_reading = {}
        self.copies_landing = [0, 0]
        self.qk_queue, self.pv_queue = [[], []], [[], []]

    # ---------------------------------------------------------------- primitives
    def wait(self, bar, k):
        """Block until phase k of bar has completed (k < 0: a phase before the first, complete)."""
        while k >= 0:
            if bar.phase < k:
                raise ProtocolViolation(f"wait for phase {k} of {bar.name} after {bar.phase}: the parity test "
                                        "passes on an older phase")
            if bar.phase > k + 1:
                raise ProtocolViolation(f"wait for phase {k} of {bar.name} after {bar.phase}: the parity test "
                                        "never passes")
            if bar.phase == k + 1:
                return
            yield "blocked"

    def parity_wait(self, bar, k):
        """A bare parity test (the planted mistake): passes whenever the current phase's parity differs."""
        while (bar.phase & 1) == (k & 1):
            yield "blocked"

    def until(self, pred):
        while not pred():
            yield "blocked"

    def write_stage(self, r, st, t, nparts):
        prev = self.stage[r][st]
        if prev is not None and prev != t and self.stage_reads[r][st] != {"qk", "pv"}:
            raise ProtocolViolation(f"CTA {r}: stage {st} written for tile {t} while tile {prev} is unread")
        d = self.stage_parts[r][st]
        d[t] = d.get(t, 0) + 1
        if d[t] == nparts:
            self.stage[r][st] = t
            self.stage_reads[r][st] = set()
            del d[t]

    # ---------------------------------------------------------------- roles
    def producer(self, r):
        it, nseg_p = 0, 0
        self.q_tma[r].arrive_expect_tx(1)

        def land_query():
            for xi in range(2):
                for q in range(4):
                    self.xr[r][xi][q] = self.stg[r][xi][q] = "Q"
            self.q_tma[r].complete_tx(1)
        self.async_ops.append(land_query)
        for n, (k, whole) in enumerate(self.segs):
            for i in range(k):
                st = it % self.NS
                yield from self.wait(self.empty[r][st], it // self.NS - 1)
                if self.mode == "dense":
                    self.full[r][st].arrive_expect_tx(1)

                    def land(t=it, st=st):
                        self.write_stage(r, st, t, 1)
                        self.full[r][st].complete_tx(1)
                    self.async_ops.append(land)
                elif self.mode == "topk":
                    def land(t=it, st=st):
                        self.write_stage(r, st, t, 2)
                        self.full[r][st].arrive()
                    self.async_ops.append(land)
                else:
                    self.full[r][st].arrive_expect_tx(1)

                    def land_rope(t=it, st=st):
                        self.write_stage(r, st, t, 3)
                        self.full[r][st].complete_tx(1)
                    self.async_ops.append(land_rope)
                    rs = it & 1
                    yield from self.wait(self.raw_empty[r][rs], (it >> 1) - 1)
                    self.raw_full[r][rs].arrive_expect_tx(1)

                    def land_raw(t=it, rs=rs):
                        if self.raw[r][rs] is not None and self.raw_reads[r][rs] != 2:
                            raise ProtocolViolation(f"CTA {r}: raw slot {rs} refilled before both converters read it")
                        self.raw[r][rs], self.raw_reads[r][rs] = t, 0
                        self.raw_full[r][rs].complete_tx(1)
                    self.async_ops.append(land_raw)
                yield
                if i == k - 1 and not whole:
                    if nseg_p > 0:
                        if self.planted == PARITY_WAIT_ON_QUERY:
                            yield from self.parity_wait(self.q_full[r], nseg_p)
                        else:
                            yield from self.until(lambda n2=nseg_p: self.q_seg[r] >= n2 + 1)
                    if self.slots_of[r] is not None and len(self.slots_read[r]) != 8:
                        raise ProtocolViolation(f"CTA {r}: slot list rewritten while segment {self.slots_of[r]}'s "
                                                "epilogue reads it")
                    self.slots_of[r], self.slots_read[r] = n, set()
                    self.is_last[r] = self.rng.random() < 0.5
                    self.last_bar[r].arrive()
                it += 1
            nseg_p += 1

    def gatherer(self, r):
        for t in range(self.ntiles):
            st = t % self.NS
            yield from self.wait(self.empty[r][st], t // self.NS - 1)

            def land(t=t, st=st):
                self.write_stage(r, st, t, 2)
                self.full[r][st].arrive()
            self.async_ops.append(land)
            yield

    def convert(self, r, t):
        rs, st = t & 1, t % self.NS
        yield from self.wait(self.raw_full[r][rs], t >> 1)
        yield from self.wait(self.empty[r][st], t // self.NS - 1)
        if self.raw[r][rs] != t:
            raise ProtocolViolation(f"CTA {r}: converter read raw slot {rs} holding {self.raw[r][rs]} for tile {t}")
        self.raw_reads[r][rs] += 1
        self.write_stage(r, st, t, 3)
        self.full[r][st].arrive()
        self.raw_empty[r][rs].arrive()

    def converter(self, r):
        for t in range(self.ntiles):
            yield from self.convert(r, t)
            yield

    def score_issuer(self, r):
        it = 0
        for n, (k, _) in enumerate(self.segs):
            yield from self.wait(self.q_full[r], n)
            for _ in range(k):
                st = it % self.NS
                yield from self.wait(self.full[r][st], it // self.NS)
                yield from self.wait(self.s_empty[r], it - 1)

                def execute(t=it, st=st, n=n):
                    if self.stage[r][st] != t:
                        raise ProtocolViolation(f"CTA {r}: S({t}) read stage {st} holding {self.stage[r][st]}")
                    if any(s != n for s in self.Q_seg[r]):
                        raise ProtocolViolation(f"CTA {r}: S({t}) read a query of segments {self.Q_seg[r]}")
                    if self.S[r] is not None and len(self.S_reads[r]) != 4:
                        raise ProtocolViolation(f"CTA {r}: S({t}) overwrote S({self.S[r]}) before the exchange read it")
                    self.stage_reads[r][st].add("qk")
                    self.S[r], self.S_reads[r], self.qk_exec[r] = t, set(), t
                    self.s_full[r].arrive()
                self.qk_queue[r].append(execute)
                it += 1
                yield

    def pv_issuer(self, r):
        if self.mode == "fp8":
            for t in range(min(2, self.ntiles)):
                yield from self.convert(r, t)
        for it in range(self.ntiles):
            st = it % self.NS
            yield from self.wait(self.p_full[r], it)

            def execute(t=it, st=st):
                if self.stage[r][st] != t or self.P[r] != t or self.pv_exec[r] != t - 1:
                    raise ProtocolViolation(f"CTA {r}: P.V({t}) on stage tile {self.stage[r][st]}, P of {self.P[r]}")
                self.P_read[r] = True
                self.stage_reads[r][st].add("pv")
                self.pv_exec[r] = t
                self.empty[r][st].arrive()
                self.pv_done[r].arrive()
            self.pv_queue[r].append(execute)
            yield
            if self.mode == "fp8" and it + 2 < self.ntiles:
                yield from self.convert(r, it + 2)

    def exchange(self, r, q):
        peer, key = 1 - r, (r, q)
        for t in range(self.ntiles):
            xi, use = t & 1, t >> 1
            yield from self.wait(self.s_full[r], t)
            if self.S[r] != t:
                raise ProtocolViolation(f"CTA {r}: exchange {q} read S({self.S[r]}) for tile {t}")
            self.S_reads[r].add(q)
            self.s_empty[r].arrive()
            yield
            yield from self.wait(self.x_free[r][xi], use)
            if self.planted != NO_STAGING_WAIT:
                yield from self.wait(self.stg_free[r][xi], use - 1)
            if q == 3:
                self.x_full[r][xi].arrive_expect_tx(4)
            prev = self.stg[r][xi][q]
            if prev == "Q" and self.q_full[r].phase < 1:
                raise ProtocolViolation(f"CTA {r}: staging overwrote the query before every softmax warp copied it")
            if isinstance(prev, int) and self.stg_read[r][xi] < prev:
                raise ProtocolViolation(f"CTA {r}: staging {xi} overwritten (tile {t}) before tile {prev} was read")
            self.stg[r][xi][q] = t
            self.copies_reading[key] = self.copies_reading.get(key, 0) + 1

            def read(t=t, xi=xi):
                if self.stg[r][xi][q] != t:
                    raise ProtocolViolation(f"CTA {r}: bulk copy read staging holding {self.stg[r][xi][q]} for {t}")
                self.copies_reading[key] -= 1
                self.copies_landing[peer] += 1

                def land():
                    self.copies_landing[peer] -= 1
                    held = self.xr[peer][xi][q]
                    if held == "Q" and not self.q_copied[peer]:
                        raise ProtocolViolation(f"CTA {peer}: partial landed on its staged query")
                    if isinstance(held, int) and self.xr_read[peer][xi] < held:
                        raise ProtocolViolation(f"CTA {peer}: partial {t} landed before tile {held} was read")
                    self.xr[peer][xi][q] = t
                    self.x_full[peer][xi].complete_tx(1)
                self.async_ops.append(land)
            self.async_ops.append(read)
            self.own_ready[r][xi].arrive()
            yield
        for t in range(max(0, self.ntiles - 2), self.ntiles):
            yield from self.wait(self.x_free[r][t & 1], (t >> 1) + 1)
        self.xch_drained[r].arrive()

    def softmax(self, r, w):
        peer, quad = 1 - r, (7 + w) & 3
        tb = npart = npub = nmd = 0
        for n, (k, whole) in enumerate(self.segs):
            if n == 0:
                yield from self.wait(self.q_tma[r], 0)
                for xi in range(2):
                    if self.xr[r][xi][quad] != "Q" or self.stg[r][xi][quad] != "Q":
                        raise ProtocolViolation(f"CTA {r}: softmax {w} found its staged query overwritten")
            elif self.qk_exec[r] != tb - 1:
                raise ProtocolViolation(f"CTA {r}: query of segment {n} written while S({self.qk_exec[r]}) pending")
            self.Q_seg[r][w] = n
            self.q_full[r].arrive()
            yield
            if w == 0:
                yield from self.wait(self.q_full[r], n)
                if n == 0:
                    self.q_copied[r] = True
                    self.x_free[peer][0].arrive()
                    self.x_free[peer][1].arrive()
                self.q_seg[r] = n + 1
            for i in range(k):
                xi, use = tb & 1, tb >> 1
                yield from self.wait(self.own_ready[r][xi], use)
                yield from self.wait(self.x_full[r][xi], use)
                if self.stg[r][xi][quad] != tb or self.xr[r][xi][quad] != tb:
                    raise ProtocolViolation(f"CTA {r}: softmax {w} tile {tb} found staging {self.stg[r][xi][quad]}"
                                            f" and receive {self.xr[r][xi][quad]}")
                self.rd_count[r][xi] += 1
                if self.rd_count[r][xi] == 8:
                    self.rd_count[r][xi] = 0
                    self.stg_read[r][xi] = self.xr_read[r][xi] = tb
                self.stg_free[r][xi].arrive()
                yield
                if w == 0:
                    yield from self.wait(self.stg_free[r][xi], use)
                    self.x_free[peer][xi].arrive()
                self.red_bar[r][xi][quad].arrive()
                yield from self.wait(self.red_bar[r][xi][quad], use)
                if i > 0:
                    yield from self.wait(self.pv_done[r], tb - 1)
                if not self.P_read[r]:
                    raise ProtocolViolation(f"CTA {r}: P({tb}) written before P.V({self.P[r]}) read P")
                self.p_writes[r][tb] = self.p_writes[r].get(tb, 0) + 1
                if self.p_writes[r][tb] == 8:
                    self.P[r], self.P_read[r] = tb, False
                self.p_full[r].arrive()
                tb += 1
                yield
            yield from self.wait(self.pv_done[r], tb - 1)
            self.sum_bar[r].arrive()
            yield from self.wait(self.sum_bar[r], n)
            last_segment = n == len(self.segs) - 1
            if last_segment and any(self.stage_parts[r][s] for s in range(self.NS)):
                raise ProtocolViolation(f"CTA {r}: staged epilogue while stage writes are in flight")
            if not whole:
                yield from self.wait(self.last_bar[r], npart)
                npart += 1
                if self.slots_of[r] != n:
                    raise ProtocolViolation(f"CTA {r}: segment {n}'s epilogue read segment {self.slots_of[r]}'s slots")
                self.slots_read[r].add(w)
                if not self.is_last[r]:
                    self.pub_bar[r].arrive()
                    if w == 0:
                        yield from self.wait(self.pub_bar[r], npub)
                    npub += 1
                else:
                    if last_segment and self.rng.random() < 0.5:  # three or more partials bulk-loaded
                        yield from self.wait(self.xch_drained[r], 0)
                        if self.copies_landing[r] or any(self.copies_reading.get((r, q), 0) for q in range(4)):
                            raise ProtocolViolation(f"CTA {r}: exchange buffers reused with copies in flight")
                    self.mrg_done[r].arrive()
                    if w == 0:
                        yield from self.wait(self.mrg_done[r], nmd)
                    nmd += 1
                yield

    # ---------------------------------------------------------------- scheduler
    def run(self, max_steps=2_000_000):
        roles = []
        for r in range(2):
            roles += [self.producer(r), self.score_issuer(r), self.pv_issuer(r)]
            roles += [self.exchange(r, q) for q in range(4)] + [self.softmax(r, w) for w in range(8)]
            if self.mode == "topk":
                roles.append(self.gatherer(r))
            if self.mode == "fp8":
                roles.append(self.converter(r))
        for _ in range(max_steps):
            if not (roles or self.async_ops or any(self.qk_queue) or any(self.pv_queue)):
                return
            choices = [("role", g) for g in roles] + [("async", i) for i in range(len(self.async_ops))]
            choices += [("mma", self.qk_queue[r]) for r in range(2) if self.qk_queue[r]]
            choices += [("mma", self.pv_queue[r]) for r in range(2) if self.pv_queue[r]]
            self.rng.shuffle(choices)
            for kind, v in choices:
                if kind == "async":
                    self.async_ops.pop(v)()
                    break
                if kind == "mma":
                    v.pop(0)()  # MMA groups of one issuer complete in issue order
                    break
                before = self.clock[0] + len(self.async_ops)
                try:
                    res = next(v)
                except StopIteration:
                    roles.remove(v)
                    break
                if res != "blocked" or self.clock[0] + len(self.async_ops) != before:
                    break
            else:
                raise ProtocolViolation("deadlock: every role waits")
        raise ProtocolViolation("no termination")


def _random_case(rng):
    segments = [(rng.randint(1, 5), rng.random() < 0.5) for _ in range(rng.randint(1, 4))]
    return segments, rng.choice(["dense", "topk", "fp8"])


def test_protocol_holds_under_random_schedules():
    """300 random segmentations of a cluster's range (1..4 segments of 1..5 tiles, whole or split),
    each decode variant, each under its own random interleaving: no violation, no deadlock."""
    rng = random.Random(2026)
    for trial in range(300):
        segments, mode = _random_case(rng)
        PairDecodeModel(trial, segments, mode).run()


def test_model_notices_a_parity_wait_on_the_query_barrier():
    """The producer deciding a later split segment after a parity test of the query barrier (instead
    of the softmax warps' segment count) can pass on an older phase after short whole segments and
    rewrite the slot list under a running epilogue; the model finds such schedules."""
    rng = random.Random(5)
    found = 0
    for trial in range(400):
        segments = [(rng.randint(1, 3), rng.random() < 0.6) for _ in range(rng.randint(2, 5))]
        try:
            PairDecodeModel(trial, segments, rng.choice(["dense", "topk", "fp8"]), PARITY_WAIT_ON_QUERY).run()
        except ProtocolViolation:
            found += 1
    assert found > 0


def test_model_notices_a_missing_staging_wait():
    """An exchange warp that refills its fp16 staging buffer without waiting for the softmax warps to
    read the tile two back is caught as an overwrite of an unread tile."""
    rng = random.Random(9)
    found = 0
    for trial in range(200):
        segments, mode = _random_case(rng)
        try:
            PairDecodeModel(trial, segments, mode, NO_STAGING_WAIT).run()
        except ProtocolViolation:
            found += 1
    assert found > 0
