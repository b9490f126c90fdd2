"""Model check of the CTA-pair decode kernel's barrier protocol (csrc/decode_pair_sm100.cu, the
multi-token decode) on the CPU, in the manner of test_decode_protocol_model.py.

The pair shares its MMAs (tcgen05 cta_group::2, issued by the even CTA): the barriers that gather
work from both CTAs live in the even CTA (stage full, query full, score read, P full, O free) and
the MMA completions arrive on both CTAs at once (score done, per-stage score done, P.V done, stage
empty, query empty).  Roles per CTA: the producer (stage rows of this CTA's positions, the query's
shared-memory slabs), the L2 reload warp (the peer positions' rows of this CTA's latent half after
the score MMA, and the split-KV arrival of a split segment), eight softmax warps (query into TMEM,
S read, row-max rendezvous per head group, V landed, tail rows zeroed, P into shared memory,
epilogue with the partial-sum rendezvous, staged stores in the range's last segment, the merge
decision); and, in the even CTA, the score and P.V issuers.  A planted mistake checks that the
model notices: the reload warp writing the peer rows into the slabs before the score MMA of the
tile has read them.  (The model also shows that the O-free barrier is implied by P full: a
segment's first P.V waits for P from every softmax warp, which each writes only after its
epilogue of the previous segment has read O.)"""

import random

from test_decode_protocol_model import Barrier, ProtocolViolation

NO_MISTAKE, NO_O_FREE_WAIT, NO_SCORE_DONE_WAIT = 0, 1, 2
NS = 2  # stages


class PairKernelModel:
    def __init__(self, seed, segments, planted=NO_MISTAKE):
        self.rng = random.Random(seed)
        self.segs = segments
        self.planted = planted
        self.ntiles = sum(k for k, _ in segments)
        self.clock = [0]
        self.async_ops = []
        B = lambda name, count: Barrier(name, count, self.clock)
        both = lambda name, count: [B(f"{name}[{r}]", count) for r in range(2)]
        # barriers of the even CTA that gather both CTAs' work
        self.full = [B(f"full[{s}]", 1) for s in range(NS)]
        self.q_full = B("q_full", 1 + 16)
        self.s_empty = B("s_empty", 16)
        self.p_full = [B(f"p_full[{i}]", 16) for i in range(2)]
        self.o_free = B("o_free", 16)
        # per-CTA barriers (MMA completions arrive on both CTAs)
        self.empty = [[B(f"empty[{r}][{s}]", 1) for s in range(NS)] for r in range(2)]
        self.qk_done = [[B(f"qk_done[{r}][{s}]", 1) for s in range(NS)] for r in range(2)]
        self.v_full = [[B(f"v_full[{r}][{s}]", 1) for s in range(NS)] for r in range(2)]
        self.s_full, self.q_empty = both("s_full", 1), both("q_empty", 1)
        self.pv_done = [[B(f"pv_done[{r}][{i}]", 1) for i in range(2)] for r in range(2)]
        self.red_bar = [[[B(f"red_bar[{r}][{i}][{g}]", 4) for g in range(2)] for i in range(2)] for r in range(2)]
        self.lsum_bar = [[B(f"lsum_bar[{r}][{g}]", 4) for g in range(2)] for r in range(2)]
        self.last_bar, self.pub_bar = both("last_bar", 1), both("pub_bar", 8)
        self.mrg_done, self.out_bar = both("mrg_done", 8), both("out_bar", 8)
        # contents
        self.own_rows = [[None] * NS for _ in range(2)]     # tile whose own-position rows the stage holds
        self.peer_rows = [[None] * NS for _ in range(2)]    # tile whose reloaded rows the stage holds
        self.stage_qk = [[None] * NS for _ in range(2)]     # tile the score MMA read from the stage
        self.stage_pv = [[None] * NS for _ in range(2)]
        self.q_smem = [None, None]                          # segment of the query slabs in shared memory
        self.q_tmem = [[None] * 8 for _ in range(2)]
        self.S = [None, None]
        self.S_reads = [0, 0]
        self.P = [[None, None] for _ in range(2)]           # [cta][buffer] tile (all 8 warps wrote)
        self.P_writes = [[{}, {}] for _ in range(2)]
        self.P_read = [[True, True] for _ in range(2)]
        self.qk_exec, self.pv_exec = -1, -1
        self.O_read_seg = [[-1] * 8 for _ in range(2)]       # segment whose O each warp has read out
        self.slots_of, self.slots_read, self.is_last = [None, None], [set(), set()], [False, False]
        self.reload_landing = [0, 0]
        self.qk_queue, self.pv_queue = [], []
        self.seg_of_tile, self.first_tile = [], set()
        t = 0
        for n, (k, _) in enumerate(segments):
            self.first_tile.add(t)
            self.seg_of_tile += [n] * k
            t += k

    def wait(self, bar, k):
        while k >= 0:
            if bar.phase < k:
                raise ProtocolViolation(f"wait for phase {k} of {bar.name} after {bar.phase}: passes early")
            if bar.phase > k + 1:
                raise ProtocolViolation(f"wait for phase {k} of {bar.name} after {bar.phase}: never passes")
            if bar.phase == k + 1:
                return
            yield "blocked"

    # ---------------------------------------------------------------- roles
    def producer(self, r):
        it = 0

        def load_q(n):
            if r == 0:
                self.q_full.arrive_expect_tx(2)

            def land():
                if self.q_smem[r] is not None and self.qk_seg_done.get(self.q_smem[r], 0) < 1:
                    raise ProtocolViolation(f"CTA {r}: query slabs of segment {n} landed while segment "
                                            f"{self.q_smem[r]}'s score MMAs may still read them")
                self.q_smem[r] = n
                self.q_full.complete_tx(1)
            self.async_ops.append(land)

        for n, (k, _) in enumerate(self.segs):
            pending = True
            if n > 0:
                yield from self.wait(self.q_empty[r], n - 1)
                load_q(n)
                pending = False
            for i in range(k):
                if pending and i == NS:
                    load_q(n)
                    pending = False
                st = it % NS
                yield from self.wait(self.empty[r][st], it // NS - 1)
                if r == 0:
                    self.full[st].arrive_expect_tx(2)

                def land(t=it, st=st):
                    if self.own_rows[r][st] is not None and self.stage_pv[r][st] != self.own_rows[r][st]:
                        raise ProtocolViolation(f"CTA {r}: stage {st} refilled (tile {t}) before P.V read tile "
                                                f"{self.own_rows[r][st]}")
                    self.own_rows[r][st] = t
                    self.full[st].complete_tx(1)
                self.async_ops.append(land)
                it += 1
                yield
            if pending:
                load_q(n)
            yield

    def reload(self, r):
        it = 0
        for n, (k, whole) in enumerate(self.segs):
            for i in range(k):
                st = it % NS
                if self.planted != NO_SCORE_DONE_WAIT:
                    yield from self.wait(self.qk_done[r][st], it // NS)
                self.v_full[r][st].arrive_expect_tx(1)
                self.reload_landing[r] += 1

                def land(t=it, st=st):
                    self.reload_landing[r] -= 1
                    if self.stage_qk[r][st] != t:
                        raise ProtocolViolation(f"CTA {r}: peer rows of tile {t} landed in slabs the score MMA "
                                                "has not read")
                    self.peer_rows[r][st] = t
                    self.v_full[r][st].complete_tx(1)
                self.async_ops.append(land)
                if i == k - 1 and not whole:
                    if self.slots_of[r] is not None and len(self.slots_read[r]) != 8:
                        raise ProtocolViolation(f"CTA {r}: slot list rewritten under segment {self.slots_of[r]}'s "
                                                "epilogue")
                    self.slots_of[r], self.slots_read[r] = n, set()
                    self.is_last[r] = self.rng.random() < 0.5
                    self.last_bar[r].arrive()
                it += 1
                yield

    def score_issuer(self):
        it = 0
        for n, (k, _) in enumerate(self.segs):
            yield from self.wait(self.q_full, n)
            for _ in range(k):
                st = it % NS
                yield from self.wait(self.full[st], it // NS)
                yield from self.wait(self.s_empty, it - 1)

                def execute(t=it, st=st, n=n):
                    for r in range(2):
                        if self.own_rows[r][st] != t:
                            raise ProtocolViolation(f"S({t}) read CTA {r}'s stage holding {self.own_rows[r][st]}")
                        if self.q_smem[r] != n or any(q != n for q in self.q_tmem[r]):
                            raise ProtocolViolation(f"S({t}) read a query of another segment in CTA {r}")
                        if self.S[r] is not None and self.S_reads[r] != 8:
                            raise ProtocolViolation(f"S({t}) overwrote CTA {r}'s S before its softmax read it")
                        self.S[r], self.S_reads[r] = t, 0
                        self.stage_qk[r][st] = t
                    self.qk_exec = t
                    for r in range(2):
                        self.s_full[r].arrive()
                        self.qk_done[r][st].arrive()
                self.qk_queue.append(execute)
                it += 1
                yield

            def seg_done(n=n):
                self.qk_seg_done[n] = 1
                for r in range(2):
                    self.q_empty[r].arrive()
            self.qk_queue.append(seg_done)

    def pv_issuer(self):
        it = 0
        for n, (k, _) in enumerate(self.segs):
            if n > 0 and self.planted != NO_O_FREE_WAIT:
                yield from self.wait(self.o_free, n - 1)
            for i in range(k):
                st, sb = it % NS, it & 1
                yield from self.wait(self.p_full[sb], it >> 1)

                def execute(t=it, st=st, sb=sb, n=n, first=(i == 0)):
                    for r in range(2):
                        if self.own_rows[r][st] != t or self.peer_rows[r][st] != t:
                            raise ProtocolViolation(f"P.V({t}) read CTA {r}'s V rows of tiles "
                                                    f"{self.own_rows[r][st]}/{self.peer_rows[r][st]}")
                        if self.P[r][sb] != t:
                            raise ProtocolViolation(f"P.V({t}) read CTA {r}'s P of tile {self.P[r][sb]}")
                        if first and n > 0 and any(s < n - 1 for s in self.O_read_seg[r]):
                            raise ProtocolViolation(f"P.V({t}) overwrote CTA {r}'s O before segment {n - 1}'s "
                                                    "epilogue read it")
                        self.P_read[r][sb] = True
                        self.stage_pv[r][st] = t
                    self.pv_exec = t
                    for r in range(2):
                        self.empty[r][st].arrive()
                        self.pv_done[r][sb].arrive()
                self.pv_queue.append(execute)
                it += 1
                yield

    def softmax(self, r, w):
        q = (4 + w) & 3
        grp = q & 1
        it = npart = npub = nmd = nout = 0
        for n, (k, whole) in enumerate(self.segs):
            if n > 0:
                yield from self.wait(self.q_empty[r], n - 1)
            self.q_tmem[r][w] = n
            self.q_full.arrive()
            yield
            for i in range(k):
                sb, st = it & 1, it % NS
                yield from self.wait(self.s_full[r], it)
                if self.S[r] != it:
                    raise ProtocolViolation(f"CTA {r}: softmax {w} read S({self.S[r]}) for tile {it}")
                self.S_reads[r] += 1
                self.s_empty.arrive()
                self.red_bar[r][sb][grp].arrive()
                yield from self.wait(self.red_bar[r][sb][grp], it >> 1)
                if i > 0:
                    yield from self.wait(self.pv_done[r][(it - 1) & 1], (it - 1) >> 1)
                    if self.pv_exec < it - 1:
                        raise ProtocolViolation("O rescaled before the previous P.V")
                yield from self.wait(self.v_full[r][st], it // NS)
                if self.peer_rows[r][st] != it:
                    raise ProtocolViolation(f"CTA {r}: V rows of tile {self.peer_rows[r][st]} at tile {it}")
                if not self.P_read[r][sb] and self.P[r][sb] is not None:
                    raise ProtocolViolation(f"CTA {r}: P buffer {sb} rewritten before P.V({self.P[r][sb]}) read it")
                d = self.P_writes[r][sb]
                d[it] = d.get(it, 0) + 1
                if d[it] == 8:
                    self.P[r][sb], self.P_read[r][sb] = it, False
                    del d[it]
                self.p_full[sb].arrive()
                it += 1
                yield
            yield from self.wait(self.pv_done[r][(it - 1) & 1], (it - 1) >> 1)
            if self.pv_exec < it - 1:
                raise ProtocolViolation("epilogue before the last P.V")
            self.lsum_bar[r][grp].arrive()
            yield from self.wait(self.lsum_bar[r][grp], n)
            self.O_read_seg[r][w] = n
            last_segment = n == len(self.segs) - 1
            if last_segment and self.reload_landing[r]:
                raise ProtocolViolation(f"CTA {r}: staged stores in the stage buffers while a reload lands there")
            if whole:
                if last_segment:
                    self.out_bar[r].arrive()
                    if w == 0:
                        yield from self.wait(self.out_bar[r], nout)
                    nout += 1
            else:
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
                    self.mrg_done[r].arrive()
                    if w == 0:
                        yield from self.wait(self.mrg_done[r], nmd)
                    nmd += 1
                    if last_segment:
                        self.out_bar[r].arrive()
                        if w == 0:
                            yield from self.wait(self.out_bar[r], nout)
                        nout += 1
            self.o_free.arrive()
            yield

    # ---------------------------------------------------------------- scheduler
    def run(self, max_steps=2_000_000):
        self.qk_seg_done = {}
        roles = [self.score_issuer(), self.pv_issuer()]
        for r in range(2):
            roles += [self.producer(r), self.reload(r)] + [self.softmax(r, w) for w in range(8)]
        for _ in range(max_steps):
            if not (roles or self.async_ops or self.qk_queue or self.pv_queue):
                return
            choices = [("role", g) for g in roles] + [("async", i) for i in range(len(self.async_ops))]
            choices += [("mma", qq) for qq in (self.qk_queue, self.pv_queue) if qq]
            self.rng.shuffle(choices)
            for kind, v in choices:
                if kind == "async":
                    self.async_ops.pop(v)()
                    break
                if kind == "mma":
                    v.pop(0)()
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


def _segments(rng):
    return [(rng.randint(1, 5), rng.random() < 0.5) for _ in range(rng.randint(1, 4))]


def test_pair_protocol_holds_under_random_schedules():
    """300 random segmentations of a cluster's range (1..4 query groups of 1..5 tiles, whole or
    split), each under its own random interleaving: no violation, no deadlock."""
    rng = random.Random(4096)
    for trial in range(300):
        PairKernelModel(trial, _segments(rng)).run()


def test_pair_model_notices_a_missing_score_done_wait():
    """A reload warp that does not wait for the tile's score MMA overwrites slabs the MMA still
    reads; the model finds such schedules."""
    rng = random.Random(17)
    found = 0
    for trial in range(200):
        try:
            PairKernelModel(trial, _segments(rng), NO_SCORE_DONE_WAIT).run()
        except ProtocolViolation:
            found += 1
    assert found > 0


def test_o_free_is_implied_by_p_full():
    """Without the O-free wait the protocol still holds: P full already orders a segment's first
    P.V after every softmax warp's epilogue of the previous segment."""
    rng = random.Random(23)
    for trial in range(200):
        segments = [(rng.randint(1, 3), rng.random() < 0.5) for _ in range(rng.randint(2, 4))]
        PairKernelModel(trial, segments, NO_O_FREE_WAIT).run()
