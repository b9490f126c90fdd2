"""Model check of the prefill attention kernel's barrier protocol (csrc/prefill_sm100.cu,
`attn_kernel`, dense causal and sparse) on the CPU, in the manner of test_decode_protocol_model.py.

One CTA takes one or two query tiles ("items") of a (sequence, head) and walks n_kv key tiles for
each; the sparse prefill takes n_kv from its key-tile lists.  Roles:

* producer (warp 0): the first item's Q, then key tiles g = 0 .. G-1 of both items through a K ring
  and a V ring of two stages each (K runs one tile ahead of V); the second item's Q replaces the
  first's once the first's score MMAs are done (q_free), issued with the first K tile of the second
  item; a drain waits for every load it issued;
* MMA issuer (warp 1): per item, the Q landed; per tile, K landed, the score MMA into one of three
  TMEM score buffers (after P.V of the tile three back), then P.V of the previous tile (P written,
  V landed); MMAs execute in issue order and each commit arrives once all earlier MMAs are done;
* four softmax warps (one TMEM lane quadrant each): S landed, the running maximum (the rescale of
  O, when a warp's maximum grows, waits for P.V of the previous tile), P written over S; the
  epilogue reads O once the item's last P.V is done.

Barriers follow the PTX rules (arrival count, transaction count, phase completion); every wait
states the phase it needs and fails if the barrier is not within one phase of it.  Every buffer
(K and V stages, Q, the score buffers per lane quadrant, O) records what it holds and fails on a
read of the wrong content or a write over content still to be read.  Two planted mistakes check
that the model notices: a rescale of O without waiting for the previous P.V, and the second item's
Q loaded without waiting for the first's score MMAs.  An item with no key tile (a sparse query tile
whose rows select no visible position, before the key-tile lists gave it its diagonal tile)
deadlocks in the model as it timed out in the kernel."""

import random

import pytest

from test_decode_protocol_model import Barrier, ProtocolViolation

NO_MISTAKE, NO_RESCALE_WAIT, NO_Q_FREE_WAIT = 0, 1, 2
STAGES, SBUF, WARPS = 2, 3, 4


class AttnModel:
    def __init__(self, seed, counts, planted=NO_MISTAKE):
        self.rng = random.Random(seed)
        self.counts = counts                 # n_kv of each item (one or two items)
        self.planted = planted
        self.G = sum(counts)
        self.item_of = [it for it, n in enumerate(counts) for _ in range(n)]
        self.first_of = [sum(counts[:it]) for it in range(len(counts))]
        self.clock = [0]
        self.async_ops = []
        self.mma_queue = []
        B = lambda name, count: Barrier(name, count, self.clock)
        self.q_tma, self.q_free = B("q_tma", 1), B("q_free", 1)
        self.kfull = [B(f"kfull[{i}]", 1) for i in range(STAGES)]
        self.kempty = [B(f"kempty[{i}]", 1) for i in range(STAGES)]
        self.vfull = [B(f"vfull[{i}]", 1) for i in range(STAGES)]
        self.vempty = [B(f"vempty[{i}]", 1) for i in range(STAGES)]
        self.s_full = [B(f"s_full[{i}]", 1) for i in range(SBUF)]
        self.p_full = [B(f"p_full[{i}]", WARPS) for i in range(SBUF)]
        self.pv_done = [B(f"pv_done[{i}]", 1) for i in range(SBUF)]
        # contents: a ring stage holds (tile, landed, read by its MMA)
        self.kst = [None] * STAGES
        self.vst = [None] * STAGES
        self.q = None                        # (item, landed)
        self.q_reads = [0] * len(counts)     # score MMAs of each item executed
        self.sbuf = [[None] * WARPS for _ in range(SBUF)]  # per quadrant: ("S" | "P", tile)
        self.sbuf_pv = [None] * SBUF         # tile whose P.V read the buffer
        self.o_item, self.o_tiles = None, []  # O: item and the tiles accumulated into it
        self.o_read = [[False] * WARPS for _ in counts]  # epilogue reads of each item's O

    # ---------------------------------------------------------------- primitives
    def wait(self, bar, k):
        """Block until phase k of bar has completed (k < 0: before the first phase, complete)."""
        while k >= 0:
            if bar.phase < k:
                raise ProtocolViolation(f"wait for phase {k} of {bar.name} after {bar.phase}: passes early")
            if bar.phase > k + 1:
                raise ProtocolViolation(f"wait for phase {k} of {bar.name} after {bar.phase}: never passes")
            if bar.phase == k + 1:
                return
            yield "blocked"

    def tma(self, bar, nbytes, land):
        bar.arrive_expect_tx(nbytes)

        def op():
            land()
            bar.complete_tx(nbytes)
        self.async_ops.append(op)

    # ---------------------------------------------------------------- roles
    def load_q(self, it):
        if self.q is not None:
            prev = self.q[0]
            if self.q_reads[prev] != self.counts[prev]:
                raise ProtocolViolation(f"Q of item {it} loaded while item {prev} has score MMAs to run")
        self.q = (it, False)

        def land():
            self.q = (it, True)
        self.tma(self.q_tma, 3, land)

    def producer(self):
        n_kv0 = self.counts[0]
        self.load_q(0)
        yield
        nk = nv = 0
        for s in range(self.G + 1):
            if s < self.G:
                g, st = s, s % STAGES
                yield from self.wait(self.kempty[st], g // STAGES - 1)
                prev = self.kst[st]
                if prev is not None and not prev[2]:
                    raise ProtocolViolation(f"K({g}) loaded over K({prev[0]}) before its score MMA read it")
                self.kst[st] = [g, False, False]

                def land_k(st=st, g=g):
                    self.kst[st][1] = True
                self.tma(self.kfull[st], 3, land_k)
                nk += 1
                yield
                if g == n_kv0 and len(self.counts) > 1:
                    if self.planted != NO_Q_FREE_WAIT:
                        yield from self.wait(self.q_free, 0)
                    self.load_q(1)
                    yield
            if s >= 1:
                g, st = s - 1, (s - 1) % STAGES
                yield from self.wait(self.vempty[st], g // STAGES - 1)
                prev = self.vst[st]
                if prev is not None and not prev[2]:
                    raise ProtocolViolation(f"V({g}) loaded over V({prev[0]}) before its P.V read it")
                self.vst[st] = [g, False, False]

                def land_v(st=st, g=g):
                    self.vst[st][1] = True
                self.tma(self.vfull[st], 2, land_v)
                nv += 1
                yield
        # drain: every load issued has landed before the CTA may exit
        for k in range(max(nk - STAGES, 0), nk):
            yield from self.wait(self.kfull[k % STAGES], k // STAGES)
        for k in range(max(nv - STAGES, 0), nv):
            yield from self.wait(self.vfull[k % STAGES], k // STAGES)
        yield from self.wait(self.q_tma, len(self.counts) - 1)

    def issue(self, execute, commits):
        def group():
            execute()
            for bar in commits:
                bar.arrive()
        self.mma_queue.append(group)

    def issue_pv(self, g, first):
        yield from self.wait(self.p_full[g % SBUF], g // SBUF)
        yield from self.wait(self.vfull[g % STAGES], g // STAGES)
        it, buf, st = self.item_of[g], g % SBUF, g % STAGES

        def execute():
            if self.vst[st][:2] != [g, True]:
                raise ProtocolViolation(f"P.V({g}) read V stage {st} holding {self.vst[st]}")
            if self.sbuf[buf] != [("P", g)] * WARPS:
                raise ProtocolViolation(f"P.V({g}) read score buffer {buf} holding {self.sbuf[buf]}")
            self.vst[st][2] = True
            self.sbuf_pv[buf] = g
            if first:
                prev = self.o_item
                if prev is not None and not all(self.o_read[prev]):
                    raise ProtocolViolation(f"P.V({g}) starts O of item {it} before item {prev}'s O was read")
                self.o_item, self.o_tiles = it, [g]
            else:
                if self.o_item != it or self.o_tiles[-1] != g - 1:
                    raise ProtocolViolation(f"P.V({g}) accumulates into O holding {self.o_item}: {self.o_tiles}")
                self.o_tiles.append(g)
        self.issue(execute, [self.vempty[st], self.pv_done[buf]])
        yield

    def mma_issuer(self):
        g = 0
        for it, n_kv in enumerate(self.counts):
            yield from self.wait(self.q_tma, it)
            for j in range(n_kv):
                st, buf = g % STAGES, g % SBUF
                yield from self.wait(self.kfull[st], g // STAGES)
                if g >= SBUF:
                    yield from self.wait(self.pv_done[buf], (g - SBUF) // SBUF)

                def execute(g=g, st=st, buf=buf, it=it):
                    if self.q != (it, True):
                        raise ProtocolViolation(f"score MMA {g} of item {it} read Q holding {self.q}")
                    if self.kst[st][:2] != [g, True]:
                        raise ProtocolViolation(f"score MMA {g} read K stage {st} holding {self.kst[st]}")
                    old = self.sbuf[buf][0]
                    if old is not None and self.sbuf_pv[buf] != old[1]:
                        raise ProtocolViolation(f"S({g}) written over buffer {buf} before P.V({old[1]}) read it")
                    self.kst[st][2] = True
                    self.q_reads[it] += 1
                    self.sbuf[buf] = [("S", g)] * WARPS
                commits = [self.s_full[buf], self.kempty[st]]
                if j == n_kv - 1 and it + 1 < len(self.counts):
                    commits.append(self.q_free)
                self.issue(execute, commits)
                yield
                if j >= 1:
                    yield from self.issue_pv(g - 1, j == 1)
                g += 1
            if n_kv > 0:
                yield from self.issue_pv(g - 1, n_kv == 1)

    def softmax(self, w):
        g = 0
        for it, n_kv in enumerate(self.counts):
            for j in range(n_kv):
                buf = g % SBUF
                yield from self.wait(self.s_full[buf], g // SBUF)
                if self.sbuf[buf][w] != ("S", g):
                    raise ProtocolViolation(f"softmax {w} read S({g}) from a buffer holding {self.sbuf[buf][w]}")
                yield
                if j > 0 and self.rng.random() < 0.4:  # this warp's running maximum grew: rescale O
                    if self.planted != NO_RESCALE_WAIT:
                        yield from self.wait(self.pv_done[(g - 1) % SBUF], (g - 1) // SBUF)
                    want = list(range(self.first_of[it], g))
                    if self.o_item != it or self.o_tiles != want:
                        raise ProtocolViolation(f"softmax {w} rescaled O holding {self.o_item}: {self.o_tiles}, "
                                                f"not tiles {want}")
                    yield
                if self.sbuf[buf][w] != ("S", g):
                    raise ProtocolViolation(f"softmax {w} wrote P({g}) over {self.sbuf[buf][w]}")
                self.sbuf[buf][w] = ("P", g)
                self.p_full[buf].arrive()
                yield
                g += 1
            if n_kv >= 1:
                yield from self.wait(self.pv_done[(g - 1) % SBUF], (g - 1) // SBUF)
                want = list(range(self.first_of[it], g))
                if self.o_item != it or self.o_tiles != want:
                    raise ProtocolViolation(f"softmax {w} read out O holding {self.o_item}: {self.o_tiles}")
                self.o_read[it][w] = True
                yield

    def run(self, max_steps=200_000):
        roles = [self.producer(), self.mma_issuer()] + [self.softmax(w) for w in range(WARPS)]
        for _ in range(max_steps):
            if not (roles or self.async_ops or self.mma_queue):
                if not all(all(r) for r in self.o_read):
                    raise ProtocolViolation("an item's rows were never written")
                return
            choices = [("role", g) for g in roles] + [("async", i) for i in range(len(self.async_ops))]
            if self.mma_queue:
                choices.append(("mma", None))
            self.rng.shuffle(choices)
            for kind, v in choices:
                if kind == "async":
                    self.async_ops.pop(v)()
                    break
                if kind == "mma":
                    self.mma_queue.pop(0)()  # in issue order
                    break
                before = self.clock[0] + len(self.async_ops) + len(self.mma_queue)
                try:
                    res = next(v)
                except StopIteration:
                    roles.remove(v)
                    break
                if res != "blocked" or self.clock[0] + len(self.async_ops) + len(self.mma_queue) != before:
                    break
            else:
                raise ProtocolViolation("deadlock: every role waits")
        raise ProtocolViolation("no termination")


def _dense_causal_counts(n_qt, pi):
    """The items of pair pi of a causal prefill with n_qt query tiles: tile n_qt - 1 - pi, then pi."""
    hi, lo = n_qt - 1 - pi, pi
    return [hi + 1] if hi == lo else [hi + 1, lo + 1]


def test_dense_causal_pairs_hold_under_random_schedules():
    """Every pair of causal prefills with 1..9 query tiles, each under several random interleavings."""
    seed = 0
    for n_qt in range(1, 10):
        for pi in range((n_qt + 1) // 2):
            for _ in range(6):
                AttnModel(seed, _dense_causal_counts(n_qt, pi)).run()
                seed += 1


def test_sparse_counts_hold_under_random_schedules():
    """400 random sparse items (one or two query tiles of 1..8 listed key tiles each)."""
    rng = random.Random(2027)
    for trial in range(400):
        counts = [rng.randint(1, 8) for _ in range(rng.choice([1, 2]))]
        AttnModel(trial, counts).run()


@pytest.mark.parametrize("counts", [[0, 3], [3, 0], [0, 0]])
def test_an_item_without_key_tiles_deadlocks(counts):
    """An empty key-tile list stalls the protocol: with the first item empty the producer waits for a
    q_free that no score MMA commits; with the second empty its Q is never loaded and the MMA issuer
    waits for it.  The key-tile lists therefore give every query tile at least its diagonal tile."""
    with pytest.raises(ProtocolViolation, match="deadlock"):
        AttnModel(1, counts).run()


def test_a_lone_item_without_key_tiles_writes_nothing():
    """A CTA whose only item has no key tile ends without an epilogue: its rows would keep whatever
    the output held, with no flag raised."""
    with pytest.raises(ProtocolViolation, match="never written"):
        AttnModel(1, [0]).run()


def test_model_notices_a_rescale_without_waiting_for_the_previous_pv():
    rng = random.Random(11)
    found = 0
    for trial in range(200):
        counts = [rng.randint(2, 6) for _ in range(rng.choice([1, 2]))]
        try:
            AttnModel(trial, counts, NO_RESCALE_WAIT).run()
        except ProtocolViolation:
            found += 1
    assert found > 0


def test_model_notices_the_second_query_loaded_without_q_free():
    rng = random.Random(12)
    found = 0
    for trial in range(200):
        counts = [rng.randint(1, 6), rng.randint(1, 6)]
        try:
            AttnModel(trial, counts, NO_Q_FREE_WAIT).run()
        except ProtocolViolation:
            found += 1
    assert found > 0
