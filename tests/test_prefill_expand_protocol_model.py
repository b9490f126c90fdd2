"""Model check of the prefill expansion GEMM's barrier protocol (csrc/prefill_sm100.cu,
`expand_kernel`) on the CPU, in the manner of test_decode_protocol_model.py.

One persistent CTA walks its output tiles (every gridDim-th of them).  Roles:

* producer (warp 0): the K slabs of every tile through a three-stage ring (A and B of one slab per
  stage, one transaction barrier each), a drain that waits for every load it issued;
* MMA issuer (warp 1): per tile, one of two TMEM accumulators once the epilogue has emptied it, the
  slab MMAs as their stages land (each slab's commit frees its stage), then the tile's commit;
* four epilogue warps: the accumulator landed; the leader waits until the previous tile's bulk
  stores have read the output tile in shared memory, and a named barrier holds the four warps until
  then; each warp writes its rows of the output tile, frees the accumulator (one arrival per warp),
  and after a second named barrier the leader issues the tile's bulk stores and commits them as a
  group; at the end it waits for every group.

Bulk stores run asynchronously: a committed group reads the output tile at some later step and then
writes global memory; `wait_group.read 0` returns once every committed group has read.  Every
buffer (stage, accumulator, output tile) records what it holds and fails on a read of the wrong
content or a write over content still to be read.  Two planted mistakes check that the model
notices: the leader skipping the read wait before the tile is rewritten, and the MMA issuer not
waiting for the accumulator to be emptied."""

import random

from test_decode_protocol_model import Barrier, ProtocolViolation

NO_MISTAKE, NO_STORE_READ_WAIT, NO_ACC_EMPTY_WAIT = 0, 1, 2
STAGES, WARPS = 3, 4


class NamedBarrier:
    """bar.sync with a fixed thread count: every participant of a generation blocks until all arrived."""

    def __init__(self, n):
        self.n, self.arrived, self.gen = n, 0, 0

    def sync(self):
        g = self.gen
        self.arrived += 1
        if self.arrived == self.n:
            self.arrived = 0
            self.gen += 1
        while self.gen == g:
            yield "blocked"


class ExpandModel:
    def __init__(self, seed, n_tiles, k_slabs, planted=NO_MISTAKE):
        self.rng = random.Random(seed)
        self.n_tiles, self.k_slabs, self.planted = n_tiles, k_slabs, planted
        self.clock = [0]
        self.async_ops = []
        self.mma_queue = []
        B = lambda name, count: Barrier(name, count, self.clock)
        self.full = [B(f"full[{i}]", 1) for i in range(STAGES)]
        self.empty = [B(f"empty[{i}]", 1) for i in range(STAGES)]
        self.acc_full = [B(f"acc_full[{a}]", 1) for a in range(2)]
        self.acc_empty = [B(f"acc_empty[{a}]", WARPS) for a in range(2)]
        self.named = NamedBarrier(WARPS)
        self.stage = [None] * STAGES              # [(tile, slab), landed, read by its MMA]
        self.acc = [None, None]                   # [tile, slabs accumulated, rows read out per warp]
        self.out_tile = [None] * WARPS            # tile whose rows each warp wrote into the output tile
        self.store_groups = []                    # committed groups whose reads are pending
        self.stored = []                          # tiles whose stores read the output tile

    def wait(self, bar, k):
        while k >= 0:
            if bar.phase < k:
                raise ProtocolViolation(f"wait for phase {k} of {bar.name} after {bar.phase}: passes early")
            if bar.phase > k + 1:
                raise ProtocolViolation(f"wait for phase {k} of {bar.name} after {bar.phase}: never passes")
            if bar.phase == k + 1:
                return
            yield "blocked"

    def producer(self):
        it = 0
        for t in range(self.n_tiles):
            for kc in range(self.k_slabs):
                st = it % STAGES
                yield from self.wait(self.empty[st], it // STAGES - 1)
                prev = self.stage[st]
                if prev is not None and not prev[2]:
                    raise ProtocolViolation(f"slab {(t, kc)} loaded over {prev[0]} before its MMA read it")
                self.stage[st] = [(t, kc), False, False]
                self.full[st].arrive_expect_tx(2)

                def land(st=st):
                    self.stage[st][1] = True
                    self.full[st].complete_tx(2)
                self.async_ops.append(land)
                it += 1
                yield
        for k in range(max(it - STAGES, 0), it):
            yield from self.wait(self.full[k % STAGES], k // STAGES)

    def mma_issuer(self):
        it = 0
        for t in range(self.n_tiles):
            a = t & 1
            if self.planted != NO_ACC_EMPTY_WAIT:
                yield from self.wait(self.acc_empty[a], t // 2 - 1)
            for kc in range(self.k_slabs):
                st = it % STAGES
                yield from self.wait(self.full[st], it // STAGES)

                def execute(t=t, kc=kc, st=st, a=a):
                    if self.stage[st][:2] != [(t, kc), True]:
                        raise ProtocolViolation(f"MMA of slab {(t, kc)} read stage {st} holding {self.stage[st]}")
                    self.stage[st][2] = True
                    if kc == 0:
                        old = self.acc[a]
                        if old is not None and old[2] != WARPS:
                            raise ProtocolViolation(f"tile {t} started in accumulator {a} before tile {old[0]} "
                                                    "was read out")
                        self.acc[a] = [t, 1, 0]
                    else:
                        if self.acc[a][:2] != [t, kc]:
                            raise ProtocolViolation(f"slab {(t, kc)} accumulated into {self.acc[a]}")
                        self.acc[a][1] += 1
                self.mma_queue.append((execute, [self.empty[st]]))
                it += 1
                yield
            self.mma_queue.append((lambda: None, [self.acc_full[a]]))
            yield

    def epilogue(self, w):
        leader = w == 0
        for t in range(self.n_tiles):
            a = t & 1
            yield from self.wait(self.acc_full[a], t // 2)
            if leader and self.planted != NO_STORE_READ_WAIT:
                while self.store_groups:  # wait_group.read 0
                    yield "blocked"
            yield from self.named.sync()
            if self.acc[a][:2] != [t, self.k_slabs]:
                raise ProtocolViolation(f"epilogue {w} read accumulator {a} holding {self.acc[a]} for tile {t}")
            prev = self.out_tile[w]
            if prev is not None and prev not in self.stored:
                raise ProtocolViolation(f"epilogue {w} rewrote the output tile of tile {prev} before its stores "
                                        "read it")
            self.out_tile[w] = t
            yield
            self.acc[a][2] += 1
            self.acc_empty[a].arrive()
            yield from self.named.sync()
            if leader:
                def read(t=t):
                    if self.out_tile != [t] * WARPS:
                        raise ProtocolViolation(f"stores of tile {t} read an output tile holding {self.out_tile}")
                    self.stored.append(t)
                    self.store_groups.remove(read)
                self.store_groups.append(read)
                self.async_ops.append(read)
                yield
        if leader:
            while self.store_groups:  # wait_group 0
                yield "blocked"

    def run(self, max_steps=200_000):
        roles = [self.producer(), self.mma_issuer()] + [self.epilogue(w) for w in range(WARPS)]
        for _ in range(max_steps):
            if not (roles or self.async_ops or self.mma_queue):
                if self.stored != list(range(self.n_tiles)):
                    raise ProtocolViolation(f"tiles stored: {self.stored}")
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
                    execute, commits = self.mma_queue.pop(0)  # in issue order
                    execute()
                    for bar in commits:
                        bar.arrive()
                    break
                before = (self.clock[0], len(self.async_ops), len(self.mma_queue), self.named.gen,
                          self.named.arrived, len(self.store_groups))
                try:
                    res = next(v)
                except StopIteration:
                    roles.remove(v)
                    break
                after = (self.clock[0], len(self.async_ops), len(self.mma_queue), self.named.gen,
                         self.named.arrived, len(self.store_groups))
                if res != "blocked" or after != before:
                    break
            else:
                raise ProtocolViolation("deadlock: every role waits")
        raise ProtocolViolation("no termination")


def test_expand_protocol_holds_under_random_schedules():
    """300 random cases (1..7 tiles per CTA, 1..9 K slabs, the prefill's 8 among them)."""
    rng = random.Random(2028)
    for trial in range(300):
        ExpandModel(trial, rng.randint(1, 7), rng.choice([1, 2, 3, 4, 8, 9])).run()


def test_model_notices_a_missing_store_read_wait():
    rng = random.Random(21)
    found = 0
    for trial in range(200):
        try:
            ExpandModel(trial, rng.randint(2, 6), rng.randint(1, 4), NO_STORE_READ_WAIT).run()
        except ProtocolViolation:
            found += 1
    assert found > 0


def test_model_notices_a_missing_accumulator_wait():
    rng = random.Random(22)
    found = 0
    for trial in range(200):
        try:
            ExpandModel(trial, rng.randint(3, 6), rng.randint(1, 4), NO_ACC_EMPTY_WAIT).run()
        except ProtocolViolation:
            found += 1
    assert found > 0
