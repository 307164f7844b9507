"""Model check of the stage-ring protocol of the fp16-operand INT4 GEMM, on
the CPU.  The kernel's roles are modelled as coroutines over mbarriers with
the hardware's phase-parity semantics:
  * a TMA producer that fills slot s for stage use u after the slot's
    previous use is consumed (asynchronous completion, as a TMA load);
  * dequantising groups that take the uses u with u % groups == g, wait on
    the slot's full barrier and publish the dequantised operand;
  * the MMA issuer that waits for each use's operand, "multiplies" it into one
    of two accumulators (asynchronous completion, as tcgen05.commit), and
    needs the low-rank operand for each tile;
  * epilogue warps that drain an accumulator, hand it back and prepare the
    next tile's low-rank operand.
Random schedules check that no wait returns on the wrong phase (each consumer
sees exactly the data of the use it waits for), that nothing deadlocks, and
that every tile's accumulator holds exactly its own uses.  A planted
mistake -- more dequantising groups than ring slots -- must be caught.
"""
import random

import pytest


class MBar:
    """mbarrier: arrival count plus transaction bytes; completed phases counted."""

    def __init__(self, count, errors):
        self.count = count
        self.pending = count
        self.tx = 0
        self.completed = 0
        self.errors = errors

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count

    def arrive(self, expect_tx=0):
        self.tx += expect_tx
        self.pending -= 1
        if self.pending < 0:  # more arrivals than the phase expects: undefined on hardware
            self.errors.append("barrier over-arrival")
            self.pending = 0
        self._check()

    def complete_tx(self, n):
        self.tx -= n
        self._check()

    def try_wait(self, parity):
        # true once the phase with this parity has completed: the current
        # (incomplete) phase has the other parity
        return (self.completed & 1) != parity


class Model:
    def __init__(self, nst, groups, ng, lr_stages, tiles, rng):
        self.nst, self.groups, self.ng, self.lr, self.tiles = nst, groups, ng, lr_stages, tiles
        self.rng = rng
        self.errors = []
        e = self.errors
        self.full = [MBar(1, e) for _ in range(nst)]
        self.ready = [MBar(1, e) for _ in range(nst)]   # one arrival per group use
        self.empty = [MBar(1, e) for _ in range(nst)]
        self.acc_full = [MBar(1, e) for _ in range(2)]
        self.acc_empty = [MBar(1, e) for _ in range(2)]
        self.lr_full = MBar(1, e)
        self.slot_codes = [None] * nst    # use id whose codes (or weight rows) are in the slot
        self.slot_operand = [None] * nst  # use id whose dequantised operand is in the slot
        self.acc = [[] for _ in range(2)]
        self.lr_operand = None
        self.tma_ops = []                 # pending TMA landings: complete in any order
        self.mma_ops = []                 # pending MMA completions: in issue order

    def uses(self):
        """(tile, use id, is_low_rank) in ring order."""
        u = 0
        for j in range(self.tiles):
            for _ in range(self.ng):
                yield j, u, False
                u += 1
            for _ in range(self.lr):
                yield j, u, True
                u += 1

    def producer(self):
        for j, u, lr in self.uses():
            s, ph = u % self.nst, (u // self.nst) & 1
            yield ("wait", self.empty[s], ph ^ 1)

            def land(s=s, u=u):
                self.slot_codes[s] = u
                self.full[s].complete_tx(1)
            self.full[s].arrive(expect_tx=1)
            self.tma_ops.append(land)

    def dequant(self, g):
        for j, u, lr in self.uses():
            if u % self.groups != g:
                continue
            s, ph = u % self.nst, (u // self.nst) & 1
            yield ("wait", self.full[s], ph)
            if self.slot_codes[s] != u:
                self.errors.append(f"group {g} read use {self.slot_codes[s]} for use {u}")
            if not lr:
                self.slot_operand[s] = u
            self.ready[s].arrive()

    def mma(self):
        uses = list(self.uses())
        for j in range(self.tiles):
            b = j & 1
            if j >= 2:
                yield ("wait", self.acc_empty[b], ((j >> 1) - 1) & 1)
            for jj, u, lr in uses:
                if jj != j:
                    continue
                s, ph = u % self.nst, (u // self.nst) & 1
                if lr and u == min(x[1] for x in uses if x[0] == j and x[2]):
                    yield ("wait", self.lr_full, j & 1)
                    if self.lr_operand != j:
                        self.errors.append(f"tile {j} low-rank operand is tile {self.lr_operand}")
                yield ("wait", self.ready[s], ph)
                if not lr and self.slot_operand[s] != u:
                    self.errors.append(f"MMA read operand of use {self.slot_operand[s]} for use {u}")
                if self.slot_codes[s] != u:
                    self.errors.append(f"MMA read weight rows of use {self.slot_codes[s]} for use {u}")

                def done(s=s, u=u, b=b, lr=lr, j=j):
                    # the tensor core reads its operands until the MMA completes
                    if self.slot_codes[s] != u or (not lr and self.slot_operand[s] != u):
                        self.errors.append(f"slot {s} overwritten before use {u} completed")
                    if lr and self.lr_operand != j:
                        self.errors.append(f"low-rank operand of tile {j} overwritten in flight")
                    self.acc[b].append(u)
                    self.empty[s].arrive()
                self.mma_ops.append(done)

            def tile_done(b=b):
                self.acc_full[b].arrive()
            self.mma_ops.append(tile_done)

    def epilogue(self):
        uses = list(self.uses())
        if self.lr:
            self.lr_operand = 0
            self.lr_full.arrive()
        for j in range(self.tiles):
            b = j & 1
            yield ("wait", self.acc_full[b], (j >> 1) & 1)
            want = [u for jj, u, _ in uses if jj == j]
            if sorted(self.acc[b]) != want:
                self.errors.append(f"tile {j} accumulator holds {sorted(self.acc[b])}")
            self.acc[b] = []
            if self.lr and j + 1 < self.tiles:
                self.lr_operand = j + 1
                self.lr_full.arrive()
            self.acc_empty[b].arrive()

    def run(self):
        agents = [self.producer(), self.mma(), self.epilogue()] + [self.dequant(g) for g in range(self.groups)]
        blocked = {i: None for i in range(len(agents))}
        live = set(range(len(agents)))
        steps = 0
        while live or self.tma_ops or self.mma_ops:
            steps += 1
            assert steps < 200000
            runnable = [i for i in live if blocked[i] is None or blocked[i][0].try_wait(blocked[i][1])]
            # asynchronous completions are scheduled like agents
            choices = runnable + (["tma"] if self.tma_ops else []) + (["mma"] if self.mma_ops else [])
            if not choices:
                return "deadlock"
            c = self.rng.choice(choices)
            if c == "tma":
                self.tma_ops.pop(self.rng.randrange(len(self.tma_ops)))()
                continue
            if c == "mma":
                self.mma_ops.pop(0)()
                continue
            blocked[c] = None
            try:
                op = next(agents[c])
                blocked[c] = (op[1], op[2])
            except StopIteration:
                live.discard(c)
        return "ok"


CONFIGS = [(nst, ng, lr, tiles) for nst in (3, 4) for ng in (1, 2, 5) for lr in (0, 1, 4) for tiles in (1, 3, 5)]


@pytest.mark.parametrize("nst,ng,lr,tiles", CONFIGS)
def test_one_group_per_slot_is_safe(nst, ng, lr, tiles):
    """The kernel's rule: as many dequantising groups as ring slots."""
    for seed in range(40):
        m = Model(nst, nst, ng, lr, tiles, random.Random(seed))
        assert m.run() == "ok"
        assert not m.errors, m.errors[:3]


@pytest.mark.parametrize("groups", [1, 2])
def test_groups_dividing_the_ring_are_safe(groups):
    for seed in range(60):
        m = Model(4, groups, 3, 1, 3, random.Random(seed))
        assert m.run() == "ok" and not m.errors, m.errors[:3]


def test_more_groups_than_slots_is_caught():
    """Planted mistake: four groups on a three-slot ring.  A group can start
    its parity wait two phases early and read another use's data."""
    bad = 0
    for seed in range(400):
        m = Model(3, 4, 5, 1, 3, random.Random(seed))
        res = m.run()
        bad += res != "ok" or bool(m.errors)
    assert bad > 0


class PairModel:
    """The SM-pair NVFP4 GEMM's protocol.  Two CTAs; the leader's full barrier
    counts both CTAs' TMA bytes; two leader copy warps move each stage's scale
    factors into tensor memory and commit to their ready barriers; the
    leader's MMA warp waits for both, multiplies, and commits the stage's
    empty barrier in both CTAs; one accumulator per SM, handed back by both
    CTAs' epilogues on the leader's barrier, which also collects both CTAs'
    low-rank operands.  ``copy_skips_lr`` plants a known mistake: copy warps
    that do not pass the low-rank stages through their ready barriers."""

    def __init__(self, nst, nks, lr_stages, tiles, rng, copy_skips_lr=False):
        self.nst, self.nks, self.lr, self.tiles, self.rng = nst, nks, lr_stages, tiles, rng
        self.copy_skips_lr = copy_skips_lr
        self.errors = []
        e = self.errors
        self.full = [MBar(1, e) for _ in range(nst)]                       # leader's
        self.empty = [[MBar(1, e) for _ in range(nst)] for _ in range(2)]  # per CTA
        self.ready = {w: [MBar(1, e) for _ in range(nst)] for w in ("a", "b")}
        self.acc_full = [MBar(1, e) for _ in range(2)]                     # per CTA
        self.acc_empty = MBar(2, e)                                        # leader's: both epilogues
        self.lr_full = MBar(2, e)                                          # leader's: both epilogues
        self.slot = [[None] * nst for _ in range(2)]                       # per CTA: use id in the slot
        self.sf = {w: [None] * nst for w in ("a", "b")}                    # tensor-memory scale slots
        self.acc = [[], []]
        self.lr_operand = [None, None]
        self.tma_ops, self.tc_ops = [], {"a": [], "b": [], "mma": []}

    def uses(self):
        u = 0
        for j in range(self.tiles):
            for _ in range(self.nks):
                yield j, u, False
                u += 1
            for _ in range(self.lr):
                yield j, u, True
                u += 1

    def producer(self, rank):
        for j, u, lr in self.uses():
            s, ph = u % self.nst, (u // self.nst) & 1
            yield ("wait", self.empty[rank][s], ph ^ 1)
            if rank == 0:
                self.full[s].arrive(expect_tx=2)

            def land(s=s, u=u, rank=rank):
                self.slot[rank][s] = u
                self.full[s].complete_tx(1)
            self.tma_ops.append(land)

    def copier(self, w):
        for j, u, lr in self.uses():
            if lr and self.copy_skips_lr:
                continue
            s, ph = u % self.nst, (u // self.nst) & 1
            yield ("wait", self.full[s], ph)
            if self.slot[0][s] != u or self.slot[1][s] != u:
                self.errors.append(f"copy warp {w} saw stage data {self.slot[0][s]}/{self.slot[1][s]} for use {u}")

            def copied(s=s, u=u, w=w, lr=lr):
                if not lr:
                    self.sf[w][s] = u
                self.ready[w][s].arrive()
            self.tc_ops[w].append(copied)

    def mma(self):
        uses = list(self.uses())
        for j in range(self.tiles):
            if j > 0:
                yield ("wait", self.acc_empty, (j - 1) & 1)
            first_lr = True
            for jj, u, lr in uses:
                if jj != j:
                    continue
                s, ph = u % self.nst, (u // self.nst) & 1
                if lr and first_lr:
                    first_lr = False
                    yield ("wait", self.lr_full, j & 1)
                yield ("wait", self.ready["a"][s], ph)
                yield ("wait", self.ready["b"][s], ph)

                def done(s=s, u=u, lr=lr, j=j):
                    if self.slot[0][s] != u or self.slot[1][s] != u:
                        self.errors.append(f"MMA of use {u} read stage data {self.slot[0][s]}/{self.slot[1][s]}")
                    if not lr and (self.sf["a"][s] != u or self.sf["b"][s] != u):
                        self.errors.append(f"MMA of use {u} read scales {self.sf['a'][s]}/{self.sf['b'][s]}")
                    if lr and self.lr_operand != [j, j]:
                        self.errors.append(f"MMA of tile {j} read low-rank operands {self.lr_operand}")
                    for r in (0, 1):
                        self.acc[r].append(u)
                        self.empty[r][s].arrive()
                self.tc_ops["mma"].append(done)

            def tile_done():
                for r in (0, 1):
                    self.acc_full[r].arrive()
            self.tc_ops["mma"].append(tile_done)

    def epilogue(self, rank):
        uses = list(self.uses())
        if self.lr:
            self.lr_operand[rank] = 0
            self.lr_full.arrive()
        for j in range(self.tiles):
            yield ("wait", self.acc_full[rank], j & 1)
            want = [u for jj, u, _ in uses if jj == j]
            if sorted(self.acc[rank]) != want:
                self.errors.append(f"CTA {rank} tile {j} accumulator holds {sorted(self.acc[rank])}")
            self.acc[rank] = []
            self.acc_empty.arrive()
            if self.lr and j + 1 < self.tiles:
                self.lr_operand[rank] = j + 1
                self.lr_full.arrive()

    def run(self):
        agents = ([self.producer(0), self.producer(1), self.copier("a"), self.copier("b"), self.mma(),
                   self.epilogue(0), self.epilogue(1)])
        blocked = {i: None for i in range(len(agents))}
        live = set(range(len(agents)))
        steps = 0
        while live or self.tma_ops or any(self.tc_ops.values()):
            steps += 1
            if steps > 400000:
                return "livelock"
            runnable = [i for i in live if blocked[i] is None or blocked[i][0].try_wait(blocked[i][1])]
            choices = (runnable + (["tma"] if self.tma_ops else [])
                       + [k for k, q in self.tc_ops.items() if q])
            if not choices:
                return "deadlock"
            c = self.rng.choice(choices)
            if c == "tma":
                self.tma_ops.pop(self.rng.randrange(len(self.tma_ops)))()
                continue
            if isinstance(c, str):
                self.tc_ops[c].pop(0)()   # each warp's tensor-core operations complete in order
                continue
            blocked[c] = None
            try:
                op = next(agents[c])
                blocked[c] = (op[1], op[2])
            except StopIteration:
                live.discard(c)
        return "ok"


PAIR_CONFIGS = [(nst, nks, lr, tiles) for nst in (4, 5) for nks in (1, 2, 5) for lr in (0, 1, 2)
                for tiles in (1, 3, 5)]


@pytest.mark.parametrize("nst,nks,lr,tiles", PAIR_CONFIGS)
def test_pair_protocol_is_safe(nst, nks, lr, tiles):
    for seed in range(30):
        m = PairModel(nst, nks, lr, tiles, random.Random(seed))
        assert m.run() == "ok"
        assert not m.errors, m.errors[:3]


def test_pair_copy_warps_skipping_low_rank_stages_is_caught():
    """Planted mistake: copy warps whose ready barriers skip the low-rank
    stages fall out of step with the ring once a tile has passed."""
    bad = 0
    for seed in range(100):
        m = PairModel(4, 3, 1, 3, random.Random(seed), copy_skips_lr=True)
        res = m.run()
        bad += res != "ok" or bool(m.errors)
    assert bad > 0


class ChainModel:
    """The fused MLP pair's epilogue hand-off (fc2's T2 = X2 . L1_2 on the
    tensor cores): 16 epilogue warps in four 64-column slices of four warps;
    each tile, the slices take turns writing their X2 rows into one shared
    buffer (x2_full: four warp arrivals per turn); warp 4 (slice 0) also
    holds the issuing thread, which waits for the tile's L1_2 rows (TMA) and
    each turn's rows, issues the turn's MMAs into the T2 accumulator (fresh
    at a row block's first MMA) and commits the buffer back; it reloads L1_2
    once the tile's MMAs have read it.  At the end of a row-block segment the
    four warps of slice 0 drain T2 (t2_drained) before the next segment's
    first MMA may overwrite it.  `shared_free` plants the single "buffer
    free" barrier that let slices two turns ahead pass on a stale parity."""

    def __init__(self, t_begin, t_end, num_n, rng, shared_free=False):
        self.t_begin, self.t_end, self.num_n = t_begin, t_end, num_n
        self.rng, self.shared = rng, shared_free
        self.errors = []
        e = self.errors
        self.x2_full = MBar(4, e)
        self.x2_free = [MBar(1, e) for _ in range(1 if shared_free else 4)]
        self.l1_full = MBar(1, e)
        self.t2_drained = MBar(4, e)
        self.buf = [None] * 4        # (tile, slice) whose rows each lane quarter wrote
        self.l1 = None               # tile whose L1_2 rows are staged
        self.t2 = set()              # (tile, slice) products accumulated in T2
        self.tma_ops = []
        self.tc_ops = []

    def seg_end(self, tile):
        return tile + 1 == self.t_end or (tile + 1) // self.num_n != tile // self.num_n

    def free_bar(self, t):
        return self.x2_free[0] if self.shared else self.x2_free[t]

    def load_l1(self, tile):
        def land():
            self.l1 = tile
            self.l1_full.complete_tx(1)
        self.l1_full.arrive(expect_tx=1)
        self.tma_ops.append(land)

    def warp(self, cs, q):
        issuer = cs == 0 and q == 0
        turn, seg, fresh = 0, 0, True
        if issuer and self.t_begin < self.t_end:
            self.load_l1(self.t_begin)
        for j, tile in enumerate(range(self.t_begin, self.t_end)):
            for t in range(4):
                if cs == t:
                    if self.shared:
                        yield ("wait", self.x2_free[0], (turn & 1) ^ 1)
                    else:
                        yield ("wait", self.x2_free[t], ((j & 1) ^ 1) if t == 0 else (j & 1))
                    self.buf[q] = (tile, t)
                    self.x2_full.arrive()
                if issuer:
                    if t == 0:
                        yield ("wait", self.l1_full, j & 1)
                        if fresh and seg > 0:
                            yield ("wait", self.t2_drained, (seg - 1) & 1)
                    yield ("wait", self.x2_full, turn & 1)
                    f = fresh

                    def mma(tile=tile, t=t, f=f):
                        if self.buf != [(tile, t)] * 4:
                            self.errors.append(f"T2 MMA of tile {tile} slice {t} read rows {self.buf}")
                        if self.l1 != tile:
                            self.errors.append(f"T2 MMA of tile {tile} read L1_2 of tile {self.l1}")
                        if f:
                            self.t2 = set()
                        self.t2.add((tile, t))
                        self.free_bar((t + 1) & 3).arrive()
                    self.tc_ops.append(mma)
                    fresh = False
                turn += 1
            if issuer and tile + 1 < self.t_end:
                if self.shared:
                    yield ("wait", self.x2_free[0], (turn - 1) & 1)
                else:
                    yield ("wait", self.x2_free[0], j & 1)
                self.load_l1(tile + 1)
            if self.seg_end(tile):
                if cs == 0:
                    if self.shared:
                        yield ("wait", self.x2_free[0], (turn - 1) & 1)
                    else:
                        yield ("wait", self.x2_free[0], j & 1)
                    mb = tile // self.num_n
                    want = {(x, s) for x in range(self.t_begin, tile + 1) if x // self.num_n == mb
                            for s in range(4)}
                    if self.t2 != want:
                        self.errors.append(f"drain of row block {mb} read {sorted(self.t2)}")
                    self.t2_drained.arrive()
                seg += 1
                fresh = True

    def run(self):
        agents = [self.warp(cs, q) for cs in range(4) for q in range(4)]
        blocked = {i: None for i in range(len(agents))}
        live = set(range(len(agents)))
        steps = 0
        while live or self.tma_ops or self.tc_ops:
            steps += 1
            if steps > 200000:
                return "livelock"
            runnable = [i for i in live if blocked[i] is None or blocked[i][0].try_wait(blocked[i][1])]
            choices = runnable + (["tma"] if self.tma_ops else []) + (["tc"] if self.tc_ops else [])
            if not choices:
                return "deadlock"
            c = self.rng.choice(choices)
            if c == "tma":
                self.tma_ops.pop(self.rng.randrange(len(self.tma_ops)))()
                continue
            if c == "tc":
                self.tc_ops.pop(0)()   # the issuer's MMAs and commits complete in order
                continue
            blocked[c] = None
            try:
                op = next(agents[c])
                blocked[c] = (op[1], op[2])
            except StopIteration:
                live.discard(c)
        return "ok"


CHAIN_CONFIGS = [(t0, n, nn) for nn in (1, 2, 3) for t0 in (0, 1, 2) for n in (1, 2, 4, 5)]


@pytest.mark.parametrize("t0,n,num_n", CHAIN_CONFIGS)
def test_chain_slice_handoff_is_safe(t0, n, num_n):
    for seed in range(12):
        m = ChainModel(t0, t0 + n, num_n, random.Random(seed))
        assert m.run() == "ok"
        assert not m.errors, m.errors[:3]


def test_chain_single_free_barrier_is_caught():
    """Planted mistake: one shared "buffer free" barrier; slices two turns
    ahead read the parity of a phase that has not begun as complete."""
    bad = 0
    for seed in range(40):
        m = ChainModel(0, 2, 2, random.Random(seed), shared_free=True)
        res = m.run()
        bad += res != "ok" or bool(m.errors)
    assert bad > 0


class QkvExchangeModel:
    """The fused QKV epilogue's per-head exchange: the two warps that hold
    the two 64-column halves of a head (same 32 rows) publish their partial
    sums of squares in shared memory and meet on one mbarrier (two warps'
    arrivals per phase), twice per tile: after writing (then each reads the
    partner's partial) and after reading (so that the next tile's write
    cannot overtake the partner's read).  Tiles whose columns are V skip the
    exchange in both warps.  `one_phase` plants the version without the
    second phase."""

    def __init__(self, tiles, rng, one_phase=False):
        self.tiles, self.rng, self.one_phase = tiles, rng, one_phase
        self.errors = []
        self.bar = MBar(2, self.errors)
        self.red = [None, None]

    def warp(self, w):
        xph = 0
        for j, is_v in enumerate(self.tiles):
            if is_v:
                yield None
                continue
            self.red[w] = (j, w)
            self.bar.arrive()
            yield (self.bar, xph & 1)
            if self.red[1 - w] != (j, 1 - w):
                self.errors.append(f"warp {w} tile {j} read the partner's {self.red[1 - w]}")
            if self.one_phase:
                xph += 1
                continue
            self.bar.arrive()
            yield (self.bar, (xph + 1) & 1)
            xph += 2

    def run(self):
        agents = [self.warp(0), self.warp(1)]
        blocked = [None, None]
        live = {0, 1}
        steps = 0
        while live:
            steps += 1
            if steps > 100000:
                return "livelock"
            runnable = [i for i in live if blocked[i] is None or blocked[i][0].try_wait(blocked[i][1])]
            if not runnable:
                return "deadlock"
            c = self.rng.choice(runnable)
            blocked[c] = None
            try:
                op = next(agents[c])
                blocked[c] = op
            except StopIteration:
                live.discard(c)
        return "ok"


@pytest.mark.parametrize("n", [1, 2, 5, 9])
def test_qkv_exchange_is_safe(n):
    for seed in range(30):
        rng = random.Random(seed)
        tiles = [rng.random() < 0.3 for _ in range(n)]
        m = QkvExchangeModel(tiles, rng)
        assert m.run() == "ok"
        assert not m.errors, m.errors[:3]


def test_qkv_exchange_single_phase_is_caught():
    """Planted mistake: one phase per tile; a warp that runs a tile ahead
    overwrites its partial before the partner has read it."""
    bad = 0
    for seed in range(40):
        m = QkvExchangeModel([False] * 4, random.Random(seed), one_phase=True)
        res = m.run()
        bad += res != "ok" or bool(m.errors)
    assert bad > 0
