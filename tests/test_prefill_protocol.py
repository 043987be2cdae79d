"""Model check of the prefill kernel's hand-off protocol (csrc/ssa_fwd.cu).

One CTA holds two query tiles (A, B) that share every K and V tile.  The roles
as the kernel writes them: warp 0 loads both query tiles once and K into a
2-slot ring (a slot is refilled once the last tile that reads it has its S);
warp 2 loads V_j into a 2-slot ring only after reading both tiles' skip votes
for step j (or hands the slot on without a load); the MMA warp issues, per
step j and tile, the first half of P.V once the softmax signals the first 64
keys' P, the second half once all of P is written, then the tile's next
QK^T; per tile four softmax warps read S, vote (one byte and one arrival per
warp in the step's vote slot, j mod 4; only a warp whose rows are all
negligible waits for the others), rescale O when the running max grew
(relying on S(j) completing after every earlier P.V of the tile), write P in
two halves with a hand-off after each, and read O out at the end.  The tensor
pipe runs in issue order; loads land in any order.

Under random interleavings, speeds, visit counts (tile B visits one key tile
more than A on causal diagonals, or none), per-warp votes and rescale
decisions, in skip mode and dense mode, every parity wait must see its own
phase, nothing may deadlock, and the buffer hazards must hold: S read after
its QK^T and overwritten only after every warp read it and its P.V ran; each
half of a P.V reads a complete half of P and a landed V tile; K and V slots
refilled only after their last reader; the vote bytes a reader sees are those
of its step; O rescaled and read out only after every earlier P.V of its
tile.  With two vote slots instead of four some schedule breaks the last-but-
one rule: after the V producer loads V_j on tile A's vote it still reads tile
B's byte of step j, and a step both tiles skip lets the MMA warp issue tile
B's QK^T two steps on, so tile B's softmax can overwrite that byte first.
With key blocks selected by bitmap the CTA walks the union of its tiles'
selections and a tile takes part only in the steps it selects: its barrier
phases and vote slots count its own steps, the V producer reads only the
taking-part tiles' votes, and the MMA warp issues a tile's next QK^T while
walking the step before it, so that the K ring never waits on a load that
a later step's release would allow.
(The model walks a list of work items with its counters running across them;
the kernel gives each CTA one.)
"""
import random

from protocol_model import Bar, ProtocolError, Sim

KST, VST, NWARP, NQT = 2, 2, 4, 2
VSLOTS = 4


class Model(Sim):
    def __init__(self, rng, items, vote_on, vslots=VSLOTS, skip=True, kst=KST, vst=VST):
        """items: list of (part [2][n], keep [2][n], grow [2][n], votes [2][n][NWARP]);
        part[t][j]: tile t takes part in step j of the CTA's walk.  A list of two
        visit counts stands for the prefix pattern (tile t takes the first n_t)."""
        super().__init__(rng)
        self.kst, self.vst = kst, vst   # ring depths (4 with 64-key tiles, where shared memory allows)
        self.items = [(_as_part(it[0]),) + tuple(it[1:]) for it in items]
        self.vote_on = vote_on
        # skip=False with votes on: key blocks by bitmap without skip-softmax.
        # Every tile that takes part keeps (a warp whose half does not select
        # the key tile still votes 0 and waits), and the V producer loads
        # without reading the votes.
        self.skip = skip
        B = Bar
        self.q_full, self.q_empty = B("q_full", 1), B("q_empty", 1)
        self.q_empty_wait = True
        self.k_full = [B(f"k_full{i}", 1) for i in range(self.kst)]
        self.k_empty = [B(f"k_empty{i}", 1) for i in range(self.kst)]
        self.v_full = [B(f"v_full{i}", 1) for i in range(self.vst)]
        self.v_empty = [B(f"v_empty{i}", 1) for i in range(self.vst)]
        self.s_full = [B(f"s_full{t}", 1) for t in range(NQT)]
        self.vs = vslots
        self.vote_bar = [[B(f"vote_bar{t}{v}", NWARP) for v in range(vslots)] for t in range(NQT)]
        self.p_half = [B(f"p_half{t}", NWARP) for t in range(NQT)]
        self.p_ready = [B(f"p_ready{t}", NWARP) for t in range(NQT)]
        self.o_done = [B(f"o_done{t}", 1) for t in range(NQT)]
        self.q_item = None                       # item whose Q tiles are in shared memory
        self.k_slot = [None] * self.kst               # (item, step) a K slot holds
        self.v_slot = [None] * self.vst
        self.qk = set()                          # (item, t, j) QK^T done
        self.s_read = {}                         # (item, t, j) -> warps that read S
        self.p_blocks = {}                       # (item, t, j) -> [warps done with half 0, half 1]
        self.pv = {}                             # (item, t, j) -> [half 0 ran, half 1 ran]
        self.vote = [[None] * vslots for _ in range(NQT)]   # per slot: (tile step, bytes written)
        self.o_read = set()                      # (item, t) epilogue read O
        self.last_s = [None] * NQT               # (item, j) of tile t's newest S
        self.live = [i for i, it in enumerate(self.items) if _steps(it[0]) > 0]

    def part(self, n, t, j):
        p = self.items[n][0][t]
        return 0 <= j < len(p) and p[j]

    def last(self, n, t):
        """Tile t's last step of item n (-1: none)."""
        p = self.items[n][0][t]
        return max((j for j in range(len(p)) if p[j]), default=-1)

    def keep(self, n, t, j):
        _, keep, _, _ = self.items[n]
        return (not self.vote_on) or (not self.skip) or j == 0 or keep[t][j]

    # ------------------------------------------------------------ roles
    def qk_producer(self):
        gk, nq = 0, 0
        for n in self.live:
            nsteps = _steps(self.items[n][0])
            if nq > 0 and self.q_empty_wait:
                yield ("wait", self.q_empty, nq - 1)
            yield ("do", lambda n=n: self._check_q_free(n))
            yield ("tma", self.q_full, lambda n=n: setattr(self, "q_item", n))
            nq += 1
            for j in range(nsteps):
                if gk >= self.kst:
                    yield ("wait", self.k_empty[gk % self.kst], gk // self.kst - 1)
                yield ("do", lambda gk=gk: self._check_k_free(gk))
                yield ("tma", self.k_full[gk % self.kst], lambda n=n, j=j, gk=gk: self.k_slot.__setitem__(gk % self.kst, (n, j)))
                gk += 1

    def v_producer(self):
        gv, gs = 0, [0, 0]   # gs[t]: tile t's steps so far (its vote slot and phase)
        for n in self.live:
            for j in range(_steps(self.items[n][0])):
                slot = gv % self.vst
                if gv >= self.vst:
                    yield ("wait", self.v_empty[slot], gv // self.vst - 1)
                loaded = False
                for t in range(NQT):
                    if not self.part(n, t, j):
                        continue
                    keep = True
                    if self.vote_on and self.skip:
                        g = gs[t]
                        yield ("wait", self.vote_bar[t][g % self.vs], g // self.vs)
                        keep = self._read_vote(n, t, j, g, "V producer")
                    gs[t] += 1
                    if keep and not loaded:
                        yield ("do", lambda gv=gv: self._check_v_free(gv))
                        yield ("tma", self.v_full[slot], lambda n=n, j=j, s=slot: self.v_slot.__setitem__(s, (n, j)))
                        loaded = True
                if not loaded:
                    yield ("arrive", self.v_full[slot])
                gv += 1

    def next_qk_early(self, n, t, j):
        """Step whose QK^T the MMA warp issues for tile t right after tile t's
        turn in step j: step j + 1 when t takes part in it."""
        return j + 1 if self.part(n, t, j + 1) else None

    def mma(self):
        gk, gv, gs, nq = 0, 0, [0, 0], 0
        k_ready = [-1]
        self.pv_slot_use = {}
        for n in self.live:
            nsteps = _steps(self.items[n][0])
            yield ("wait", self.q_full, nq)
            nq += 1
            qk_left = [sum(1 for t in range(NQT) if self.last(n, t) >= 0)]
            issued = set()

            def issue_qk(t, j, gk=gk, n=n):
                kg = gk + j
                if k_ready[0] < kg:
                    yield ("wait", self.k_full[kg % self.kst], kg // self.kst)
                    k_ready[0] = kg
                issued.add((t, j))
                yield ("op", lambda: self._exec_qk(n, t, j, kg))
                yield ("commit", self.s_full[t])

            def after_qk(t, j, gk=gk, n=n):
                # the last QK^T on K tile j: tile B's when B takes part in step j
                if (1 if self.part(n, 1, j) else 0) == t:
                    yield ("commit", self.k_empty[(gk + j) % self.kst])
                if j == self.last(n, t):
                    qk_left[0] -= 1
                    if qk_left[0] == 0:
                        yield ("commit", self.q_empty)

            for t in range(NQT):
                if self.part(n, t, 0):
                    yield from issue_qk(t, 0)
                    yield from after_qk(t, 0)
            for j in range(nsteps):
                slot = gv % self.vst
                v_seen = any_pv = False
                for t in range(NQT):
                    if self.part(n, t, j):
                        g = gs[t]
                        gs[t] += 1
                        yield ("wait", self.p_half[t], g)
                        keep = self._read_vote(n, t, j, g, "MMA") if self.vote_on else True
                        if keep:
                            if not v_seen:
                                yield ("wait", self.v_full[slot], gv // self.vst)
                                v_seen = True
                            yield ("op", lambda n=n, t=t, j=j, s=slot: self._exec_pv(n, t, j, 0, s))
                        yield ("wait", self.p_ready[t], g)
                        if keep:
                            yield ("op", lambda n=n, t=t, j=j, s=slot: self._exec_pv(n, t, j, 1, s))
                            any_pv = True
                        if j == self.last(n, t):
                            yield ("commit", self.o_done[t])
                    nxt = self.next_qk_early(n, t, j)
                    if nxt is not None and (t, nxt) not in issued:
                        yield from issue_qk(t, nxt)
                        yield from after_qk(t, nxt)
                if not v_seen:
                    yield ("wait", self.v_full[slot], gv // self.vst)
                if any_pv:
                    yield ("commit", self.v_empty[slot])
                else:
                    yield ("arrive", self.v_empty[slot])
                gv += 1
            gk += nsteps

    def softmax(self, t, w):
        gs, oi = 0, 0
        for n in range(len(self.items)):
            _, _, grow, votes = self.items[n]
            n_pv = 0
            for j in range(_steps(self.items[n][0])):
                if not self.part(n, t, j):
                    continue
                g = gs
                gs += 1
                yield ("wait", self.s_full[t], g)
                yield ("do", lambda n=n, j=j: self._read_s(n, t, j))
                keep = self.keep(n, t, j)
                if self.vote_on:
                    # a warp keeps when some row of it does; the tile keeps iff a warp does
                    wkeep = votes[t][j][w] if keep else False
                    if j == 0:
                        wkeep = True
                    yield ("do", lambda g=g: self._write_vote(t, g))
                    yield ("arrive", self.vote_bar[t][g % self.vs])
                    if not wkeep:
                        yield ("wait", self.vote_bar[t][g % self.vs], g // self.vs)
                        yield ("do", lambda n=n, j=j, g=g: self._read_vote(n, t, j, g, f"softmax{t}{w}"))
                if keep:
                    if grow[t][j] and n_pv > 0:
                        yield ("do", lambda n=n, j=j: self._check_o(n, t, j, "rescaled"))
                    yield ("do", lambda n=n, j=j: self._p_done(n, t, j, 0))
                yield ("arrive", self.p_half[t])
                if keep:
                    yield ("do", lambda n=n, j=j: self._p_done(n, t, j, 1))
                    n_pv += 1
                yield ("arrive", self.p_ready[t])
            if self.last(n, t) >= 0:
                yield ("wait", self.o_done[t], oi)
                yield ("do", lambda n=n: self._check_o(n, t, _steps(self.items[n][0]), "read out"))
                yield ("do", lambda n=n: self.o_read.add((n, t, w)))
                oi += 1

    def run(self):
        roles = [("qk_producer", self.qk_producer()), ("v_producer", self.v_producer()), ("mma", self.mma())]
        roles += [(f"softmax{t}{w}", self.softmax(t, w)) for t in range(NQT) for w in range(NWARP)]
        Sim.run(self, roles)

    # ------------------------------------------------------------ state and checks
    def _write_vote(self, t, g):
        v = self.vote[t][g % self.vs]
        step, cnt = v if v and v[0] == g else (g, 0)
        self.vote[t][g % self.vs] = (step, cnt + 1)

    def _read_vote(self, n, t, j, g, who):
        v = self.vote[t][g % self.vs]
        self.check(v is not None and v == (g, NWARP), f"{who} read tile {t}'s votes {v} at its step {g}")
        return self.keep(n, t, j)

    def _check_q_free(self, n):
        prev = [m for m in self.live if m < n]
        if prev:
            m = prev[-1]
            for t in range(NQT):
                for j in range(_steps(self.items[m][0])):
                    if self.part(m, t, j):
                        self.check((m, t, j) in self.qk, f"Q of item {n} loaded before QK^T({m},{t},{j}) ran")

    def _check_k_free(self, gk):
        if gk >= self.kst:
            prev = self.k_slot[gk % self.kst]
            self.check(prev is not None, "K slot refilled before its first load landed")
            m, j = prev
            for t in range(NQT):
                if self.part(m, t, j):
                    self.check((m, t, j) in self.qk, f"K slot of ({m},{j}) refilled before QK^T({m},{t},{j})")

    def _check_v_free(self, gv):
        if gv >= self.vst:
            prev = self.v_slot[gv % self.vst]
            if prev is not None:
                m, j = prev
                for t in range(NQT):
                    if self.part(m, t, j) and self.keep(m, t, j):
                        self.check(all(self.pv.get((m, t, j), [False, False])),
                                   f"V slot of ({m},{j}) refilled before its P.V")

    def _exec_qk(self, n, t, j, kg):
        self.check(self.q_item == n, f"QK^T({n},{t},{j}) read Q tiles of item {self.q_item}")
        self.check(self.k_slot[kg % self.kst] == (n, j), f"QK^T({n},{t},{j}) read a K slot holding {self.k_slot[kg % self.kst]}")
        prev = self.last_s[t]
        if prev is not None:
            m, i = prev
            self.check(self.s_read.get((m, t, i), 0) == NWARP, f"S({n},{t},{j}) overwrote S({m},{t},{i}) unread")
            self.check(not self.keep(m, t, i) or all(self.pv.get((m, t, i), [False, False])),
                       f"S({n},{t},{j}) overwrote P({m},{t},{i}) before its P.V")
        self.last_s[t] = (n, j)
        self.qk.add((n, t, j))

    def _read_s(self, n, t, j):
        self.check((n, t, j) in self.qk, f"softmax read S({n},{t},{j}) before its QK^T ran")
        self.s_read[(n, t, j)] = self.s_read.get((n, t, j), 0) + 1

    def _p_done(self, n, t, j, half):
        b = self.p_blocks.setdefault((n, t, j), [0, 0])
        b[half] += 1

    def _exec_pv(self, n, t, j, half, slot):
        self.check(self.p_blocks.get((n, t, j), [0, 0])[half] == NWARP, f"P.V half {half} of ({n},{t},{j}) read an incomplete P")
        self.check(self.v_slot[slot] == (n, j), f"P.V({n},{t},{j}) read a V slot holding {self.v_slot[slot]}")
        if not any(self.pv.get((n, t, i), [False, False])[0] for i in range(j)) and half == 0:
            # the item's first P.V of this tile overwrites O: the previous item's O must be read out
            prev = [m for m in self.live if m < n and self.last(m, t) >= 0]
            if prev:
                self.check(all((prev[-1], t, w) in self.o_read for w in range(NWARP)),
                           f"first P.V of ({n},{t}) overwrote O of item {prev[-1]} before its epilogue read it")
        self.pv.setdefault((n, t, j), [False, False])[half] = True

    def _check_o(self, n, t, j, what):
        for h in range(j):
            if self.part(n, t, h) and self.keep(n, t, h):
                self.check(all(self.pv.get((n, t, h), [False, False])),
                           f"O of tile {t} of item {n} {what} at step {j} before the P.V of step {h}")


def _as_part(p):
    """Two visit counts -> the prefix pattern; a pattern passes through."""
    if all(isinstance(x, int) for x in p):
        n = max(p)
        return [[j < p[t] for j in range(n)] for t in range(NQT)]
    return p


def _steps(part):
    return max(len(p) for p in part)


def _random_items(rng, count, selected=False):
    """Random work items.  selected=False: each tile visits a prefix of the
    steps (causal diagonals: tile B one more than A, or none); True: key
    blocks selected by bitmap, the walk is the union of two random
    selections, with runs that only one tile takes part in."""
    items = []
    for _ in range(count):
        if selected:
            n = rng.randint(1, 8)
            dens = [rng.choice([0.2, 0.5, 0.9]) for _ in range(NQT)]
            part = [[False] * n for _ in range(NQT)]
            for j in range(n):
                pick = [rng.random() < dens[t] for t in range(NQT)]
                if not any(pick):
                    pick[rng.randrange(NQT)] = True   # the walk lists only selected key tiles
                for t in range(NQT):
                    part[t][j] = pick[t]
            if rng.random() < 0.15:
                # a tile with nothing selected: the walk is the other tile's selection
                t = rng.randrange(NQT)
                part[t] = [False] * n
                part[1 - t] = [True] * n
        else:
            a = rng.randint(0, 5)
            b = rng.choice([a, a + 1, a + 1, 0 if a > 0 else 1])
            part = [a, b]
        keep = [[rng.random() < 0.6 for _ in range(8)] for _ in range(NQT)]
        grow = [[rng.random() < 0.3 for _ in range(8)] for _ in range(NQT)]
        votes = [[[rng.random() < 0.5 for _ in range(NWARP)] for _ in range(8)] for _ in range(NQT)]
        for t in range(NQT):
            for j in range(8):
                if not any(votes[t][j]):
                    votes[t][j][rng.randrange(NWARP)] = True   # a kept tile has a keeping warp
        items.append((part, keep, grow, votes))
    return items


def test_prefill_protocol_holds_under_random_schedules():
    for seed in range(500):
        rng = random.Random(1000 + seed)
        items = _random_items(rng, 1)   # the kernel gives each CTA one item
        m = Model(rng, items, rng.random() < 0.8)
        m.run()
        for n in m.live:
            for t in range(NQT):
                assert all((n, t, j) in m.qk for j in range(items[n][0][t])), seed


def test_protocol_holds_with_selected_key_blocks():
    """Key blocks selected by bitmap: each tile takes part in its own steps of
    the union walk, in skip mode and without skipping."""
    for seed in range(500):
        rng = random.Random(3000 + seed)
        items = _random_items(rng, 1, selected=True)
        m = Model(rng, items, rng.random() < 0.8)
        m.run()
        part = m.items[0][0]
        for t in range(NQT):
            assert all((0, t, j) in m.qk for j in range(len(part[t])) if part[t][j]), seed
            assert not any((0, t, j) in m.qk for j in range(len(part[t])) if not part[t][j]), seed
    for seed in range(100):
        rng = random.Random(4000 + seed)
        Model(rng, _random_items(rng, rng.choice([2, 3]), selected=True), True).run()
    for seed in range(300):
        # without skip-softmax: the V producer does not read the votes
        rng = random.Random(4500 + seed)
        Model(rng, _random_items(rng, 1, selected=True), True, skip=False).run()


def test_checker_finds_a_qk_issued_steps_ahead():
    """Issuing a tile's next QK^T as soon as its turn in the previous step it
    took part in ends (rather than while walking the step just before) waits
    on a K load that only a later step's release allows: must be caught."""
    class Ahead(Model):
        def next_qk_early(self, n, t, j):
            if not self.part(n, t, j):
                return None
            p = self.items[n][0][t]
            return next((i for i in range(j + 1, len(p)) if p[i]), None)

    found = 0
    for seed in range(300):
        rng = random.Random(seed)
        items = _random_items(rng, 1, selected=True)
        n = 6
        items[0] = ([[j in (0, 5) for j in range(n)], [True] * n],) + items[0][1:]
        try:
            Ahead(rng, items, rng.random() < 0.5).run()
        except ProtocolError:
            found += 1
    assert found > 0


def test_checker_finds_votes_counted_by_walk_step():
    """The V producer taking a tile's vote slot and phase from the step of the
    union walk instead of the tile's own step count must be caught."""
    class WalkSlots(Model):
        def v_producer(self):
            gv = 0
            for n in self.live:
                for j in range(_steps(self.items[n][0])):
                    slot = gv % VST
                    if gv >= VST:
                        yield ("wait", self.v_empty[slot], gv // VST - 1)
                    loaded = False
                    for t in range(NQT):
                        if not self.part(n, t, j):
                            continue
                        yield ("wait", self.vote_bar[t][j % self.vs], j // self.vs)
                        keep = self._read_vote(n, t, j, j, "V producer")
                        if keep and not loaded:
                            yield ("tma", self.v_full[slot], lambda n=n, j=j, s=slot: self.v_slot.__setitem__(s, (n, j)))
                            loaded = True
                    if not loaded:
                        yield ("arrive", self.v_full[slot])
                    gv += 1

    found = 0
    for seed in range(200):
        rng = random.Random(seed)
        items = _random_items(rng, 1, selected=True)
        items[0] = ([[j % 2 == 0 for j in range(6)], [True] * 6],) + items[0][1:]
        try:
            WalkSlots(rng, items, True).run()
        except ProtocolError:
            found += 1
    assert found > 0


def test_protocol_holds_with_four_deep_rings():
    """The 4-deep K and V rings of the shapes whose tiles leave room for them."""
    for seed in range(300):
        rng = random.Random(7000 + seed)
        sel = rng.random() < 0.5
        Model(rng, _random_items(rng, 1, selected=sel), rng.random() < 0.8, skip=rng.random() < 0.7,
              kst=4, vst=4).run()


def test_protocol_counters_run_across_items():
    """The same roles walking several items with their counters running on
    (q_empty guarding the query tiles) stay consistent as well."""
    for seed in range(200):
        rng = random.Random(5000 + seed)
        Model(rng, _random_items(rng, rng.choice([2, 3, 4])), rng.random() < 0.8).run()


def test_checker_finds_two_vote_slots_too_few():
    found = 0
    for seed in range(600):
        rng = random.Random(seed)
        # long items with many steps skipped by both tiles
        items = _random_items(rng, 1)
        items[0][0][0], items[0][0][1] = 7, 8
        for t in range(NQT):
            items[0][1][t] = [j % 3 == 0 for j in range(8)]
        try:
            Model(rng, items, True, vslots=2).run()
        except ProtocolError:
            found += 1
    assert found > 0


def test_checker_finds_a_missing_q_empty_wait():
    """Loading the next item's Q without waiting for the previous item's last
    QK^T must be caught."""
    class NoQEmpty(Model):
        def qk_producer(self):
            for cmd in Model.qk_producer(self):
                if cmd[0] == "wait" and cmd[1] is self.q_empty:
                    continue
                yield cmd

    found = 0
    for seed in range(300):
        rng = random.Random(seed)
        items = _random_items(rng, 3)
        for it in items:
            it[0][0], it[0][1] = 2, 3
        try:
            NoQEmpty(rng, items, False).run()
        except ProtocolError:
            found += 1
    assert found > 0


def test_checker_finds_a_missing_p_half_wait():
    """The MMA warp issuing the first half of P.V without waiting for the
    softmax's first-half hand-off must be caught."""
    class NoHalfWait(Model):
        def mma(self):
            for cmd in Model.mma(self):
                if cmd[0] == "wait" and cmd[1] in self.p_half:
                    continue
                yield cmd

        def softmax(self, t, w):
            for cmd in Model.softmax(self, t, w):
                if cmd[0] == "arrive" and cmd[1] in self.p_half:
                    continue  # nobody waits for it any more
                yield cmd

    found = 0
    for seed in range(300):
        rng = random.Random(seed)
        items = _random_items(rng, 1)
        items[0][0][0], items[0][0][1] = 4, 5
        try:
            NoHalfWait(rng, items, False).run()
        except ProtocolError:
            found += 1
    assert found > 0
