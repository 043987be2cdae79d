"""Model check of the decode kernel's hand-off protocol (csrc/ssa_decode.cu).

The split kernel's roles talk through mbarriers that a waiter tests by phase
parity only: a wait for the k-th completion of a barrier is right only if,
whenever it is polled, the barrier has completed k or k + 1 phases.  With
fewer it may return early (parity k - 1 looks like k + 1), with more it has
missed its phase.  Which of these can happen depends on every role's speed, so
this test runs the protocol as the kernel writes it -- the TMA producer (3 K
and 2 V ring slots), the query loader (two query tiles), the MMA issuer (S two
tiles ahead, P.V after the hand-off), the four softmax warps (named barrier per
tile, rescale after the previous P.V, epilogue per split) and an in-order
tensor pipe whose commits arrive once every earlier operation is done -- under
many random interleavings, with random per-role speeds, random keep / skip and
rescale decisions and random split sizes (empty splits included), and checks:

* every poll of every wait sees k or k + 1 completed phases (no early return,
  no missed phase) and the run ends without deadlock;
* data hazards: S_g is read after it is computed and overwritten (S_{g+2})
  only after all four warps read it and its P.V ran; P.V reads a complete P
  and a landed V tile; a K / V / query slot is refilled only after its last
  reader ran; an O buffer is reused only after the split that used it was read
  out; O is rescaled and read out only after every earlier P.V of its split;
  the MMA warp reads the keep flag of the tile it is working on.

The checker is itself checked: with the P hand-off on one barrier instead of
one per tile parity (the form that gave up waits on the GPU) it must find a
missed phase.
"""
import random

from protocol_model import Bar, ProtocolError, Sim

KST, VST, NWARP = 3, 2, 4


class Model(Sim):
    def __init__(self, rng, items, per_parity_p_ready=True):
        super().__init__(rng)
        self.items = items  # per split: list of (keep, grow) per tile; [] = empty split
        self.per_parity = per_parity_p_ready
        self.nonempty = [n for n, it in enumerate(items) if it]
        self.tiles = [(n, t) for n in self.nonempty for t in range(len(items[n]))]
        B = Bar
        self.kfull = [B(f"kfull{i}", 1) for i in range(KST)]
        self.kempty = [B(f"kempty{i}", 1) for i in range(KST)]
        self.vfull = [B(f"vfull{i}", 1) for i in range(VST)]
        self.vempty = [B(f"vempty{i}", 1) for i in range(VST)]
        self.q_full = [B(f"q_full{i}", 1) for i in range(2)]
        self.q_empty = [B(f"q_empty{i}", 1) for i in range(2)]
        self.s_full = [B(f"s_full{i}", 1) for i in range(2)]
        self.o_done = [B(f"o_done{i}", 1) for i in range(2)]
        self.p_ready = [B(f"p_ready{i}", NWARP) for i in range(2 if per_parity_p_ready else 1)]
        self.pv_done = B("pv_done", 1)
        # state for the hazard checks
        G = len(self.tiles)
        self.keep = [items[n][t][0] or t == 0 for n, t in self.tiles]
        self.s_exec = [False] * G
        self.s_read = [0] * G
        self.p_written = [0] * G
        self.pv_exec = [False] * G
        self.mma_done_tile = [False] * G  # the MMA warp handed the tile's V slot back
        self.k_slot = [None] * KST
        self.v_slot = [None] * VST
        self.q_buf = [None, None]
        self.o_read = {}
        self.keep_word = [None, None]

    # ------------------------------------------------------------ roles
    def producer(self):
        for g in range(len(self.tiles)):
            if g >= KST:
                yield ("wait", self.kempty[g % KST], g // KST - 1)
            yield ("do", lambda g=g: self.check(g < KST or self.s_exec[g - KST], f"K slot of tile {g} refilled early"))
            yield ("tma", self.kfull[g % KST], lambda g=g: self.k_slot.__setitem__(g % KST, g))
            if g >= VST:
                yield ("wait", self.vempty[g % VST], g // VST - 1)
            yield ("do", lambda g=g: self.check(g < VST or (self.mma_done_tile[g - VST] and (self.pv_exec[g - VST] or not self.keep[g - VST])),
                                              f"V slot of tile {g} refilled early"))
            yield ("tma", self.vfull[g % VST], lambda g=g: self.v_slot.__setitem__(g % VST, g))

    def loader(self):
        for i, n in enumerate(self.nonempty):
            if i >= 2:
                yield ("wait", self.q_empty[i % 2], i // 2 - 1)
            yield ("do", lambda i=i: self._write_q(i))
            yield ("arrive", self.q_full[i % 2])

    def _write_q(self, i):
        if i >= 2:
            prev = [g for g, (n, t) in enumerate(self.tiles) if n == self.nonempty[i - 2]]
            self.check(all(self.s_exec[g] for g in prev), f"query tile of split {i} written before S of split {i - 2} ran")
        self.q_buf[i % 2] = i

    def mma(self):
        tiles, items = self.tiles, self.items
        split_index = {n: i for i, n in enumerate(self.nonempty)}
        cur = {"s": 0}

        def issue_s():
            g = cur["s"]
            n, t = tiles[g]
            i = split_index[n]
            if t == 0:
                yield ("wait", self.q_full[i % 2], i // 2)
            yield ("wait", self.kfull[g % KST], g // KST)
            yield ("op", lambda g=g, i=i: self._exec_s(g, i))
            yield ("commit", self.s_full[g % 2])
            yield ("commit", self.kempty[g % KST])
            if t == len(items[n]) - 1:
                yield ("commit", self.q_empty[i % 2])
            cur["s"] += 1

        for _ in range(2):
            if cur["s"] < len(tiles):
                yield from issue_s()
        pv_count = 0
        for g, (n, t) in enumerate(tiles):
            i = split_index[n]
            if self.per_parity:
                yield ("wait", self.p_ready[g % 2], g // 2)
            else:
                yield ("wait", self.p_ready[0], g)
            yield ("wait", self.vfull[g % VST], g // VST)
            kw = self.keep_word[g % 2]
            self.check(kw is not None and kw[0] == g, f"MMA read the keep flag of tile {kw and kw[0]} for tile {g}")
            if kw[1]:
                yield ("op", lambda g=g, i=i, first=(pv_count == 0): self._exec_pv(g, i, first))
                pv_count += 1
            yield ("do", lambda g=g: self.mma_done_tile.__setitem__(g, True))
            yield ("commit", self.vempty[g % VST])
            yield ("commit", self.pv_done)
            if t == len(items[n]) - 1:
                yield ("commit", self.o_done[i % 2])
                pv_count = 0
            if cur["s"] < len(tiles):
                yield from issue_s()

    def softmax(self, w):
        g, i = 0, 0
        for n, tiles in enumerate(self.items):
            n_pv = 0
            for t, (keep, grow) in enumerate(tiles):
                keep = keep or t == 0
                yield ("wait", self.s_full[g % 2], g // 2)
                yield ("do", lambda g=g: self._read_s(g))
                yield ("nbar",)
                if keep:
                    yield ("do", lambda g=g: self.p_written.__setitem__(g, self.p_written[g] + 1))
                    if grow and n_pv > 0:
                        yield ("wait", self.pv_done, g - 1)
                        yield ("do", lambda g=g, n=n: self._check_o_current(g, n, "rescaled"))
                    n_pv += 1
                if w == 0:
                    yield ("do", lambda g=g, keep=keep: self.keep_word.__setitem__(g % 2, (g, keep)))
                if self.per_parity:
                    yield ("arrive", self.p_ready[g % 2])
                else:
                    yield ("arrive", self.p_ready[0])
                g += 1
            if tiles:
                yield ("wait", self.o_done[i % 2], i // 2)
                yield ("do", lambda n=n, i=i: self._read_o(n, i))
                i += 1

    # ------------------------------------------------------------ checks run by the pipe and the roles
    def _exec_s(self, g, i):
        n, t = self.tiles[g]
        self.check(self.k_slot[g % KST] == g, f"S_{g} read a K slot holding tile {self.k_slot[g % KST]}")
        self.check(self.q_buf[i % 2] == i, f"S_{g} read the query tile of split {self.q_buf[i % 2]}")
        if g >= 2:
            self.check(self.s_read[g - 2] == NWARP, f"S_{g} overwrote S_{g - 2} before every warp read it")
            self.check(self.pv_exec[g - 2] or not self.keep[g - 2], f"S_{g} overwrote P_{g - 2} before its P.V")
        self.s_exec[g] = True

    def _read_s(self, g):
        self.check(self.s_exec[g], f"softmax read S_{g} before it was computed")
        self.s_read[g] += 1

    def _exec_pv(self, g, i, first):
        self.check(self.p_written[g] == NWARP, f"P.V of tile {g} read an incomplete P")
        self.check(self.v_slot[g % VST] == g, f"P.V of tile {g} read a V slot holding tile {self.v_slot[g % VST]}")
        if first and i >= 2:
            self.check(self.o_read.get(i - 2, 0) == NWARP, f"split {i} overwrote the O of split {i - 2} before it was read")
        self.pv_exec[g] = True

    def _check_o_current(self, g, n, what):
        for h, (m, t) in enumerate(self.tiles):
            if m == n and h < g and self.keep[h]:
                self.check(self.pv_exec[h], f"O {what} at tile {g} before the P.V of tile {h}")

    def _read_o(self, n, i):
        self._check_o_current(len(self.tiles), n, "read out")
        self.o_read[i] = self.o_read.get(i, 0) + 1

    def run(self):
        roles = [("producer", self.producer()), ("loader", self.loader()), ("mma", self.mma())]
        roles += [(f"softmax{w}", self.softmax(w)) for w in range(NWARP)]
        Sim.run(self, roles, nbar_size=NWARP)


def _random_items(rng):
    items = []
    for _ in range(rng.randint(1, 5)):
        nt = rng.choice([0, 1, 1, 2, 3, 4, 6])
        items.append([(rng.random() < 0.6, rng.random() < 0.3) for _ in range(nt)])
    return items


def test_protocol_holds_under_random_schedules():
    for seed in range(600):
        rng = random.Random(seed)
        m = Model(rng, _random_items(rng))
        m.run()
        assert all(m.s_exec) and m.o_read == {i: NWARP for i in range(len(m.nonempty))}, seed


def test_checker_finds_the_single_p_ready_barrier_race():
    found = 0
    for seed in range(600):
        rng = random.Random(seed)
        items = [[(rng.random() < 0.5, False) for _ in range(8)]]
        try:
            Model(rng, items, per_parity_p_ready=False).run()
        except ProtocolError as e:
            assert "p_ready" in str(e), e
            found += 1
    assert found > 0
