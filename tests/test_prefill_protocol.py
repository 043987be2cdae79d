"""Model check of the prefill kernel's hand-off protocol (csrc/ssa_fwd.cu).

One CTA holds two query tiles (A, B) that share every K and V tile.  The roles
as the kernel writes them: warp 0 loads both query tiles once and K into a
2-slot ring (a slot is refilled once the last tile that reads it has its S);
warp 2 loads V_j into a 2-slot ring only after reading both tiles' skip votes
for step j (or hands the slot on without a load); the MMA warp issues, per
step j and tile, the first half of P.V once the softmax signals the first 64
keys' P, the second half once all of P is written, then the tile's next
QK^T; per tile four softmax warps read S, vote (one byte and one arrival per
warp on the step parity's vote barrier), wait for the vote, rescale O when
the running max grew (relying on S(j) completing after every earlier P.V of
the tile), write P in two halves with a hand-off after each, and read O out
at the end.  The tensor pipe runs in issue order; loads land in any order.

Under random interleavings, speeds, visit counts (tile B visits one key tile
more than A on causal diagonals, or none) and keep / rescale decisions, in
skip mode and dense mode, every parity wait must see its own phase, nothing
may deadlock, and the buffer hazards must hold: S read after its QK^T and
overwritten only after every warp read it and its P.V ran; each half of a P.V
reads a complete half of P and a landed V tile; K and V slots refilled only
after their last reader; the vote bytes a reader sees are those of its step;
O rescaled and read out only after every earlier P.V of its tile.
"""
import random

from protocol_model import Bar, ProtocolError, Sim

KST, VST, NWARP, NQT = 2, 2, 4, 2


class Model(Sim):
    def __init__(self, rng, nvis_t, keep, grow, vote_on):
        super().__init__(rng)
        self.nvis_t = nvis_t          # key steps each query tile visits
        self.nvis = max(nvis_t)
        self.vote_on = vote_on
        # keep[t][j]: the tile's decision at step j (its first step is always kept)
        self.keep = [[(not vote_on) or j == 0 or keep[t][j] for j in range(nvis_t[t])] for t in range(NQT)]
        self.grow = grow
        B = Bar
        self.q_full = B("q_full", 1)
        self.k_full = [B(f"k_full{i}", 1) for i in range(KST)]
        self.k_empty = [B(f"k_empty{i}", 1) for i in range(KST)]
        self.v_full = [B(f"v_full{i}", 1) for i in range(VST)]
        self.v_empty = [B(f"v_empty{i}", 1) for i in range(VST)]
        self.s_full = [B(f"s_full{t}", 1) for t in range(NQT)]
        self.vote_bar = [[B(f"vote_bar{t}{par}", NWARP) for par in range(2)] for t in range(NQT)]
        self.p_half = [B(f"p_half{t}", NWARP) for t in range(NQT)]
        self.p_ready = [B(f"p_ready{t}", NWARP) for t in range(NQT)]
        self.o_done = [B(f"o_done{t}", 1) for t in range(NQT)]
        n = self.nvis
        self.q_landed = False
        self.k_slot = [None] * KST
        self.v_slot = [None] * VST
        self.qk_exec = [[False] * n for _ in range(NQT)]
        self.s_read = [[0] * n for _ in range(NQT)]
        self.p_blocks = [[[0, 0] for _ in range(n)] for _ in range(NQT)]
        self.pv_exec = [[[False, False] for _ in range(n)] for _ in range(NQT)]
        self.vote = [[None, None] for _ in range(NQT)]  # (step, bytes written) per parity
        self.v_needed = [any(j < nvis_t[t] and self.keep[t][j] for t in range(NQT)) for j in range(n)]

    def users(self, j):
        return [t for t in range(NQT) if j < self.nvis_t[t]]

    # ------------------------------------------------------------ roles
    def qk_producer(self):
        if self.nvis == 0:
            return
        yield ("tma", self.q_full, lambda: setattr(self, "q_landed", True))
        for j in range(self.nvis):
            if j >= KST:
                yield ("wait", self.k_empty[j % KST], j // KST - 1)
            yield ("do", lambda j=j: self.check(j < KST or all(self.qk_exec[t][j - KST] for t in self.users(j - KST)),
                                                f"K slot of step {j} refilled before its last QK^T"))
            yield ("tma", self.k_full[j % KST], lambda j=j: self.k_slot.__setitem__(j % KST, j))

    def v_producer(self):
        for j in range(self.nvis):
            slot = j % VST
            if j >= VST:
                yield ("wait", self.v_empty[slot], j // VST - 1)
            loaded = False
            for t in self.users(j):
                keep = True
                if self.vote_on:
                    yield ("wait", self.vote_bar[t][j & 1], j >> 1)
                    keep = self._read_vote(t, j, "V producer")
                if keep and not loaded:
                    yield ("do", lambda j=j: self._check_v_free(j))
                    yield ("tma", self.v_full[slot], lambda j=j: self.v_slot.__setitem__(j % VST, j))
                    loaded = True
            if not loaded:
                yield ("arrive", self.v_full[slot])

    def mma(self):
        if self.nvis == 0:
            return
        yield ("wait", self.q_full, 0)
        k_ready = [-1]

        def issue_qk(t, j):
            if k_ready[0] < j:
                yield ("wait", self.k_full[j % KST], j // KST)
                k_ready[0] = j
            yield ("op", lambda t=t, j=j: self._exec_qk(t, j))
            yield ("commit", self.s_full[t])

        def k_last_user(j):
            return 1 if j < self.nvis_t[1] else 0

        for t in range(NQT):
            if self.nvis_t[t] > 0:
                yield from issue_qk(t, 0)
                if k_last_user(0) == t:
                    yield ("commit", self.k_empty[0])
        for j in range(self.nvis):
            slot = j % VST
            v_seen = any_pv = False
            for t in range(NQT):
                if j >= self.nvis_t[t]:
                    continue
                yield ("wait", self.p_half[t], j)
                keep = self._read_vote(t, j, "MMA") if self.vote_on else True
                if keep:
                    if not v_seen:
                        yield ("wait", self.v_full[slot], j // VST)
                        v_seen = True
                    yield ("op", lambda t=t, j=j: self._exec_pv(t, j, 0))
                yield ("wait", self.p_ready[t], j)
                if keep:
                    yield ("op", lambda t=t, j=j: self._exec_pv(t, j, 1))
                    any_pv = True
                if j == self.nvis_t[t] - 1:
                    yield ("commit", self.o_done[t])
                if j + 1 < self.nvis_t[t]:
                    yield from issue_qk(t, j + 1)
                    if k_last_user(j + 1) == t:
                        yield ("commit", self.k_empty[(j + 1) % KST])
            if not v_seen:
                yield ("wait", self.v_full[slot], j // VST)
            if any_pv:
                yield ("commit", self.v_empty[slot])
            else:
                yield ("arrive", self.v_empty[slot])

    def softmax(self, t, w):
        n_pv = 0
        for j in range(self.nvis_t[t]):
            yield ("wait", self.s_full[t], j)
            yield ("do", lambda j=j: self._read_s(t, j))
            keep = self.keep[t][j]
            if self.vote_on:
                yield ("do", lambda j=j: self._write_vote(t, j))
                yield ("arrive", self.vote_bar[t][j & 1])
                yield ("wait", self.vote_bar[t][j & 1], j >> 1)
            if keep:
                if self.grow[t][j] and n_pv > 0:
                    yield ("do", lambda j=j: self._check_o(t, j, "rescaled"))
                yield ("do", lambda j=j: self.p_blocks[t][j].__setitem__(0, self.p_blocks[t][j][0] + 1))
            yield ("arrive", self.p_half[t])
            if keep:
                yield ("do", lambda j=j: self.p_blocks[t][j].__setitem__(1, self.p_blocks[t][j][1] + 1))
                n_pv += 1
            yield ("arrive", self.p_ready[t])
        if self.nvis_t[t] > 0:
            yield ("wait", self.o_done[t], 0)
            yield ("do", lambda: self._check_o(t, self.nvis_t[t], "read out"))

    def run(self):
        roles = [("qk_producer", self.qk_producer()), ("v_producer", self.v_producer()), ("mma", self.mma())]
        roles += [(f"softmax{t}{w}", self.softmax(t, w)) for t in range(NQT) for w in range(NWARP)]
        Sim.run(self, roles)

    # ------------------------------------------------------------ state and checks
    def _write_vote(self, t, j):
        step, n = self.vote[t][j & 1] if self.vote[t][j & 1] and self.vote[t][j & 1][0] == j else (j, 0)
        self.vote[t][j & 1] = (step, n + 1)

    def _read_vote(self, t, j, who):
        v = self.vote[t][j & 1]
        self.check(v is not None and v == (j, NWARP), f"{who} read tile {t}'s votes {v} at step {j}")
        return self.keep[t][j]

    def _check_v_free(self, j):
        if j >= VST:
            for t in self.users(j - VST):
                if self.keep[t][j - VST]:
                    self.check(all(self.pv_exec[t][j - VST]), f"V slot of step {j} refilled before the P.V of step {j - VST}")

    def _exec_qk(self, t, j):
        self.check(self.q_landed, "QK^T before the query tiles landed")
        self.check(self.k_slot[j % KST] == j, f"QK^T({t},{j}) read a K slot holding step {self.k_slot[j % KST]}")
        if j >= 1:
            self.check(self.s_read[t][j - 1] == NWARP, f"S({t},{j}) overwrote S({t},{j - 1}) before every warp read it")
            self.check(not self.keep[t][j - 1] or all(self.pv_exec[t][j - 1]),
                       f"S({t},{j}) overwrote P({t},{j - 1}) before its P.V")
        self.qk_exec[t][j] = True

    def _read_s(self, t, j):
        self.check(self.qk_exec[t][j], f"softmax read S({t},{j}) before its QK^T ran")
        self.s_read[t][j] += 1

    def _exec_pv(self, t, j, half):
        self.check(self.p_blocks[t][j][half] == NWARP, f"P.V half {half} of ({t},{j}) read an incomplete P")
        self.check(self.v_slot[j % VST] == j, f"P.V({t},{j}) read a V slot holding step {self.v_slot[j % VST]}")
        self.pv_exec[t][j][half] = True

    def _check_o(self, t, j, what):
        for h in range(j):
            if self.keep[t][h]:
                self.check(all(self.pv_exec[t][h]), f"O of tile {t} {what} at step {j} before the P.V of step {h}")


def _random_case(rng):
    a = rng.randint(0, 6)
    b = rng.choice([a, a + 1, a + 1, 0 if a > 0 else 1])
    nvis_t = [a, b]
    keep = [[rng.random() < 0.6 for _ in range(8)] for _ in range(NQT)]
    grow = [[rng.random() < 0.3 for _ in range(8)] for _ in range(NQT)]
    return nvis_t, keep, grow, rng.random() < 0.8


def test_prefill_protocol_holds_under_random_schedules():
    runs = 0
    for seed in range(500):
        rng = random.Random(1000 + seed)
        nvis_t, keep, grow, vote_on = _random_case(rng)
        m = Model(rng, nvis_t, keep, grow, vote_on)
        m.run()
        for t in range(NQT):
            assert all(m.qk_exec[t][:nvis_t[t]]), seed
        runs += 1
    assert runs == 500


def test_checker_finds_a_missing_p_half_wait():
    """The same protocol with the MMA warp issuing the first half of P.V
    without waiting for the softmax's first-half hand-off must be caught."""
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
        try:
            NoHalfWait(rng, [4, 5], [[True] * 8] * 2, [[False] * 8] * 2, True).run()
        except ProtocolError:
            found += 1
    assert found > 0
