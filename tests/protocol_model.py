"""A small discrete-event model of mbarrier hand-offs between a kernel's roles,
for the protocol tests (test_decode_protocol.py, test_prefill_protocol.py).

Roles are Python generators that yield commands:
  ("wait", bar, k)    wait for the k-th completion (0-based) of `bar`, tested by
                      phase parity as mbarrier.try_wait.parity does;
  ("arrive", bar)     one arrival;
  ("tma", bar, land)  start a load: it lands later, in any order with other
                      loads, runs `land()` and arrives on `bar`;
  ("op", fn)          enqueue a tensor-core operation: the pipe runs `fn()` in
                      issue order;
  ("commit", bar)     enqueue a commit: `bar` gets its arrival once every
                      earlier operation of the pipe has run;
  ("nbar",)           named barrier over the `nbar_size` roles that use it;
  ("do", fn)          run `fn()` now (state updates and hazard checks).
The scheduler picks, step by step, a random role (or the pipe, or the load
engine) with per-run random speeds.  A wait is polled each time its role is
picked: seeing k + 1 completed phases ends it; seeing k + 2 or more (the phase
was missed) or k - 1 (same parity as k + 1: an early return) is an error, as
is a state in which nothing can move.
"""


class ProtocolError(AssertionError):
    pass


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.phase = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending < 0:
            raise ProtocolError(f"{self.name}: more arrivals than expected")
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count


class Sim:
    def __init__(self, rng):
        self.rng = rng
        self.queue = []   # tensor pipe: ("op", fn) / ("commit", bar), in issue order
        self.tma = []     # loads in flight: (bar, land)
        self.nbar_gen, self.nbar_count = 0, 0

    def check(self, ok, what):
        if not ok:
            raise ProtocolError(what)

    def run(self, roles, nbar_size=0, max_steps=500000):
        rng = self.rng
        gens = dict(roles)
        pend = {name: None for name in gens}
        done = set()
        nbar_wait = {}
        speed = {name: rng.uniform(0.05, 1.0) for name in gens}
        speed["pipe"], speed["tma"] = rng.uniform(0.05, 1.0), rng.uniform(0.05, 1.0)
        idle = 0
        for _ in range(max_steps):
            cands = [n for n in gens if n not in done]
            if self.queue:
                cands.append("pipe")
            if self.tma:
                cands.append("tma")
            if not cands:
                return
            who = rng.choices(cands, weights=[speed[c] for c in cands])[0]
            progressed = False
            if who == "pipe":
                kind, x = self.queue.pop(0)
                x() if kind == "op" else x.arrive()
                progressed = True
            elif who == "tma":
                bar, land = self.tma.pop(rng.randrange(len(self.tma)))
                land()
                bar.arrive()
                progressed = True
            else:
                if pend[who] is None:
                    try:
                        pend[who] = next(gens[who])
                    except StopIteration:
                        done.add(who)
                        continue
                cmd = pend[who]
                if cmd[0] == "wait":
                    bar, k = cmd[1], cmd[2]
                    if bar.phase >= k + 2:
                        raise ProtocolError(f"{who} waits for completion {k} of {bar.name}, "
                                            f"which has completed {bar.phase} phases: missed")
                    if bar.phase == k + 1:
                        pend[who], progressed = None, True
                    elif bar.phase % 2 != k % 2:
                        raise ProtocolError(f"{who} waits for completion {k} of {bar.name} "
                                            f"at phase {bar.phase}: early return")
                elif cmd[0] == "nbar":
                    if who not in nbar_wait:
                        nbar_wait[who] = self.nbar_gen
                        self.nbar_count += 1
                        if self.nbar_count == nbar_size:
                            self.nbar_gen += 1
                            self.nbar_count = 0
                        progressed = True
                    if nbar_wait[who] < self.nbar_gen:
                        del nbar_wait[who]
                        pend[who], progressed = None, True
                else:
                    if cmd[0] == "arrive":
                        cmd[1].arrive()
                    elif cmd[0] == "tma":
                        self.tma.append((cmd[1], cmd[2]))
                    elif cmd[0] in ("op", "commit"):
                        self.queue.append((cmd[0], cmd[1]))
                    elif cmd[0] == "do":
                        cmd[1]()
                    else:
                        raise ValueError(cmd)
                    pend[who], progressed = None, True
            idle = 0 if progressed else idle + 1
            if idle > 5000:
                blocked = [(n, pend[n][0], getattr(pend[n][1], "name", None))
                           for n in gens if n not in done and pend[n]]
                raise ProtocolError(f"deadlock: {blocked}")
        raise ProtocolError("step limit")
