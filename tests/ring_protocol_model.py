"""A model of the ring protocol of the tensor-core decode kernel
(paged_kv_cache_339_b200/csrc/pa_decode_tc.cu), run under random
interleavings on the CPU.

Roles, as in the kernel: the scheduler describes ring positions through an
8-entry descriptor queue; the producer copies each position's K (with the
chunk metadata) and V into stage c % 3; per stream, an MMA issuer and a
softmax group consume the positions of their stream. Position c belongs to
stream c & 1 until one stream has ended; from the position after its END the
other stream takes every position (its first chunk there is marked SOLO).
Barriers are mbarriers with phase parity and transaction counts; copies and
MMA commits complete asynchronously (commits in issue order per issuer).

Checked in every schedule: no deadlock; every chunk of a stream is consumed
once, in order, by that stream's consumers; no stage's K or V and no
metadata slot is overwritten while a consumer still needs it. A scheduler
that starves one role for a while is part of the interleavings, so lagging
consumers are explored.

`rules` switches individual protocol rules off, to show that the checks catch
a broken protocol.
"""

from __future__ import annotations

import random

KNST, KQD = 3, 8
END, STOP, SOLO, DATA = "END", "STOP", "SOLO", "DATA"

RULES = ("solo_switch",        # consumers take every position after a SOLO chunk
         "issuer_exits_at_end",  # an MMA issuer stops at its stream's END
         "end_waits_ack",       # END releases K only after the softmax group saw it
         "end_waits_v")         # END releases V only after the producer passed its V half


class Bar:
    """mbarrier: arrival count per phase, transaction bytes, phase parity."""

    def __init__(self, count):
        self.count, self.pending, self.tx, self.phase = count, count, 0, 0

    def arrive(self, tx=0):
        self.tx += tx
        self.pending -= 1
        assert self.pending >= 0, "more arrivals than the barrier's count"
        self._step()

    def complete_tx(self, n):
        self.tx -= n
        assert self.tx >= 0
        self._step()

    def _step(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):
        """try_wait.parity: the phase with this parity has completed."""
        return (self.phase & 1) != parity


class RingModel:
    def __init__(self, rng, items, rules=RULES):
        self.rng, self.items, self.rules = rng, items, set(rules)
        b = self.bar = {}
        for s in range(KNST):
            b["kempty", s] = Bar(1)
            b["vempty", s] = Bar(1)
        for i in range(2 * KNST):
            b["kfull", i] = Bar(1)
            b["vfull", i] = Bar(1)
        for t in range(2):
            for n in ("s_full", "s_free", "p_full", "o_full", "o_free"):
                b[n, t] = Bar(1)
        for q in range(KQD):
            b["desc_full", q] = Bar(1)
            b["desc_empty", q] = Bar(1)
        self.desc = [None] * KQD
        self.meta = [None] * (2 * KNST)   # [position, flags, payload, readers]
        self.kreg = [None] * KNST         # [position, state] of the stage's K
        self.vreg = [None] * KNST
        self.copies = []                  # copies in flight
        self.commits = {0: [], 1: []}     # MMA commits in flight, per issuer
        self.consumed = {0: [], 1: []}

    # -------------------------------------------------------------- roles
    def scheduler(self):
        b = self.bar
        nxt = [[0, 0], [0, 0]]            # per stream: item index, chunk index
        ended = [False, False]
        c, solo, mark, stops = 0, -1, False, 0

        def next_chunk(t):
            it = nxt[t]
            while it[0] < len(self.items[t]) and it[1] >= self.items[t][it[0]]:
                it[0], it[1] = it[0] + 1, 0
            if it[0] >= len(self.items[t]):
                return None
            it[1] += 1
            return (t, it[0], it[1] - 1)

        while True:
            t = solo if solo >= 0 else (c & 1)
            if ended[t]:
                assert ended[1 - t], "a position for an ended stream while the other runs"
                flags, payload = {STOP}, None
            else:
                payload = next_chunk(t)
                if payload is None:
                    ended[t] = True
                    flags = {END}
                    if not ended[1 - t]:
                        solo, mark = 1 - t, True
                else:
                    flags = {DATA}
                    if mark:
                        flags.add(SOLO)
                        mark = False
            q = c % KQD
            yield lambda q=q, c=c: b["desc_empty", q].done(((c // KQD) & 1) ^ 1)
            self.desc[q] = (c, flags, payload)
            b["desc_full", q].arrive()
            c += 1
            if STOP in flags:
                stops += 1
                if stops == 2:
                    return

    def producer(self):
        b = self.bar
        stops, c = 0, 0
        while True:
            q = c % KQD
            yield lambda q=q, c=c: b["desc_full", q].done((c // KQD) & 1)
            pos, flags, payload = self.desc[q]
            assert pos == c
            b["desc_empty", q].arrive()
            s, epar, bi = c % KNST, ((c // KNST) & 1) ^ 1, 2 * (c % KNST) + (c & 1)
            data = DATA in flags
            yield lambda s=s, epar=epar: b["kempty", s].done(epar)
            assert self.kreg[s] is None or self.kreg[s][1] == "free", ("K overwritten", c)
            m = self.meta[bi]
            assert m is None or {"mma", "softmax"} <= m[3] or not ({DATA, END} & m[1]), \
                ("metadata overwritten before it was read", c, m)
            self.meta[bi] = [c, flags, payload, set()]
            self.kreg[s] = [c, "loading" if data else "free"]
            if data:
                b["kfull", bi].arrive(tx=1)
                self.copies.append(("k", s, bi, c))
            else:
                b["kfull", bi].arrive()
            yield lambda s=s, epar=epar: b["vempty", s].done(epar)
            assert self.vreg[s] is None or self.vreg[s][1] == "free", ("V overwritten", c)
            self.vreg[s] = [c, "loading" if data else "free"]
            if data:
                b["vfull", bi].arrive(tx=1)
                self.copies.append(("v", s, bi, c))
            else:
                b["vfull", bi].arrive()
            if STOP in flags:
                stops += 1
                if stops == 2:
                    return
            c += 1

    def _read_meta(self, c, bi, who):
        m = self.meta[bi]
        assert m[0] == c, (who, "read the metadata of another position", c, m[0])
        m[3].add(who)
        return m[1], m[2]

    def issuer(self, t):
        b = self.bar
        n, c, step = 0, t, 2
        while True:
            s, fpar, bi = c % KNST, (c // (2 * KNST)) & 1, 2 * (c % KNST) + (c & 1)
            yield lambda bi=bi, fpar=fpar: b["kfull", bi].done(fpar)
            flags, payload = self._read_meta(c, bi, "mma")
            if STOP in flags:
                return
            if SOLO in flags and "solo_switch" in self.rules:
                step = 1
            par = n & 1
            if END in flags:
                if "end_waits_ack" in self.rules:
                    yield lambda par=par: b["p_full", t].done(par)
                self.kreg[s][1] = "free"
                b["kempty", s].arrive()
                if "end_waits_v" in self.rules:
                    yield lambda bi=bi, fpar=fpar: b["vfull", bi].done(fpar)
                self.vreg[s][1] = "free"
                b["vempty", s].arrive()
                if "issuer_exits_at_end" in self.rules:
                    return
                c += 2
                continue
            assert payload[0] == t, ("a chunk of the other stream", t, payload)
            yield lambda par=par: b["s_free", t].done(par ^ 1)
            assert self.kreg[s] == [c, "ready"], ("K not landed", c, self.kreg[s])
            self.kreg[s][1] = "reading"
            self.commits[t].append(("score", s, c))
            yield lambda par=par: b["p_full", t].done(par)
            yield lambda par=par: b["o_free", t].done(par ^ 1)
            yield lambda bi=bi, fpar=fpar: b["vfull", bi].done(fpar)
            assert self.vreg[s] == [c, "ready"], ("V not landed", c, self.vreg[s])
            self.vreg[s][1] = "reading"
            self.commits[t].append(("pv", s, c))
            n += 1
            c += step

    def softmax(self, t):
        b = self.bar
        n, c, step = 0, t, 2
        while True:
            bi, fpar = 2 * (c % KNST) + (c & 1), (c // (2 * KNST)) & 1
            yield lambda bi=bi, fpar=fpar: b["kfull", bi].done(fpar)
            flags, payload = self._read_meta(c, bi, "softmax")
            if SOLO in flags and "solo_switch" in self.rules:
                step = 1
            if END in flags:
                b["p_full", t].arrive()   # acknowledges END
                return
            assert payload[0] == t, ("a chunk of the other stream", t, payload)
            self.consumed[t].append(payload)
            par = n & 1
            yield lambda par=par: b["s_full", t].done(par)
            b["s_free", t].arrive()
            b["p_full", t].arrive()
            yield lambda par=par: b["o_full", t].done(par)
            b["o_free", t].arrive()
            n += 1
            c += step

    # ------------------------------------------------------------- engine
    def _complete_one(self):
        opts = [("copy", x) for x in self.copies] + [("commit", t) for t in (0, 1) if self.commits[t]]
        if not opts:
            return False
        kind, x = self.rng.choice(opts)
        b = self.bar
        if kind == "commit":
            what, s, c = self.commits[x].pop(0)
            if what == "score":
                b["s_full", x].arrive()
                self.kreg[s][1] = "free"
                b["kempty", s].arrive()
            else:
                b["o_full", x].arrive()
                self.vreg[s][1] = "free"
                b["vempty", s].arrive()
        else:
            self.copies.remove(x)
            half, s, bi, c = x
            reg = self.kreg if half == "k" else self.vreg
            assert reg[s] == [c, "loading"]
            reg[s][1] = "ready"
            b["kfull" if half == "k" else "vfull", bi].complete_tx(1)
        return True

    def run(self, max_steps=10 ** 6):
        roles = {"scheduler": self.scheduler(), "producer": self.producer(),
                 "mma0": self.issuer(0), "mma1": self.issuer(1),
                 "softmax0": self.softmax(0), "softmax1": self.softmax(1)}
        waits = {k: next(g) for k, g in roles.items()}
        victim, starve, steps = None, 0, 0
        while roles:
            ready = [k for k in roles if waits[k]()]
            if starve == 0 and self.rng.random() < 0.02:
                victim, starve = self.rng.choice(sorted(roles)), self.rng.randint(20, 400)
            if starve > 0:
                starve -= 1
                if victim in ready and len(ready) > 1:
                    ready.remove(victim)
            if (not ready or self.rng.random() < 0.3) and self._complete_one():
                continue
            assert ready, f"deadlock: {sorted(roles)} wait"
            k = self.rng.choice(ready)
            try:
                waits[k] = roles[k].send(None)
            except StopIteration:
                del roles[k]
            steps += 1
            assert steps < max_steps
        while self._complete_one():
            pass
        for t in (0, 1):
            want = [(t, j, k) for j, n in enumerate(self.items[t]) for k in range(n)]
            assert self.consumed[t] == want, ("chunks lost or reordered", t)


def random_items(rng):
    """Items per stream, each 1-4 chunks; a stream may have none."""
    return [[rng.randint(1, 4) for _ in range(rng.randint(0, 6))] for _ in range(2)]


def run_schedules(n, seed, rules=RULES):
    rng = random.Random(seed)
    for _ in range(n):
        RingModel(rng, random_items(rng), rules).run()
