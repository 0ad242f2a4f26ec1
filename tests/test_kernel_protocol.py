"""A model check of the attention kernel's whole synchronisation protocol (CPU only).

Every role of one block is an actor: the list builder (single-launch path), the producer (Q tile
and K/V chunk fills), the two tensor-core issuers, the two softmax groups and the two V-tile
warps.  Copies and MMAs complete asynchronously through a hardware actor: MMAs in issue order per
issuer, copies in issue order per ring slot (fills of different slots may land in any order).  Every barrier of
the kernel is modelled with mbarrier parity semantics: a waiter keeps one phase bit per barrier,
exactly as the kernel does, and a wait passes when the barrier's phase parity differs from it.
Besides that, the model tracks which phase each wait is *meant* to see, and fails when a wait
passes before that phase completed, or when a schedule can make no progress.  It also tracks who
owns each group's TMEM buffers -- S (written by Q K^T, read by the softmax), P (written by the
softmax, read by the PV MMA) and O (accumulated by PV, rescaled and read out by the softmax) --
and fails when a writer or reader touches a buffer another role still owns.

On the single-launch path each copier warp is an actor of its own running the producer loop; the
Q and K/V full barriers complete a phase after one arrival per copier, and an arrival must land in
the phase of the fill it belongs to (checked for two copiers, the kernel, and three).

The roles' orders of waits and arrivals restate the kernel's (csrc/attend.cu): item n belongs to
softmax group n % 2 and uses Q slot n % 2 and kept-row list slot n % 4; K/V chunks go round a
4-slot ring in production order, with one "full" barrier per slot and group (the 3-slot ring of an
earlier design is checked too).
"""
import random

import pytest


class Bar:
    def __init__(self, name, count=1):
        self.name = name
        self.done = 0  # completed phases
        self.count = count  # arrivals that complete a phase
        self.pending = 0

    def passes(self, bit):
        return self.done % 2 != bit

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.done += 1


class Model:
    def __init__(self, nkc, fused, rng, early_qk=False, shared_v_ready=False, v_mode="slot", stages=4, starve=(),
                 copiers=1, full_count=None):
        self.nkc, self.fused, self.rng = nkc, fused, rng
        # single-launch path: `copiers` warps each run the producer loop and each arrives once per
        # fill on the Q / K/V full barriers, whose phases complete after `full_count` arrivals (the
        # kernel: 32 * kCopyWarps lanes, modelled as one arrival per warp); planted mistake: a count
        # that assumes fewer copiers than run
        self.copiers = copiers if fused else 1
        full_count = self.copiers if full_count is None else full_count
        self.stages = stages  # K/V ring slots (the kernel's kKVStages)
        self.early_qk = early_qk  # planted mistake: the next S = Q K^T before the softmax released S
        self.shared_v_ready = shared_v_ready  # planted mistake: one V-ready barrier per group
        # V warps: "slot" -- warp w owns ring slots s = w (mod 2), waits for and prepares every fill of
        # them (the kernel); planted mistakes: "observe_all" -- warp w prepares fills w, w + 2, ... and
        # waits for every fill; "alt_skip" -- it prepares fills w, w + 2, ... and waits only for those
        self.v_mode = v_mode
        self.starve = set(starve)  # actors scheduled only when nothing else can move
        self.v_fill = {}  # fill -> "landed" / "ready" (what the V warps may rely on)
        self.items = len(nkc)
        B = {}

        def bar(name, count=1):
            B[name] = Bar(name, count)
            return B[name]

        self.q_full = [bar(f"q_full{s}", full_count) for s in range(2)]
        self.q_empty = [bar(f"q_empty{s}") for s in range(2)]
        self.kv_full = [[bar(f"kv_full{s}.{g}", full_count) for g in range(2)] for s in range(stages)]
        self.kv_empty = [bar(f"kv_empty{s}") for s in range(stages)]
        self.s_full = [bar(f"s_full{g}") for g in range(2)]
        self.p_full = [bar(f"p_full{g}") for g in range(2)]
        self.pv_done = [bar(f"pv_done{g}") for g in range(2)]
        self.v_ready = [[bar(f"v_ready{s}.{g}") for g in range(2)] for s in range(stages)]
        if shared_v_ready:
            one = [bar("v_ready0"), bar("v_ready1")]
            self.v_ready = [[one[0], one[1]] for _ in range(stages)]
        self.o_free = [bar(f"o_free{g}") for g in range(2)]
        # buffer ownership per group: S "free" / "qk" (MMA writing) / "softmax"; P "free" /
        # "softmax" (written) / "pv" (MMA reading); O: PVs in flight, and whether the epilogue holds it
        self.S = ["free", "free"]
        self.P = ["free", "free"]
        self.pv_flight = [0, 0]
        self.o_reading = [False, False]
        self.error = None
        self.idx_full = [bar(f"idx_full{s}") for s in range(4)]
        self.idx_free = [bar(f"idx_free{s}") for s in range(4)]
        self.hw = []  # pending asynchronous completions: (source, barrier, check) in issue order
        # chunk slots in production order
        self.slot = {}
        t = 0
        for n, k in enumerate(nkc):
            for c in range(k):
                self.slot[(n, c)] = t % stages
                t += 1
        self.actors = [self.list_builder()] + [self.producer(j) for j in range(self.copiers)] + [
            self.issuer(0), self.issuer(1), self.softmax(0), self.softmax(1), self.v_warp(0), self.v_warp(1)]
        self.finished = [False] * len(self.actors)

    # -- helpers: a generator yields ("wait", barrier, bit, expected_phase) or ("step",)
    def wait(self, bar, bit, phase):
        """Wait for completed phase `phase` (0-based) of `bar` with the waiter's parity `bit`."""
        return ("wait", bar, bit, phase)

    def complete_async(self, source, bar, effect=None):
        self.hw.append((source, bar, effect))

    def check(self, cond, what):
        if not cond and self.error is None:
            self.error = what

    def list_builder(self):
        if not self.fused:
            return
        free_bits = 0
        for n in range(self.items):
            s = n % 4
            if n >= 4:  # slot reuse: the epilogue of item n - 4 released it
                yield self.wait(self.idx_free[s], ((free_bits >> s) & 1) ^ 1, n // 4 - 1)
            free_bits ^= 1 << s
            yield ("step",)
            self.idx_full[s].done += 1

    def arrival(self, bar, fill):
        """An arrival for fill `fill` (0-based) of a full barrier: it must land in that phase."""
        def effect():
            self.check(bar.done == fill, f"an arrival for fill {fill} of {bar.name} landed in phase {bar.done}")
        return effect

    def producer(self, j=0):
        qb = kb = fb = 0
        qfill = [0, 0]
        kvfill = [0] * self.stages
        kvseen = {}  # fills of kv_full[s][g] issued so far
        for n in range(self.items):
            g = n % 2
            if self.fused:
                s = n % 4
                yield self.wait(self.idx_full[s], (fb >> s) & 1, n // 4)
                fb ^= 1 << s
            qs = n % 2
            if qfill[qs] >= 1:
                yield self.wait(self.q_empty[qs], ((qb >> qs) & 1) ^ 1, qfill[qs] - 1)
            qb ^= 1 << qs
            qfill[qs] += 1
            self.complete_async(f"copy{j}_q{qs}", self.q_full[qs], self.arrival(self.q_full[qs], qfill[qs] - 1))
            for c in range(self.nkc[n]):
                s = self.slot[(n, c)]
                if kvfill[s] >= 1:
                    yield self.wait(self.kv_empty[s], ((kb >> s) & 1) ^ 1, kvfill[s] - 1)
                kb ^= 1 << s
                kvfill[s] += 1
                f = kvseen.get((s, g), 0)
                kvseen[(s, g)] = f + 1
                # bulk copies into different slots may land in any order
                self.complete_async(f"copy{j}_kv{s}", self.kv_full[s][g], self.arrival(self.kv_full[s][g], f))
            yield ("step",)

    def v_warp(self, vw):
        """V warp vw (of two), in production order, as each fill lands (see v_mode)."""
        kb = 0
        seen = {}  # fills of kv_full[s][g] seen so far
        fill = 0
        for n in range(self.items):
            g = n % 2
            for c in range(self.nkc[n]):
                s = self.slot[(n, c)]
                k = seen.get((s, g), 0)
                if self.v_mode == "slot":
                    mine = watch = s % 2 == vw
                else:
                    mine = fill % 2 == vw
                    watch = mine or self.v_mode == "observe_all"
                if watch:
                    yield self.wait(self.kv_full[s][g], (kb >> (2 * s + g)) & 1, k)
                kb ^= 1 << (2 * s + g)
                seen[(s, g)] = k + 1
                if mine:
                    yield ("step",)
                    self.v_ready[s][g].done += 1
                fill += 1

    def v_wait(self, g, s, bits, seen):
        """A group's wait for the V tile of its next chunk in slot s (per-slot parity bits)."""
        if self.shared_v_ready:
            k = sum(seen.values())
            b = bits.get("all", 0)
            bits["all"] = b ^ 1
        else:
            k = seen.get(s, 0)
            b = bits.get(s, 0)
            bits[s] = b ^ 1
        seen[s] = seen.get(s, 0) + 1
        return self.wait(self.v_ready[s][g], b, k)

    def issuer(self, g):
        qb = kb = pb = ob = 0
        vbits, vseen = {}, {}
        own_kv = [0] * self.stages  # fills of kv_full[s][g] seen so far
        qseen = 0
        p_seen = 0
        items_done = 0

        def qk(qs, last):
            self.check(self.S[g] == "free", f"QK into S{g} while {self.S[g]} owns it")
            self.S[g] = "qk"

            def done():
                self.S[g] = "softmax"
            self.complete_async(f"mma{g}", self.s_full[g], done)
            if last:
                self.complete_async(f"mma{g}", self.q_empty[qs], None)

        def pv(s):
            self.check(self.P[g] == "softmax", f"PV reads P{g} in state {self.P[g]}")
            self.check(not self.o_reading[g], f"PV into O{g} while the epilogue reads it")
            self.P[g] = "pv"
            self.pv_flight[g] += 1

            def done():
                self.P[g] = "free"
                self.pv_flight[g] -= 1
            self.complete_async(f"mma{g}", self.pv_done[g], done)
            self.complete_async(f"mma{g}", self.kv_empty[s], None)

        for n in range(self.items):
            if n % 2 != g:
                continue
            qs = n % 2
            yield self.wait(self.q_full[qs], (qb >> qs) & 1, qseen)
            qb ^= 1 << qs
            qseen += 1
            s0 = self.slot[(n, 0)]
            yield self.wait(self.kv_full[s0][g], (kb >> s0) & 1, own_kv[s0])
            kb ^= 1 << s0
            own_kv[s0] += 1
            qk(qs, self.nkc[n] == 1)
            for c in range(self.nkc[n]):
                s = self.slot[(n, c)]
                if self.early_qk and c + 1 < self.nkc[n]:
                    sn = self.slot[(n, c + 1)]
                    yield self.wait(self.kv_full[sn][g], (kb >> sn) & 1, own_kv[sn])
                    kb ^= 1 << sn
                    own_kv[sn] += 1
                    qk(qs, c + 1 == self.nkc[n] - 1)
                yield self.wait(self.p_full[g], pb, p_seen)
                pb ^= 1
                p_seen += 1
                if c + 1 < self.nkc[n] and not self.early_qk:
                    sn = self.slot[(n, c + 1)]
                    yield self.wait(self.kv_full[sn][g], (kb >> sn) & 1, own_kv[sn])
                    kb ^= 1 << sn
                    own_kv[sn] += 1
                    qk(qs, c + 1 == self.nkc[n] - 1)
                if c == 0 and items_done >= 1:
                    yield self.wait(self.o_free[g], ob, items_done - 1)
                    ob ^= 1
                yield self.v_wait(g, s, vbits, vseen)
                pv(s)
            items_done += 1

    def softmax(self, g):
        sb = pvb = fb = 0
        s_seen = pv_seen = 0
        vbits, vseen = {}, {}
        for n in range(self.items):
            if n % 2 != g:
                continue
            for c in range(self.nkc[n]):
                yield self.wait(self.s_full[g], sb, s_seen)
                sb ^= 1
                s_seen += 1
                self.check(self.S[g] == "softmax", f"softmax reads S{g} in state {self.S[g]}")
                if c > 0:
                    yield self.wait(self.pv_done[g], pvb, pv_seen)
                    pvb ^= 1
                    pv_seen += 1
                    self.check(self.pv_flight[g] == 0, f"O{g} rescaled while a PV is in flight")
                yield self.v_wait(g, self.slot[(n, c)], vbits, vseen)
                self.check(self.P[g] == "free", f"softmax writes P{g} in state {self.P[g]}")
                yield ("step",)
                self.check(self.S[g] == "softmax", f"S{g} overwritten during the softmax")
                self.S[g] = "free"
                self.P[g] = "softmax"
                self.p_full[g].done += 1
            yield self.wait(self.pv_done[g], pvb, pv_seen)
            pvb ^= 1
            pv_seen += 1
            self.check(self.pv_flight[g] == 0, f"O{g} read out while a PV is in flight")
            if self.fused:
                s = n % 4
                yield self.wait(self.idx_full[s], (fb >> s) & 1, n // 4)
                fb ^= 1 << s
            self.o_reading[g] = True
            yield ("step",)
            self.o_reading[g] = False
            self.o_free[g].done += 1
            if self.fused:
                self.idx_free[n % 4].done += 1

    def run(self):
        pending = [None] * len(self.actors)  # the wait an actor is blocked on
        for _ in range(200000):
            choices = []
            for i, a in enumerate(self.actors):
                if self.finished[i]:
                    continue
                w = pending[i]
                if w is None or w[1].passes(w[2]):
                    choices.append(("actor", i))
            if self.error is not None:
                return f"hazard:{self.error}"
            sources = []
            for src, _, _ in self.hw:
                if src not in sources:
                    sources.append(src)
            choices += [("hw", src) for src in sources]
            if not choices:
                return "ok" if all(self.finished) and not self.hw else "stuck"
            preferred = [c for c in choices if not (c[0] == "actor" and c[1] in self.starve)]
            kind, who = self.rng.choice(preferred or choices)
            if kind == "hw":
                k = next(j for j, (src, _, _) in enumerate(self.hw) if src == who)  # in order per source
                _, bar, effect = self.hw.pop(k)
                if effect is not None:
                    effect()
                bar.arrive()
                continue
            w = pending[who]
            if w is not None and w[1].done <= w[3]:
                return f"early:{w[1].name}"
            pending[who] = None
            try:
                nxt = next(self.actors[who])
            except StopIteration:
                self.finished[who] = True
                continue
            if nxt[0] == "wait":
                pending[who] = nxt
        return "stuck" if self.error is None else f"hazard:{self.error}"


def random_cases(count, seed):
    rng = random.Random(seed)
    for _ in range(count):
        nkc = [rng.randint(1, 3) for _ in range(rng.randint(1, 10))]
        yield nkc, random.Random(rng.random())


ACTORS = ["list", "producer", "issuer0", "issuer1", "softmax0", "softmax1", "v0", "v1"]


@pytest.mark.parametrize("stages", [4, 3])
@pytest.mark.parametrize("fused", [False, True])
def test_protocol_never_passes_early_or_hangs(fused, stages):
    """Random schedules, some of them starving one role (it moves only when nothing else can)."""
    bad = []
    for i, (nkc, rng) in enumerate(random_cases(1500, 7 + fused)):
        starve = () if i % 3 == 0 else (i % len(ACTORS),)
        out = Model(nkc, fused, rng, stages=stages, starve=starve).run()
        if out != "ok":
            bad.append((nkc, starve, out))
    assert not bad, bad[:5]


def test_model_sees_a_shared_kv_barrier_fail():
    """With one K/V full barrier per slot shared by both groups (each issuer waiting only on its
    own chunks), some schedule passes a wait early or hangs: the check has teeth."""
    bad = 0
    for nkc, rng in random_cases(1500, 11):
        m = Model(nkc, False, rng)
        shared = [Bar(f"kv_full{s}") for s in range(m.stages)]
        m.kv_full = [[shared[s], shared[s]] for s in range(m.stages)]
        m.actors = [m.list_builder(), m.producer(), m.issuer(0), m.issuer(1), m.softmax(0), m.softmax(1), m.v_warp(0),
                    m.v_warp(1)]
        m.finished = [False] * len(m.actors)
        if m.run() != "ok":
            bad += 1
    assert bad > 0


def test_model_sees_an_early_qk_fail():
    """Issuing the next chunk's S = Q K^T before the softmax has released S (p_full) is caught as a
    buffer hazard in some schedule: the ownership checks have teeth."""
    bad = 0
    for nkc, rng in random_cases(800, 13):
        if max(nkc) < 2:
            continue
        if Model(nkc, False, rng, early_qk=True).run() != "ok":
            bad += 1
    assert bad > 0


def test_model_sees_a_shared_v_ready_fail():
    """With one V-ready barrier per group (the V warp may prepare two of a group's chunks before
    that group waits for the first), some schedule sees a phase early or hangs."""
    bad = 0
    for nkc, rng in random_cases(800, 17):
        if Model(nkc, False, rng, shared_v_ready=True).run() != "ok":
            bad += 1
    assert bad > 0


def test_model_sees_v_warps_skipping_fills_fail():
    """V warps that prepare alternate fills and wait only for those: with a 3-slot ring a slot's
    fills alternate between the warps, so a parity wait can pass on the fill before (still in
    flight) and some schedule fails."""
    bad = 0
    for nkc, rng in random_cases(800, 19):
        if Model(nkc, False, rng, v_mode="alt_skip", stages=3).run() != "ok":
            bad += 1
    assert bad > 0


def test_model_sees_observing_v_warps_lapped():
    """V warps that prepare alternate fills but wait for every fill: a warp that only looks at a fill
    the other one prepares can be lapped -- the slot is released and refilled for the same group
    before it looks, and its parity wait then sees two phases at once and never passes.  A schedule
    that starves one V warp finds it; owning whole slots (the kernel) cannot be lapped."""
    bad = 0
    for i, (nkc, rng) in enumerate(random_cases(600, 23)):
        if Model(nkc, i % 2 == 1, rng, v_mode="observe_all", starve=(6 + i % 2,)).run() != "ok":
            bad += 1
    assert bad > 0


@pytest.mark.parametrize("copiers", [2, 3])
def test_protocol_with_several_copier_warps(copiers):
    """The single-launch path with two copier warps (the kernel) and three (a tried variant):
    every copier runs the producer loop and arrives once per fill; random schedules, some
    starving one role or one copier, never pass a wait early, never land an arrival in the wrong
    phase, and never hang -- nothing in the protocol assumes two copiers."""
    bad = []
    for i, (nkc, rng) in enumerate(random_cases(1200, 29 + copiers)):
        n_actors = 1 + copiers + 6
        starve = () if i % 3 == 0 else (i % n_actors,)
        out = Model(nkc, True, rng, copiers=copiers, starve=starve).run()
        if out != "ok":
            bad.append((nkc, starve, out))
    assert not bad, bad[:5]


def test_model_sees_a_copier_count_mistake():
    """Three copiers against full barriers that complete after two arrivals (a constant that
    assumes two copiers): some schedule lands an arrival in the wrong phase, passes a wait early
    or hangs -- the check has teeth for the mistake it is meant to rule out."""
    bad = 0
    for nkc, rng in random_cases(600, 31):
        if Model(nkc, True, rng, copiers=3, full_count=2).run() != "ok":
            bad += 1
    assert bad > 0
