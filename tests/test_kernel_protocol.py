"""A model check of the attention kernel's whole synchronisation protocol (CPU only).

Every role of one block is an actor: the list builder (single-launch path), the producer (Q tile
and K/V chunk fills), the two tensor-core issuers and the two softmax groups.  Copies and MMAs
complete asynchronously, in issue order per issuer, through a hardware actor.  Every barrier of
the kernel is modelled with mbarrier parity semantics: a waiter keeps one phase bit per barrier,
exactly as the kernel does, and a wait passes when the barrier's phase parity differs from it.
Besides that, the model tracks which phase each wait is *meant* to see, and fails when a wait
passes before that phase completed, or when a schedule can make no progress.

The roles' orders of waits and arrivals restate the kernel's (csrc/attend.cu): item n belongs to
softmax group n % 2 and uses Q slot n % 2 and kept-row list slot n % 4; K/V chunks go round a
3-slot ring in production order, with one "full" barrier per slot and group.
"""
import random

import pytest


class Bar:
    def __init__(self, name):
        self.name = name
        self.done = 0  # completed phases

    def passes(self, bit):
        return self.done % 2 != bit


class Model:
    def __init__(self, nkc, fused, rng):
        self.nkc, self.fused, self.rng = nkc, fused, rng
        self.items = len(nkc)
        B = {}

        def bar(name):
            B[name] = Bar(name)
            return B[name]

        self.q_full = [bar(f"q_full{s}") for s in range(2)]
        self.q_empty = [bar(f"q_empty{s}") for s in range(2)]
        self.kv_full = [[bar(f"kv_full{s}.{g}") for g in range(2)] for s in range(3)]
        self.kv_empty = [bar(f"kv_empty{s}") for s in range(3)]
        self.s_full = [bar(f"s_full{g}") for g in range(2)]
        self.p_full = [bar(f"p_full{g}") for g in range(2)]
        self.s_free = [bar(f"s_free{g}") for g in range(2)]
        self.o_full = [bar(f"o_full{g}") for g in range(2)]
        self.o_free = [bar(f"o_free{g}") for g in range(2)]
        self.idx_full = [bar(f"idx_full{s}") for s in range(4)]
        self.idx_free = [bar(f"idx_free{s}") for s in range(4)]
        self.hw = []  # pending asynchronous completions: (source, barrier, check) in issue order
        # chunk slots in production order
        self.slot = {}
        t = 0
        for n, k in enumerate(nkc):
            for c in range(k):
                self.slot[(n, c)] = t % 3
                t += 1
        self.actors = [self.list_builder(), self.producer(), self.issuer(0), self.issuer(1),
                       self.softmax(0), self.softmax(1)]
        self.finished = [False] * len(self.actors)

    # -- helpers: a generator yields ("wait", barrier, bit, expected_phase) or ("step",)
    def wait(self, bar, bit, phase):
        """Wait for completed phase `phase` (0-based) of `bar` with the waiter's parity `bit`."""
        return ("wait", bar, bit, phase)

    def complete_async(self, source, bar):
        self.hw.append((source, bar))

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

    def producer(self):
        qb = kb = fb = 0
        qfill = [0, 0]
        kvfill = [0, 0, 0]
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
            self.complete_async("copy", self.q_full[qs])
            for c in range(self.nkc[n]):
                s = self.slot[(n, c)]
                if kvfill[s] >= 1:
                    yield self.wait(self.kv_empty[s], ((kb >> s) & 1) ^ 1, kvfill[s] - 1)
                kb ^= 1 << s
                kvfill[s] += 1
                self.complete_async("copy", self.kv_full[s][g])
            yield ("step",)

    def issuer(self, g):
        qb = kb = pb = sb = ob = 0
        own_kv = [0, 0, 0]  # fills of kv_full[s][g] seen so far
        qseen = 0
        s_busy = False
        pv_done = 0
        items_done = 0
        for n in range(self.items):
            if n % 2 != g:
                continue
            qs = n % 2
            yield self.wait(self.q_full[qs], (qb >> qs) & 1, qseen)
            qb ^= 1 << qs
            qseen += 1
            for c in range(self.nkc[n]):
                s = self.slot[(n, c)]
                yield self.wait(self.kv_full[s][g], (kb >> s) & 1, own_kv[s])
                kb ^= 1 << s
                own_kv[s] += 1
                if s_busy:
                    yield self.wait(self.s_free[g], sb, pv_done - 1)
                    sb ^= 1
                self.complete_async(f"mma{g}", self.s_full[g])
                if c == self.nkc[n] - 1:
                    self.complete_async(f"mma{g}", self.q_empty[qs])
                yield self.wait(self.p_full[g], pb, pv_done)
                pb ^= 1
                if c == 0 and items_done >= 1:
                    yield self.wait(self.o_free[g], ob, items_done - 1)
                    ob ^= 1
                self.complete_async(f"mma{g}", self.o_full[g])
                self.complete_async(f"mma{g}", self.s_free[g])
                self.complete_async(f"mma{g}", self.kv_empty[s])
                pv_done += 1
                s_busy = True
            items_done += 1

    def softmax(self, g):
        sb = ob = fb = 0
        s_seen = o_seen = 0
        for n in range(self.items):
            if n % 2 != g:
                continue
            for c in range(self.nkc[n]):
                yield self.wait(self.s_full[g], sb, s_seen)
                sb ^= 1
                s_seen += 1
                if c > 0:
                    yield self.wait(self.o_full[g], ob, o_seen)
                    ob ^= 1
                    o_seen += 1
                yield ("step",)
                self.p_full[g].done += 1
            yield self.wait(self.o_full[g], ob, o_seen)
            ob ^= 1
            o_seen += 1
            if self.fused:
                s = n % 4
                yield self.wait(self.idx_full[s], (fb >> s) & 1, n // 4)
                fb ^= 1 << s
            yield ("step",)
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
            sources = []
            for src, _ in self.hw:
                if src not in sources:
                    sources.append(src)
            choices += [("hw", src) for src in sources]
            if not choices:
                return "ok" if all(self.finished) and not self.hw else "stuck"
            kind, who = self.rng.choice(choices)
            if kind == "hw":
                k = next(j for j, (src, _) in enumerate(self.hw) if src == who)  # in order per source
                _, bar = self.hw.pop(k)
                bar.done += 1
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
        return "stuck"


def random_cases(count, seed):
    rng = random.Random(seed)
    for _ in range(count):
        nkc = [rng.randint(1, 3) for _ in range(rng.randint(1, 10))]
        yield nkc, random.Random(rng.random())


@pytest.mark.parametrize("fused", [False, True])
def test_protocol_never_passes_early_or_hangs(fused):
    bad = []
    for nkc, rng in random_cases(1500, 7 + fused):
        out = Model(nkc, fused, rng).run()
        if out != "ok":
            bad.append((nkc, out))
    assert not bad, bad[:5]


def test_model_sees_a_shared_kv_barrier_fail():
    """With one K/V full barrier per slot shared by both groups (each issuer waiting only on its
    own chunks), some schedule passes a wait early or hangs: the check has teeth."""
    bad = 0
    for nkc, rng in random_cases(1500, 11):
        m = Model(nkc, False, rng)
        shared = [Bar(f"kv_full{s}") for s in range(3)]
        m.kv_full = [[shared[s], shared[s]] for s in range(3)]
        m.actors = [m.list_builder(), m.producer(), m.issuer(0), m.issuer(1), m.softmax(0), m.softmax(1)]
        if m.run() != "ok":
            bad += 1
    assert bad > 0
