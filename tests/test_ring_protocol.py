"""A model check of the K/V ring protocol of the attention kernel (CPU only).

The kernel's producer fills a 3-slot K/V ring in item order; each work item belongs to one of two
softmax groups (item n to group n % 2), and each group's tensor-core issuer consumes only its
own items' chunks and releases each slot with its PV.  Waits are mbarrier parity waits, which
pass when the barrier's current phase parity differs from the awaited one -- so a waiter that is
a phase ahead (or two behind) of the barrier would pass early (or hang).

The model runs the producer and both issuers under random interleavings and checks that every
wait that passes corresponds to the fill it was waiting for, and that the schedule always
completes.  With one "full" barrier per slot per group (the kernel's protocol) it must hold for
every schedule; with one shared "full" barrier per slot and the other group's fills skipped by
flipping the phase bit, some schedule must break it (the model can see the failure it guards
against).
"""
import random

import pytest


class Barrier:
    """mbarrier phases: `done` completed phases; a parity wait for phase k passes iff done % 2 != k % 2."""

    def __init__(self):
        self.done = 0

    def passes(self, parity):
        return self.done % 2 != parity


def run(nkc, per_group, rng, max_release_lag=3):
    """One random schedule.  Returns 'ok', 'early' (a wait passed before its fill) or 'stuck'."""
    S = 3
    chunks = [(n, c) for n, k in enumerate(nkc) for c in range(k)]  # production order
    slot_of = [t % S for t in range(len(chunks))]
    full = {(s, g): Barrier() for s in range(S) for g in range(2)} if per_group else {s: Barrier() for s in range(S)}
    empty = [Barrier() for _ in range(S)]
    filled = set()  # chunk indices whose data has landed

    def full_bar(t):
        return full[(slot_of[t], chunks[t][0] % 2)] if per_group else full[slot_of[t]]

    # producer state
    prod = {"t": 0, "fills": [0] * S}
    # issuer state: chunk cursor over all chunks, phase bits, pending releases
    iss = [{"t": 0, "ph": [0] * S, "pending": []} for _ in range(2)]

    def producer_step():
        t = prod["t"]
        if t >= len(chunks):
            return False
        s = slot_of[t]
        j = prod["fills"][s]  # this is fill j of slot s: wait for release j - 1 (parity idiom)
        if not empty[s].passes(((j & 1) ^ 1)):
            return False
        prod["fills"][s] += 1
        filled.add(t)
        full_bar(t).done += 1
        prod["t"] += 1
        return True

    def issuer_step(g):
        st = iss[g]

        def release():
            t = st["pending"].pop(0)  # its PV completes: the slot is free again
            empty[slot_of[t]].done += 1
            return True

        # sometimes let a release happen first (PVs complete with some lag)
        if st["pending"] and (len(st["pending"]) > max_release_lag or rng.random() < 0.5):
            return release()
        t = st["t"]
        if t < len(chunks):
            s = slot_of[t]
            if chunks[t][0] % 2 != g:
                if not per_group:
                    st["ph"][s] ^= 1  # the shared barrier's phase moves with the other group's fill
                st["t"] += 1
                return True
            if full_bar(t).passes(st["ph"][s]):
                if t not in filled:
                    raise AssertionError("early")
                st["ph"][s] ^= 1
                st["pending"].append(t)
                st["t"] += 1
                return True
        # blocked or finished: an outstanding PV can still complete
        return release() if st["pending"] else False

    actors = [producer_step, lambda: issuer_step(0), lambda: issuer_step(1)]
    for _ in range(100000):
        order = actors[:]
        rng.shuffle(order)
        progressed = False
        for a in order:
            try:
                if a():
                    progressed = True
                    break
            except AssertionError:
                return "early"
        done = prod["t"] == len(chunks) and all(st["t"] == len(chunks) and not st["pending"] for st in iss)
        if done:
            return "ok"
        if not progressed:
            return "stuck"
    return "stuck"


def schedules(count, seed):
    rng = random.Random(seed)
    for _ in range(count):
        items = rng.randint(1, 9)
        nkc = [rng.randint(1, 4) for _ in range(items)]
        yield nkc, random.Random(rng.random())


@pytest.mark.parametrize("lag", [0, 3])  # 0: a group's chunk is released before it takes the next, as in the kernel
def test_per_group_full_barriers_never_pass_early_or_hang(lag):
    outcomes = {run(nkc, True, r, max_release_lag=lag) for nkc, r in schedules(3000, 1)}
    assert outcomes == {"ok"}, outcomes


def test_shared_full_barrier_can_pass_early():
    outcomes = [run(nkc, False, r) for nkc, r in schedules(3000, 2)]
    assert any(o != "ok" for o in outcomes)


@pytest.mark.parametrize("nkc", [[1] * 8, [2] * 8, [4, 1, 4, 1, 4, 1], [3, 3, 1, 2, 4]])
def test_fixed_shapes(nkc):
    for seed in range(200):
        assert run(nkc, True, random.Random(seed)) == "ok"
