"""A model of the tensor-core forward kernel's mbarrier protocol, run under
random interleavings on the CPU.

Each role of the kernel's CTA is a generator: the Q/K and V TMA producers,
one MMA issuer per tensor-memory buffer, one softmax warpgroup per buffer,
and the epilogue warpgroup, which takes every pair in order and receives
each pair's row sums through shared memory.  Every role waits and arrives
exactly as the kernel does (a warpgroup's arrivals are one arrival here).  The
asynchronous completions -- a TMA load landing, an MMA chain finishing --
fire after random delays.  A barrier holds a completed-phase count, and a
parity wait succeeds when the current phase's parity differs from the parity
waited for, as mbarrier.try_wait.parity does.  The model checks that:

  * every successful wait observes exactly the phase it was meant for (no
    parity aliasing);
  * no shared-memory slot is overwritten while an MMA still reads it, and
    every MMA reads the pair it was meant for;
  * no tensor-memory S, P or O buffer is reused while still in use, and no
    shared-memory row-sum slot is overwritten before the epilogue read it;
  * nothing deadlocks.

This covers every combination the kernel builds: 1-3 stages, 1-2 buffers,
and V sharing the K slot.  O overlays the dead part of its buffer's S.  The
last tests plant two protocol mistakes -- one "full" barrier per stage
shared by both issuers (met while building the kernel), and an epilogue that
releases a buffer before reading its O -- and check that the model catches
them.
"""
import random

import pytest


class Barrier:
    def __init__(self, name, count=1):
        self.name, self.count, self.completed, self.pending = name, count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.completed += 1

    def try_wait(self, phase):
        """Wait for the completion of `phase` (parity phase & 1)."""
        ok = (self.completed & 1) != (phase & 1)
        if ok and self.completed != phase + 1:
            raise AssertionError(f"{self.name}: wait for phase {phase} passed with {self.completed} completed")
        return ok


class ProtocolError(AssertionError):
    pass


def simulate(stages, nbuf, alias, npairs, seed, split_full=True, early_release=False):
    rnd = random.Random(seed)
    lcm = stages if stages % nbuf == 0 else stages * nbuf
    # split_full: one Q/K and one V "full" barrier per (stage, buffer), as in the kernel
    fkey = (lambda n: (n % stages, n % nbuf)) if split_full else (lambda n: (n % stages, 0))
    fphase = (lambda n: n // lcm) if split_full else (lambda n: n // stages)
    kfull = {(s, b): Barrier(f"kfull{s}{b}") for s in range(stages) for b in range(nbuf)}
    vfull = {(s, b): Barrier(f"vfull{s}{b}") for s in range(stages) for b in range(nbuf)}
    kempty = [Barrier(f"kempty{s}") for s in range(stages)]
    vempty = [Barrier(f"vempty{s}") for s in range(stages)]
    s_full = [Barrier(f"s_full{b}") for b in range(nbuf)]
    p_full = [Barrier(f"p_full{b}") for b in range(nbuf)]
    o_full = [Barrier(f"o_full{b}") for b in range(nbuf)]
    o_empty = [Barrier(f"o_empty{b}") for b in range(nbuf)]
    l_full = {(b, par): Barrier(f"l_full{b}{par}") for b in range(nbuf) for par in (0, 1)}
    lsum = {}                                                # row sums in shared memory, per buffer and parity

    kslot, vslot = [None] * stages, [None] * stages          # pair held by each slot
    kreaders, vreaders = [set() for _ in range(stages)], [set() for _ in range(stages)]
    S, O = [None] * nbuf, [None] * nbuf                      # pair held by each buffer's S and O
    events, clock, seq = [], [0], [0]

    def later(fn, delay=None):
        seq[0] += 1
        events.append((clock[0] + (rnd.randint(1, 20) if delay is None else delay), seq[0], fn))

    def check(cond, what):
        if not cond:
            raise ProtocolError(what)

    def qk_producer():
        for n in range(npairs):
            s = n % stages
            if n >= stages:  # the slot's previous user is done with it
                prev = vempty[s] if alias else kempty[s]
                while not prev.try_wait(n // stages - 1):
                    yield
            check(not kreaders[s] and not (alias and vreaders[s]), f"Q/K slot {s} reused while read")

            def land(n=n, s=s):
                check(not kreaders[s] and not (alias and vreaders[s]), f"Q/K slot {s} landed while read")
                kslot[s] = n
                kfull[fkey(n)].arrive()
            later(land)
        yield "done"

    def v_producer():
        for n in range(npairs):
            s = n % stages
            if alias:  # V goes into the K slot once S = QK^T has read this pair's K
                while not kempty[s].try_wait(n // stages):
                    yield
            elif n >= stages:
                while not vempty[s].try_wait(n // stages - 1):
                    yield
            check(not vreaders[s] and not (alias and kreaders[s]), f"V slot {s} reused while read")

            def land(n=n, s=s):
                check(not vreaders[s] and not (alias and kreaders[s]), f"V slot {s} landed while read")
                vslot[s] = n
                vfull[fkey(n)].arrive()
            later(land)
        yield "done"

    def issuer(b):
        for use, n in enumerate(range(b, npairs, nbuf)):
            s = n % stages
            while not kfull[fkey(n)].try_wait(fphase(n)):
                yield
            check(kslot[s] == n, f"QK({n}) reads Q/K of pair {kslot[s]}")
            if use > 0:  # the epilogue has read the buffer's O, which overlays S
                while not o_empty[b].try_wait(use - 1):
                    yield
            check(S[b] is None, f"QK({n}) overwrites S of pair {S[b]}")
            kreaders[s].add(n)
            qk_time = rnd.randint(1, 10)

            def qk_done(n=n, s=s, b=b):
                check(kslot[s] == n, f"Q/K slot of pair {n} changed under QK")
                check(O[b] is None, f"QK({n}) overwrites O of pair {O[b]} before the epilogue read it")
                kreaders[s].discard(n)
                S[b] = n
                s_full[b].arrive()
                kempty[s].arrive()
            later(qk_done, qk_time)

            while not p_full[b].try_wait(use):
                yield
            while not vfull[fkey(n)].try_wait(fphase(n)):
                yield
            check(vslot[s] == n, f"PV({n}) reads V of pair {vslot[s]}")
            check(S[b] == n, f"PV({n}) reads P of pair {S[b]}")
            check(O[b] is None, f"PV({n}) overwrites O of pair {O[b]}")
            vreaders[s].add(n)

            def pv_done(n=n, s=s, b=b):
                check(vslot[s] == n, f"V slot of pair {n} changed under PV")
                vreaders[s].discard(n)
                O[b] = n
                o_full[b].arrive()
                vempty[s].arrive()
            later(pv_done, qk_time + rnd.randint(1, 10))
        yield "done"

    def softmax_group(g):
        for use, n in enumerate(range(g, npairs, nbuf)):
            while not s_full[g].try_wait(use):
                yield
            check(S[g] == n, f"softmax of pair {n} finds S of pair {S[g]}")
            for _ in range(rnd.randint(0, 15)):
                yield
            slot = (g, use & 1)
            check(lsum.get(slot, "read") == "read", f"row sums of pair {n} overwrite unread ones")
            lsum[slot] = n
            l_full[slot].arrive()
            p_full[g].arrive()
        yield "done"

    def epilogue():
        for n in range(npairs):
            b, use = n % nbuf, n // nbuf
            while not l_full[(b, use & 1)].try_wait(use >> 1):
                yield
            check(lsum[(b, use & 1)] == n, f"epilogue of pair {n} reads the row sums of pair {lsum[(b, use & 1)]}")
            lsum[(b, use & 1)] = "read"
            while not o_full[b].try_wait(use):
                yield
            if early_release:  # planted mistake: the buffer is released before O is read
                o_empty[b].arrive()
                for _ in range(rnd.randint(0, 20)):
                    yield
            check(O[b] == n, f"epilogue of pair {n} finds O of pair {O[b]}")
            O[b] = None
            S[b] = None
            if not early_release:
                o_empty[b].arrive()
            for _ in range(rnd.randint(0, 5)):
                yield
        yield "done"

    roles = [qk_producer(), v_producer()] + [issuer(b) for b in range(nbuf)] + [softmax_group(g)
                                                                                 for g in range(nbuf)] + [epilogue()]
    done = [False] * len(roles)
    for _ in range(10 ** 6):
        if all(done):
            return
        events.sort()
        while events and events[0][0] <= clock[0]:
            events.pop(0)[2]()
        i = rnd.randrange(len(roles))
        if not done[i] and next(roles[i]) == "done":
            done[i] = True
        clock[0] += 1
    raise ProtocolError("deadlock")


COMBOS = [(st, nb, al) for st in (1, 2, 3) for nb in (1, 2) for al in (False, True)]


@pytest.mark.parametrize("stages,nbuf,alias", COMBOS)
def test_protocol_under_random_interleavings(stages, nbuf, alias):
    for seed in range(60):
        for npairs in (1, 2, 3, 5, 8, 13):
            simulate(stages, nbuf, alias, npairs, seed * 100 + npairs)


def test_model_catches_a_full_barrier_shared_by_both_issuers():
    # one "full" barrier per stage, waited on by both issuers: with one stage the
    # second issuer's parity wait passes a phase early
    with pytest.raises(AssertionError):
        for seed in range(40):
            simulate(1, 2, False, 6, seed, split_full=False)


def test_model_catches_a_buffer_released_before_its_o_is_read():
    # the epilogue arrives on o_empty before it has read O: the buffer's next
    # S = Q K^T, which overwrites the columns O overlays, may then land first
    with pytest.raises(AssertionError):
        for seed in range(200):
            for npairs in (3, 5, 8):
                simulate(2, 2, False, npairs, seed, early_release=True)
