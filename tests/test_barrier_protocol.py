"""A model of the tensor-core forward kernel's mbarrier protocol, run under
random interleavings on the CPU.

Each role of the kernel's CTA is a generator: the Q/K and V TMA producers,
one MMA issuer per tensor-memory buffer, one softmax warpgroup per buffer,
and the epilogue warpgroup, which takes every pair in order and receives
each pair's row sums through shared memory.  Every role waits and arrives exactly as the kernel does.  The
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
O shared or overlaying S, and V sharing the K slot.  The last tests plant
the two protocol mistakes met while building the kernel -- one "full"
barrier per stage shared by both issuers, and one "O read" barrier for a
shared O although the epilogue may lag a use behind -- and check that the
model catches them.
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


def simulate(stages, nbuf, shared_o, alias, npairs, seed, split_full=True, split_o_empty=True):
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
    s_free = [Barrier(f"s_free{b}") for b in range(nbuf)]
    # O overlaying S: one o_empty per buffer.  A shared O: one per pair parity,
    # since the epilogue may lag a buffer's softmax by a use
    n_oe = (2 if split_o_empty else 1) if shared_o else nbuf
    o_empty = [Barrier(f"o_empty{o}") for o in range(n_oe)]
    o_empty_of = lambda n: o_empty[n % n_oe]                # o_empty pair n arrives on
    o_slot = (lambda b: 0) if shared_o else (lambda b: b)
    l_full = {(b, par): Barrier(f"l_full{b}{par}") for b in range(nbuf) for par in (0, 1)}
    lsum = {}                                                # row sums in shared memory, per buffer and parity

    kslot, vslot = [None] * stages, [None] * stages          # pair held by each slot
    kreaders, vreaders = [set() for _ in range(stages)], [set() for _ in range(stages)]
    S, O = [None] * nbuf, [None] * (1 if shared_o else nbuf)  # pair held by each buffer
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
            if use > 0:  # S of this buffer is free
                free = s_free[b] if shared_o else o_empty[b]
                while not free.try_wait(use - 1):
                    yield
            check(S[b] is None, f"QK({n}) overwrites S of pair {S[b]}")
            kreaders[s].add(n)
            qk_time = rnd.randint(1, 10)

            def qk_done(n=n, s=s, b=b):
                check(kslot[s] == n, f"Q/K slot of pair {n} changed under QK")
                kreaders[s].discard(n)
                S[b] = n
                s_full[b].arrive()
                kempty[s].arrive()
            later(qk_done, qk_time)

            while not p_full[b].try_wait(use):
                yield
            if shared_o and n > 0:  # the previous pair's epilogue has read O
                while not o_empty_of(n - 1).try_wait((n - 1) // n_oe):
                    yield
            while not vfull[fkey(n)].try_wait(fphase(n)):
                yield
            check(vslot[s] == n, f"PV({n}) reads V of pair {vslot[s]}")
            o = 0 if shared_o else b
            check(O[o] is None, f"PV({n}) overwrites O of pair {O[o]}")
            vreaders[s].add(n)

            def pv_done(n=n, s=s, b=b, o=o):
                check(vslot[s] == n, f"V slot of pair {n} changed under PV")
                vreaders[s].discard(n)
                O[o] = n
                if shared_o:
                    S[b] = None
                o_full[b].arrive()
                vempty[s].arrive()
                if shared_o:
                    s_free[b].arrive()
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
            o = o_slot(b)
            check(O[o] == n, f"epilogue of pair {n} finds O of pair {O[o]}")
            O[o] = None
            if not shared_o:
                S[b] = None
            o_empty_of(n).arrive()
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


COMBOS = [(st, nb, sh, al) for st in (1, 2, 3) for nb in (1, 2) for sh in ((False, True) if nb == 2 else (False,))
          for al in (False, True)]


@pytest.mark.parametrize("stages,nbuf,shared_o,alias", COMBOS)
def test_protocol_under_random_interleavings(stages, nbuf, shared_o, alias):
    for seed in range(40):
        for npairs in (1, 2, 3, 5, 8, 13):
            simulate(stages, nbuf, shared_o, alias, npairs, seed * 100 + npairs)


def test_model_catches_a_full_barrier_shared_by_both_issuers():
    # one "full" barrier per stage, waited on by both issuers: with one stage the
    # second issuer's parity wait passes a phase early
    with pytest.raises(AssertionError):
        for seed in range(40):
            simulate(1, 2, True, False, 6, seed, split_full=False)


def test_model_catches_a_single_o_empty_for_a_shared_o():
    # one barrier for "the epilogue has read the shared O": the epilogue may lag
    # the softmax of a buffer by a use, and the issuer's parity wait passes early
    with pytest.raises(AssertionError):
        for seed in range(200):
            for npairs in (5, 8, 13):
                simulate(3, 2, True, False, npairs, seed, split_o_empty=False)
